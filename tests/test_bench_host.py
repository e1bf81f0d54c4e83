"""Host-side logic of bench.py (CPU): the algorithmic units behind every
throughput it prints, the DRAM-traffic figures tied to the kernel sources
they were captured on, the decode row's inputs exceeding L2, and the
reading of the clock record."""

import hashlib
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_row_units_are_the_closed_forms(bench):
    N, K, g, Md, Mp = bench.N_W, bench.K_W, bench.GROUP, bench.M_DECODE, bench.M_PREFILL
    assert (N, K, g, Md, Mp) == (28672, 8192, 128, 1, 8192)
    u = bench._row_units()
    packed = N * K // 2                 # 0.5 B per weight
    scales = 2 * N * (K // g)           # one fp16 per (row, group)
    assert u["quantize"]["bytes"] == 2 * N * K + packed + scales == 590_872_576
    assert u["unpack"]["bytes"] == packed + N * K == 352_321_536
    assert u["decode"]["bytes"] == packed == 117_440_512
    assert u["decode"]["bytes_total"] == packed + scales + 2 * K + 4 * N
    assert u["prefill"]["flops"] == 2 * Mp * N * K
    # the affine quantizer also writes one uint8 zero point per (row, group)
    assert u["quantize_affine"]["bytes"] == u["quantize"]["bytes"] + N * (K // g)
    assert {r["bound"] for r in u.values()} == {"hbm", "tensor"}


def test_decode_row_inputs_exceed_l2(bench):
    # The decode row streams DECODE_COPIES distinct weight buffers back to
    # back; together they must exceed B200's 126 MB L2 (here: twice over), so
    # that no call finds its weights there.
    assert bench.DECODE_COPIES >= 2
    assert bench.DECODE_COPIES * bench.N_W * bench.K_W // 2 > 126 * 2**20 * 2


def test_traffic_follows_the_source_hash(bench, tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_bytes(b"// kernel source\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_TRAFFIC", {"k": (1234, "kernel.cu", digest)})
    assert bench._traffic("k") == 1234
    src.write_bytes(b"// kernel source, edited\n")
    assert bench._traffic("k") is None           # stale once the source changes
    assert bench._traffic("missing") is None
    src.unlink()
    assert bench._traffic("k") is None


def test_traffic_entries_name_existing_sources(bench):
    for name, (nbytes, path, digest) in bench.KERNEL_TRAFFIC.items():
        assert nbytes > 0 and len(digest) == 64, name
        assert os.path.isfile(os.path.join(ROOT, path)), path


def test_peaks_fall_back_without_the_measured_file(bench, tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench._peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0


def test_clock_summary_reads_the_samples(bench, tmp_path):
    """The clock record of a run: the median SM clock of the samples taken
    under load (idle samples below half the highest are left out), the
    highest max clock, and every throttle reason seen active."""
    rows = [
        "0, 345, 1965, 120.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1965, 1965, 900.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 950.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, [N/A], 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    path = tmp_path / "clocks.csv"
    path.write_text("\n".join(rows) + "\n")
    clk = bench.ClockSampler(0)
    clk.proc, clk.path = object(), str(path)
    s = clk.summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 4
    assert not path.exists()   # the record is removed once read


def test_clock_summary_without_samples(bench, tmp_path):
    path = tmp_path / "clocks.csv"
    path.write_text("")
    clk = bench.ClockSampler(0)
    clk.proc, clk.path = object(), str(path)
    assert clk.summary()["reasons"] == ["no samples"]
    clk2 = bench.ClockSampler(0)
    assert clk2.summary()["reasons"] == ["nvidia-smi unavailable"]

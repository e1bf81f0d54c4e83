"""Helpers for the GPU parity tests: move tensors to NumPy and compare the
CUDA library's outputs with the CPU oracle."""

import numpy as np
import torch

import oracle

# Matmul tolerance factors c in |y - y_ref| <= c * sum_k |x||w_hat|.
TOL_F32 = 1e-5
TOL_HALF = 4e-3


def to_np(t: torch.Tensor) -> np.ndarray:
    """Exact host copy; bf16 is widened to fp32 (exact), fp16 stays fp16."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def oracle_quantize(w: torch.Tensor, group: int):
    wn = to_np(w)
    if wn.dtype == np.float16:
        wn = wn.astype(np.float32)
    return oracle.quantize_int4(wn, group)


def assert_quantize_exact(w, packed, scales, group, rows=None):
    """Bit-exact packed bytes and fp16 scale bits (optionally on sampled rows)."""
    if rows is not None:
        idx = torch.as_tensor(rows, device=w.device)
        w = w.index_select(0, idx)
        packed = packed.index_select(0, idx)
        scales = scales.index_select(0, idx)
    p_ref, s_ref, K = oracle_quantize(w, group)
    p = packed.cpu().numpy()
    s = scales.cpu().view(torch.int16).numpy().view(np.uint16)
    sr = s_ref.view(np.uint16)
    bad_s = np.argwhere(s != sr)
    assert bad_s.size == 0, f"scale mismatch at {bad_s[:5].tolist()}: {s[tuple(bad_s[0])]:#06x} vs {sr[tuple(bad_s[0])]:#06x}"
    bad_p = np.argwhere(p != p_ref)
    assert bad_p.size == 0, f"packed mismatch at {bad_p[:5].tolist()}: {p[tuple(bad_p[0])]:#04x} vs {p_ref[tuple(bad_p[0])]:#04x}"


def assert_matmul_close(y, x, packed, scales, K, group, c, rows=None, cols=None):
    """|y - y_ref| <= c * sum|x||w_hat| elementwise (optionally on a sampled grid)."""
    if rows is not None:
        ri = torch.as_tensor(rows, device=x.device)
        x = x.index_select(0, ri)
        y = y.index_select(0, ri)
    if cols is not None:
        ci = torch.as_tensor(cols, device=x.device)
        packed = packed.index_select(0, ci)
        scales = scales.index_select(0, ci)
        y = y.index_select(1, ci)
    xn = to_np(x).astype(np.float64)
    pn = packed.cpu().numpy()
    sn = scales.cpu().numpy()
    y_ref = oracle.int4_matmul_ref(xn, pn, sn, K, group)
    bound = oracle.matmul_error_bound(xn, pn, sn, K, group, c)
    yn = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(yn).all()
    err = np.abs(yn - y_ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert (err <= bound).all(), (
        f"matmul error {err[worst]:.3e} > bound {bound[worst]:.3e} at {worst} "
        f"(y={yn[worst]:.6e}, ref={y_ref[worst]:.6e})")
    return float((err / np.maximum(bound, 1e-300)).max())


def assert_matmul_lines(y, x, packed, scales, K, group, c, rows, cols, chunk=4096):
    """Whole lines of y against the oracle: every column of the sampled rows
    `rows` and every row of the sampled columns `cols`, the oracle computed
    over chunks of weight rows (so full-size matrices fit in host memory)."""
    xn_rows = to_np(x.index_select(0, torch.as_tensor(rows, device=x.device))).astype(np.float64)
    pn_all = packed.cpu().numpy()
    sn_all = scales.cpu().numpy()
    y_rows = y.index_select(0, torch.as_tensor(rows, device=y.device)).cpu().numpy()
    N = pn_all.shape[0]
    worst = 0.0
    for n0 in range(0, N, chunk):
        n1 = min(n0 + chunk, N)
        ref = oracle.int4_matmul_ref(xn_rows, pn_all[n0:n1], sn_all[n0:n1], K, group)
        bound = oracle.matmul_error_bound(xn_rows, pn_all[n0:n1], sn_all[n0:n1], K, group, c)
        err = np.abs(y_rows[:, n0:n1].astype(np.float64) - ref)
        assert (err <= bound).all(), f"rows: error above the bound in columns {n0}..{n1}"
        worst = max(worst, float((err / np.maximum(bound, 1e-300)).max()))
    xn = to_np(x).astype(np.float64)
    ci = torch.as_tensor(cols, device=y.device)
    y_cols = y.index_select(1, ci).cpu().numpy().astype(np.float64)
    ref = oracle.int4_matmul_ref(xn, pn_all[cols], sn_all[cols], K, group)
    bound = oracle.matmul_error_bound(xn, pn_all[cols], sn_all[cols], K, group, c)
    err = np.abs(y_cols - ref)
    assert (err <= bound).all(), "columns: error above the bound"
    return max(worst, float((err / np.maximum(bound, 1e-300)).max()))

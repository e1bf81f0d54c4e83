"""Writes tests/golden/tiny_case_expected.json from the CPU oracle alone.

Run from the repository root: ``python tests/golden/make_golden.py``.
It imports only ``oracle`` and the seeded input generator ``workloads``.
"""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from workloads import tiny_case  # noqa: E402


def main():
    case = tiny_case()
    packed, scales, K = oracle.quantize_int4(case["w"], case["group"])
    y = oracle.int4_matmul_ref(case["x"], packed, scales, K, case["group"])
    out = {
        "source": "oracle.quantize_int4 / oracle.int4_matmul_ref on workloads.tiny_case()",
        "K": K,
        "group": case["group"],
        "packed_hex": packed.tobytes().hex(),
        "scales_fp16_bits": scales.view(np.uint16).tolist(),
        "y": y.tolist(),
    }
    with open(os.path.join(HERE, "tiny_case_expected.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()

"""Writes the stored expected values under tests/golden/.

Calls only the CPU oracle (``oracle/``) on the seeded ``tiny`` workload
(W 256x512 ~ N(0, 0.02^2), E2M1, group 128, fp32 scales; x 1x512 ~ N(0, 1);
seed 0).  Run from the repository root:  python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from w4a16_gemm_fp4_b200 import synth  # noqa: E402


def main():
    case = synth.tiny()
    r = oracle.quantize(case["W"], 128, oracle.E2M1, False, None, "f32")
    Y = oracle.gemm(case["X"], r["packed"], r["scales"], oracle.E2M1, 128)
    out = {
        "workload": "tiny: W 256x512 N(0,0.02^2) seed 0, E2M1, group 128, fp32 scales, x 1x512",
        "packed_sha256": hashlib.sha256(r["packed"].tobytes()).hexdigest(),
        "scales_sha256": hashlib.sha256(r["scales"].tobytes()).hexdigest(),
        "y_first8": [float(v) for v in Y[0, :8]],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_digest.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()

"""Writes tests/golden/tiny_oracle.json from the oracle alone.

The pages print no worked numeric example, so the stored values here are a
regression fixture of the oracle itself on the tiny workload (B=1, H=2,
N=256, d=64, fp16, INT8/FP8 mode, seed 0): digests of the pre-pass codes
and scales and a fixed sample of output values.  Run from the repo root:

    python tests/golden/make_golden.py
"""

import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import attention as att  # noqa: E402
from oracle import prepass as pp  # noqa: E402
from quantized_attention_quant_b200.workloads import WORKLOADS, make_qkv, to_numpy32  # noqa: E402


def digest(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def compute():
    w = WORKLOADS["tiny"]
    q, k, v = [to_numpy32(t) for t in make_qkv(w)]
    qk = pp.quant_qk_int8(q, k)
    vc, vs = pp.quant_v_fp8(v)
    o = att.sage_attention_output(q, k, v, w.causal, w.sm_scale, "int8_fp8", w.dtype)
    idx = [(0, 0, 0, 0), (0, 0, 17, 5), (0, 1, 128, 63), (0, 1, 255, 31), (0, 0, 200, 40)]
    return {
        "workload": "tiny B=1 H=2 N=256 d=64 f16 int8_fp8 seed=0",
        "q_codes": digest(qk["q_codes"]), "q_scales": digest(qk["q_scales"]),
        "k_codes": digest(qk["k_codes"]), "k_scales": digest(qk["k_scales"]),
        "k_mean": digest(qk["k_mean"]), "v_codes": digest(vc), "v_scales": digest(vs),
        "o_samples": [[list(i), float(o[i])] for i in idx],
    }


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(out, "w") as f:
        json.dump(compute(), f, indent=1)
    print("wrote", out)

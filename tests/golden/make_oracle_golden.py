"""Write tests/golden/oracle_tiny.json: digests and a few values of the
oracle's outputs on the seeded tiny workload (quant emulation with smoothing,
with K-residual quantization and with a fixed tile mask; exact attention; the
codes; the tile scores and the tau = 0.5 selection).  It calls only the oracle and
the seeded input generator; test_golden.py recomputes and compares, so any
change to the oracle's arithmetic shows up (and must be justified when the
file is regenerated)."""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from quantized_attention_qk_b200.inputs import WORKLOADS, make_qkv  # noqa: E402


def digests():
    w = WORKLOADS["tiny"]
    q, k, v, _ = make_qkv(w)
    _, quant_bits = oracle.attn_quant(q, k, v, w.sm_scale)
    exact = oracle.attn_exact(q, k, v, w.sm_scale)
    codes = oracle.quantize(q, k, v)
    _, kres_bits = oracle.attn_quant(q, k, v, w.sm_scale, k_residual=True)
    keep = np.ones((w.B, w.H, 2, 2), dtype=np.uint8)   # N = 256: two 128-token tiles
    keep[:, :, 0, 1] = 0                               # query tile 0 skips key tile 1
    keep[:, 1, 1, 0] = 0                               # head 1, query tile 1 skips key tile 0
    _, masked_bits = oracle.attn_quant(q, k, v, w.sm_scale, kv_keep=keep)
    sbar = oracle.block_scores(q, k, v, w.sm_scale)
    sel = oracle.block_select(sbar, w.N, 0.5)
    return {
        "workload": "tiny: B=1 H=2 N=256 d=64, seed 1001",
        "quant_bf16_sha256": hashlib.sha256(np.ascontiguousarray(quant_bits).tobytes()).hexdigest(),
        "exact_f64_sha256": hashlib.sha256(np.ascontiguousarray(exact).tobytes()).hexdigest(),
        "codes_sha256": {kk: hashlib.sha256(np.ascontiguousarray(vv).tobytes()).hexdigest()
                         for kk, vv in sorted(codes.items())},
        "kres_bf16_sha256": hashlib.sha256(np.ascontiguousarray(kres_bits).tobytes()).hexdigest(),
        "masked_bf16_sha256": hashlib.sha256(np.ascontiguousarray(masked_bits).tobytes()).hexdigest(),
        "block_scores": [float(x) for x in np.asarray(sbar, dtype=np.float64).ravel()],
        "block_select_tau_0.5": [int(x) for x in np.asarray(sel).ravel()],
        "quant_bf16_samples": {f"{h},{r},{c}": int(quant_bits[0, h, r, c])
                               for (h, r, c) in [(0, 0, 0), (0, 127, 63), (1, 128, 5), (1, 255, 31)]},
        "exact_samples": {f"{h},{r},{c}": float(exact[0, h, r, c])
                          for (h, r, c) in [(0, 0, 0), (0, 127, 63), (1, 128, 5), (1, 255, 31)]},
    }


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")
    with open(out, "w") as f:
        json.dump(digests(), f, indent=1, ensure_ascii=False)
        f.write("\n")
    print("wrote", out)

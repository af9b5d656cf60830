"""Fit the scale of the Zipf router bias of the skewed workload and freeze it.

Workload: T=8192, d=2880, E=32, K=4, bf16, router bias alpha * (e+1)^(-1.2)
added to the logits; "top experts get about 5x the mean load". This script
finds alpha by bisection so that max_e counts_e / (T*K/E) = 5.0 +- 0.1 with
no capacity limit, on the oracle's own router logits (seed 0), and writes
``tests/golden/zipf_bias_alpha.json``. It calls only the oracle for the
routing arithmetic (``moe_inputs`` supplies x, W_r and the bias shape).

Run:  python oracle/fit_zipf_bias.py
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, _ROOT)

import moe_inputs as mi  # noqa: E402
from oracle import moe_oracle as orc  # noqa: E402

TARGET, TOL = 5.0, 0.1


def load_ratio(x, w_r, cfg, alpha: float) -> float:
    bias = mi.zipf_bias(cfg.E, cfg.zipf_s, alpha).numpy()
    lg = orc.router_logits(x, w_r, bias)
    ids = orc.topk_ids(lg, cfg.K)
    counts, _, _, _ = orc.permute(ids, cfg.E, None)
    return float(counts.max()) / (cfg.T * cfg.K / cfg.E)


def main() -> None:
    cfg = mi.SKEWED_CAPACITY_BF16
    cfg0 = mi.MoEConfig(**{**cfg.__dict__, "zipf_s": 0.0})
    inp = mi.make_inputs(cfg0, with_experts=False)
    x, w_r = orc.as_f64(inp.x), orc.as_f64(inp.w_r)
    lo, hi = 0.0, 16.0
    r_hi = load_ratio(x, w_r, cfg, hi)
    assert r_hi > TARGET, r_hi
    alpha, r = hi, r_hi
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        r = load_ratio(x, w_r, cfg, mid)
        alpha = mid
        if abs(r - TARGET) <= TOL:
            break
        if r < TARGET:
            lo = mid
        else:
            hi = mid
    assert abs(r - TARGET) <= TOL, (alpha, r)
    out = {
        "alpha": round(alpha, 6),
        "max_over_mean_load": round(load_ratio(x, w_r, cfg, round(alpha, 6)), 4),
        "workload": "T=8192 d=2880 E=32 K=4 bf16, seed 0, Zipf s=1.2, no capacity",
        "how": "bisection on alpha for max_e counts_e / (T*K/E) = 5.0 +- 0.1, oracle logits",
        "written_by": "oracle/fit_zipf_bias.py",
    }
    with open(mi.ZIPF_ALPHA_FILE, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print(json.dumps(out))


if __name__ == "__main__":
    main()

"""Calibrate the coarse scale of each synthetic workload with the fp64 oracle.

Writes ``coarse_scale.json`` beside this file.  Only the oracle and the seeded input
generator are called: no value here comes from the CUDA path.

Sparsity is the fraction of (row, past block) pairs whose entmax weight is zero, over
all rows (b, h, t) -- own (diagonal) blocks excluded.  The scale is found by bisection
on log(scale) until the sparsity of a sample of rows is within 0.5 % of the target,
then the realised sparsity is measured on a larger sample (every row where that is
cheap) and recorded with the seed and a SHA-256 of the bf16 inputs.

Usage: python tests/golden/calibrate.py [name ...]
"""
from __future__ import annotations

import json
import math
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from sparse_hierarchical_attention_pool_b200 import inputs  # noqa: E402

OUT = os.path.join(HERE, "coarse_scale.json")


def sparsity(q_rows, k, rows, Hq, blk, alpha, cs):
    r = oracle.select_rows(q_rows, k, rows, Hq, blk, alpha, cs)
    return 1.0 - r["nsel"].sum() / max(1, r["bt"].sum()), r


def rows_for(wl, n, seed_off):
    if wl.kind == "decode":
        return [(b, h, wl.T - 1) for b in range(wl.B) for h in range(wl.Hq)]
    return inputs.sample_rows(wl.B, wl.Hq, wl.T, n, seed=wl.seed + seed_off, t_lo=wl.block)


def calibrate(name):
    wl, tens = inputs.make(name)
    q, k = tens[0], tens[1]
    if wl.kind == "decode":
        q = q.reshape(wl.B, wl.Hq, 1, wl.d)
    rows = rows_for(wl, 8192, 100)
    if wl.kind == "decode":
        qr = q[:, :, 0].reshape(-1, wl.d)
    else:
        qr = oracle.gather_q_rows(q, rows)
    rec = {"workload": wl.name, "seed": wl.seed, "alpha": wl.alpha, "n_topics": wl.n_topics,
           "shape": {"B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "T": wl.T, "d": wl.d, "block": wl.block},
           "sha256_bf16_inputs": inputs.sha256(*tens[:3])}
    if wl.target_sparsity is None:
        cs = 1.0
    else:
        lo, hi = math.log(1e-4), math.log(10.0)
        cs = None
        for _ in range(60):
            mid = 0.5 * (lo + hi)
            rho, _ = sparsity(qr, k, rows, wl.Hq, wl.block, wl.alpha, math.exp(mid))
            if abs(rho - wl.target_sparsity) <= 0.005:
                cs = math.exp(mid)
                break
            if rho < wl.target_sparsity:
                lo = mid
            else:
                hi = mid
        if cs is None:
            raise RuntimeError(f"{name}: calibration did not reach the target")
        cs = float(f"{cs:.6g}")
    rec["coarse_scale"] = cs
    rec["calibration_rows"] = len(rows)
    # realised sparsity on a larger sample (all rows when the workload is small)
    if wl.kind == "decode":
        mrows, mq = rows, qr
    elif wl.B * wl.Hq * wl.T <= 300_000:
        mrows = [(b, h, t) for b in range(wl.B) for h in range(wl.Hq) for t in range(wl.T)]
        mq = q.reshape(-1, wl.d)
    else:
        mrows = rows_for(wl, 65536, 200)
        mq = oracle.gather_q_rows(q, mrows)
    alphas = [1.25, 1.5, 2.0] if name == "32k" else [wl.alpha]
    rec["realised_sparsity"] = {}
    for a in alphas:
        rho, r = sparsity(mq, k, mrows, wl.Hq, wl.block, a, cs)
        nsel = r["nsel"]
        rec["realised_sparsity"][str(a)] = {
            "sparsity": round(float(rho), 6),
            "selected_per_row_p10_p50_p90": [float(x) for x in np.percentile(nsel, [10, 50, 90])],
        }
    rec["measured_rows"] = len(mrows)
    return rec


def main(names):
    data = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            data = json.load(f)
    for name in names:
        t0 = time.time()
        data[name] = calibrate(name)
        print(name, json.dumps(data[name]["realised_sparsity"]), data[name]["coarse_scale"],
              f"{time.time() - t0:.1f}s", flush=True)
        with open(OUT, "w") as f:
            json.dump(data, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:] or list(inputs.WORKLOADS))

"""Fits the analytic tactic scorer's constants to measured candidate times.

    python -m precision_quantized_gemm_b200.fit_scorer [--data tables/b200_candidates.txt]

The data is the tuner's log of every timed candidate (``tune_tables.py
--log``): one line per (format, M, N, K, split_k, swap_ab, tile_n, stages,
reduce_mode, [variant, rows,] µs); the tile kernel's model is fitted to its
own lines (variant 0; logs from before the decode kernel have no variant
column).  The model is the one csrc/scorer.cu evaluates (see the
comment at its top): Little's-law streaming per CTA under per-SM and HBM
caps, MMA-loop cycles per K tile (Block_FP8: plus promotion cycles per
column a thread promotes), waves over the SMs, and the split-K
reduction cost of each mode.  Fitting minimises log-time residuals with a
free offset per shape (ranking within a shape ignores per-shape constants
such as the quantiser's time), with the HBM bandwidth held at the measured
copy bandwidth.  Prints the constants for scorer.cu and the ranking quality:
the measured time of the top-ranked configuration over the shape's best,
and of the best among the top N.  Needs numpy and scipy; no GPU.
"""
from __future__ import annotations

import argparse
import collections
import json
import math
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SMS = 148
SMEM_PER_SM = 233472
HBM_GBS = 6450.9


def tmem_columns(f, tn):
    used = (2 if tn >= 256 else 4) * tn if f == 2 else (tn + 16 + 16 * (2 if tn > 128 else 1) if f == 3 else tn)
    cols = 32
    while cols < used:
        cols *= 2
    return cols


def smem_estimate(f, M, sk, sw, tn, st, rm, nkt):
    """Dynamic shared memory of a launch (the carve-up of gemm_kernel.cuh, rounded)."""
    ring = st * (16384 + tn * 128)
    if f == 3:
        ring += st * (2048 + 2048 * (2 if tn > 128 else 1))
    push = sk > 1 and rm == 0 and tn <= 64
    recv = 512 * (min(tn, M) if sw else tn) if push else 0
    scales = 4 * ((tn if sw else 128) + (2 if (not sw and tn > 128) else 1)) * nkt if f == 2 else 0
    epis = 4 * (128 + tn) if f in (0, 1) else 0
    fuse = 4 * 9 * tn if (sw and f != 3) else 0
    return ring + recv + scales + epis + fuse + 8 * (2 * st + 12) + 2048


def features(rows):
    out = collections.defaultdict(list)
    for r in rows:
        f, M, N, K, sk, sw, tn, st, rm = (int(x) for x in r[:9])
        rb = K // 2 if f == 3 else K
        kt = (rb + 127) // 128
        nkt = (kt + sk - 1) // sk
        rows_p, rows_q = (N, M) if sw else (M, N)
        ctas = ((rows_p + 127) // 128) * ((rows_q + tn - 1) // tn) * sk
        blk = f == 2
        regcap = 3 if (not blk and tn <= 64) else (2 if (not blk or tn <= 64) else 1)
        cps = max(1, min(regcap, 512 // tmem_columns(f, tn),
                         SMEM_PER_SM // (smem_estimate(f, M, sk, sw, tn, st, rm, nkt) + 1024)))
        mt = min(M, tn) if sw else min(M, 128)
        # Block_FP8 promotion runs on 4, 8 or 16 epilogue warps (tile_n < 128,
        # 128, 256): columns each thread promotes per K tile
        pcols = tn // (4 if tn >= 256 else 2 if tn >= 128 else 1) if blk else 0
        vals = dict(M=M, N=N, sk=sk, tn=tn, st=st, rm=rm, nkt=nkt, blk=float(blk), cps=cps, pcols=pcols,
                    waves=math.ceil(ctas / (SMS * cps)), rb=rb, mt=mt, pushed=mt if sw else tn)
        for k, v in vals.items():
            out[k].append(v)
    return {k: np.array(v, float) for k, v in out.items()}


NAMES = ["lat_us", "sm_gbs", "a0", "a1", "a2", "a3", "e0", "e1", "e2", "e3", "e4", "e5"]


def model(p, V):
    lat, smbw, a0, a1, a2, a3, e0, e1, e2, e3, e4, e5 = p
    stage = (128 + V["tn"]) * 128
    rate = np.minimum(np.minimum(V["st"], V["nkt"]) * stage / lat, smbw * 1e3 / V["cps"])
    t_str = stage * V["nkt"] / rate
    t_mma = V["nkt"] * (a0 + a1 * V["tn"] + V["blk"] * (a2 * V["pcols"] + a3)) / 1900.0
    hbm = V["N"] * V["rb"] + np.where(V["M"] >= 1024, V["M"] * V["rb"], 0.0)
    body = np.maximum(hbm / (HBM_GBS * 1e3), V["waves"] * np.maximum(t_str, t_mma))
    split = V["sk"] > 1
    cl = split & (V["rm"] == 0)
    ws = split & (V["rm"] > 0)
    epi = (e0 * V["pushed"] / 16.0
           + cl * V["waves"] * (e1 + V["sk"] * 128 * V["pushed"] * 4 / (e2 * 1e3))
           + ws * (np.where(V["rm"] == 1, e3, e4) + 2 * V["sk"] * V["M"] * V["N"] * 4 / (e5 * 1e3)))
    return body + epi


def main(argv=None):
    from scipy.optimize import least_squares
    ap = argparse.ArgumentParser()
    ap.add_argument("--data", default=os.path.join(HERE, "tables", "b200_candidates.txt"))
    a = ap.parse_args(argv)
    rows = []
    for line in open(a.data):
        v = [float(x) for x in line.split()]
        if len(v) == 12 and v[9] != 0:         # the decode kernel: not this model
            continue
        if len(v) in (10, 12):
            rows.append(v[:9] + [v[-1]])
    rows = np.array(rows)
    t = rows[:, 9]
    V = features(rows)
    shapes = collections.defaultdict(list)
    for i, r in enumerate(rows):
        shapes[tuple(int(x) for x in r[:4])].append(i)
    keys = list(shapes)
    sid = np.empty(len(rows), int)
    for j, k in enumerate(keys):
        sid[shapes[k]] = j
    p0 = [1.5, 100.0, 300.0, 1.0, 3.0, 100.0, 0.3, 0.5, 50.0, 2.0, 3.0, 3000.0]
    lo = [0.05, 5, 0, 0, 0, 0, 0, 0, 1, 0, 0, 100]
    hi = [20, 5000, 5000, 50, 50, 5000, 10, 10, 50000, 30, 30, 50000]
    off0 = [max(0.5, 0.4 * t[shapes[k]].min()) for k in keys]

    def resid(q):
        return np.log(q[len(p0):][sid] + model(q[:len(p0)], V)) - np.log(t)

    fit = least_squares(resid, np.array(p0 + off0), bounds=(lo + [0] * len(keys), hi + [5000] * len(keys)),
                        loss="soft_l1", f_scale=0.1, max_nfev=400)
    p = fit.x[:len(p0)]
    print(json.dumps({n: float(v) for n, v in zip(NAMES, p)}, indent=1))
    pred = model(p, V)
    for n in (1, 2, 4, 8, 16):
        reg = np.array([t[np.array(ix)[np.argsort(pred[ix])[:n]]].min() / t[ix].min() for ix in shapes.values()])
        print(f"top-{n}: measured time over the best, geomean {np.exp(np.mean(np.log(reg))):.4f}, "
              f"p90 {np.percentile(reg, 90):.3f}, max {reg.max():.3f}")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())

"""Regenerates the ahead-of-time per-shape configuration table.

    python -m precision_quantized_gemm_b200.tune_tables [--out PATH] [--suites a,b]
                                                        [--budget SECONDS] [--resume]

Runs qgemm_tune (the library's tuner: enumerate split_k / swap_ab / tile_n /
stages / reduce_mode, reject candidates whose output disagrees with the
default configuration, select on one graph-timed pass, record an
independent second pass) over the decode and prefill shapes of the
quantized linear layers this library serves, and writes the table that
qgemm_dispatch reads.  ``--top-n N`` times only the analytic scorer's N
best-ranked configurations per shape (qgemm_tune_ranked) plus the best four
of each kernel variant; ``--log`` keeps every candidate's time (the data
fit_scorer.py fits the scorer to); ``--objective`` chooses what a timed
step is (the GEMM alone, the default, or quantisation + GEMM).
Needs a B200.
"""
from __future__ import annotations

import argparse
import os
import sys

import precision_quantized_gemm_b200 as qg

HERE = os.path.dirname(os.path.abspath(__file__))
DEFAULT_OUT = os.path.join(HERE, "tables", "b200.qgt")

# (format, token counts, (N, K) pairs): LLM projection shapes.
SWEEP_NK = [(896, 5120), (1024, 7168), (1280, 8192), (1792, 5120), (2560, 8192), (4096, 4096),
            (4608, 7168), (5120, 640), (5120, 2048), (6144, 4096), (7168, 2048), (8192, 8192)]
MEDIUM_M = [64, 128, 256, 512, 1024, 2048]
MEDIUM_NK = [(1792, 5120), (4096, 4096), (5120, 2048), (8192, 8192)]
SHAPES = {
    "fp8_tiny": [(qg.QG_FP8_DYNAMIC, [16], [(2048, 2048)])],
    "int8": [(qg.QG_W8A8_INT8, [1, 8, 32], [(4096, 4096)])],
    "block_fp8": [(qg.QG_BLOCK_FP8, [1, 4, 16, 32], [(512, 7168), (4608, 7168), (5120, 640), (2560, 8192)])],
    "nvfp4": [(qg.QG_NVFP4, [1, 8, 64, 512], [(896, 1024), (1792, 5120), (5120, 2048), (1280, 8192)])],
    "sweep": [(qg.QG_FP8_DYNAMIC, [1, 2, 4, 8, 16, 32], SWEEP_NK),
              (qg.QG_BLOCK_FP8, [1, 2, 4, 8, 16, 32], SWEEP_NK)],
    "large_m": [(qg.QG_BLOCK_FP8, [4096, 16384], [(5120, 5120)])],
    # medium token counts (prefill chunks, batched decode): the buckets between
    # decode and large M, and the 4096-token bucket above them (where the
    # persistent and CTA-pair kernels compete with the tile kernel)
    "medium_m": [(qg.QG_FP8_DYNAMIC, MEDIUM_M + [4096], MEDIUM_NK), (qg.QG_BLOCK_FP8, MEDIUM_M + [4096], MEDIUM_NK),
                 (qg.QG_W8A8_INT8, [256, 512, 1024, 2048, 4096], MEDIUM_NK)],
}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=DEFAULT_OUT)
    ap.add_argument("--suites", default="fp8_tiny,int8,block_fp8,nvfp4,large_m,sweep,medium_m")
    ap.add_argument("--budget", type=float, default=20.0, help="seconds per shape")
    ap.add_argument("--resume", action="store_true", help="start from the existing table, skip tuned shapes")
    ap.add_argument("--log", default=None, help="append every timed candidate to this file")
    ap.add_argument("--top-n", type=int, default=0,
                    help="time only the analytic scorer's top-N configurations per shape (0: the whole grid)")
    ap.add_argument("--objective", choices=["gemm", "step"], default="gemm",
                    help="time each candidate as back-to-back GEMMs (the per-shape metric) or as "
                         "activation-quantisation + GEMM steps")
    a = ap.parse_args(argv)
    if a.log:
        qg.qgemm_set_tune_log(a.log)
    qg.qgemm_set_tune_objective(a.objective == "gemm")
    table = qg.Table(a.out) if (a.resume and os.path.exists(a.out)) else qg.Table()
    for name in [s.strip() for s in a.suites.split(",") if s.strip()]:
        for fmt, Ms, NK in SHAPES[name]:
            table.tune(fmt, Ms, NK, budget_s_per_shape=a.budget, verbose=True, top_n=a.top_n)
            table.save(a.out)            # checkpoint after every family
    print(f"wrote {len(table)} entries to {a.out}", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())

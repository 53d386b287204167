"""The scaled quantized contraction y = dequant(A_q) . dequant(W_q)^T (oracle).

Test infrastructure only.  A_q is [M, K] (tokens x reduction), W_q is
[N, K] (output channels x reduction, the "NT" layout of a linear layer), and
y is [M, N] in bf16.  The contraction of codes is exact:

* int8 codes are summed in int64;
* e4m3 products are exact in fp64 and every partial sum of at most 2^13 of
  them is a multiple of 2^-18 below 2^31, so fp64 accumulation in any order
  is exact (the library matmul serves as that sum);
* NVFP4 decodes each element with its block scale (a product of at most
  6 significant bits, exact in fp64) and accumulates in fp64.

Scales are applied in fp64 and the result is rounded once to bf16 (nearest
even).  The variants of "Helion in the vLLM backend" (second paragraph):
Split-K sums K-slices of the same exact contraction, Swap-AB computes
(W_q . A_q^T)^T; both reach the same exact sums, which the tests check.
"""
from __future__ import annotations

import numpy as np

from .formats import bf16_round, decode_e2m1, decode_e4m3


# ----------------------------------------------------------------- cores --
def acc_int8(qa: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """Exact int64 sums  acc[m, n] = sum_k qa[m, k] * qw[n, k]."""
    return qa.astype(np.int64) @ qw.astype(np.int64).T


def acc_e4m3(qa: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """Exact fp64 sums of e4m3 products."""
    return decode_e4m3(qa) @ decode_e4m3(qw).T


def acc_e4m3_groups(qa: np.ndarray, qw: np.ndarray, group: int = 128) -> np.ndarray:
    """Exact per-group sums  p[g, m, n] = sum_{k in group g} a_q * w_q."""
    a = decode_e4m3(qa)
    w = decode_e4m3(qw)
    G = a.shape[1] // group
    return np.stack([a[:, g * group:(g + 1) * group] @ w[:, g * group:(g + 1) * group].T
                     for g in range(G)])


def nvfp4_dequant(q: np.ndarray, sf: np.ndarray, sf_vec: int = 16) -> np.ndarray:
    """Element values dec(q) * dec(block scale), without the tensor scale."""
    R, K = q.shape
    return decode_e2m1(q) * np.repeat(decode_e4m3(sf), sf_vec, axis=1)[:, :K]


# ------------------------------------------------------------ full GEMMs --
def fp8_dynamic(qa, sa, qw, sw):
    """FP8_Dynamic: y = (sum a_q w_q) * s_a[m] * s_w[n] -> bf16 (fp64 values)."""
    acc = acc_e4m3(qa, qw)
    return bf16_round(acc * sa.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :])


def w8a8_int8(qa, sa, qw, sw):
    """W8A8_INT8: exact int64 accumulators, fp64 scale epilogue -> bf16."""
    acc = acc_int8(qa, qw)
    return bf16_round(acc.astype(np.float64) * sa.astype(np.float64)[:, None]
                      * sw.astype(np.float64)[None, :])


def block_fp8(qa, sa_groups, qw, sw_blocks, group: int = 128):
    """Block_FP8: y = sum_g p_g * s_a[m, g] * s_w[n // 128, g] -> bf16."""
    p = acc_e4m3_groups(qa, qw, group)                         # [G, M, N]
    N = qw.shape[0]
    sw_n = sw_blocks.astype(np.float64)[np.arange(N) // group, :]   # [N, G]
    sa = sa_groups.astype(np.float64)                          # [M, G]
    y = np.einsum("gmn,mg,ng->mn", p, sa, sw_n)
    return bf16_round(y)


def nvfp4(qa, sfa, ga, qw, sfw, gw):
    """NVFP4: y = (sum_k dec(a) dec(sfa) dec(w) dec(sfw)) * g_a * g_w -> bf16."""
    acc = nvfp4_dequant(qa, sfa) @ nvfp4_dequant(qw, sfw).T
    return bf16_round(acc * float(ga) * float(gw))


# -------------------------------------------------------------- variants --
def split_k_partials(qa, qw, splits: int, acc_fn=acc_e4m3):
    """Split-K: the exact contraction over each of ``splits`` equal K slices."""
    K = qa.shape[1]
    assert K % splits == 0
    ks = K // splits
    return [acc_fn(qa[:, s * ks:(s + 1) * ks], qw[:, s * ks:(s + 1) * ks])
            for s in range(splits)]


def swap_ab(qa, qw, acc_fn=acc_e4m3):
    """Swap-AB: (W_q . A_q^T)^T, the weight filling the row role."""
    return acc_fn(qw, qa).T


def grouped(gemm_fn, qa, sa, qw, sw, offsets, n_per_expert: int, w_rows_per_scale: int = 1):
    """Mixture-of-experts grouped GEMM ("Helion in the vLLM backend", last
    paragraph: the MoE backend is the next target): the tokens are sorted by
    expert, expert e owns token rows [offsets[e], offsets[e + 1]) of A and y
    and weight rows [e N, (e + 1) N) of the stacked W; its rows of y are the
    plain GEMM ``gemm_fn`` (one of the four above, taking (qa, sa, qw, sw))
    of those slices.  ``w_rows_per_scale`` is 1 for per-channel weight scales
    and 128 for 128x128 block scales (N is then a multiple of 128).  Returns
    y [T, N] in fp64 values of bf16."""
    T = qa.shape[0]
    N = n_per_expert
    y = np.zeros((T, N), np.float64)
    for e in range(len(offsets) - 1):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 <= r0:
            continue
        w0, w1 = e * N, (e + 1) * N
        s0, s1 = w0 // w_rows_per_scale, w1 // w_rows_per_scale
        y[r0:r1] = gemm_fn(qa[r0:r1], sa[r0:r1], qw[w0:w1], sw[s0:s1])
    return y


def grouped_nvfp4(qa, sfa, ga, qw, sfw, gw, offsets, n_per_expert: int):
    """The grouped GEMM above for NVFP4 operands.  Each expert's weight is a
    tensor of its own (a mixture-of-experts layer holds one linear layer per
    expert), so expert e contributes its own tensor scale gw[e]; the
    activations of all tokens are one tensor with one scale ga.  Expert e's
    rows of y are nvfp4(qa[r0:r1], sfa[r0:r1], ga, qw[eN:(e+1)N],
    sfw[eN:(e+1)N], gw[e]).  Returns y [T, N] in fp64 values of bf16."""
    T = qa.shape[0]
    N = n_per_expert
    y = np.zeros((T, N), np.float64)
    for e in range(len(offsets) - 1):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 <= r0:
            continue
        w0, w1 = e * N, (e + 1) * N
        y[r0:r1] = nvfp4(qa[r0:r1], sfa[r0:r1], ga, qw[w0:w1], sfw[w0:w1], gw[e])
    return y


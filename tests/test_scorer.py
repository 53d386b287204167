"""The analytic tactic scorer (qgemm_score_config / qgemm_rank_configs), on the
CPU: its ranking is valid, deterministic and what qgemm_default_config
returns, and, evaluated on the tuner's measured time of every candidate on a
B200 (tables/b200_candidates.txt), its top-ranked configuration is close to
each shape's measured best and its top 16 contain it (FlashInfer PR 3948:
rank tactics with a heuristic, tune only the top N)."""
import collections
import math
import os

import pytest

import precision_quantized_gemm_b200 as qg

DATA = os.path.join(os.path.dirname(qg.__file__), "tables", "b200_candidates.txt")
FAKE = 0x100000


def _measured():
    shapes = collections.defaultdict(list)
    for line in open(DATA):
        v = line.split()
        if len(v) == 10:
            f, M, N, K, sk, sw, tn, st, rm = (int(x) for x in v[:9])
            shapes[(f, M, N, K)].append((qg.make_config(sk, sw, tn, st, rm), float(v[9])))
    return shapes


@pytest.mark.parametrize("fmt,M,N,K", [(1, 8, 4096, 4096), (0, 1, 896, 5120), (2, 4096, 5120, 5120),
                                       (3, 512, 5120, 2048), (2, 32, 512, 7168), (0, 16, 2048, 2048)])
def test_ranking_is_valid_sorted_and_the_default(fmt, M, N, K):
    ranked = qg.qgemm_rank_configs(fmt, M, N, K, max_out=64)
    assert len(ranked) > 4
    est = [e for _, e in ranked]
    assert est == sorted(est) and all(e > 0 for e in est)
    torch = pytest.importorskip("torch")
    for c, e in ranked:
        assert qg.qgemm_score_config(fmt, M, N, K, c) == pytest.approx(e)
        if torch.cuda.is_available():
            continue                            # fake pointers: host checks only without a device
        # every ranked configuration passes qgemm_run's host checks and stops
        # at the device check
        ws = FAKE if qg.qgemm_workspace_size(fmt, M, N, K, c) else None
        st = qg.qgemm_run(fmt, qg.qg_operand(FAKE, FAKE, FAKE, M, K), qg.qg_operand(FAKE, FAKE, FAKE, N, K),
                          M, N, K, c, ws, 1 << 40, FAKE, N, 0, None)
        assert st == qg.QG_ERR_NO_DEVICE, (c, st)
    assert qg.qgemm_default_config(fmt, M, N, K).as_dict() == ranked[0][0].as_dict()
    again = qg.qgemm_rank_configs(fmt, M, N, K, max_out=64)
    assert [c.as_dict() for c, _ in again] == [c.as_dict() for c, _ in ranked]


def _variants(fmt, M, N, K):
    ranked = qg.qgemm_rank_configs(fmt, M, N, K, max_out=4096)
    return collections.Counter(c.variant for c, _ in ranked), ranked


def test_large_m_candidates_per_kernel():
    # persistent rings deep enough for one CTA per SM: 256 x 4 and 128 x 6
    # for FP8_Dynamic / W8A8_INT8, 256 x 3 for Block_FP8; CTA pairs (256 x 256
    # tiles, rings of 3, 4, 6) for Block_FP8 only, and only with at least 60
    # pair tiles
    for fmt in (qg.QG_FP8_DYNAMIC, qg.QG_W8A8_INT8):
        v, ranked = _variants(fmt, 4096, 5120, 5120)
        assert v[3] == 0
        assert sorted((c.tile_n, c.stages) for c, _ in ranked if c.variant == 2) == [(128, 6), (256, 4)]
    v, ranked = _variants(qg.QG_BLOCK_FP8, 4096, 5120, 5120)
    assert sorted((c.tile_n, c.stages) for c, _ in ranked if c.variant == 2) == [(256, 3)]
    assert sorted((c.tile_n, c.stages) for c, _ in ranked if c.variant == 3) == [(256, 3), (256, 4), (256, 6)]
    assert qg.qgemm_default_config(qg.QG_BLOCK_FP8, 4096, 5120, 5120).variant == 3
    # 4 x 16 = 64 pair tiles: offered; 2 x 16 = 32: not
    assert _variants(qg.QG_BLOCK_FP8, 1024, 4096, 4096)[0][3] == 3
    assert _variants(qg.QG_BLOCK_FP8, 512, 4096, 4096)[0][3] == 0
    assert _variants(qg.QG_NVFP4, 4096, 5120, 5120)[0][2] == 0
    assert _variants(qg.QG_NVFP4, 4096, 5120, 5120)[0][3] == 0


def test_scoring_an_invalid_config_returns_its_status():
    with pytest.raises(qg.QGemmError) as e:
        qg.qgemm_score_config(1, 8, 4096, 4096, qg.make_config(split_k=3))
    assert e.value.status == qg.QG_ERR_UNSUPPORTED


def test_scorer_ranking_against_measured_candidates():
    # the C++ model itself, scored on every measured candidate of every shape
    top1, top16, rule = [], [], []
    for (f, M, N, K), cands in _measured().items():
        best = min(t for _, t in cands)
        scored = sorted(((qg.qgemm_score_config(f, M, N, K, c), t) for c, t in cands), key=lambda x: x[0])
        top1.append(scored[0][1] / best)
        top16.append(min(t for _, t in scored[:16]) / best)
    geo = lambda xs: math.exp(sum(math.log(x) for x in xs) / len(xs))
    assert len(top1) >= 200
    assert geo(top1) <= 1.10, geo(top1)          # fitted: 1.071 (the fixed rule it replaced: 1.32)
    assert geo(top16) <= 1.01, geo(top16)        # fitted: 1.003
    # the worst shape's best configuration lies outside the top 16 (fitted:
    # 1.22x, a medium-M bucket)
    assert max(top16) <= 1.30

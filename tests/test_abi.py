"""C-ABI boundary tests that need no GPU: the library loads, exports every
symbol the header declares, sizes its buffers, rejects bad arguments on the
host before any launch, and round-trips its per-shape table."""
import ctypes
import os
import re

import numpy as np
import pytest

import precision_quantized_gemm_b200 as qg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qgemm.h")

FAKE = 0x100000  # an aligned, never-dereferenced stand-in for a device pointer


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"\b(qgemm_[a-z_0-9]+)\s*\(", txt)))


def test_every_declared_symbol_is_exported():
    L = qg.lib()
    names = _declared()
    assert len(names) >= 18
    for n in names:
        assert hasattr(L, n), n
    assert sorted(qg.EXPORTS) == names


def test_abi_version_and_status_strings():
    assert qg.lib().qgemm_abi_version() == 1
    for s in range(9):
        assert qg.status_string(s)
    assert qg.status_string(0) == "ok"


@pytest.mark.parametrize("fmt,is_w,rows,K,q,s", [
    (qg.QG_FP8_DYNAMIC, 0, 16, 2048, 16 * 2048, 16 * 4),
    (qg.QG_W8A8_INT8, 1, 4096, 4096, 4096 * 4096, 4096 * 4),
    (qg.QG_BLOCK_FP8, 0, 4, 7168, 4 * 7168, 4 * 56 * 4),
    (qg.QG_BLOCK_FP8, 1, 4608, 7168, 4608 * 7168, 36 * 56 * 4),
    (qg.QG_BLOCK_FP8, 1, 200, 256, 200 * 256, 2 * 2 * 4),
    (qg.QG_NVFP4, 0, 8, 1024, 8 * 512, 128 * 64),
    (qg.QG_NVFP4, 1, 1280, 8192, 1280 * 4096, 1280 * 512),
    (qg.QG_NVFP4, 1, 130, 96, 130 * 48, 256 * 16),
])
def test_operand_bytes(fmt, is_w, rows, K, q, s):
    assert qg.qgemm_operand_bytes(fmt, is_w, rows, K) == (q, s)


@pytest.mark.parametrize("fmt,K", [(qg.QG_FP8_DYNAMIC, 24), (qg.QG_BLOCK_FP8, 192),
                                   (qg.QG_NVFP4, 48), (7, 128)])
def test_operand_bytes_rejects_bad_k_or_format(fmt, K):
    with pytest.raises(qg.QGemmError):
        qg.qgemm_operand_bytes(fmt, 0, 4, K)


def test_workspace_sizes():
    c = qg.make_config(split_k=1)
    assert qg.qgemm_workspace_size(qg.QG_FP8_DYNAMIC, 16, 2048, 2048, c) == 0
    c = qg.make_config(split_k=8, swap_ab=1, tile_n=16, reduce_mode=0)
    assert qg.qgemm_workspace_size(qg.QG_FP8_DYNAMIC, 16, 2048, 2048, c) == 0   # cluster: none
    c = qg.make_config(split_k=8, swap_ab=1, tile_n=16, reduce_mode=1)
    assert qg.qgemm_workspace_size(qg.QG_FP8_DYNAMIC, 16, 2048, 2048, c) == 8 * 16 * 2048 * 4
    c = qg.make_config(split_k=8, swap_ab=1, tile_n=16, reduce_mode=2)
    ws = qg.qgemm_workspace_size(qg.QG_FP8_DYNAMIC, 16, 2048, 2048, c)
    assert ws == 8 * 16 * 2048 * 4 + 256          # partials + 16 tile counters padded to 256
    assert qg.qgemm_quant_workspace_size(qg.QG_NVFP4, 8, 1024) > 0
    assert qg.qgemm_quant_workspace_size(qg.QG_W8A8_INT8, 8, 1024) == 0


def test_default_config_follows_the_swap_rule_and_fills_sms():
    # the scored default (qgemm_rank_configs' first): decode shapes swap A and
    # B and split K over a cluster until tiles x split covers most SMs; large
    # M keeps the standard orientation with wide tiles and no split
    for fmt, M in ((qg.QG_W8A8_INT8, 8), (qg.QG_FP8_DYNAMIC, 1), (qg.QG_BLOCK_FP8, 16)):
        c = qg.qgemm_default_config(fmt, M, 4096, 4096)
        assert c.swap_ab == 1 and c.tile_n <= 32
        if c.variant == 1:                             # the decode kernel: rows per CTA fill the SMs
            assert c.split_k == 1 and 74 <= 4096 // c.rows * ((M + c.tile_n - 1) // c.tile_n) <= 4 * 148
            continue
        assert c.split_k >= 2 and (c.split_k & (c.split_k - 1)) == 0
        assert 74 <= 32 * c.split_k * ((M + c.tile_n - 1) // c.tile_n) <= 2 * 148
        assert c.reduce_mode == 0                      # cluster reduction: no workspace
    c = qg.qgemm_default_config(qg.QG_BLOCK_FP8, 4096, 5120, 5120)
    assert c.swap_ab == 0 and c.tile_n == 256 and c.split_k == 1


def _op(rows, K, q=FAKE, s=FAKE, g=FAKE):
    return qg.qg_operand(q, s, g, rows, K)


def _run(fmt=qg.QG_FP8_DYNAMIC, M=16, N=256, K=512, cfg=None, A=None, W=None, ws=None, wsb=0,
         Y=FAKE, ldy=None, out_kind=0):
    cfg = cfg or qg.make_config(split_k=1, swap_ab=1, tile_n=16, stages=4)
    A = A or _op(M, K)
    W = W or _op(N, K)
    return qg.qgemm_run(fmt, A, W, M, N, K, cfg, ws, wsb, Y, ldy if ldy is not None else N, out_kind, None)


@pytest.mark.parametrize("kw,status", [
    (dict(M=0), qg.QG_ERR_INVALID_ARG),                         # zero dimension
    (dict(N=0), qg.QG_ERR_INVALID_ARG),
    (dict(K=0), qg.QG_ERR_INVALID_ARG),
    (dict(K=520), qg.QG_ERR_INVALID_ARG),                       # K % 16
    (dict(fmt=qg.QG_BLOCK_FP8, K=384 + 64), qg.QG_ERR_INVALID_ARG),
    (dict(Y=None), qg.QG_ERR_INVALID_ARG),
    (dict(Y=FAKE + 8), qg.QG_ERR_INVALID_ARG),                  # misaligned output
    (dict(ldy=100), qg.QG_ERR_INVALID_ARG),                     # ldy < N
    (dict(out_kind=5), qg.QG_ERR_INVALID_ARG),
    (dict(A=_op(16, 512, q=FAKE + 4)), qg.QG_ERR_INVALID_ARG),  # misaligned codes
    (dict(A=_op(8, 512)), qg.QG_ERR_INVALID_ARG),               # rows != M
    (dict(W=_op(256, 256)), qg.QG_ERR_INVALID_ARG),             # K mismatch
    (dict(fmt=qg.QG_NVFP4, A=_op(16, 512, g=0)), qg.QG_ERR_INVALID_ARG),  # no tensor scale
    (dict(fmt=qg.QG_NVFP4, M=64, A=_op(64, 512), cfg=qg.make_config(tile_n=32, stages=4)),
     qg.QG_ERR_UNSUPPORTED),                                    # second 32-token tile: odd SF word
    (dict(fmt=qg.QG_NVFP4, M=20, A=_op(20, 512), cfg=qg.make_config(tile_n=16, stages=4)),
     qg.QG_ERR_UNSUPPORTED),
    (dict(fmt=9), qg.QG_ERR_INVALID_ARG),
    (dict(cfg=qg.make_config(split_k=3)), qg.QG_ERR_UNSUPPORTED),      # not a power of two
    (dict(cfg=qg.make_config(split_k=512)), qg.QG_ERR_UNSUPPORTED),    # above 256
    (dict(cfg=qg.make_config(split_k=8)), qg.QG_ERR_UNSUPPORTED),      # > 4 K tiles of 128 B
    (dict(cfg=qg.make_config(tile_n=48)), qg.QG_ERR_UNSUPPORTED),
    (dict(cfg=qg.make_config(stages=1)), qg.QG_ERR_UNSUPPORTED),
    (dict(cfg=qg.make_config(tile_n=256, stages=12)), qg.QG_ERR_UNSUPPORTED),  # smem
    (dict(fmt=qg.QG_BLOCK_FP8, K=8192 * 2, cfg=qg.make_config(tile_n=256, stages=3)), qg.QG_ERR_UNSUPPORTED),
    (dict(cfg=qg.make_config(swap_ab=2)), qg.QG_ERR_INVALID_ARG),
    (dict(cfg=qg.make_config(split_k=2, stages=4, reduce_mode=2), ws=None), qg.QG_ERR_WORKSPACE),
    (dict(cfg=qg.make_config(split_k=2, stages=4, reduce_mode=1), ws=FAKE, wsb=64), qg.QG_ERR_WORKSPACE),
    (dict(cfg=qg.make_config(split_k=4, stages=4, reduce_mode=3)), qg.QG_ERR_INVALID_ARG),
    (dict(K=4096, cfg=qg.make_config(split_k=16, stages=4, reduce_mode=0)), qg.QG_ERR_UNSUPPORTED),
])
def test_run_rejects_bad_arguments_before_any_launch(kw, status):
    assert _run(**kw) == status


def test_run_reserved_fields_must_be_zero():
    c = qg.make_config()
    c.reserved = 7
    assert _run(cfg=c) == qg.QG_ERR_INVALID_ARG
    c = qg.make_config()
    c.rows = 32                                     # rows belongs to the decode kernel only
    assert _run(cfg=c) == qg.QG_ERR_INVALID_ARG
    c = qg.make_config(variant=4)                   # no such kernel
    assert _run(cfg=c) == qg.QG_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,status", [
    (dict(), qg.QG_ERR_NO_DEVICE),                                  # valid: reaches the device check
    (dict(stages=6), qg.QG_ERR_NO_DEVICE),
    (dict(stages=1), qg.QG_ERR_UNSUPPORTED),
    (dict(stages=13), qg.QG_ERR_UNSUPPORTED),
    (dict(stages=8), qg.QG_ERR_NO_DEVICE),                          # 8 x 24 KB + the 32 KB y slice fit
    (dict(stages=9), qg.QG_ERR_UNSUPPORTED),                        # 9 x 24 KB + 32 KB: beyond smem
    (dict(tile_n=256, stages=6), qg.QG_ERR_NO_DEVICE),              # 256-wide pair tiles: 32 KB per stage
    (dict(tile_n=256, stages=7), qg.QG_ERR_UNSUPPORTED),
])
def test_pair_config_checks(kw, status):
    c = qg.pair_config(**({"tile_n": 128} | kw))
    assert _run(fmt=qg.QG_BLOCK_FP8, M=512, N=512, K=5120, cfg=c) == status
    for bad in (dict(split_k=2), dict(swap_ab=1), dict(reduce_mode=1), dict(rows=16), dict(tile_n=64)):
        c2 = qg.pair_config(**({"tile_n": 128} | kw))
        for k, v in bad.items():
            setattr(c2, k, v)
        assert _run(fmt=qg.QG_BLOCK_FP8, M=512, N=512, K=5120, cfg=c2) == qg.QG_ERR_UNSUPPORTED
    # only Block_FP8 runs on CTA pairs
    for fmt in (qg.QG_FP8_DYNAMIC, qg.QG_W8A8_INT8, qg.QG_NVFP4):
        assert _run(fmt=fmt, M=512, N=512, K=5120, cfg=qg.pair_config(128)) == qg.QG_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw,status", [
    (dict(), qg.QG_ERR_NO_DEVICE),                                  # valid: reaches the device check
    (dict(tile_n=128, stages=4), qg.QG_ERR_NO_DEVICE),
    (dict(tile_n=64), qg.QG_ERR_UNSUPPORTED),                       # 128- or 256-wide tiles only
    (dict(stages=13), qg.QG_ERR_UNSUPPORTED),
    (dict(tile_n=256, stages=5), qg.QG_ERR_UNSUPPORTED),            # 5 x 48 KB + 64 KB of y boxes: beyond smem
])
def test_persistent_config_checks(kw, status):
    c = qg.persist_config(**kw)
    assert _run(M=512, N=512, cfg=c) == status
    for bad in (dict(split_k=2), dict(swap_ab=1), dict(reduce_mode=1), dict(rows=16)):
        c2 = qg.persist_config(**kw)
        for k, v in bad.items():
            setattr(c2, k, v)
        assert _run(M=512, N=512, cfg=c2) == qg.QG_ERR_UNSUPPORTED
    # NVFP4 has no persistent kernel; Block_FP8's keeps a share of shared
    # memory for the tile's scales (more the longer K)
    assert _run(fmt=qg.QG_NVFP4, M=512, N=512, cfg=qg.persist_config()) == qg.QG_ERR_UNSUPPORTED
    assert _run(fmt=qg.QG_BLOCK_FP8, M=512, N=512, K=5120, cfg=qg.persist_config(256, 3)) == qg.QG_ERR_NO_DEVICE
    assert _run(fmt=qg.QG_BLOCK_FP8, M=512, N=512, K=65536, cfg=qg.persist_config(256, 3)) == qg.QG_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw,status", [
    (dict(tile_n=16, rows=32, stages=32), qg.QG_ERR_NO_DEVICE),     # valid: reaches the device check
    (dict(tile_n=32, rows=8, stages=16), qg.QG_ERR_NO_DEVICE),
    (dict(tile_n=8, rows=16, stages=8), qg.QG_ERR_NO_DEVICE),      # up to 8 tokens: weights as A
    (dict(tile_n=8, rows=8, stages=16), qg.QG_ERR_UNSUPPORTED),     # ... needs 16 rows per warp
    (dict(tile_n=8, rows=32, stages=6), qg.QG_ERR_UNSUPPORTED),     # 4 K groups: ring a multiple of 4
    (dict(tile_n=64, rows=32, stages=32), qg.QG_ERR_UNSUPPORTED),   # tokens per CTA: 8, 16 or 32
    (dict(tile_n=16, rows=24, stages=32), qg.QG_ERR_UNSUPPORTED),   # rows: 8, 16, 32, 64
    (dict(tile_n=16, rows=8, stages=12), qg.QG_ERR_UNSUPPORTED),    # ring depth a multiple of 64/rows
    (dict(tile_n=16, rows=64, stages=65), qg.QG_ERR_UNSUPPORTED),
    (dict(tile_n=32, rows=64, stages=20), qg.QG_ERR_UNSUPPORTED),   # 20 x 12 KB: beyond shared memory
])
def test_skinny_config_checks(kw, status):
    c = qg.skinny_config(**kw)
    assert _run(cfg=c) == status
    for bad in (dict(split_k=2), dict(swap_ab=0), dict(reduce_mode=1)):
        c2 = qg.skinny_config(**kw)
        for k, v in bad.items():
            setattr(c2, k, v)
        assert _run(cfg=c2) == qg.QG_ERR_UNSUPPORTED


def test_skinny_refuses_nvfp4_and_the_fused_and_grouped_launches():
    assert _run(fmt=qg.QG_NVFP4, K=1024, cfg=qg.skinny_config()) == qg.QG_ERR_UNSUPPORTED


def test_quantize_rejects_bad_arguments():
    out = _op(4, 512)
    assert qg.qgemm_quantize_act(qg.QG_FP8_DYNAMIC, FAKE, 4, 512, 100, None, out, None, 0, None) == qg.QG_ERR_INVALID_ARG
    assert qg.qgemm_quantize_act(qg.QG_FP8_DYNAMIC, FAKE + 2, 4, 512, 512, None, out, None, 0, None) == qg.QG_ERR_INVALID_ARG
    assert qg.qgemm_quantize_act(qg.QG_FP8_DYNAMIC, FAKE, 5, 512, 512, None, out, None, 0, None) == qg.QG_ERR_INVALID_ARG
    assert qg.qgemm_quantize_act(qg.QG_NVFP4, FAKE, 4, 512, 512, None, out, None, 0, None) == qg.QG_ERR_WORKSPACE
    assert qg.qgemm_quantize_weight(qg.QG_W8A8_INT8, None, 4, 512, out, None, 0, None) == qg.QG_ERR_INVALID_ARG


def test_valid_arguments_reach_the_device_check():
    # Everything is valid on the host: without a GPU the call stops at the
    # device check (with one, this test does not run: fake pointers).
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("needs a machine without a GPU")
    assert _run() in (qg.QG_ERR_NO_DEVICE, qg.QG_ERR_UNSUPPORTED)


def test_table_roundtrip_and_dispatch(tmp_path):
    t = qg.Table()
    c8 = qg.make_config(split_k=4, swap_ab=1, tile_n=16, stages=8)
    c32 = qg.make_config(split_k=2, swap_ab=1, tile_n=32, stages=6, reduce_mode=1)
    c2 = qg.make_config(split_k=8, swap_ab=1, tile_n=16, stages=4, reduce_mode=2)
    t.put(qg.QG_W8A8_INT8, 2, 4096, 4096, c2, 3.0)           # every reduce mode is storable
    t.put(qg.QG_W8A8_INT8, 8, 4096, 4096, c8, 3.5)
    t.put(qg.QG_W8A8_INT8, 32, 4096, 4096, c32, 4.25)
    assert len(t) == 3
    p = str(tmp_path / "table.txt")
    t.save(p)
    t2 = qg.Table(p)
    assert len(t2) == 3
    c, hit = t2.dispatch(qg.QG_W8A8_INT8, 2, 4096, 4096)
    assert hit == 1 and c.as_dict() == c2.as_dict()
    c, hit = t2.dispatch(qg.QG_W8A8_INT8, 8, 4096, 4096)
    assert hit == 1 and c.as_dict() == c8.as_dict()
    c, hit = t2.dispatch(qg.QG_W8A8_INT8, 20, 4096, 4096)         # rounds up to M=32
    assert hit == 2 and c.as_dict() == c32.as_dict()
    c, hit = t2.dispatch(qg.QG_W8A8_INT8, 1, 4096, 4096)          # rounds up to M=2
    assert hit == 2 and c.as_dict() == c2.as_dict()
    c, hit = t2.dispatch(qg.QG_W8A8_INT8, 64, 4096, 4096)         # beyond the table: default
    assert hit == 0 and c.as_dict() == qg.qgemm_default_config(qg.QG_W8A8_INT8, 64, 4096, 4096).as_dict()
    c, hit = t2.dispatch(qg.QG_FP8_DYNAMIC, 8, 4096, 4096)        # other format: default
    assert hit == 0


def test_table_version1_files_load_as_the_tile_kernel_and_decode_entries_roundtrip(tmp_path):
    p = tmp_path / "v1.qgt"
    p.write_text("qgemm-table 1\ndevice x sms 148\n1 8 4096 4096 4 1 16 8 0 3.5\n")
    c, hit = qg.Table(str(p)).dispatch(qg.QG_W8A8_INT8, 8, 4096, 4096)
    assert hit == 1 and c.as_dict() == qg.make_config(4, 1, 16, 8, 0).as_dict()
    t = qg.Table()
    sk = qg.skinny_config(tile_n=16, rows=32, stages=32)
    t.put(qg.QG_FP8_DYNAMIC, 1, 4096, 4096, sk, 2.5)
    q = str(tmp_path / "v2.qgt")
    t.save(q)
    assert open(q).readline().split() == ["qgemm-table", "2"]
    c, hit = qg.Table(q).dispatch(qg.QG_FP8_DYNAMIC, 1, 4096, 4096)
    assert hit == 1 and c.as_dict() == sk.as_dict()


def test_table_roundtrips_persistent_and_pair_entries(tmp_path):
    t = qg.Table()
    t.put(qg.QG_FP8_DYNAMIC, 2048, 4096, 4096, qg.persist_config(256, 4), 29.3)
    t.put(qg.QG_BLOCK_FP8, 4096, 5120, 5120, qg.pair_config(256, 4), 132.9)
    t.put(qg.QG_BLOCK_FP8, 1024, 4096, 4096, qg.pair_config(128, 6), 30.0)
    q = str(tmp_path / "v2.qgt")
    t.save(q)
    t2 = qg.Table(q)
    for fmt, M, N, K, cfg in [(qg.QG_FP8_DYNAMIC, 2048, 4096, 4096, qg.persist_config(256, 4)),
                              (qg.QG_BLOCK_FP8, 4096, 5120, 5120, qg.pair_config(256, 4)),
                              (qg.QG_BLOCK_FP8, 1024, 4096, 4096, qg.pair_config(128, 6))]:
        c, hit = t2.dispatch(fmt, M, N, K)
        assert hit == 1 and c.as_dict() == cfg.as_dict()


@pytest.mark.parametrize("content", [
    "",
    "qgemm-table 3\ndevice x sms 148\n",                                    # unknown version
    "qgemm-table 2\ndevice x sms 148\n2 4096 5120 5120 1 0 64 4 0 3 0 1.0\n",  # CTA pairs: 128 or 256 wide
    "qgemm-table 2\ndevice x sms 148\n2 4096 5120 5120 1 0 256 4 0 4 0 1.0\n", # no variant 4
    "qgemm-table 1\ndevice x sms 148\n1 8 4096 4096 4 1 16 8 0\n",          # missing field
    "qgemm-table 2\ndevice x sms 148\n1 8 4096 4096 4 1 16 8 0 1.0\n",      # version 2: variant, rows missing
    "qgemm-table 2\ndevice x sms 148\n1 8 4096 4096 1 1 16 24 0 1 12 1.0\n",  # decode kernel: bad rows
    "qgemm-table 2\ndevice x sms 148\n1 8 4096 4096 4 1 16 8 0 0 32 1.0\n",   # rows on the tile kernel
    "qgemm-table 1\ndevice x sms 148\n1 8 4096 4096 4 3 16 8 0 1.0\n",      # bad swap
    "qgemm-table 1\ndevice x sms 148\n1 8 4096 4096 4 1 16 8 3 1.0\n",      # bad reduce mode
    "not a table\n",
])
def test_table_load_rejects_corrupt_files(tmp_path, content):
    p = tmp_path / "bad.txt"
    p.write_text(content)
    with pytest.raises(qg.QGemmError) as e:
        qg.Table(str(p))
    assert e.value.status == qg.QG_ERR_TABLE_IO


def test_table_load_missing_file():
    with pytest.raises(qg.QGemmError) as e:
        qg.Table("/nonexistent/qgemm_table.txt")
    assert e.value.status == qg.QG_ERR_TABLE_IO


def _fused(fmt=qg.QG_W8A8_INT8, M=8, N=256, K=512, cfg=None, A=FAKE, lda=None, W=None, ws=None, wsb=0,
           Y=FAKE, ldy=None, out_kind=0, scales=None):
    cfg = cfg or qg.make_config(split_k=2, swap_ab=1, tile_n=16, stages=4, reduce_mode=0)
    W = W or _op(N, K)
    return qg.qgemm_run_fused_act(fmt, A, lda if lda is not None else K, W, M, N, K, cfg, ws, wsb, Y,
                                  ldy if ldy is not None else N, out_kind, scales, None)


@pytest.mark.parametrize("kw,status", [
    (dict(M=0), qg.QG_ERR_INVALID_ARG),
    (dict(A=None), qg.QG_ERR_INVALID_ARG),
    (dict(A=FAKE + 8), qg.QG_ERR_INVALID_ARG),                  # activations not 16-byte aligned
    (dict(lda=500), qg.QG_ERR_INVALID_ARG),                     # lda < K
    (dict(lda=516), qg.QG_ERR_INVALID_ARG),                     # row stride not a multiple of 16 bytes
    (dict(K=520), qg.QG_ERR_INVALID_ARG),
    (dict(scales=FAKE + 2), qg.QG_ERR_INVALID_ARG),             # misaligned scale output
    (dict(W=_op(128, 512)), qg.QG_ERR_INVALID_ARG),             # W rows != N
    (dict(fmt=qg.QG_NVFP4), qg.QG_ERR_UNSUPPORTED),             # tensor amax spans all of A
    (dict(cfg=qg.make_config(split_k=1, swap_ab=0, tile_n=128, stages=4)), qg.QG_ERR_UNSUPPORTED),
    (dict(cfg=qg.make_config(split_k=2, swap_ab=1, tile_n=16, stages=4, reduce_mode=1), ws=FAKE,
          wsb=1 << 20), qg.QG_ERR_UNSUPPORTED),                 # per-token amax needs a cluster
    (dict(fmt=qg.QG_FP8_DYNAMIC, cfg=qg.make_config(split_k=2, swap_ab=1, tile_n=16, stages=4,
                                                     reduce_mode=2), ws=FAKE, wsb=1 << 20),
     qg.QG_ERR_UNSUPPORTED),
    (dict(fmt=qg.QG_BLOCK_FP8, cfg=qg.make_config(split_k=2, swap_ab=1, tile_n=16, stages=4,
                                                   reduce_mode=1)), qg.QG_ERR_WORKSPACE),
    (dict(cfg=qg.make_config(split_k=3, swap_ab=1, tile_n=16, stages=4)), qg.QG_ERR_UNSUPPORTED),
])
def test_fused_rejects_bad_arguments_before_any_launch(kw, status):
    assert _fused(**kw) == status


def test_fused_valid_arguments_reach_the_device_check():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("needs a machine without a GPU")
    # Block_FP8 groups are local to a K tile: any split and reduce mode
    ok = [dict(),
          dict(fmt=qg.QG_BLOCK_FP8, cfg=qg.make_config(split_k=2, swap_ab=1, tile_n=16, stages=4,
                                                        reduce_mode=1), ws=FAKE, wsb=1 << 20),
          dict(fmt=qg.QG_FP8_DYNAMIC, cfg=qg.make_config(split_k=1, swap_ab=1, tile_n=32, stages=4))]
    for kw in ok:
        assert _fused(**kw) in (qg.QG_ERR_NO_DEVICE, qg.QG_ERR_UNSUPPORTED)


@pytest.mark.parametrize("kw,status", [
    # NVFP4: a 16-token tile below row 16 of a scale atom is refused (T = 24 > 16)
    (dict(fmt=qg.QG_NVFP4), qg.QG_ERR_UNSUPPORTED),
    (dict(E=0), qg.QG_ERR_INVALID_ARG),
    (dict(E=300), qg.QG_ERR_UNSUPPORTED),                       # more than 256 experts
    (dict(offsets=None), qg.QG_ERR_INVALID_ARG),
    (dict(offsets=FAKE + 2), qg.QG_ERR_INVALID_ARG),
    (dict(N=200), qg.QG_ERR_INVALID_ARG),                       # experts must fill 128-row blocks
    (dict(Wrows=4 * 256 + 128), qg.QG_ERR_INVALID_ARG),         # W rows != experts * N
    (dict(cfg=qg.make_config(split_k=1, swap_ab=0, tile_n=128, stages=4)), qg.QG_ERR_UNSUPPORTED),
    (dict(cfg=qg.make_config(split_k=2, swap_ab=1, tile_n=16, stages=4, reduce_mode=2), ws=FAKE),
     qg.QG_ERR_UNSUPPORTED),                                     # last-CTA counters are per tile
])
def test_grouped_rejects_bad_arguments_before_any_launch(kw, status):
    fmt = kw.get("fmt", qg.QG_FP8_DYNAMIC)
    E, N, K, T = kw.get("E", 4), kw.get("N", 256), 512, 24
    cfg = kw.get("cfg", qg.make_config(split_k=1, swap_ab=1, tile_n=16, stages=4))
    W = _op(kw.get("Wrows", E * N), K)
    st = qg.qgemm_run_grouped(fmt, E, kw.get("offsets", FAKE), _op(T, K), W, N, K, cfg, kw.get("ws", None),
                              1 << 30, FAKE, N, 0, None)
    assert st == status


@pytest.mark.parametrize("fmt", [qg.QG_FP8_DYNAMIC, qg.QG_W8A8_INT8, qg.QG_BLOCK_FP8, qg.QG_NVFP4])
@pytest.mark.parametrize("E,T,N,K", [(128, 8, 1536, 2048), (128, 512, 2048, 768), (4, 3, 256, 512),
                                     (256, 4096, 1024, 4096)])
def test_grouped_default_config_is_accepted_by_the_grouped_launch(fmt, E, T, N, K):
    c = qg.qgemm_grouped_default_config(fmt, E, T, N, K)
    assert c.swap_ab == 1 and c.reduce_mode in (0, 1)
    assert c.split_k >= 1 and c.split_k & (c.split_k - 1) == 0 and c.tile_n in (16, 32, 64, 128, 256)
    if fmt == qg.QG_NVFP4:
        assert c.tile_n >= 64 or T <= c.tile_n
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        return                     # the fake pointers below must never reach a launch
    # the arguments pass every host check of qgemm_run_grouped: only the device is missing here
    wsb = qg.qgemm_workspace_size(fmt, T, N, K, c)
    st = qg.qgemm_run_grouped(fmt, E, FAKE, _op(T, K), _op(E * N, K), N, K, c, FAKE if wsb else None, wsb, FAKE,
                              N, 0, None)
    assert st == qg.QG_ERR_NO_DEVICE


def test_grouped_default_config_rejects_bad_sizes():
    c = qg.qg_config()
    assert qg.lib().qgemm_grouped_default_config(qg.QG_FP8_DYNAMIC, 0, 8, 256, 512, c) == qg.QG_ERR_INVALID_ARG
    assert qg.lib().qgemm_grouped_default_config(qg.QG_FP8_DYNAMIC, 8, 8, 256, 100, c) == qg.QG_ERR_INVALID_ARG


def test_wait_expiry_selftest_rejects_limits_before_the_device():
    # checked on the host before any device work (no GPU needed)
    assert qg.lib().qgemm_selftest_wait_expiry(0, None) == qg.QG_ERR_INVALID_ARG
    assert qg.lib().qgemm_selftest_wait_expiry(10 ** 9, None) == qg.QG_ERR_INVALID_ARG
    qg.qgemm_set_wait_limit(5_000_000)
    qg.qgemm_set_wait_limit(0)


@pytest.mark.parametrize("E,T,K", [(8, 1, 512), (8, 300, 512), (256, 200, 1024), (4, 4096, 256), (1, 128, 64)])
def test_grouped_act_bytes_bound_every_routing(E, T, K):
    # NVFP4: floor((T - a) / 128) + a atoms, a = min(E, T), is the most any
    # routing of T tokens over E experts needs (brute force over the extremes)
    q, s = qg.qgemm_grouped_act_bytes(qg.QG_NVFP4, E, T, K)
    q1, s1 = qg.qgemm_operand_bytes(qg.QG_NVFP4, 0, T, K)
    C = (K + 255) // 256 * 16
    a = min(E, T)
    assert q == q1 and s == ((T - a) // 128 + a) * 128 * C and s >= s1
    rng = np.random.default_rng(T)
    worst = 0
    for counts in ([T] + [0] * (E - 1), [1] * (a - 1) + [T - a + 1] + [0] * (E - a),
                   rng.multinomial(T, [1 / E] * E)):
        worst = max(worst, sum((c + 127) // 128 for c in counts))
    assert worst * 128 * C <= s
    # the 8-bit formats' scales do not depend on the routing
    for f in (qg.QG_FP8_DYNAMIC, qg.QG_W8A8_INT8, qg.QG_BLOCK_FP8):
        if K % 128 == 0 or f != qg.QG_BLOCK_FP8:
            assert qg.qgemm_grouped_act_bytes(f, E, T, K) == qg.qgemm_operand_bytes(f, 0, T, K)


def test_grouped_quantisers_check_arguments_before_the_device():
    L = qg.lib()
    T, K, E, N = 24, 512, 4, 256
    qb, sb = qg.qgemm_grouped_act_bytes(qg.QG_NVFP4, E, T, K)
    out = _op(T, K)
    assert L.qgemm_grouped_act_bytes(qg.QG_NVFP4, 0, T, K, None, None) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_grouped_act_bytes(qg.QG_NVFP4, 300, T, K, None, None) == qg.QG_ERR_UNSUPPORTED
    args = lambda **kw: (kw.get("f", qg.QG_NVFP4), kw.get("E", E), kw.get("off", FAKE), kw.get("A", FAKE),
                         kw.get("T", T), K, kw.get("lda", K), None, kw.get("out", out), FAKE, 1 << 20, None)
    assert L.qgemm_quantize_act_grouped(*args(off=None)) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_quantize_act_grouped(*args(off=FAKE + 2)) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_quantize_act_grouped(*args(E=0)) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_quantize_act_grouped(*args(E=300)) == qg.QG_ERR_UNSUPPORTED
    assert L.qgemm_quantize_act_grouped(*args(lda=K - 1)) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_quantize_act_grouped(*args(out=_op(T + 1, K))) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_quantize_act_grouped(*args(out=_op(T, K, g=0))) == qg.QG_ERR_INVALID_ARG
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        assert L.qgemm_quantize_act_grouped(*args()) == qg.QG_ERR_NO_DEVICE
        assert L.qgemm_quantize_act_grouped(*args(f=qg.QG_W8A8_INT8)) == qg.QG_ERR_NO_DEVICE
    W = _op(E * N, K)
    wargs = lambda **kw: (kw.get("f", qg.QG_NVFP4), kw.get("E", E), FAKE, kw.get("N", N), K, kw.get("out", W),
                          FAKE, kw.get("wsb", 1 << 20), None)
    assert L.qgemm_quantize_weight_grouped(*wargs(N=200)) == qg.QG_ERR_INVALID_ARG     # N % 128
    assert L.qgemm_quantize_weight_grouped(*wargs(E=0)) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_quantize_weight_grouped(*wargs(E=300)) == qg.QG_ERR_UNSUPPORTED
    assert L.qgemm_quantize_weight_grouped(*wargs(out=_op(E * N - 128, K))) == qg.QG_ERR_INVALID_ARG
    assert L.qgemm_quantize_weight_grouped(*wargs(wsb=0)) == qg.QG_ERR_WORKSPACE
    if not torch.cuda.is_available():
        assert L.qgemm_quantize_weight_grouped(*wargs()) == qg.QG_ERR_NO_DEVICE


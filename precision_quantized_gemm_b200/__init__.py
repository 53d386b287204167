"""Python binding of libqgemm.so — the B200 quantized linear-layer GEMM.

Argument marshalling only: every step of the quantized path (activation
quantisation, the tcgen05 GEMM, split-K reduction, dispatch, tuning) runs in
the C-ABI library ``libqgemm.so`` built from ``csrc/``.  PyTorch supplies
device memory and streams.  If the library is missing this module raises on
first use; there is no fallback.

The ctypes entry points carry the C names (``qgemm_run`` ...).  ``Operand``,
``quantize_act``, ``quantize_weight``, ``run`` and ``Linear`` are
conveniences over them that allocate the caller-owned buffers with torch.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_int, c_int32, c_size_t, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqgemm.so")

# formats
QG_FP8_DYNAMIC, QG_W8A8_INT8, QG_BLOCK_FP8, QG_NVFP4 = 0, 1, 2, 3
FORMATS = {"fp8_dynamic": 0, "w8a8_int8": 1, "block_fp8": 2, "nvfp4": 3}
# statuses
QG_OK = 0
QG_ERR_INVALID_ARG = 1
QG_ERR_UNSUPPORTED = 2
QG_ERR_WORKSPACE = 3
QG_ERR_TABLE_IO = 4
QG_ERR_TABLE_MISS = 5
QG_ERR_CUDA = 6
QG_ERR_DEVICE_TIMEOUT = 7
QG_ERR_NO_DEVICE = 8
# output kinds
QG_OUT_BF16, QG_OUT_ACC = 0, 1

EXPORTS = [
    "qgemm_abi_version", "qgemm_set_pdl", "qgemm_status_string", "qgemm_operand_bytes",
    "qgemm_quant_workspace_size", "qgemm_workspace_size", "qgemm_workspace_clear",
    "qgemm_quantize_act", "qgemm_quantize_weight", "qgemm_run", "qgemm_default_config",
    "qgemm_table_load", "qgemm_table_create", "qgemm_table_put", "qgemm_table_save",
    "qgemm_table_free", "qgemm_table_size", "qgemm_dispatch", "qgemm_tune", "qgemm_device_error",
    "qgemm_run_noalloc", "qgemm_set_trace", "qgemm_run_fused_act", "qgemm_set_tune_log",
    "qgemm_score_config", "qgemm_rank_configs", "qgemm_tune_ranked", "qgemm_table_validate",
    "qgemm_run_grouped", "qgemm_grouped_default_config", "qgemm_set_wait_limit", "qgemm_selftest_wait_expiry",
    "qgemm_set_tune_objective", "qgemm_grouped_act_bytes", "qgemm_quantize_act_grouped",
    "qgemm_quantize_weight_grouped", "qgemm_set_tma_store",
]


class qg_config(ctypes.Structure):
    _fields_ = [("split_k", c_int32), ("swap_ab", c_int32), ("tile_n", c_int32),
                ("stages", c_int32), ("reduce_mode", c_int32), ("variant", c_int32), ("rows", c_int32),
                ("reserved", c_int32)]

    def as_dict(self):
        return {k: getattr(self, k) for k in ("split_k", "swap_ab", "tile_n", "stages", "reduce_mode", "variant",
                                               "rows")}

    def __repr__(self):
        return f"qg_config({self.as_dict()})"


def make_config(split_k=1, swap_ab=1, tile_n=16, stages=8, reduce_mode=0, variant=0, rows=0) -> qg_config:
    c = qg_config()
    c.split_k, c.swap_ab, c.tile_n, c.stages, c.reduce_mode = split_k, swap_ab, tile_n, stages, reduce_mode
    c.variant, c.rows = variant, rows
    return c


def persist_config(tile_n=256, stages=3) -> qg_config:
    """Configuration of the persistent kernel (8-bit formats; large M): one
    CTA per SM walks the 128 x tile_n output tiles, overlapping a tile's
    epilogue with the next tile's MMAs."""
    return make_config(split_k=1, swap_ab=0, tile_n=tile_n, stages=stages, reduce_mode=0, variant=2)


def pair_config(tile_n=256, stages=4) -> qg_config:
    """Configuration of the CTA-pair kernel (Block_FP8, large M): clusters of
    two CTAs walk 256 x tile_n output tiles (tile_n 128 or 256) with one
    two-SM MMA per K step."""
    return make_config(split_k=1, swap_ab=0, tile_n=tile_n, stages=stages, reduce_mode=0, variant=3)


def skinny_config(tile_n=16, rows=32, stages=32) -> qg_config:
    """Configuration of the decode ("skinny") kernel: `rows` weight rows per
    CTA over the whole of K, `tile_n` tokens, a ring of `stages` K tiles."""
    return make_config(split_k=1, swap_ab=1, tile_n=tile_n, stages=stages, reduce_mode=0, variant=1, rows=rows)


class qg_operand(ctypes.Structure):
    _fields_ = [("q", c_void_p), ("scale", c_void_p), ("global_scale", c_void_p),
                ("rows", c_int32), ("K", c_int32)]


class QGemmError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libqgemm.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m precision_quantized_gemm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "qgemm_abi_version": (c_int, []),
            "qgemm_set_pdl": (None, [c_int]),
            "qgemm_set_tma_store": (None, [c_int]),
            "qgemm_status_string": (c_char_p, [c_int]),
            "qgemm_operand_bytes": (c_int, [c_int, c_int, c_int, c_int, POINTER(c_size_t), POINTER(c_size_t)]),
            "qgemm_quant_workspace_size": (c_size_t, [c_int, c_int, c_int]),
            "qgemm_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int, POINTER(qg_config)]),
            "qgemm_workspace_clear": (c_int, [c_void_p, c_size_t, c_void_p]),
            "qgemm_quantize_act": (c_int, [c_int, c_void_p, c_int, c_int, c_int, c_void_p,
                                           POINTER(qg_operand), c_void_p, c_size_t, c_void_p]),
            "qgemm_quantize_weight": (c_int, [c_int, c_void_p, c_int, c_int, POINTER(qg_operand),
                                              c_void_p, c_size_t, c_void_p]),
            "qgemm_run": (c_int, [c_int, POINTER(qg_operand), POINTER(qg_operand), c_int, c_int, c_int,
                                  POINTER(qg_config), c_void_p, c_size_t, c_void_p, c_int, c_int, c_void_p]),
            "qgemm_default_config": (c_int, [c_int, c_int, c_int, c_int, POINTER(qg_config)]),
            "qgemm_table_load": (c_int, [c_char_p, POINTER(c_void_p)]),
            "qgemm_table_create": (c_int, [POINTER(c_void_p)]),
            "qgemm_table_put": (c_int, [c_void_p, c_int, c_int, c_int, c_int, POINTER(qg_config), c_double]),
            "qgemm_table_save": (c_int, [c_void_p, c_char_p]),
            "qgemm_table_free": (None, [c_void_p]),
            "qgemm_table_size": (c_int, [c_void_p]),
            "qgemm_dispatch": (c_int, [c_void_p, c_int, c_int, c_int, c_int, POINTER(qg_config), POINTER(c_int)]),
            "qgemm_tune": (c_int, [c_void_p, c_int, POINTER(c_int), c_int, POINTER(c_int), c_int, c_double, c_int]),
            "qgemm_device_error": (c_int, []),
            "qgemm_set_wait_limit": (None, [ctypes.c_ulonglong]),
            "qgemm_selftest_wait_expiry": (c_int, [ctypes.c_ulonglong, c_void_p]),
            "qgemm_set_trace": (None, [c_void_p, c_size_t]),
            "qgemm_set_tune_log": (None, [c_char_p]),
            "qgemm_set_tune_objective": (None, [c_int]),
            "qgemm_score_config": (c_int, [c_int, c_int, c_int, c_int, POINTER(qg_config), POINTER(c_double)]),
            "qgemm_rank_configs": (c_int, [c_int, c_int, c_int, c_int, POINTER(qg_config), c_int,
                                           POINTER(c_double), POINTER(c_int)]),
            "qgemm_tune_ranked": (c_int, [c_void_p, c_int, POINTER(c_int), c_int, POINTER(c_int), c_int, c_int,
                                          c_double, c_int]),
            "qgemm_table_validate": (c_int, [c_void_p, POINTER(c_int), POINTER(c_int), c_int]),
            "qgemm_grouped_default_config": (c_int, [c_int, c_int, c_int, c_int, c_int, POINTER(qg_config)]),
            "qgemm_grouped_act_bytes": (c_int, [c_int, c_int, c_int, c_int, POINTER(c_size_t), POINTER(c_size_t)]),
            "qgemm_quantize_act_grouped": (c_int, [c_int, c_int, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p,
                                                   POINTER(qg_operand), c_void_p, c_size_t, c_void_p]),
            "qgemm_quantize_weight_grouped": (c_int, [c_int, c_int, c_void_p, c_int, c_int, POINTER(qg_operand),
                                                      c_void_p, c_size_t, c_void_p]),
            "qgemm_run_grouped": (c_int, [c_int, c_int, c_void_p, POINTER(qg_operand), POINTER(qg_operand), c_int,
                                          c_int, POINTER(qg_config), c_void_p, c_size_t, c_void_p, c_int, c_int,
                                          c_void_p]),
            "qgemm_run_noalloc": (c_int, [c_int, POINTER(qg_operand), POINTER(qg_operand), c_int, c_int, c_int,
                                          POINTER(qg_config), c_void_p, c_int, c_int, c_void_p]),
            "qgemm_run_fused_act": (c_int, [c_int, c_void_p, c_int, POINTER(qg_operand), c_int, c_int, c_int,
                                            POINTER(qg_config), c_void_p, c_size_t, c_void_p, c_int, c_int,
                                            c_void_p, c_void_p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().qgemm_status_string(status).decode()


def check(status: int, what: str = "qgemm") -> None:
    if status != QG_OK:
        raise QGemmError(status, what)


# ------------------------------------------------------- C-named entry points --
def qgemm_operand_bytes(fmt, is_weight, rows, K):
    q, s = c_size_t(), c_size_t()
    st = lib().qgemm_operand_bytes(fmt, int(is_weight), rows, K, ctypes.byref(q), ctypes.byref(s))
    check(st, "qgemm_operand_bytes")
    return q.value, s.value


def qgemm_quant_workspace_size(fmt, rows, K):
    return lib().qgemm_quant_workspace_size(fmt, rows, K)


def qgemm_workspace_size(fmt, M, N, K, cfg: qg_config):
    return lib().qgemm_workspace_size(fmt, M, N, K, ctypes.byref(cfg))


def qgemm_workspace_clear(ws_ptr, ws_bytes, stream=None):
    return lib().qgemm_workspace_clear(ws_ptr, ws_bytes, stream)


def qgemm_quantize_act(fmt, A_ptr, M, K, lda, static_amax_ptr, out: qg_operand, ws_ptr, ws_bytes, stream):
    return lib().qgemm_quantize_act(fmt, A_ptr, M, K, lda, static_amax_ptr, ctypes.byref(out),
                                    ws_ptr, ws_bytes, stream)


def qgemm_quantize_weight(fmt, W_ptr, N, K, out: qg_operand, ws_ptr, ws_bytes, stream):
    return lib().qgemm_quantize_weight(fmt, W_ptr, N, K, ctypes.byref(out), ws_ptr, ws_bytes, stream)


def qgemm_run(fmt, A: qg_operand, W: qg_operand, M, N, K, cfg: qg_config, ws_ptr, ws_bytes,
              Y_ptr, ldy, out_kind, stream):
    return lib().qgemm_run(fmt, ctypes.byref(A), ctypes.byref(W), M, N, K, ctypes.byref(cfg),
                           ws_ptr, ws_bytes, Y_ptr, ldy, out_kind, stream)


def qgemm_run_noalloc(fmt, A: qg_operand, W: qg_operand, M, N, K, cfg: qg_config, Y_ptr, ldy, out_kind,
                      stream):
    """qgemm_run with the library's own fixed scratch instead of a caller workspace."""
    return lib().qgemm_run_noalloc(fmt, ctypes.byref(A), ctypes.byref(W), M, N, K, ctypes.byref(cfg),
                                   Y_ptr, ldy, out_kind, stream)


def qgemm_run_fused_act(fmt, A_ptr, lda, W: qg_operand, M, N, K, cfg: qg_config, ws_ptr, ws_bytes,
                        Y_ptr, ldy, out_kind, act_scale_ptr, stream):
    """GEMM on bf16 activations, quantised inside the kernel (Swap-AB decode path)."""
    return lib().qgemm_run_fused_act(fmt, A_ptr, lda, ctypes.byref(W), M, N, K, ctypes.byref(cfg), ws_ptr,
                                     ws_bytes, Y_ptr, ldy, out_kind, act_scale_ptr, stream)


def qgemm_run_grouped(fmt, experts, offsets_ptr, A: qg_operand, W: qg_operand, N, K, cfg: qg_config, ws_ptr,
                      ws_bytes, Y_ptr, ldy, out_kind, stream):
    """Grouped (mixture-of-experts) GEMM over tokens sorted by expert."""
    return lib().qgemm_run_grouped(fmt, experts, offsets_ptr, ctypes.byref(A), ctypes.byref(W), N, K,
                                   ctypes.byref(cfg), ws_ptr, ws_bytes, Y_ptr, ldy, out_kind, stream)


def qgemm_grouped_act_bytes(fmt, experts, T, K):
    """Bytes of the q and scale buffers of a grouped activation operand."""
    q, s = c_size_t(), c_size_t()
    check(lib().qgemm_grouped_act_bytes(fmt, experts, T, K, ctypes.byref(q), ctypes.byref(s)),
          "qgemm_grouped_act_bytes")
    return q.value, s.value


def qgemm_quantize_act_grouped(fmt, experts, offsets_ptr, A_ptr, T, K, lda, static_amax_ptr, out: qg_operand,
                               ws_ptr, ws_bytes, stream):
    """Activation quantisation for a grouped launch (NVFP4: per-expert scale layout)."""
    return lib().qgemm_quantize_act_grouped(fmt, experts, offsets_ptr, A_ptr, T, K, lda, static_amax_ptr,
                                            ctypes.byref(out), ws_ptr, ws_bytes, stream)


def qgemm_quantize_weight_grouped(fmt, experts, W_ptr, N, K, out: qg_operand, ws_ptr, ws_bytes, stream):
    """Stacked expert weights (NVFP4: one tensor scale per expert)."""
    return lib().qgemm_quantize_weight_grouped(fmt, experts, W_ptr, N, K, ctypes.byref(out), ws_ptr, ws_bytes,
                                               stream)


def qgemm_default_config(fmt, M, N, K) -> qg_config:
    c = qg_config()
    check(lib().qgemm_default_config(fmt, M, N, K, ctypes.byref(c)), "qgemm_default_config")
    return c


def qgemm_grouped_default_config(fmt, experts, T, N, K) -> qg_config:
    c = qg_config()
    check(lib().qgemm_grouped_default_config(fmt, experts, T, N, K, ctypes.byref(c)), "qgemm_grouped_default_config")
    return c


def qgemm_score_config(fmt, M, N, K, cfg: qg_config) -> float:
    """The analytic scorer's estimated µs for one configuration (raises if it is invalid)."""
    est = c_double()
    check(lib().qgemm_score_config(fmt, M, N, K, ctypes.byref(cfg), ctypes.byref(est)), "qgemm_score_config")
    return est.value


def qgemm_rank_configs(fmt, M, N, K, max_out=16):
    """The scorer's ranking: [(qg_config, estimated µs)], best first."""
    out = (qg_config * max(max_out, 1))()
    est = (c_double * max(max_out, 1))()
    n = c_int(0)
    check(lib().qgemm_rank_configs(fmt, M, N, K, out, max_out, est, ctypes.byref(n)), "qgemm_rank_configs")
    return [(out[i], est[i]) for i in range(n.value)]


def qgemm_dispatch(table, fmt, M, N, K):
    c = qg_config()
    hit = c_int(0)
    check(lib().qgemm_dispatch(table, fmt, M, N, K, ctypes.byref(c), ctypes.byref(hit)), "qgemm_dispatch")
    return c, hit.value


def qgemm_device_error():
    return lib().qgemm_device_error()


def qgemm_set_wait_limit(limit_ns: int):
    """Limit (ns) of every bounded in-kernel wait of later launches (0: the 200 ms default)."""
    lib().qgemm_set_wait_limit(int(limit_ns))


def qgemm_selftest_wait_expiry(limit_ns: int, stream=None) -> int:
    """Launches a wait on an mbarrier nothing arrives on, bounded by limit_ns;
    the next qgemm_device_error() reports QG_ERR_DEVICE_TIMEOUT."""
    return lib().qgemm_selftest_wait_expiry(int(limit_ns), _stream(stream))


def qgemm_set_trace(buf_ptr, nbytes):
    """Debug: record per-CTA phase timestamps of later launches into a device buffer."""
    lib().qgemm_set_trace(buf_ptr, nbytes)


def qgemm_set_tune_log(path):
    """Tuning instrumentation: log every timed candidate of qgemm_tune to `path` (None: off)."""
    lib().qgemm_set_tune_log(path.encode() if path else None)


def qgemm_set_tune_objective(gemm_only: bool):
    """Tuner timing: quantise + GEMM steps (False, the default) or GEMMs alone (True)."""
    lib().qgemm_set_tune_objective(1 if gemm_only else 0)


def qgemm_set_pdl(enable: bool):
    lib().qgemm_set_pdl(1 if enable else 0)


def qgemm_set_tma_store(enable: bool):
    """TMA stores of direct standard-orientation output tiles (default on)."""
    lib().qgemm_set_tma_store(1 if enable else 0)


class Table:
    """Owning wrapper of a qgemm table handle."""

    def __init__(self, path: str | None = None):
        h = c_void_p()
        if path is None:
            check(lib().qgemm_table_create(ctypes.byref(h)), "qgemm_table_create")
        else:
            check(lib().qgemm_table_load(path.encode(), ctypes.byref(h)), f"qgemm_table_load({path})")
        self.handle = h

    def __len__(self):
        return lib().qgemm_table_size(self.handle)

    def put(self, fmt, M, N, K, cfg: qg_config, us: float = 0.0):
        check(lib().qgemm_table_put(self.handle, fmt, M, N, K, ctypes.byref(cfg), us), "qgemm_table_put")

    def save(self, path: str):
        check(lib().qgemm_table_save(self.handle, path.encode()), "qgemm_table_save")

    def dispatch(self, fmt, M, N, K):
        return qgemm_dispatch(self.handle, fmt, M, N, K)

    def tune(self, fmt, Ms, NK, budget_s_per_shape=30.0, verbose=True, top_n=0):
        """qgemm_tune over the whole candidate grid, or (top_n > 0) qgemm_tune_ranked
        over the scorer's top_n configurations."""
        Ms_arr = (c_int * len(Ms))(*Ms)
        flat = [v for nk in NK for v in nk]
        NK_arr = (c_int * len(flat))(*flat)
        if top_n > 0:
            check(lib().qgemm_tune_ranked(self.handle, fmt, Ms_arr, len(Ms), NK_arr, len(NK), int(top_n),
                                          float(budget_s_per_shape), 1 if verbose else 0), "qgemm_tune_ranked")
            return
        check(lib().qgemm_tune(self.handle, fmt, Ms_arr, len(Ms), NK_arr, len(NK),
                               float(budget_s_per_shape), 1 if verbose else 0), "qgemm_tune")

    def validate(self, verbose=False):
        """qgemm_table_validate: run every entry next to the scored default and drop
        the ones refused or out of tolerance; returns (checked, rejected)."""
        checked, rejected = c_int(0), c_int(0)
        check(lib().qgemm_table_validate(self.handle, ctypes.byref(checked), ctypes.byref(rejected),
                                         1 if verbose else 0), "qgemm_table_validate")
        return checked.value, rejected.value

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            lib().qgemm_table_free(self.handle)
            self.handle = c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------ torch helpers --
def _torch():
    import torch
    return torch


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return c_void_p(s.cuda_stream)


class Operand:
    """Caller-owned buffers of a quantized operand, allocated with torch.
    ``sizes`` overrides the (q, scale) byte counts and ``n_global`` the number
    of tensor scales (grouped operands)."""

    def __init__(self, fmt: int, is_weight: bool, rows: int, K: int, device="cuda", sizes=None, n_global=1):
        torch = _torch()
        qb, sb = sizes or qgemm_operand_bytes(fmt, is_weight, rows, K)
        self.fmt, self.is_weight, self.rows, self.K = fmt, is_weight, rows, K
        self.q = torch.empty(qb, dtype=torch.uint8, device=device)
        self.scale = torch.zeros(sb, dtype=torch.uint8, device=device)
        self.global_scale = torch.zeros(max(n_global, 4), dtype=torch.float32, device=device)
        self.c = qg_operand(self.q.data_ptr(), self.scale.data_ptr(), self.global_scale.data_ptr(), rows, K)


def quantize_act(fmt: int, A, out: Operand | None = None, static_amax=None, stream=None) -> Operand:
    """Dynamic activation quantisation of bf16 A [M, K] (row stride A.stride(0))."""
    torch = _torch()
    M, K = A.shape
    out = out or Operand(fmt, False, M, K, A.device)
    wsb = qgemm_quant_workspace_size(fmt, M, K)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=A.device)
    sa = static_amax.data_ptr() if static_amax is not None else None
    check(qgemm_quantize_act(fmt, A.data_ptr(), M, K, A.stride(0), sa, out.c, ws.data_ptr(), wsb,
                             _stream(stream)), "qgemm_quantize_act")
    out._ws = ws
    return out


def quantize_act_grouped(fmt: int, A, offsets, static_amax=None, stream=None) -> Operand:
    """Activation quantisation of bf16 A [T, K], tokens sorted by expert
    (``offsets``: device int32 [experts + 1]), for run_grouped."""
    torch = _torch()
    T, K = A.shape
    experts = offsets.numel() - 1
    out = Operand(fmt, False, T, K, A.device, sizes=qgemm_grouped_act_bytes(fmt, experts, T, K))
    wsb = qgemm_quant_workspace_size(fmt, T, K)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=A.device)
    sa = static_amax.data_ptr() if static_amax is not None else None
    check(qgemm_quantize_act_grouped(fmt, experts, offsets.data_ptr(), A.data_ptr(), T, K, A.stride(0), sa,
                                     out.c, ws.data_ptr(), wsb, _stream(stream)), "qgemm_quantize_act_grouped")
    out._ws = ws
    return out


def quantize_weight_grouped(fmt: int, W, experts: int, stream=None) -> Operand:
    """Stacked expert weights bf16 [experts * N, K] for run_grouped (NVFP4:
    each expert its own tensor, one tensor scale per expert)."""
    torch = _torch()
    R, K = W.shape
    N = R // experts
    out = Operand(fmt, True, R, K, W.device, n_global=experts)
    wsb = qgemm_quant_workspace_size(fmt, N, K)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=W.device)
    check(qgemm_quantize_weight_grouped(fmt, experts, W.contiguous().data_ptr(), N, K, out.c, ws.data_ptr(), wsb,
                                        _stream(stream)), "qgemm_quantize_weight_grouped")
    out._ws = ws
    return out


def quantize_weight(fmt: int, W, stream=None) -> Operand:
    torch = _torch()
    N, K = W.shape
    out = Operand(fmt, True, N, K, W.device)
    wsb = qgemm_quant_workspace_size(fmt, N, K)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=W.device)
    check(qgemm_quantize_weight(fmt, W.contiguous().data_ptr(), N, K, out.c, ws.data_ptr(), wsb,
                                _stream(stream)), "qgemm_quantize_weight")
    out._ws = ws
    return out


class Workspace:
    """A zeroed run workspace that grows on demand."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = None

    def get(self, nbytes: int):
        torch = _torch()
        if nbytes == 0:
            return None, 0
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        return self.buf.data_ptr(), self.buf.numel()


def run(fmt: int, A: Operand, W: Operand, cfg: qg_config | None = None, out=None,
        out_kind: int = QG_OUT_BF16, workspace: Workspace | None = None, stream=None):
    """y = dequant(A_q) . dequant(W_q)^T through qgemm_run; returns y [M, N]."""
    torch = _torch()
    M, N, K = A.rows, W.rows, A.K
    cfg = cfg or qgemm_default_config(fmt, M, N, K)
    if out is None:
        dt = torch.bfloat16 if out_kind == QG_OUT_BF16 else (torch.int32 if fmt == QG_W8A8_INT8 else torch.float32)
        out = torch.empty(M, N, dtype=dt, device=A.q.device)
    workspace = workspace or Workspace(A.q.device)
    wsp, wsb = workspace.get(qgemm_workspace_size(fmt, M, N, K, cfg))
    check(qgemm_run(fmt, A.c, W.c, M, N, K, cfg, wsp, wsb, out.data_ptr(), out.stride(0), out_kind,
                    _stream(stream)), "qgemm_run")
    return out


def run_fused(fmt: int, A, W: Operand, cfg: qg_config | None = None, out=None,
              out_kind: int = QG_OUT_BF16, workspace: Workspace | None = None, act_scale_out=None,
              stream=None):
    """y = dequant(quant(A)) . dequant(W_q)^T for bf16 A [M, K] through
    qgemm_run_fused_act (activation quantisation inside the GEMM); returns y."""
    torch = _torch()
    M, K = A.shape
    N = W.rows
    cfg = cfg or qgemm_default_config(fmt, M, N, K)
    if out is None:
        dt = torch.bfloat16 if out_kind == QG_OUT_BF16 else (torch.int32 if fmt == QG_W8A8_INT8 else torch.float32)
        out = torch.empty(M, N, dtype=dt, device=A.device)
    workspace = workspace or Workspace(A.device)
    wsp, wsb = workspace.get(qgemm_workspace_size(fmt, M, N, K, cfg))
    sp = act_scale_out.data_ptr() if act_scale_out is not None else None
    check(qgemm_run_fused_act(fmt, A.data_ptr(), A.stride(0), W.c, M, N, K, cfg, wsp, wsb, out.data_ptr(),
                              out.stride(0), out_kind, sp, _stream(stream)), "qgemm_run_fused_act")
    return out


def run_grouped(fmt: int, A: Operand, W: Operand, offsets, N: int, cfg: qg_config | None = None, out=None,
                out_kind: int = QG_OUT_BF16, workspace: Workspace | None = None, stream=None):
    """y = per-expert dequant(A_q) . dequant(W_q[e])^T through qgemm_run_grouped.
    ``offsets``: device int32 [experts + 1] token offsets (tokens sorted by
    expert); W: the experts' weights stacked, W.rows = experts * N."""
    torch = _torch()
    T, K = A.rows, A.K
    experts = offsets.numel() - 1
    cfg = cfg or qgemm_grouped_default_config(fmt, experts, T, N, K)
    if out is None:
        dt = torch.bfloat16 if out_kind == QG_OUT_BF16 else (torch.int32 if fmt == QG_W8A8_INT8 else torch.float32)
        out = torch.empty(T, N, dtype=dt, device=A.q.device)
    workspace = workspace or Workspace(A.q.device)
    wsp, wsb = workspace.get(qgemm_workspace_size(fmt, T, N, K, cfg))
    check(qgemm_run_grouped(fmt, experts, offsets.data_ptr(), A.c, W.c, N, K, cfg, wsp, wsb, out.data_ptr(),
                            out.stride(0), out_kind, _stream(stream)), "qgemm_run_grouped")
    return out


class Linear:
    """A quantized linear layer: weights quantised once, activations per call,
    configuration from a tuned table (or the default), optional CUDA-graph
    replay per token count (``capture(M)``)."""

    def __init__(self, fmt: int, W, table: Table | None = None):
        self.fmt = fmt
        self.N, self.K = W.shape
        self.Wq = quantize_weight(fmt, W)
        self.table = table
        self.ws = Workspace(W.device)
        self._act = {}
        self.graphs = {}

    def config(self, M):
        if self.table is not None:
            return self.table.dispatch(self.fmt, M, self.N, self.K)[0]
        return qgemm_default_config(self.fmt, M, self.N, self.K)

    def __call__(self, A, out=None, stream=None):
        M = A.shape[0]
        act = self._act.get(M)
        if act is None:
            act = self._act[M] = Operand(self.fmt, False, M, self.K, A.device)
        quantize_act(self.fmt, A, out=act, stream=stream)
        return run(self.fmt, act, self.Wq, self.config(M), out=out, workspace=self.ws, stream=stream)


class GraphStep:
    """One captured decode step of a quantized linear layer for a fixed token
    count M: activation quantisation + GEMM replayed as a single CUDA graph
    ("Helion in the vLLM backend", fourth paragraph: shapes up to
    max_helion_size run under CUDA-graph replay).  Write the input into
    ``A`` (bf16 [M, K]), call ``replay()``, read ``Y`` (bf16 [M, N]).
    ``fused=True`` captures the one-launch path (qgemm_run_fused_act).
    ``host_io=True`` adds pinned host buffers ``A_host`` / ``Y_host`` whose
    copies to and from the device are captured in the same graph: a replay
    then moves the step's input in and its result out with no further call
    (synchronize the stream before reading ``Y_host``).  ``A`` / ``Y`` may be
    given: caller-owned contiguous device tensors of those shapes (e.g. views
    of one buffer shared by several steps, so that one copy fills them all)."""

    def __init__(self, layer: "Linear", M: int, W: Operand | None = None, cfg: qg_config | None = None,
                 fused: bool = False, host_io: bool = False, A=None, Y=None):
        torch = _torch()
        self.fused = fused
        self.host_io = host_io
        dev = layer.Wq.q.device
        self.M, self.N, self.K = M, layer.N, layer.K
        self.fmt = layer.fmt
        self.W = W or layer.Wq
        self.cfg = cfg or layer.config(M)
        for t, shape in ((A, (M, self.K)), (Y, (M, self.N))):
            if t is not None and (tuple(t.shape) != shape or t.dtype != torch.bfloat16 or not t.is_contiguous()):
                raise ValueError(f"GraphStep buffers must be contiguous bf16 {shape}")
        self.A = A if A is not None else torch.zeros(M, self.K, dtype=torch.bfloat16, device=dev)
        self.Y = Y if Y is not None else torch.empty(M, self.N, dtype=torch.bfloat16, device=dev)
        self.act = Operand(self.fmt, False, M, self.K, dev)
        self.ws = Workspace(dev)
        self.ws.get(qgemm_workspace_size(self.fmt, M, self.N, self.K, self.cfg))
        self.qws = torch.zeros(max(qgemm_quant_workspace_size(self.fmt, M, self.K), 16), dtype=torch.uint8,
                               device=dev)
        if host_io:
            self.A_host = torch.zeros(M, self.K, dtype=torch.bfloat16, pin_memory=True)
            self.Y_host = torch.empty(M, self.N, dtype=torch.bfloat16, pin_memory=True)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self._launch()                     # warm-up: configures kernels before capture
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._body()

    def _body(self):
        """The captured work: [input copy in], quantisation + GEMM, [result copy out]."""
        if self.host_io:
            self.A.copy_(self.A_host, non_blocking=True)
        self._launch()
        if self.host_io:
            self.Y_host.copy_(self.Y, non_blocking=True)

    def _launch(self):
        st = _stream(None)
        if self.fused:
            wsp, wsb = self.ws.get(qgemm_workspace_size(self.fmt, self.M, self.N, self.K, self.cfg))
            check(qgemm_run_fused_act(self.fmt, self.A.data_ptr(), self.K, self.W.c, self.M, self.N, self.K,
                                      self.cfg, wsp, wsb, self.Y.data_ptr(), self.N, QG_OUT_BF16, None, st),
                  "qgemm_run_fused_act")
            return
        check(qgemm_quantize_act(self.fmt, self.A.data_ptr(), self.M, self.K, self.K, None, self.act.c,
                                 self.qws.data_ptr(), self.qws.numel(), st), "qgemm_quantize_act")
        wsp, wsb = self.ws.get(qgemm_workspace_size(self.fmt, self.M, self.N, self.K, self.cfg))
        check(qgemm_run(self.fmt, self.act.c, self.W.c, self.M, self.N, self.K, self.cfg, wsp, wsb,
                        self.Y.data_ptr(), self.N, QG_OUT_BF16, st), "qgemm_run")

    def replay(self):
        self.graph.replay()
        return self.Y_host if self.host_io else self.Y


def capture_steps(steps) -> "torch.cuda.CUDAGraph":
    """One CUDA graph that runs the given captured steps back to back (as a
    decode forward runs its layers), so that each step's kernels overlap the
    previous step's tail through programmatic dependent launch instead of
    waiting for a graph launch.  The steps keep their own buffers; replay
    the returned graph instead of the steps one by one."""
    torch = _torch()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for st in steps:
            st._body()
    return g


def _linear_capture(self, M: int, W: Operand | None = None, cfg: qg_config | None = None,
                    fused: bool = False, host_io: bool = False) -> GraphStep:
    g = GraphStep(self, M, W=W, cfg=cfg, fused=fused, host_io=host_io)
    self.graphs[M] = g
    return g


Linear.capture = _linear_capture

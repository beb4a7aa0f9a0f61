"""Thin ctypes binding of liblyc.so (declared in include/lyc.h).

Every step of the decode path runs in the library's CUDA kernels; this module
only marshals arguments.  The functions ``lyc_*`` mirror the C entry points
one to one (raw pointers and sizes); ``Lyc`` is a convenience wrapper that
takes torch tensors and passes their device pointers.  Importing this module
on a machine where the library is not built raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblyc.so")

LYC_OK = 0
LYC_ERR_INVALID_ARG = -1
LYC_ERR_UNSUPPORTED = -2
LYC_ERR_OOM = -3
LYC_ERR_CUDA = -4
LYC_ERR_BAD_INDEX = -5
LYC_ERR_TIMEOUT = -6
LYC_ERR_SCRATCH_LIMIT = -7

LYC_NOALLOC_MAX_SETS = 256
LYC_NOALLOC_MAX_CTAS = 32

LYC_BF16 = 0
LYC_FP32 = 1
LYC_SELECT_PER_QHEAD = 0
LYC_SELECT_KVGROUP_MEAN = 1

LYC_CFG_TMA_GATHER = 0x1
LYC_CFG_TCGEN05 = 0x2

LYC_STEP_S_IN = 0x1
LYC_STEP_NO_GRAPH = 0x2
LYC_STEP_VALIDATE_S = 0x4

LYC_TIMING_OFF = 0
LYC_TIMING_ON = 1

LYC_RULE_TOPK = 0
LYC_RULE_RATIO = 1
LYC_RULE_BLOCK_TOPK = 2
LYC_RULE_TOPP = 3
LYC_RULE_THRESHOLD = 4

LYC_TOPK_FIXED = 0
LYC_TOPK_RULES = 1

EXPORTED = ["lyc_create", "lyc_decode_step", "lyc_decode_step_host", "lyc_decode_step_batch",
            "lyc_sync_status",
            "lyc_set_s_trace", "lyc_step_bytes", "lyc_step_launches", "lyc_topk_f32", "lyc_topk_f32_ex",
            "lyc_set_timing",
            "lyc_kernel_times", "lyc_set_timeline", "lyc_status_string", "lyc_last_error",
            "lyc_destroy", "lyc_sparse_attention_noalloc", "lyc_set_selection", "lyc_cache_correction"]


class lyc_config(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int), ("batch", ctypes.c_int),
                ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("max_ctx", ctypes.c_int64),
                ("max_k", ctypes.c_int), ("dtype", ctypes.c_int),
                ("select_mode", ctypes.c_int), ("device", ctypes.c_int),
                ("flags", ctypes.c_uint32)]


class lyc_kv_cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("n", ctypes.c_int64),
                ("s_layer", ctypes.c_int64), ("s_batch", ctypes.c_int64),
                ("s_head", ctypes.c_int64), ("s_token", ctypes.c_int64)]


class lyc_kv_batch(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("n", ctypes.c_void_p),
                ("s_layer", ctypes.c_int64), ("s_batch", ctypes.c_int64),
                ("s_head", ctypes.c_int64), ("s_token", ctypes.c_int64),
                ("s_page", ctypes.c_int64), ("block_table", ctypes.c_void_p),
                ("page_rows", ctypes.c_int32), ("max_blocks", ctypes.c_int32),
                ("num_pages", ctypes.c_int64), ("k_new", ctypes.c_void_p),
                ("v_new", ctypes.c_void_p)]


class lyc_selection(ctypes.Structure):
    _fields_ = [("rule", ctypes.c_int32), ("block", ctypes.c_int32),
                ("ratio_num", ctypes.c_int64), ("ratio_den", ctypes.c_int64),
                ("p", ctypes.c_double), ("tau", ctypes.c_double)]


class lyc_kernel_time(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("layer", ctypes.c_int), ("ms", ctypes.c_float)]


class LycError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str = ""):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code}) {detail}".rstrip())


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblyc.so.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m hybrid_head_sparse_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    L.lyc_create.argtypes = [ctypes.POINTER(lyc_config), ctypes.POINTER(P)]
    L.lyc_decode_step.argtypes = [P, P, ctypes.POINTER(lyc_kv_cache), P, I, P, P, P, ctypes.c_uint32]
    L.lyc_decode_step_host.argtypes = [P, P, ctypes.POINTER(lyc_kv_cache), P, I, P, P, P,
                                       ctypes.c_uint32]
    L.lyc_decode_step_batch.argtypes = [P, P, ctypes.POINTER(lyc_kv_batch), P, I, P, P, P,
                                        ctypes.c_uint32]
    L.lyc_sync_status.argtypes = [P]
    L.lyc_set_selection.argtypes = [P, ctypes.POINTER(lyc_selection)]
    L.lyc_cache_correction.argtypes = [P, P, ctypes.POINTER(lyc_kv_cache), I, P, P, P, P]
    L.lyc_set_s_trace.argtypes = [P, P]
    L.lyc_step_bytes.argtypes = [ctypes.POINTER(lyc_config), P, ctypes.c_int64, I, I,
                                 ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64)]
    L.lyc_step_launches.argtypes = [P, ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(I)]
    L.lyc_topk_f32.argtypes = [P, P, ctypes.c_int64, I, P, P]
    L.lyc_topk_f32_ex.argtypes = [P, P, ctypes.c_int64, I, P, I, I, P]
    L.lyc_set_timing.argtypes = [P, I]
    L.lyc_set_timeline.argtypes = [P, P, I]
    L.lyc_kernel_times.argtypes = [P, ctypes.POINTER(lyc_kernel_time), I, ctypes.POINTER(I)]
    L.lyc_status_string.argtypes = [I]
    L.lyc_status_string.restype = ctypes.c_char_p
    L.lyc_last_error.argtypes = [P]
    L.lyc_last_error.restype = ctypes.c_char_p
    L.lyc_destroy.argtypes = [P]
    L.lyc_destroy.restype = None
    L.lyc_sparse_attention_noalloc.argtypes = [P, ctypes.POINTER(lyc_kv_cache), I, I, I, I, P, I,
                                               P, P, P]
    for name in EXPORTED:
        if name not in ("lyc_status_string", "lyc_last_error", "lyc_destroy"):
            getattr(L, name).restype = I
    _lib = L
    return L


# ------------------------------------------------------------ C-named functions


def lyc_create(cfg: lyc_config) -> int:
    ctx = ctypes.c_void_p()
    rc = load().lyc_create(ctypes.byref(cfg), ctypes.byref(ctx))
    if rc != LYC_OK:
        raise LycError(rc, "lyc_create")
    return ctx.value


def lyc_decode_step(ctx, q, kv: lyc_kv_cache, role_mask, k, out, S, stream, flags) -> int:
    return load().lyc_decode_step(ctx, q, ctypes.byref(kv), role_mask, k, out, S, stream, flags)


def lyc_decode_step_host(ctx, q, kv: lyc_kv_cache, role_mask, k, out, S, stream, flags) -> int:
    return load().lyc_decode_step_host(ctx, q, ctypes.byref(kv), role_mask, k, out, S, stream,
                                       flags)


def lyc_decode_step_batch(ctx, q, kv: lyc_kv_batch, role_mask, k, out, S, stream, flags) -> int:
    return load().lyc_decode_step_batch(ctx, q, ctypes.byref(kv), role_mask, k, out, S, stream,
                                        flags)


def lyc_sparse_attention_noalloc(q, kv: lyc_kv_cache, batch, num_q_heads, num_kv_heads,
                                 head_dim, S, k, out, status, stream) -> int:
    """The allocation-free sparse attention of one layer (include/lyc.h).
    Pointers are ints (device addresses); status may be None."""
    return load().lyc_sparse_attention_noalloc(q, ctypes.byref(kv), batch, num_q_heads,
                                               num_kv_heads, head_dim, S, k, out, status,
                                               stream)


def lyc_sync_status(ctx) -> int:
    return load().lyc_sync_status(ctx)


def lyc_set_selection(ctx, sel: lyc_selection | None) -> int:
    return load().lyc_set_selection(ctx, None if sel is None else ctypes.byref(sel))


def lyc_cache_correction(ctx, q, kv: lyc_kv_cache, T, k_new, v_new, out, stream) -> int:
    return load().lyc_cache_correction(ctx, q, ctypes.byref(kv), T, k_new, v_new, out, stream)


def lyc_set_s_trace(ctx, trace) -> int:
    return load().lyc_set_s_trace(ctx, trace)


def lyc_step_bytes(cfg: lyc_config, role_mask: np.ndarray, n: int, k: int, s_in: bool = False):
    a = ctypes.c_uint64()
    d = ctypes.c_uint64()
    role_mask = np.ascontiguousarray(role_mask, dtype=np.uint8)
    rc = load().lyc_step_bytes(ctypes.byref(cfg), role_mask.ctypes.data, n, k, int(s_in),
                               ctypes.byref(a), ctypes.byref(d))
    if rc != LYC_OK:
        raise LycError(rc, "lyc_step_bytes")
    return a.value, d.value


def lyc_topk_f32(ctx, keys, n, k, S, stream) -> int:
    return load().lyc_topk_f32(ctx, keys, n, k, S, stream)


def lyc_topk_f32_ex(ctx, keys, n, k, S, cluster, variant, stream) -> int:
    return load().lyc_topk_f32_ex(ctx, keys, n, k, S, cluster, variant, stream)


def lyc_set_timing(ctx, mode: int) -> int:
    return load().lyc_set_timing(ctx, mode)


def lyc_kernel_times(ctx, cap: int = 1 << 16):
    arr = (lyc_kernel_time * cap)()
    cnt = ctypes.c_int()
    rc = load().lyc_kernel_times(ctx, arr, cap, ctypes.byref(cnt))
    if rc != LYC_OK:
        raise LycError(rc, "lyc_kernel_times")
    return [(arr[i].kind, arr[i].layer, arr[i].ms) for i in range(cnt.value)]


def lyc_set_timeline(ctx, buf, cap: int) -> int:
    return load().lyc_set_timeline(ctx, buf, cap)


def lyc_status_string(code: int) -> str:
    return load().lyc_status_string(code).decode()


def status_string(code: int) -> str:
    try:
        return lyc_status_string(code)
    except Exception:  # library missing: still format the error
        return "status"


def lyc_last_error(ctx) -> str:
    return load().lyc_last_error(ctx).decode()


def lyc_destroy(ctx) -> None:
    load().lyc_destroy(ctx)


# ------------------------------------------------------------ torch wrapper


def _dtype_code(dtype) -> int:
    import torch
    if dtype in ("bf16", torch.bfloat16, LYC_BF16):
        return LYC_BF16
    if dtype in ("fp32", torch.float32, LYC_FP32):
        return LYC_FP32
    raise ValueError(f"unsupported dtype {dtype}")


def _mode_code(mode) -> int:
    if mode in ("per_qhead", LYC_SELECT_PER_QHEAD):
        return LYC_SELECT_PER_QHEAD
    if mode in ("kvgroup_mean", LYC_SELECT_KVGROUP_MEAN):
        return LYC_SELECT_KVGROUP_MEAN
    raise ValueError(f"unknown select mode {mode}")


def _stream_ptr(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


class Lyc:
    """One library context.  Tensors are passed by device pointer."""

    def __init__(self, L, B, Hq, Hkv, d, max_ctx, max_k, dtype="bf16", select_mode="per_qhead",
                 device=0, flags=0):
        self.cfg = lyc_config(L, B, Hq, Hkv, d, max_ctx, max_k, _dtype_code(dtype),
                              _mode_code(select_mode), device, flags)
        self.ctx = lyc_create(self.cfg)
        self.Hs = Hkv if self.cfg.select_mode == LYC_SELECT_KVGROUP_MEAN else Hq
        self._trace = None

    def close(self):
        if self.ctx:
            lyc_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, rc, where):
        if rc != LYC_OK:
            raise LycError(rc, where, lyc_last_error(self.ctx))

    @staticmethod
    def kv_cache(K, V, n) -> lyc_kv_cache:
        """Describe [L][B][Hkv][rows][d]-strided torch tensors K, V."""
        assert K.stride() == V.stride() and K.shape == V.shape and K.stride(-1) == 1
        s = K.stride()
        return lyc_kv_cache(K.data_ptr(), V.data_ptr(), n, s[0], s[1], s[2], s[3])

    def decode_step(self, q, K, V, n, role_mask, k, out, S, stream=None, s_in=False,
                    no_graph=False, validate_s=False):
        role = np.ascontiguousarray(role_mask, dtype=np.uint8)
        self._role = role  # keep alive while the call runs
        flags = ((LYC_STEP_S_IN if s_in else 0) | (LYC_STEP_NO_GRAPH if no_graph else 0)
                 | (LYC_STEP_VALIDATE_S if validate_s else 0))
        kv = self.kv_cache(K, V, n)
        rc = lyc_decode_step(self.ctx, q.data_ptr(), kv, role.ctypes.data, k, out.data_ptr(),
                             S.data_ptr(), _stream_ptr(stream), flags)
        self._check(rc, "lyc_decode_step")

    def decode_step_batch(self, q, K, V, n, role_mask, k, out, S, stream=None, s_in=False,
                          validate_s=False, k_new=None, v_new=None, block_table=None,
                          page_rows=0, strides=None):
        """The serving form: n is a sequence of B row counts.  Contiguous cache:
        K, V are [L][B][Hkv][rows][d]-strided tensors.  Paged cache: K, V are
        [L][pages][page_rows][Hkv][d] tensors and block_table a device int32
        [B][max_blocks] tensor.  k_new/v_new: [L][B][Hkv][d] rows appended at
        n[b]-1 before attention, or None.  strides: optional (s_layer, s_batch,
        s_head, s_token, s_page) override in elements."""
        role = np.ascontiguousarray(role_mask, dtype=np.uint8)
        nn = np.ascontiguousarray(np.asarray(n, dtype=np.int64))
        self._role, self._n = role, nn  # keep alive while the call runs
        flags = (LYC_STEP_S_IN if s_in else 0) | (LYC_STEP_VALIDATE_S if validate_s else 0)
        assert K.stride() == V.stride() and K.shape == V.shape and K.stride(-1) == 1
        st = K.stride()
        if strides is not None:
            s_layer, s_batch, s_head, s_token, s_page = strides
        elif block_table is None:
            s_layer, s_batch, s_head, s_token, s_page = st[0], st[1], st[2], st[3], 0
        else:
            s_layer, s_batch, s_head, s_token, s_page = st[0], 0, st[3], st[2], st[1]
        kv = lyc_kv_batch(K.data_ptr(), V.data_ptr(), nn.ctypes.data, s_layer, s_batch, s_head,
                          s_token, s_page,
                          None if block_table is None else block_table.data_ptr(),
                          int(page_rows), 0 if block_table is None else int(block_table.shape[1]),
                          0 if block_table is None else int(K.shape[1]),
                          None if k_new is None else k_new.data_ptr(),
                          None if v_new is None else v_new.data_ptr())
        rc = lyc_decode_step_batch(self.ctx, q.data_ptr(), kv, role.ctypes.data, k,
                                   out.data_ptr(), S.data_ptr(), _stream_ptr(stream), flags)
        self._check(rc, "lyc_decode_step_batch")

    def decode_step_host(self, q_host, K, V, n, role_mask, k, out_host, S_host, stream=None,
                         s_in=False):
        role = np.ascontiguousarray(role_mask, dtype=np.uint8)
        self._role = role
        kv = self.kv_cache(K, V, n)
        flags = LYC_STEP_S_IN if s_in else 0
        rc = lyc_decode_step_host(self.ctx, q_host.data_ptr(), kv, role.ctypes.data, k,
                                  out_host.data_ptr(), S_host.data_ptr(), _stream_ptr(stream), flags)
        self._check(rc, "lyc_decode_step_host")

    def sync_status(self) -> int:
        return lyc_sync_status(self.ctx)

    def set_selection(self, rule=LYC_RULE_TOPK, block=64, ratio=(1, 2), p=0.9, tau=1e-3):
        """The selection rule of the steps that follow (lyc_set_selection)."""
        sel = lyc_selection(int(rule), int(block), int(ratio[0]), int(ratio[1]), float(p),
                            float(tau))
        self._check(lyc_set_selection(self.ctx, sel), "lyc_set_selection")

    def cache_correction(self, q, K, V, n, out, k_new=None, v_new=None, stream=None):
        """Cache Correction's dense causal attention: q [L][B][Hq][T][d] bf16,
        out [L][B][Hq][T][d] fp32, K/V as in decode_step (n counts the T
        positions); k_new/v_new [L][B][Hkv][T][d] written at rows n-T..n-1 first."""
        kv = self.kv_cache(K, V, n)
        rc = lyc_cache_correction(self.ctx, q.data_ptr(), kv, int(q.shape[3]),
                                  None if k_new is None else k_new.data_ptr(),
                                  None if v_new is None else v_new.data_ptr(), out.data_ptr(),
                                  _stream_ptr(stream))
        self._check(rc, "lyc_cache_correction")

    def set_trace(self, trace):
        self._trace = trace
        self._check(lyc_set_s_trace(self.ctx, None if trace is None else trace.data_ptr()),
                    "lyc_set_s_trace")

    def set_timing(self, on: bool):
        self._check(lyc_set_timing(self.ctx, LYC_TIMING_ON if on else LYC_TIMING_OFF),
                    "lyc_set_timing")

    def kernel_times(self):
        return lyc_kernel_times(self.ctx)

    def set_timeline(self, buf, cap: int):
        """buf: device int64 tensor of 1 + 3*cap words (word 0 zeroed), or None."""
        self._timeline = buf
        self._check(lyc_set_timeline(self.ctx, None if buf is None else buf.data_ptr(), cap),
                    "lyc_set_timeline")

    def topk_f32(self, keys, n, k, S, stream=None, cluster=None, variant=LYC_TOPK_FIXED):
        """The selection kernel alone; cluster (4, 8, 16) and variant choose its
        launch form (lyc_topk_f32_ex), None the context's default."""
        if cluster is None and variant == LYC_TOPK_FIXED:
            self._check(lyc_topk_f32(self.ctx, keys.data_ptr(), n, k, S.data_ptr(),
                                     _stream_ptr(stream)), "lyc_topk_f32")
        else:
            self._check(lyc_topk_f32_ex(self.ctx, keys.data_ptr(), n, k, S.data_ptr(),
                                        cluster or 0, variant, _stream_ptr(stream)),
                        "lyc_topk_f32_ex")

    def step_bytes(self, role_mask, n, k, s_in=False):
        return lyc_step_bytes(self.cfg, role_mask, n, k, s_in)

    def step_launches(self):
        """(attention, selection, other) kernel launches of the most recent step."""
        a, t, o = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        self._check(load().lyc_step_launches(self.ctx, ctypes.byref(a), ctypes.byref(t), ctypes.byref(o)),
                    "lyc_step_launches")
        return a.value, t.value, o.value

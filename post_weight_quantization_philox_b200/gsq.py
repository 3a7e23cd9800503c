"""Thin ctypes binding of libgsq (the C ABI in include/gsq.h).

Argument marshalling only: every step of the GSQ reconstruction path runs in
the library's CUDA kernels.  PyTorch supplies device memory and the current
stream; numpy arrays are accepted as host buffers.  There is no fallback: if
the shared library is missing or fails to load, importing raises.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgsq.so")

GSQ_GRID_2BIT, GSQ_GRID_TERNARY, GSQ_GRID_3BIT_LOCAL = 0, 1, 2
GSQ_F32, GSQ_BF16 = 0, 1
GSQ_OK = 0
GSQ_ERR_INVALID_ARG, GSQ_ERR_CUDA, GSQ_ERR_OOM = -1, -2, -3
GSQ_ERR_NONFINITE, GSQ_ERR_STATE, GSQ_ERR_UNSUPPORTED, GSQ_ERR_TIMEOUT = -4, -5, -6, -7
GSQ_RECON_HARD, GSQ_RECON_SOFT = 0, 1
GSQ_NOALLOC_MAX_COORDS = 65536
(GSQ_DBG_LOGITS, GSQ_DBG_MOM, GSQ_DBG_SCALES, GSQ_DBG_SMOM, GSQ_DBG_I0,
 GSQ_DBG_WHAT, GSQ_DBG_WSOFT32, GSQ_DBG_DW, GSQ_DBG_DYT, GSQ_DBG_YREFT,
 GSQ_DBG_DL, GSQ_DBG_DS) = range(12)
GSQ_MLP_STAGE = 3
GSQ_ATTN_STAGE = 2
(GSQ_ATTN_DBG_P, GSQ_ATTN_DBG_PT, GSQ_ATTN_DBG_VT, GSQ_ATTN_DBG_O, GSQ_ATTN_DBG_DPT,
 GSQ_ATTN_DBG_DV, GSQ_ATTN_DBG_RT) = range(7)
(GSQ_MLP_DBG_AT, GSQ_MLP_DBG_BT, GSQ_MLP_DBG_HT, GSQ_MLP_DBG_DPT, GSQ_MLP_DBG_DHT,
 GSQ_MLP_DBG_DAT, GSQ_MLP_DBG_DBT, GSQ_MLP_DBG_RT) = range(8)

NUM_LOGITS = {GSQ_GRID_2BIT: 4, GSQ_GRID_TERNARY: 4, GSQ_GRID_3BIT_LOCAL: 5}

# every symbol include/gsq.h declares (checked by the CPU tests)
EXPORTS = [
    "gsq_init", "gsq_step", "gsq_run", "gsq_last_loss", "gsq_loss_history",
    "gsq_packed_bytes", "gsq_harden_pack", "gsq_recon_error",
    "gsq_state_bytes", "gsq_export_state", "gsq_import_state", "gsq_get_step",
    "gsq_destroy", "gsq_error_string", "gsq_set_timing", "gsq_phase_times",
    "gsq_debug_uniforms", "gsq_debug_noise_log2", "gsq_debug_get", "gsq_debug_set", "gsq_debug_noise",
    "gsq_debug_soft_weight", "gsq_debug_forward", "gsq_debug_weight_grad",
    "gsq_debug_backward", "gsq_gemm_bf16_abt", "gsq_gemm_bf16_abt_sub", "gsq_uniforms_noalloc",
    "gsq_scale_step", "gsq_scale_run", "gsq_debug_scale_backward",
    "gsq_gptq", "gsq_release_cached_memory", "gsq_set_cached_memory_limit", "gsq_init_gptq", "gsq_init_bf16_state",
    "gsq_init_rows", "gsq_step_next", "gsq_mlp_set_timing", "gsq_mlp_phase_times", "gsq_attn_set_timing",
    "gsq_attn_phase_times", "gsq_debug_stall_probe", "gsq_debug_fail_alloc", "gsq_debug_pool_used",
    "gsq_mlp_init", "gsq_mlp_step", "gsq_mlp_run", "gsq_mlp_last_loss",
    "gsq_mlp_recon_error", "gsq_mlp_harden_pack", "gsq_mlp_debug_get",
    "gsq_mlp_debug_set", "gsq_mlp_get_step", "gsq_mlp_destroy",
    "gsq_attn_init", "gsq_attn_step", "gsq_attn_run", "gsq_attn_last_loss",
    "gsq_attn_recon_error", "gsq_attn_harden_pack", "gsq_attn_debug_get",
    "gsq_attn_debug_set", "gsq_attn_get_step", "gsq_attn_destroy",
    "gsq_dequant", "gsq_block_forward", "gsq_block_quantize",
    "gsq_kq_block_bytes", "gsq_kq_init", "gsq_kq_step", "gsq_kq_run", "gsq_kq_last_loss",
    "gsq_kq_export", "gsq_kq_start_blocks", "gsq_kq_recon_error", "gsq_kq_dequant",
    "gsq_kq_debug_get", "gsq_kq_debug_set", "gsq_kq_debug_soft_weight",
    "gsq_kq_debug_backward", "gsq_kq_debug_noise", "gsq_kq_get_step", "gsq_kq_destroy",
]


class GSQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {error_string(status)} ({status})")


_i32, _i64, _u32, _u64 = C.c_int, C.c_int64, C.c_uint32, C.c_uint64
_f32, _p, _sz = C.c_float, C.c_void_p, C.c_size_t
_pp = C.POINTER(C.c_void_p)

_SIGS = {
    "gsq_init": [_pp, _p, _i32, _p, _i32, _i64, _i64, _i64, _i32, _i32, _p, _u64, _p],
    "gsq_debug_stall_probe": [_p],
    "gsq_mlp_set_timing": [_p, _i32],
    "gsq_mlp_phase_times": [_p, _p, _p],
    "gsq_attn_set_timing": [_p, _i32],
    "gsq_attn_phase_times": [_p, _p, _p],
    "gsq_debug_fail_alloc": [_i64],
    "gsq_debug_pool_used": [_i32, C.POINTER(_u64)],
    "gsq_init_rows": [_pp, _p, _i32, _p, _i32, _i64, _i64, _i64, _i32, _i32, _p, _u64, _i64,
                      _i32, _p],
    "gsq_step": [_p, _f32, _f32, _f32, _f32],
    "gsq_step_next": [_p, _f32, _f32, _f32, _f32, _f32],
    "gsq_run": [_p, _p, _i64, _f32, _f32, _f32],
    "gsq_last_loss": [_p, C.POINTER(C.c_double)],
    "gsq_loss_history": [_p, _u64, _i64, _p],
    "gsq_packed_bytes": [_i32, _i64, _i64, C.POINTER(_sz)],
    "gsq_harden_pack": [_p, _p, _p, _p],
    "gsq_recon_error": [_p, _i32, _f32, C.POINTER(C.c_double), C.POINTER(C.c_double)],
    "gsq_state_bytes": [_p, C.POINTER(_sz)],
    "gsq_export_state": [_p, _p, _sz],
    "gsq_import_state": [_p, _p, _sz],
    "gsq_get_step": [_p, C.POINTER(_u64)],
    "gsq_destroy": [_p],
    "gsq_error_string": [_i32],
    "gsq_set_timing": [_p, _i32],
    "gsq_phase_times": [_p, _p, _p],
    "gsq_debug_uniforms": [_p, _u32, _u64, _i64, _p],
    "gsq_debug_noise_log2": [_p, _u32, _i64, _p],
    "gsq_debug_get": [_p, _i32, _p, _sz],
    "gsq_debug_set": [_p, _i32, _p, _sz],
    "gsq_debug_noise": [_p, _i32],
    "gsq_debug_soft_weight": [_p, _f32],
    "gsq_debug_forward": [_p, C.POINTER(C.c_double)],
    "gsq_debug_weight_grad": [_p],
    "gsq_debug_backward": [_p, _f32, _f32, _f32, _f32],
    "gsq_scale_step": [_p, _f32, _f32, _f32],
    "gsq_gptq": [_p, _i32, _p, _i32, _i64, _i64, _i64, _i32, _i32, _f32, _p, _p, _p],
    "gsq_release_cached_memory": [],
    "gsq_set_cached_memory_limit": [_u64],
    "gsq_init_gptq": [_pp, _p, _i32, _p, _i32, _i64, _i64, _i64, _i32, _i32, _f32, _u64, _p],
    "gsq_init_bf16_state": [_pp, _p, _i32, _p, _i32, _i64, _i64, _i64, _i32, _i32, _p, _u64,
                            _p],
    "gsq_scale_run": [_p, _i64, _f32, _f32, _f32],
    "gsq_debug_scale_backward": [_p, _f32, _f32, _f32],
    "gsq_gemm_bf16_abt": [_p, _p, _p, _i64, _i64, _i64, _p],
    "gsq_gemm_bf16_abt_sub": [_p, _p, _p, _i64, _i64, _i64, _p],
    "gsq_uniforms_noalloc": [_i32, _u64, _u32, _u64, _i64, _p, _p],
    "gsq_mlp_init": [_pp, _p, _i32, _p, _i32, _p, _p, _p, _i32, _i64, _i64, _i64,
                     _i32, _i32, _u64, _p],
    "gsq_mlp_step": [_p, _f32, _f32, _f32, _f32],
    "gsq_mlp_run": [_p, _p, _i64, _f32, _f32, _f32],
    "gsq_mlp_last_loss": [_p, C.POINTER(C.c_double)],
    "gsq_mlp_recon_error": [_p, _i32, _f32, C.POINTER(C.c_double), C.POINTER(C.c_double)],
    "gsq_mlp_harden_pack": [_p, _i32, _p, _p, _p],
    "gsq_mlp_debug_get": [_p, _i32, _i32, _p, _sz],
    "gsq_mlp_debug_set": [_p, _i32, _i32, _p, _sz],
    "gsq_mlp_get_step": [_p, C.POINTER(_u64)],
    "gsq_mlp_destroy": [_p],
    "gsq_attn_init": [_pp, _p, _i32, _p, _i32, _p, _p, _p, _p, _i32, _i64, _i64, _i64,
                      _i64, _i64, C.c_double, _i32, _i32, _u64, _p],
    "gsq_attn_step": [_p, _f32, _f32, _f32, _f32],
    "gsq_attn_run": [_p, _p, _i64, _f32, _f32, _f32],
    "gsq_attn_last_loss": [_p, C.POINTER(C.c_double)],
    "gsq_attn_recon_error": [_p, _i32, _f32, C.POINTER(C.c_double), C.POINTER(C.c_double)],
    "gsq_attn_harden_pack": [_p, _i32, _p, _p, _p],
    "gsq_attn_debug_get": [_p, _i32, _i32, _p, _sz],
    "gsq_attn_debug_set": [_p, _i32, _i32, _p, _sz],
    "gsq_attn_get_step": [_p, C.POINTER(_u64)],
    "gsq_attn_destroy": [_p],
    "gsq_dequant": [_i32, _p, _p, _i64, _i64, _i32, _p, _p],
    "gsq_kq_block_bytes": [_i32, _i64, _i64, C.POINTER(_sz)],
    "gsq_kq_init": [_pp, _p, _i32, _p, _i32, _i64, _i64, _i64, _i32, _p, _u64, _p],
    "gsq_kq_step": [_p, _f32, _f32, _f32, _f32],
    "gsq_kq_run": [_p, _p, _i64, _f32, _f32, _f32],
    "gsq_kq_last_loss": [_p, C.POINTER(C.c_double)],
    "gsq_kq_export": [_p, _p],
    "gsq_kq_start_blocks": [_p, _p],
    "gsq_kq_recon_error": [_p, _i32, C.POINTER(C.c_double), C.POINTER(C.c_double)],
    "gsq_kq_dequant": [_i32, _p, _i64, _i64, _p, _p],
    "gsq_kq_debug_get": [_p, _i32, _p, _sz],
    "gsq_kq_debug_set": [_p, _i32, _p, _sz],
    "gsq_kq_debug_soft_weight": [_p, _f32],
    "gsq_kq_debug_backward": [_p, _f32, _f32, _f32, _f32],
    "gsq_kq_debug_noise": [_p, _i32],
    "gsq_kq_get_step": [_p, C.POINTER(_u64)],
    "gsq_kq_destroy": [_p],
    "gsq_block_forward": [_p, _p, _i64, _i64, _i64, _i64, _i64, _i64, C.c_double, _f32,
                          _p, _p, _p],
    "gsq_block_quantize": [_p, _p, _i64, _i64, _i64, _i64, _i64, _i64, C.c_double, _f32,
                           _i32, _i32, _p, _p, _f32, _f32, _f32, _u64, _p, _p, _p, _p, _p,
                           _p],
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libgsq.so not found at {LIB_PATH}; build it with "
            "`python -m post_weight_quantization_philox_b200.build`")
    lib = C.CDLL(LIB_PATH)
    for name, args in _SIGS.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = C.c_char_p if name == "gsq_error_string" else C.c_int
    return lib


_lib = _load()


def lib():
    return _lib


def error_string(status: int) -> str:
    return _lib.gsq_error_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != GSQ_OK:
        raise GSQError(status, where)


def _ptr_dtype(a):
    """(pointer, GSQ dtype, keep-alive object) of a numpy array or torch tensor."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            if not a.is_contiguous():
                a = a.contiguous()
            if a.dtype == torch.float32:
                return a.data_ptr(), GSQ_F32, a
            if a.dtype == torch.bfloat16:
                return a.data_ptr(), GSQ_BF16, a
            raise TypeError(f"unsupported tensor dtype {a.dtype}")
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a.ctypes.data, GSQ_F32, a


def _stream_ptr(stream):
    if stream is not None:
        return int(getattr(stream, "cuda_stream", stream))
    import torch
    if torch.cuda.is_available():
        return torch.cuda.current_stream().cuda_stream
    return None


def _host_ptr(a):
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.data_ptr()
    except ImportError:  # pragma: no cover
        pass
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# --------------------------------------------------------------- C-ABI names

def gsq_packed_bytes(grid_mode: int, N: int, K: int) -> int:
    b = C.c_size_t()
    _check(_lib.gsq_packed_bytes(grid_mode, N, K, C.byref(b)), "gsq_packed_bytes")
    return b.value


def gsq_init(W, X, group: int = 128, grid_mode: int = GSQ_GRID_2BIT,
             init_idx=None, seed: int = 0, stream=None, state_bf16: bool = False,
             row0=None) -> "Layer":
    """W (N x K) and X (T x K): numpy fp32 or torch fp32/bf16, host or device.
    state_bf16 selects gsq_init_bf16_state (bf16 logits and momenta).  With
    row0, W holds the rows [row0, row0 + N) of a larger layer
    (gsq_init_rows: the noise is keyed by the global coordinate)."""
    wp, wdt, wk = _ptr_dtype(W)
    xp, xdt, xk = _ptr_dtype(X)
    N, K = int(W.shape[0]), int(W.shape[1])
    T = int(X.shape[0])
    if int(X.shape[1]) != K:
        raise ValueError("X and W disagree on K")
    ip, ik = None, None
    if init_idx is not None:
        try:
            import torch
            if isinstance(init_idx, torch.Tensor):
                ik = init_idx.to(torch.int8).contiguous()
                ip = ik.data_ptr()
        except ImportError:  # pragma: no cover
            pass
        if ip is None:
            ik = np.ascontiguousarray(init_idx, dtype=np.int8)
            ip = ik.ctypes.data
    ctx = C.c_void_p()
    st = _stream_ptr(stream)
    if row0 is not None:
        _check(_lib.gsq_init_rows(C.byref(ctx), wp, wdt, xp, xdt, N, K, T, group, grid_mode,
                                  ip, seed & 0xFFFFFFFFFFFFFFFF, int(row0), int(bool(state_bf16)),
                                  st), "gsq_init_rows")
    else:
        fn = _lib.gsq_init_bf16_state if state_bf16 else _lib.gsq_init
        _check(fn(C.byref(ctx), wp, wdt, xp, xdt, N, K, T, group,
                  grid_mode, ip, seed & 0xFFFFFFFFFFFFFFFF, st),
               "gsq_init_bf16_state" if state_bf16 else "gsq_init")
    del wk, xk, ik
    return Layer(ctx, grid_mode, N, K, T, group, state16=state_bf16)


def gsq_gptq(W, X, group: int = 128, grid_mode: int = GSQ_GRID_2BIT, damp: float = 0.01,
             stream=None, levels=None, scales=None):
    """GPTQ initial levels (N x K int8) and group scales (N x K/group fp32).
    W, X as for gsq_init.  Returned as host numpy arrays, or written into
    `levels` / `scales` (contiguous int8 / fp32 torch tensors or numpy arrays
    of those shapes, host or device) when both are given."""
    wp, wdt, wk = _ptr_dtype(W)
    xp, xdt, xk = _ptr_dtype(X)
    N, K = int(W.shape[0]), int(W.shape[1])
    T = int(X.shape[0])
    if int(X.shape[1]) != K:
        raise ValueError("X and W disagree on K")
    if (levels is None) != (scales is None):
        raise ValueError("give both levels and scales, or neither")
    if levels is None:
        levels = np.zeros((N, K), np.int8)
        scales = np.zeros((N, K // group), np.float32)
    if tuple(levels.shape) != (N, K) or tuple(scales.shape) != (N, K // group):
        raise ValueError("levels / scales have the wrong shape")
    _check(_lib.gsq_gptq(wp, wdt, xp, xdt, N, K, T, group, grid_mode, damp,
                         _host_ptr(levels), _host_ptr(scales), _stream_ptr(stream)),
           "gsq_gptq")
    del wk, xk
    return levels, scales


def gsq_set_cached_memory_limit(nbytes: int) -> None:
    """Keep at most nbytes of freed device memory reserved per device."""
    _check(_lib.gsq_set_cached_memory_limit(int(nbytes)), "gsq_set_cached_memory_limit")


def gsq_release_cached_memory() -> None:
    """Return the device memory the library's pools keep in reserve."""
    _check(_lib.gsq_release_cached_memory(), "gsq_release_cached_memory")


def gsq_init_gptq(W, X, group: int = 128, grid_mode: int = GSQ_GRID_2BIT,
                  damp: float = 0.01, seed: int = 0, stream=None) -> "Layer":
    """gsq_init with the GPTQ levels and scales as the starting point."""
    wp, wdt, wk = _ptr_dtype(W)
    xp, xdt, xk = _ptr_dtype(X)
    N, K = int(W.shape[0]), int(W.shape[1])
    T = int(X.shape[0])
    if int(X.shape[1]) != K:
        raise ValueError("X and W disagree on K")
    ctx = C.c_void_p()
    _check(_lib.gsq_init_gptq(C.byref(ctx), wp, wdt, xp, xdt, N, K, T, group, grid_mode,
                              damp, seed & 0xFFFFFFFFFFFFFFFF, _stream_ptr(stream)),
           "gsq_init_gptq")
    del wk, xk
    return Layer(ctx, grid_mode, N, K, T, group)


def gsq_step(layer: "Layer", tau: float, lr: float, beta1: float = 0.9,
             beta2: float = 0.99) -> None:
    _check(_lib.gsq_step(layer.ctx, tau, lr, beta1, beta2), "gsq_step")


def gsq_scale_step(layer: "Layer", lr: float, beta1: float = 0.9, beta2: float = 0.99) -> None:
    _check(_lib.gsq_scale_step(layer.ctx, lr, beta1, beta2), "gsq_scale_step")


def gsq_scale_run(layer: "Layer", n: int, lr: float, beta1: float = 0.9,
                  beta2: float = 0.99) -> None:
    _check(_lib.gsq_scale_run(layer.ctx, n, lr, beta1, beta2), "gsq_scale_run")


def gsq_run(layer: "Layer", taus, lr: float, beta1: float = 0.9,
            beta2: float = 0.99) -> None:
    t = np.ascontiguousarray(taus, dtype=np.float32).ravel()
    _check(_lib.gsq_run(layer.ctx, t.ctypes.data, t.size, lr, beta1, beta2),
           "gsq_run")


def gsq_last_loss(layer: "Layer") -> float:
    v = C.c_double()
    _check(_lib.gsq_last_loss(layer.ctx, C.byref(v)), "gsq_last_loss")
    return v.value


def gsq_harden_pack(layer: "Layer", packed=None, scales_f16=None,
                    scales_f32=None):
    """Into the given buffers (host numpy or device tensors); allocates host
    numpy outputs when none are given.  Returns (packed, scales_f16, scales_f32)."""
    if packed is None:
        packed = np.zeros(gsq_packed_bytes(layer.mode, layer.N, layer.K) // 4,
                          np.uint32)
        scales_f16 = np.zeros((layer.N, layer.G), np.uint16)
        scales_f32 = np.zeros((layer.N, layer.G), np.float32)
    _check(_lib.gsq_harden_pack(
        layer.ctx, _host_ptr(packed),
        None if scales_f16 is None else _host_ptr(scales_f16),
        None if scales_f32 is None else _host_ptr(scales_f32)), "gsq_harden_pack")
    return packed, scales_f16, scales_f32


def gsq_recon_error(layer: "Layer", mode: int = GSQ_RECON_HARD,
                    tau: float = 1.0):
    a, r = C.c_double(), C.c_double()
    _check(_lib.gsq_recon_error(layer.ctx, mode, tau, C.byref(a), C.byref(r)),
           "gsq_recon_error")
    return a.value, r.value


def gsq_export_state(layer: "Layer") -> np.ndarray:
    n = C.c_size_t()
    _check(_lib.gsq_state_bytes(layer.ctx, C.byref(n)), "gsq_state_bytes")
    buf = np.zeros(n.value, np.uint8)
    _check(_lib.gsq_export_state(layer.ctx, buf.ctypes.data, n.value),
           "gsq_export_state")
    return buf


def gsq_import_state(layer: "Layer", buf: np.ndarray) -> None:
    buf = np.ascontiguousarray(buf, np.uint8)
    _check(_lib.gsq_import_state(layer.ctx, buf.ctypes.data, buf.size),
           "gsq_import_state")


def gsq_get_step(layer: "Layer") -> int:
    t = C.c_uint64()
    _check(_lib.gsq_get_step(layer.ctx, C.byref(t)), "gsq_get_step")
    return t.value


def gsq_destroy(layer: "Layer") -> None:
    if layer.ctx:
        _check(_lib.gsq_destroy(layer.ctx), "gsq_destroy")
        layer.ctx = None


def gsq_set_timing(layer: "Layer", on: bool) -> None:
    _check(_lib.gsq_set_timing(layer.ctx, int(on)), "gsq_set_timing")


def gsq_phase_times(layer: "Layer"):
    ms = np.zeros(5, np.float64)
    n = np.zeros(5, np.int64)
    _check(_lib.gsq_phase_times(layer.ctx, ms.ctypes.data, n.ctypes.data),
           "gsq_phase_times")
    return ms, n


def gsq_gemm_bf16_abt(A, B, Cout, stream=None) -> None:
    """Cout (M x N fp32) = A (M x Kc bf16) . B (N x Kc bf16)^T; torch device tensors."""
    M, Kc = A.shape
    N = B.shape[0]
    _check(_lib.gsq_gemm_bf16_abt(A.data_ptr(), B.data_ptr(), Cout.data_ptr(),
                                  M, N, Kc, _stream_ptr(stream)),
           "gsq_gemm_bf16_abt")


def gsq_gemm_bf16_abt_sub(A, B, C, stream=None) -> None:
    """C (M x N fp32) -= A (M x Kc bf16) . B (N x Kc bf16)^T in place; torch
    device tensors."""
    M, Kc = A.shape
    N = B.shape[0]
    _check(_lib.gsq_gemm_bf16_abt_sub(A.data_ptr(), B.data_ptr(), C.data_ptr(),
                                      M, N, Kc, _stream_ptr(stream)),
           "gsq_gemm_bf16_abt_sub")


class Layer:
    """A GSQ context for one linear layer (owner of the C handle)."""

    def __init__(self, ctx, mode, N, K, T, group, state16=False):
        self.ctx, self.mode, self.N, self.K, self.T, self.group = ctx, mode, N, K, T, group
        self.state16 = bool(state16)
        self.G = K // group
        self.L = NUM_LOGITS[mode]
        self.Tp = (T + 63) // 64 * 64

    # debug accessors ---------------------------------------------------
    _SHAPES = {
        GSQ_DBG_LOGITS: ("L,N,K", np.float32), GSQ_DBG_MOM: ("L,N,K", np.float32),
        GSQ_DBG_SCALES: ("N,G", np.float32), GSQ_DBG_SMOM: ("N,G", np.float32),
        GSQ_DBG_I0: ("N,K", np.int8), GSQ_DBG_WHAT: ("N,K", np.uint16),
        GSQ_DBG_WSOFT32: ("N,K", np.float32), GSQ_DBG_DW: ("N,K", np.float32),
        GSQ_DBG_DYT: ("N,Tp", np.uint16), GSQ_DBG_YREFT: ("N,Tp", np.float32),
        GSQ_DBG_DL: ("L,N,K", np.float32), GSQ_DBG_DS: ("N,G", np.float32),
    }

    def _shape(self, which):
        spec, dt = self._SHAPES[which]
        if self.state16 and which in (GSQ_DBG_LOGITS, GSQ_DBG_MOM):
            dt = np.uint16  # bf16 bit patterns
        return tuple(getattr(self, d) for d in spec.split(",")), dt

    def get(self, which) -> np.ndarray:
        shape, dt = self._shape(which)
        out = np.zeros(shape, dt)
        _check(_lib.gsq_debug_get(self.ctx, which, out.ctypes.data, out.nbytes),
               "gsq_debug_get")
        return out

    def set(self, which, arr) -> None:
        shape, dt = self._shape(which)
        a = np.ascontiguousarray(arr, dtype=dt).reshape(shape)
        _check(_lib.gsq_debug_set(self.ctx, which, a.ctypes.data, a.nbytes),
               "gsq_debug_set")

    def uniforms(self, t: int, coord0: int, count: int) -> np.ndarray:
        out = np.zeros((count, self.L), np.float32)
        _check(_lib.gsq_debug_uniforms(self.ctx, t, coord0, count, out.ctypes.data),
               "gsq_debug_uniforms")
        return out

    def noise_log2(self, m0: int, count: int) -> np.ndarray:
        out = np.zeros(count, np.float32)
        _check(_lib.gsq_debug_noise_log2(self.ctx, m0, count, out.ctypes.data),
               "gsq_debug_noise_log2")
        return out

    def noise(self, on: bool) -> None:
        _check(_lib.gsq_debug_noise(self.ctx, int(on)), "gsq_debug_noise")

    def soft_weight(self, tau: float) -> None:
        _check(_lib.gsq_debug_soft_weight(self.ctx, tau), "gsq_debug_soft_weight")

    def forward(self) -> float:
        v = C.c_double()
        _check(_lib.gsq_debug_forward(self.ctx, C.byref(v)), "gsq_debug_forward")
        return v.value

    def weight_grad(self) -> None:
        _check(_lib.gsq_debug_weight_grad(self.ctx), "gsq_debug_weight_grad")

    def backward(self, tau, lr, beta1=0.9, beta2=0.99) -> None:
        _check(_lib.gsq_debug_backward(self.ctx, tau, lr, beta1, beta2),
               "gsq_debug_backward")

    def debug_scale_backward(self, lr, beta1=0.9, beta2=0.99):
        _check(_lib.gsq_debug_scale_backward(self.ctx, lr, beta1, beta2),
               "gsq_debug_scale_backward")

    # convenience -------------------------------------------------------
    def step(self, tau, lr, beta1=0.9, beta2=0.99, tau_next=None):
        """One step; with tau_next, gsq_step_next (the backward also forms the
        next step's soft weight at tau_next)."""
        if tau_next is None:
            gsq_step(self, tau, lr, beta1, beta2)
        else:
            _check(_lib.gsq_step_next(self.ctx, tau, tau_next, lr, beta1, beta2),
                   "gsq_step_next")

    def scale_step(self, lr, beta1=0.9, beta2=0.99):
        gsq_scale_step(self, lr, beta1, beta2)

    def scale_run(self, n, lr, beta1=0.9, beta2=0.99):
        gsq_scale_run(self, n, lr, beta1, beta2)

    def run(self, taus, lr, beta1=0.9, beta2=0.99):
        gsq_run(self, taus, lr, beta1, beta2)

    def last_loss(self):
        return gsq_last_loss(self)

    def close(self):
        gsq_destroy(self)

    def __del__(self):
        try:
            if self.ctx:
                _lib.gsq_destroy(self.ctx)
                self.ctx = None
        except Exception:
            pass


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32 values (exact)."""
    return (b.astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------ block stage: SwiGLU MLP

def gsq_mlp_init(Xn, R, Wg, Wu, Wd, group: int = 128,
                 grid_mode: int = GSQ_GRID_2BIT, seed: int = 0, stream=None) -> "Mlp":
    """Xn, R (T x H); Wg, Wu (F x H); Wd (H x F): numpy fp32 or torch fp32/bf16."""
    xp, xdt, xk = _ptr_dtype(Xn)
    rp, rdt, rk = _ptr_dtype(R)
    gp, wdt, gk = _ptr_dtype(Wg)
    up, udt, uk = _ptr_dtype(Wu)
    dp, ddt, dk = _ptr_dtype(Wd)
    if not (wdt == udt == ddt):
        raise TypeError("Wg, Wu and Wd must share a dtype")
    T, H = int(Xn.shape[0]), int(Xn.shape[1])
    F = int(Wg.shape[0])
    ctx = C.c_void_p()
    _check(_lib.gsq_mlp_init(C.byref(ctx), xp, xdt, rp, rdt, gp, up, dp, wdt, T, H, F,
                             group, grid_mode, seed & 0xFFFFFFFFFFFFFFFF,
                             _stream_ptr(stream)), "gsq_mlp_init")
    del xk, rk, gk, uk, dk
    return Mlp(ctx, grid_mode, T, H, F, group)


class Mlp:
    """Context of the SwiGLU MLP stage (gate, up, down quantized jointly)."""

    def __init__(self, ctx, mode, T, H, F, group):
        self.ctx, self.mode, self.T, self.H, self.F, self.group = ctx, mode, T, H, F, group
        self.L = NUM_LOGITS[mode]
        self.shapes = ((F, H), (F, H), (H, F))

    def step(self, tau, lr, beta1=0.9, beta2=0.99):
        _check(_lib.gsq_mlp_step(self.ctx, tau, lr, beta1, beta2), "gsq_mlp_step")

    def run(self, taus, lr, beta1=0.9, beta2=0.99):
        t = np.ascontiguousarray(taus, dtype=np.float32).ravel()
        _check(_lib.gsq_mlp_run(self.ctx, t.ctypes.data, t.size, lr, beta1, beta2),
               "gsq_mlp_run")

    def set_timing(self, on: bool) -> None:
        _check(_lib.gsq_mlp_set_timing(self.ctx, int(bool(on))), "gsq_mlp_set_timing")

    def phase_times(self):
        """(ms[4], launches[4]) of soft weights, GEMMs, elementwise, backward
        since the last call (syncs)."""
        ms = np.zeros(4, np.float64)
        n = np.zeros(4, np.int64)
        _check(_lib.gsq_mlp_phase_times(self.ctx, ms.ctypes.data, n.ctypes.data),
               "gsq_mlp_phase_times")
        return ms, n

    def last_loss(self):
        v = C.c_double()
        _check(_lib.gsq_mlp_last_loss(self.ctx, C.byref(v)), "gsq_mlp_last_loss")
        return v.value

    def recon_error(self, mode=GSQ_RECON_HARD, tau=1.0):
        a, r = C.c_double(), C.c_double()
        _check(_lib.gsq_mlp_recon_error(self.ctx, mode, tau, C.byref(a), C.byref(r)),
               "gsq_mlp_recon_error")
        return a.value, r.value

    def harden_pack(self, which):
        N, K = self.shapes[which]
        packed = np.zeros(gsq_packed_bytes(self.mode, N, K) // 4, np.uint32)
        h16 = np.zeros((N, K // self.group), np.uint16)
        f32 = np.zeros((N, K // self.group), np.float32)
        _check(_lib.gsq_mlp_harden_pack(self.ctx, which, packed.ctypes.data,
                                        h16.ctypes.data, f32.ctypes.data),
               "gsq_mlp_harden_pack")
        return packed, h16, f32

    def _shape(self, which, buf):
        if which < 3:
            N, K = self.shapes[which]
            G = K // self.group
            return {GSQ_DBG_LOGITS: ((self.L, N, K), np.float32),
                    GSQ_DBG_MOM: ((self.L, N, K), np.float32),
                    GSQ_DBG_SCALES: ((N, G), np.float32), GSQ_DBG_SMOM: ((N, G), np.float32),
                    GSQ_DBG_I0: ((N, K), np.int8), GSQ_DBG_WHAT: ((N, K), np.uint16),
                    GSQ_DBG_DW: ((N, K), np.float32)}[buf]
        F, H, T = self.F, self.H, self.T
        return {GSQ_MLP_DBG_AT: ((F, T), np.float32), GSQ_MLP_DBG_BT: ((F, T), np.float32),
                GSQ_MLP_DBG_HT: ((F, T), np.uint16), GSQ_MLP_DBG_DPT: ((H, T), np.uint16),
                GSQ_MLP_DBG_DHT: ((F, T), np.float32), GSQ_MLP_DBG_DAT: ((F, T), np.uint16),
                GSQ_MLP_DBG_DBT: ((F, T), np.uint16), GSQ_MLP_DBG_RT: ((H, T), np.float32)}[buf]

    def get(self, which, buf):
        shape, dt = self._shape(which, buf)
        out = np.zeros(shape, dt)
        _check(_lib.gsq_mlp_debug_get(self.ctx, which, buf, out.ctypes.data, out.nbytes),
               "gsq_mlp_debug_get")
        return out

    def set(self, which, buf, arr):
        shape, dt = self._shape(which, buf)
        a = np.ascontiguousarray(arr, dtype=dt).reshape(shape)
        _check(_lib.gsq_mlp_debug_set(self.ctx, which, buf, a.ctypes.data, a.nbytes),
               "gsq_mlp_debug_set")

    def get_step(self):
        t = C.c_uint64()
        _check(_lib.gsq_mlp_get_step(self.ctx, C.byref(t)), "gsq_mlp_get_step")
        return t.value

    def close(self):
        if self.ctx:
            _check(_lib.gsq_mlp_destroy(self.ctx), "gsq_mlp_destroy")
            self.ctx = None

    def __del__(self):
        try:
            if self.ctx:
                _lib.gsq_mlp_destroy(self.ctx)
                self.ctx = None
        except Exception:
            pass


# ----------------------------------------- block stage: attention V/O

def gsq_attn_init(Xa, R, Wq, Wk, Wv, Wo, n_seq, seq_len, n_heads, n_kv_heads,
                  head_dim=128, rope_theta=500000.0, group=128,
                  grid_mode=GSQ_GRID_2BIT, seed=0, stream=None) -> "Attn":
    """Xa, R (T x H); Wq, Wo (H x H); Wk, Wv (n_kv_heads head_dim x H)."""
    xp, xdt, xk = _ptr_dtype(Xa)
    rp, rdt, rk = _ptr_dtype(R)
    ws = [_ptr_dtype(W) for W in (Wq, Wk, Wv, Wo)]
    if len({w[1] for w in ws}) != 1:
        raise TypeError("Wq, Wk, Wv and Wo must share a dtype")
    ctx = C.c_void_p()
    _check(_lib.gsq_attn_init(C.byref(ctx), xp, xdt, rp, rdt, ws[0][0], ws[1][0], ws[2][0],
                              ws[3][0], ws[0][1], n_seq, seq_len, n_heads, n_kv_heads,
                              head_dim, rope_theta, group, grid_mode,
                              seed & 0xFFFFFFFFFFFFFFFF, _stream_ptr(stream)),
           "gsq_attn_init")
    del xk, rk, ws
    return Attn(ctx, grid_mode, n_seq, seq_len, n_heads, n_kv_heads, head_dim, group)


class Attn:
    """Context of the attention V/O stage (value and output quantized jointly)."""

    def __init__(self, ctx, mode, nseq, S, nh, nkv, d, group):
        self.ctx, self.mode, self.group = ctx, mode, group
        self.nseq, self.S, self.nh, self.nkv, self.d = nseq, S, nh, nkv, d
        self.T, self.H, self.Hk = nseq * S, nh * d, nkv * d
        self.L = NUM_LOGITS[mode]
        self.shapes = ((self.Hk, self.H), (self.H, self.H))

    def step(self, tau, lr, beta1=0.9, beta2=0.99):
        _check(_lib.gsq_attn_step(self.ctx, tau, lr, beta1, beta2), "gsq_attn_step")

    def run(self, taus, lr, beta1=0.9, beta2=0.99):
        t = np.ascontiguousarray(taus, dtype=np.float32).ravel()
        _check(_lib.gsq_attn_run(self.ctx, t.ctypes.data, t.size, lr, beta1, beta2),
               "gsq_attn_run")

    def set_timing(self, on: bool) -> None:
        _check(_lib.gsq_attn_set_timing(self.ctx, int(bool(on))), "gsq_attn_set_timing")

    def phase_times(self):
        """(ms[4], launches[4]) of soft weights, GEMMs, elementwise, backward
        since the last call (syncs)."""
        ms = np.zeros(4, np.float64)
        n = np.zeros(4, np.int64)
        _check(_lib.gsq_attn_phase_times(self.ctx, ms.ctypes.data, n.ctypes.data),
               "gsq_attn_phase_times")
        return ms, n

    def last_loss(self):
        v = C.c_double()
        _check(_lib.gsq_attn_last_loss(self.ctx, C.byref(v)), "gsq_attn_last_loss")
        return v.value

    def recon_error(self, mode=GSQ_RECON_HARD, tau=1.0):
        a, r = C.c_double(), C.c_double()
        _check(_lib.gsq_attn_recon_error(self.ctx, mode, tau, C.byref(a), C.byref(r)),
               "gsq_attn_recon_error")
        return a.value, r.value

    def harden_pack(self, which):
        N, K = self.shapes[which]
        packed = np.zeros(gsq_packed_bytes(self.mode, N, K) // 4, np.uint32)
        h16 = np.zeros((N, K // self.group), np.uint16)
        f32 = np.zeros((N, K // self.group), np.float32)
        _check(_lib.gsq_attn_harden_pack(self.ctx, which, packed.ctypes.data,
                                         h16.ctypes.data, f32.ctypes.data),
               "gsq_attn_harden_pack")
        return packed, h16, f32

    def _shape(self, which, buf):
        if which < 2:
            N, K = self.shapes[which]
            G = K // self.group
            return {GSQ_DBG_LOGITS: ((self.L, N, K), np.float32),
                    GSQ_DBG_MOM: ((self.L, N, K), np.float32),
                    GSQ_DBG_SCALES: ((N, G), np.float32), GSQ_DBG_SMOM: ((N, G), np.float32),
                    GSQ_DBG_I0: ((N, K), np.int8), GSQ_DBG_WHAT: ((N, K), np.uint16),
                    GSQ_DBG_DW: ((N, K), np.float32)}[buf]
        P = (self.nseq, self.nh, self.S, self.S)
        return {GSQ_ATTN_DBG_P: (P, np.uint16), GSQ_ATTN_DBG_PT: (P, np.uint16),
                GSQ_ATTN_DBG_VT: ((self.Hk, self.T), np.uint16),
                GSQ_ATTN_DBG_O: ((self.T, self.H), np.uint16),
                GSQ_ATTN_DBG_DPT: ((self.H, self.T), np.uint16),
                GSQ_ATTN_DBG_DV: ((self.T, self.Hk), np.uint16),
                GSQ_ATTN_DBG_RT: ((self.H, self.T), np.float32)}[buf]

    def get(self, which, buf):
        shape, dt = self._shape(which, buf)
        out = np.zeros(shape, dt)
        _check(_lib.gsq_attn_debug_get(self.ctx, which, buf, out.ctypes.data, out.nbytes),
               "gsq_attn_debug_get")
        return out

    def set(self, which, buf, arr):
        shape, dt = self._shape(which, buf)
        a = np.ascontiguousarray(arr, dtype=dt).reshape(shape)
        _check(_lib.gsq_attn_debug_set(self.ctx, which, buf, a.ctypes.data, a.nbytes),
               "gsq_attn_debug_set")

    def close(self):
        if self.ctx:
            _check(_lib.gsq_attn_destroy(self.ctx), "gsq_attn_destroy")
            self.ctx = None

    def __del__(self):
        try:
            if self.ctx:
                _lib.gsq_attn_destroy(self.ctx)
                self.ctx = None
        except Exception:
            pass


# ------------------------------------------------------ staged block pipeline

BLOCK_WEIGHTS = ("q", "k", "v", "o", "gate", "up", "down")
BLOCK_STAGES = ("q", "k", "vo", "mlp")


def block_weight_shapes(n_heads, n_kv_heads, head_dim, ffn):
    H, Hk = n_heads * head_dim, n_kv_heads * head_dim
    return {"q": (H, H), "k": (Hk, H), "v": (Hk, H), "o": (H, H),
            "gate": (ffn, H), "up": (ffn, H), "down": (H, ffn)}


def _block_shapes_ok(x, W, n_seq, seq_len, n_heads, n_kv_heads, head_dim, ffn):
    """The C entry points see raw pointers: check every extent here."""
    shapes = block_weight_shapes(n_heads, n_kv_heads, head_dim, ffn)
    if tuple(x.shape) != (n_seq * seq_len, n_heads * head_dim):
        raise ValueError(f"x has shape {tuple(x.shape)}, expected "
                         f"{(n_seq * seq_len, n_heads * head_dim)}")
    for name in BLOCK_WEIGHTS:
        if tuple(W[name].shape) != shapes[name]:
            raise ValueError(f"weight {name} has shape {tuple(W[name].shape)}, "
                             f"expected {shapes[name]}")


def _bf16_weights(W):
    """Keep-alive list and a C array of the seven bf16 weight pointers."""
    import torch
    keep = []
    for name in BLOCK_WEIGHTS:
        w = W[name]
        if not isinstance(w, torch.Tensor):
            w = torch.from_numpy(np.ascontiguousarray(w, np.float32))
        w = w.to(torch.bfloat16).contiguous()
        keep.append(w)
    arr = (C.c_void_p * 7)(*[w.data_ptr() for w in keep])
    return keep, arr


def _f32_tensor(x):
    import torch
    if not isinstance(x, torch.Tensor):
        x = torch.from_numpy(np.ascontiguousarray(x, np.float32))
    return x.to(torch.float32).contiguous()


def gsq_dequant(grid_mode, packed, scales_f32, N, K, group=128, out=None, stream=None):
    """bf16 weight (N x K) of a packed code stream and its fp32 group scales.
    Returns `out` (a torch bf16 tensor, host or device) or a new device tensor."""
    import torch
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    if (tuple(out.shape) != (N, K) or out.dtype != torch.bfloat16
            or int(np.prod(scales_f32.shape)) != N * (K // group)
            or int(packed.nbytes if hasattr(packed, "nbytes") else
                   packed.numel() * packed.element_size()) != gsq_packed_bytes(grid_mode, N, K)):
        raise ValueError("gsq_dequant: buffer sizes do not match N x K")
    _check(_lib.gsq_dequant(grid_mode, _host_ptr(packed), _host_ptr(scales_f32), N, K, group,
                            out.data_ptr(), _stream_ptr(stream)), "gsq_dequant")
    return out


def gsq_block_forward(x, W, n_seq, seq_len, n_heads, n_kv_heads, head_dim, ffn,
                      rope_theta=500000.0, rms_eps=1e-5, stream=None):
    """(h, y) of the pre-norm block on the fp32 residual stream x (T x H) with
    bf16 weights W (dict of the seven projections); device tensors."""
    import torch
    x = _f32_tensor(x)
    _block_shapes_ok(x, W, n_seq, seq_len, n_heads, n_kv_heads, head_dim, ffn)
    keep, arr = _bf16_weights(W)
    T, H = int(x.shape[0]), int(x.shape[1])
    dev = x.device if x.is_cuda else torch.device("cuda")
    h = torch.empty((T, H), dtype=torch.float32, device=dev)
    y = torch.empty((T, H), dtype=torch.float32, device=dev)
    _check(_lib.gsq_block_forward(x.data_ptr(), arr, n_seq, seq_len, n_heads, n_kv_heads,
                                  head_dim, ffn, rope_theta, rms_eps, h.data_ptr(),
                                  y.data_ptr(), _stream_ptr(stream)), "gsq_block_forward")
    del keep
    return h, y


def gsq_block_quantize(x, W, n_seq, seq_len, n_heads, n_kv_heads, head_dim, ffn, taus,
                       lr, beta1=0.9, beta2=0.99, seed=0, grid_mode=GSQ_GRID_2BIT,
                       group=128, rope_theta=500000.0, rms_eps=1e-5, stream=None,
                       host_outputs=False):
    """GSQ's staged reconstruction of one block (Q, K, then V/O, then the MLP
    on the block output).  taus: four temperature schedules (one per stage).
    Returns a dict: x_out (fp32, the next block's input), packed and
    scales_f32 per weight, stats per stage (first loss, last loss, hard abs /
    rel error, ms).  Outputs are device tensors, or pinned host tensors with
    host_outputs (the library writes them through unified addressing)."""
    import torch
    x = _f32_tensor(x)
    _block_shapes_ok(x, W, n_seq, seq_len, n_heads, n_kv_heads, head_dim, ffn)
    keep, arr = _bf16_weights(W)
    T, H = int(x.shape[0]), int(x.shape[1])
    dev = x.device if x.is_cuda else torch.device("cuda")
    if host_outputs:
        dev = torch.device("cpu")
    shapes = block_weight_shapes(n_heads, n_kv_heads, head_dim, ffn)
    pin = dict(pin_memory=True) if host_outputs else {}
    x_out = torch.empty((T, H), dtype=torch.float32, device=dev, **pin)
    packed, scales = {}, {}
    for name in BLOCK_WEIGHTS:
        N, K = shapes[name]
        packed[name] = torch.empty(gsq_packed_bytes(grid_mode, N, K) // 4, dtype=torch.int32,
                                   device=dev, **pin)
        scales[name] = torch.empty((N, K // group), dtype=torch.float32, device=dev, **pin)
    tau_arr = [np.ascontiguousarray(t, np.float32) for t in taus]
    if len(tau_arr) != 4:
        raise ValueError("taus: one schedule per stage (4)")
    tp = (C.c_void_p * 4)(*[t.ctypes.data if t.size else None for t in tau_arr])
    ns = (C.c_int64 * 4)(*[int(t.size) for t in tau_arr])
    pk = (C.c_void_p * 7)(*[packed[n].data_ptr() for n in BLOCK_WEIGHTS])
    sc = (C.c_void_p * 7)(*[scales[n].data_ptr() for n in BLOCK_WEIGHTS])
    stats = np.zeros(20, np.float64)
    _check(_lib.gsq_block_quantize(x.data_ptr(), arr, n_seq, seq_len, n_heads, n_kv_heads,
                                   head_dim, ffn, rope_theta, rms_eps, group, grid_mode, tp,
                                   ns, lr, beta1, beta2, seed & 0xFFFFFFFFFFFFFFFF,
                                   x_out.data_ptr(), pk, None, sc, stats.ctypes.data,
                                   _stream_ptr(stream)), "gsq_block_quantize")
    del keep, tau_arr
    st = {name: dict(first_loss=stats[5 * j], last_loss=stats[5 * j + 1],
                     recon=(stats[5 * j + 2], stats[5 * j + 3]), ms=stats[5 * j + 4])
          for j, name in enumerate(BLOCK_STAGES)}
    return {"x_out": x_out, "packed": packed, "scales": scales, "stats": st}


# ------------------------------------------------------- GGUF K-Quant formats

GSQ_KQ_Q2_K, GSQ_KQ_Q3_K = 0, 1
(GSQ_KQ_DBG_LOGITS, GSQ_KQ_DBG_MOM, GSQ_KQ_DBG_A, GSQ_KQ_DBG_MA, GSQ_KQ_DBG_B, GSQ_KQ_DBG_MB,
 GSQ_KQ_DBG_Q0, GSQ_KQ_DBG_WHAT, GSQ_KQ_DBG_DW, GSQ_KQ_DBG_DL, GSQ_KQ_DBG_DA, GSQ_KQ_DBG_DB,
 GSQ_KQ_DBG_WSOFT32) = range(13)


def gsq_kq_block_bytes(fmt: int, N: int, K: int) -> int:
    b = C.c_size_t()
    _check(_lib.gsq_kq_block_bytes(fmt, N, K, C.byref(b)), "gsq_kq_block_bytes")
    return b.value


def gsq_kq_init(W, X, fmt: int = GSQ_KQ_Q2_K, start_blocks=None, seed: int = 0,
                stream=None) -> "KqLayer":
    """GSQ on a K-Quant format: W (N x K), X (T x K) as for gsq_init;
    start_blocks (uint8 numpy array or torch tensor of gsq_kq_block_bytes
    bytes) or None for the min-max K-Quant of W."""
    wp, wdt, wk = _ptr_dtype(W)
    xp, xdt, xk = _ptr_dtype(X)
    N, K = int(W.shape[0]), int(W.shape[1])
    T = int(X.shape[0])
    if int(X.shape[1]) != K:
        raise ValueError("X and W disagree on K")
    sp, sk = None, None
    if start_blocks is not None:
        sk = start_blocks if hasattr(start_blocks, "data_ptr") else np.ascontiguousarray(
            start_blocks, np.uint8)
        nb = sk.numel() * sk.element_size() if hasattr(sk, "numel") else sk.nbytes
        if nb != gsq_kq_block_bytes(fmt, N, K):
            raise ValueError("start_blocks has the wrong size")
        sp = _host_ptr(sk)
    ctx = C.c_void_p()
    _check(_lib.gsq_kq_init(C.byref(ctx), wp, wdt, xp, xdt, N, K, T, fmt, sp,
                            seed & 0xFFFFFFFFFFFFFFFF, _stream_ptr(stream)), "gsq_kq_init")
    del wk, xk, sk
    return KqLayer(ctx, fmt, N, K, T)


def gsq_kq_dequant(fmt: int, blocks, N: int, K: int, out=None, stream=None):
    """bf16 weight (N x K) of K-Quant blocks; a device tensor unless `out` is given."""
    import torch
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    b = blocks if hasattr(blocks, "data_ptr") else np.ascontiguousarray(blocks, np.uint8)
    nb = b.numel() * b.element_size() if hasattr(b, "numel") else b.nbytes
    if nb != gsq_kq_block_bytes(fmt, N, K) or tuple(out.shape) != (N, K):
        raise ValueError("gsq_kq_dequant: sizes do not match N x K")
    _check(_lib.gsq_kq_dequant(fmt, _host_ptr(b), N, K, out.data_ptr(), _stream_ptr(stream)),
           "gsq_kq_dequant")
    return out


class KqLayer:
    """A GSQ context on a K-Quant format (owner of the C handle)."""

    def __init__(self, ctx, fmt, N, K, T):
        self.ctx, self.fmt, self.N, self.K, self.T = ctx, fmt, N, K, T
        self.L = 4 if fmt == GSQ_KQ_Q2_K else 5
        self.S = K // 16

    _SHAPES = {GSQ_KQ_DBG_LOGITS: ("L,N,K", np.float32), GSQ_KQ_DBG_MOM: ("L,N,K", np.float32),
               GSQ_KQ_DBG_A: ("N,S", np.float32), GSQ_KQ_DBG_MA: ("N,S", np.float32),
               GSQ_KQ_DBG_B: ("N,S", np.float32), GSQ_KQ_DBG_MB: ("N,S", np.float32),
               GSQ_KQ_DBG_Q0: ("N,K", np.int8), GSQ_KQ_DBG_WHAT: ("N,K", np.uint16),
               GSQ_KQ_DBG_DW: ("N,K", np.float32), GSQ_KQ_DBG_DL: ("L,N,K", np.float32),
               GSQ_KQ_DBG_DA: ("N,S", np.float32), GSQ_KQ_DBG_DB: ("N,S", np.float32),
               GSQ_KQ_DBG_WSOFT32: ("N,K", np.float32)}

    def _shape(self, which):
        spec, dt = self._SHAPES[which]
        return tuple(getattr(self, d) for d in spec.split(",")), dt

    def get(self, which) -> np.ndarray:
        shape, dt = self._shape(which)
        out = np.zeros(shape, dt)
        _check(_lib.gsq_kq_debug_get(self.ctx, which, out.ctypes.data, out.nbytes),
               "gsq_kq_debug_get")
        return out

    def set(self, which, arr) -> None:
        shape, dt = self._shape(which)
        a = np.ascontiguousarray(arr, dtype=dt).reshape(shape)
        _check(_lib.gsq_kq_debug_set(self.ctx, which, a.ctypes.data, a.nbytes),
               "gsq_kq_debug_set")

    def step(self, tau, lr, beta1=0.9, beta2=0.99):
        _check(_lib.gsq_kq_step(self.ctx, tau, lr, beta1, beta2), "gsq_kq_step")

    def run(self, taus, lr, beta1=0.9, beta2=0.99):
        t = np.ascontiguousarray(taus, np.float32)
        _check(_lib.gsq_kq_run(self.ctx, t.ctypes.data, t.size, lr, beta1, beta2), "gsq_kq_run")

    def last_loss(self) -> float:
        v = C.c_double()
        _check(_lib.gsq_kq_last_loss(self.ctx, C.byref(v)), "gsq_kq_last_loss")
        return v.value

    def export(self) -> np.ndarray:
        out = np.zeros(gsq_kq_block_bytes(self.fmt, self.N, self.K), np.uint8)
        _check(_lib.gsq_kq_export(self.ctx, out.ctypes.data), "gsq_kq_export")
        return out

    def start_blocks(self) -> np.ndarray:
        out = np.zeros(gsq_kq_block_bytes(self.fmt, self.N, self.K), np.uint8)
        _check(_lib.gsq_kq_start_blocks(self.ctx, out.ctypes.data), "gsq_kq_start_blocks")
        return out

    def recon_error(self, which: int = 0):
        a, r = C.c_double(), C.c_double()
        _check(_lib.gsq_kq_recon_error(self.ctx, which, C.byref(a), C.byref(r)),
               "gsq_kq_recon_error")
        return a.value, r.value

    def soft_weight(self, tau: float) -> None:
        _check(_lib.gsq_kq_debug_soft_weight(self.ctx, tau), "gsq_kq_debug_soft_weight")

    def backward(self, tau, lr, beta1=0.9, beta2=0.99) -> None:
        _check(_lib.gsq_kq_debug_backward(self.ctx, tau, lr, beta1, beta2),
               "gsq_kq_debug_backward")

    def noise(self, on: bool) -> None:
        _check(_lib.gsq_kq_debug_noise(self.ctx, int(on)), "gsq_kq_debug_noise")

    def close(self):
        if self.ctx:
            _lib.gsq_kq_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # pragma: no cover
            pass

"""Thin Python binding of libhq.so, the sm_100a Hadamard-domain quantized
linear layer (HadaNorm identity X W + b = X~ W~ + b~; see include/hq.h).

Every function marshals torch tensors (device memory, owned by the caller) and
the current CUDA stream into the C ABI of the same name; all computation runs
in the library's CUDA kernels.  There is no CPU fallback: if libhq.so is
missing or the device is not sm_100, the calls raise.

    hq_calib_act_absmax(desc, X, absmax)
    hq_prepare_weights(desc, W, bias, act_absmax, alpha, w_codes, w_scale, colsum, sigma_inv, bias_f32)
    hq_quantize_act(desc, X, sigma_inv, a_codes, a_scale, a_mean, workspace)
    hq_linear(desc, a_codes, a_scale, a_mean, w_codes, w_scale, colsum, bias_f32, Y, acc_debug)
    hq_check_device_error()

The group-wise 4-bit form with a 16-bit low-rank branch (include/hq_gw.h):

    hq_gw_sigma_inv(desc, W, act_absmax, alpha, sigma_inv)
    hq_gw_prepare_weights(desc, W, bias, sigma_inv, L1, L2, w_codes, w_scale, l1s, l2b, bias_f32)
    hq_gw_quantize_act(desc, X, sigma_inv, l1s, a_codes, a_scale, u, workspace)
    hq_gw_linear(desc, a_codes, a_scale, u, w_codes, w_scale, l2b, bias_f32, Y)

`HadamardQuantLinear` and `GroupWiseQuantLinear` bundle the caller-side
buffers of one layer of each form.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "HQError", "LayerDesc", "load_library", "library_path", "exported_symbols",
    "HQ_PER_TOKEN", "HQ_PER_TENSOR_DYNAMIC", "HQ_PER_TENSOR_STATIC",
    "HQ_CENTER_NONE", "HQ_CENTER_TOKEN_MEAN", "HQ_CENTER_TOKEN_MEAN_PRE", "HQ_CODES_I8",
    "HQ_CODES_I4_PACKED",
    "HQ_FAULT_NONE", "HQ_FAULT_QUANT_WITHHOLD_ROW", "STATUS_NAMES",
    "hq_version", "hq_status_string", "hq_calib_act_absmax", "hq_prepare_weights",
    "hq_quantize_act_workspace_bytes", "hq_quantize_act", "hq_linear", "hq_forward_host",
    "hq_check_device_error", "hq_debug_set_wait_limit", "hq_debug_inject_fault",
    "hq_debug_set_gemm_variant", "HQ_GEMM_AUTO", "HQ_GEMM_SINGLE_CTA", "HQ_GEMM_CTA_PAIR",
    "hq_quantize_act_noalloc", "hq_debug_plan", "hq_debug_mma_ceiling", "hq_debug_tmap_cache",
    "HadamardQuantLinear", "GwDesc", "hq_gw_scale_ld", "hq_gw_sigma_inv", "hq_gw_prepare_weights",
    "hq_gw_quantize_act", "hq_gw_linear", "hq_gw_debug_linear_f32", "GroupWiseQuantLinear",
    "hq_debug_last_cuda_error", "hq_gw_quantize_act_workspace_bytes",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libhq.so")

HQ_PER_TOKEN, HQ_PER_TENSOR_DYNAMIC, HQ_PER_TENSOR_STATIC = 0, 1, 2
HQ_CENTER_NONE, HQ_CENTER_TOKEN_MEAN, HQ_CENTER_TOKEN_MEAN_PRE = 0, 1, 2
HQ_CODES_I8, HQ_CODES_I4_PACKED = 0, 1
HQ_FAULT_NONE, HQ_FAULT_QUANT_WITHHOLD_ROW = 0, 1
HQ_GEMM_AUTO, HQ_GEMM_SINGLE_CTA, HQ_GEMM_CTA_PAIR = 0, 1, 2
STATUS_NAMES = {0: "HQ_OK", 1: "HQ_ERR_INVALID_ARGUMENT", 2: "HQ_ERR_UNSUPPORTED",
                3: "HQ_ERR_MISALIGNED", 4: "HQ_ERR_CUDA", 5: "HQ_ERR_TIMEOUT",
                6: "HQ_ERR_DEVICE"}
EXPORTED = ("hq_status_string", "hq_version", "hq_calib_act_absmax", "hq_prepare_weights",
            "hq_quantize_act_workspace_bytes", "hq_quantize_act", "hq_linear", "hq_forward_host",
            "hq_check_device_error", "hq_debug_set_wait_limit", "hq_debug_inject_fault",
            "hq_debug_set_gemm_variant", "hq_quantize_act_noalloc", "hq_debug_plan",
            "hq_debug_mma_ceiling", "hq_debug_tmap_cache", "hq_gw_scale_ld", "hq_gw_sigma_inv",
            "hq_gw_prepare_weights", "hq_gw_quantize_act", "hq_gw_linear",
            "hq_gw_debug_linear_f32", "hq_debug_last_cuda_error",
            "hq_gw_quantize_act_workspace_bytes")


class HQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class LayerDesc(ctypes.Structure):
    """hq_layer_desc (host memory)."""
    _fields_ = [("K", ctypes.c_int32), ("N", ctypes.c_int32), ("had_order", ctypes.c_int32),
                ("a_bits", ctypes.c_int32), ("w_bits", ctypes.c_int32),
                ("act_gran", ctypes.c_int32), ("centering", ctypes.c_int32),
                ("code_format", ctypes.c_int32), ("out_order", ctypes.c_int32)]

    def __init__(self, K, N, had_order, a_bits=4, w_bits=4, act_gran=HQ_PER_TOKEN,
                 centering=HQ_CENTER_TOKEN_MEAN, code_format=HQ_CODES_I8, out_order=0):
        """out_order > 1 selects the weight-only Hadamard form (had_order 1,
        centering HQ_CENTER_NONE): W rotated along N in blocks of out_order."""
        super().__init__(K, N, had_order, a_bits, w_bits, act_gran, centering, code_format,
                         out_order)


class GwDesc(ctypes.Structure):
    """hq_gw_desc (host memory): the group-wise form's layer description."""
    _fields_ = [("K", ctypes.c_int32), ("N", ctypes.c_int32), ("group", ctypes.c_int32),
                ("rank", ctypes.c_int32), ("a_bits", ctypes.c_int32), ("w_bits", ctypes.c_int32)]

    def __init__(self, K, N, group=64, rank=32, a_bits=4, w_bits=4):
        super().__init__(K, N, group, rank, a_bits, w_bits)


_lib = None
_lock = threading.Lock()
_vp = ctypes.c_void_p


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Loads libhq.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: run hadamard_rotated_bit_token_b200/build.py "
                              "(or __graft_entry__.build()) first; there is no fallback path")
        lib = ctypes.CDLL(_LIB_PATH)
        desc_p = ctypes.POINTER(LayerDesc)
        lib.hq_status_string.argtypes = [ctypes.c_int]
        lib.hq_status_string.restype = ctypes.c_char_p
        lib.hq_version.argtypes = []
        lib.hq_version.restype = ctypes.c_int
        lib.hq_calib_act_absmax.argtypes = [desc_p, _vp, ctypes.c_int64, _vp, _vp]
        lib.hq_prepare_weights.argtypes = [desc_p, _vp, _vp, _vp, ctypes.c_float, _vp, _vp, _vp,
                                           _vp, _vp, _vp]
        lib.hq_quantize_act_workspace_bytes.argtypes = [desc_p, ctypes.c_int64]
        lib.hq_quantize_act_workspace_bytes.restype = ctypes.c_size_t
        lib.hq_quantize_act.argtypes = [desc_p, _vp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp,
                                        ctypes.c_size_t, _vp]
        lib.hq_linear.argtypes = [desc_p, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                  _vp, _vp]
        lib.hq_forward_host.argtypes = [desc_p, _vp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp, _vp,
                                        ctypes.c_size_t, _vp, _vp, _vp, _vp, _vp, _vp,
                                        ctypes.c_int, _vp]
        lib.hq_quantize_act_noalloc.argtypes = [desc_p, _vp, ctypes.c_int64, _vp, _vp, _vp, _vp,
                                                _vp]
        lib.hq_check_device_error.argtypes = [_vp]
        lib.hq_debug_set_wait_limit.argtypes = [ctypes.c_uint64]
        lib.hq_debug_inject_fault.argtypes = [ctypes.c_int]
        lib.hq_debug_set_gemm_variant.argtypes = [ctypes.c_int]
        _i32p = ctypes.POINTER(ctypes.c_int32)
        lib.hq_debug_plan.argtypes = [desc_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                      _i32p, _i32p, _i32p, _i32p]
        lib.hq_debug_mma_ceiling.argtypes = [ctypes.c_int, ctypes.c_int64, _i32p, _vp]
        _u64p = ctypes.POINTER(ctypes.c_uint64)
        lib.hq_debug_tmap_cache.argtypes = [_u64p, _u64p]
        lib.hq_debug_last_cuda_error.argtypes = []
        lib.hq_debug_last_cuda_error.restype = ctypes.c_int
        gw_p = ctypes.POINTER(GwDesc)
        lib.hq_gw_scale_ld.argtypes = [ctypes.c_int64]
        lib.hq_gw_scale_ld.restype = ctypes.c_int64
        lib.hq_gw_sigma_inv.argtypes = [gw_p, _vp, _vp, ctypes.c_float, _vp, _vp]
        lib.hq_gw_prepare_weights.argtypes = [gw_p, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                              _vp, _vp]
        lib.hq_gw_quantize_act_workspace_bytes.argtypes = [gw_p, ctypes.c_int64]
        lib.hq_gw_quantize_act_workspace_bytes.restype = ctypes.c_size_t
        lib.hq_gw_quantize_act.argtypes = [gw_p, _vp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp,
                                           _vp, ctypes.c_size_t, _vp]
        lib.hq_gw_linear.argtypes = [gw_p, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                     _vp, _vp]
        lib.hq_gw_debug_linear_f32.argtypes = list(lib.hq_gw_linear.argtypes)
        for name in ("hq_gw_sigma_inv", "hq_gw_prepare_weights", "hq_gw_quantize_act",
                     "hq_gw_linear", "hq_gw_debug_linear_f32"):
            getattr(lib, name).restype = ctypes.c_int
        for name in ("hq_calib_act_absmax", "hq_prepare_weights", "hq_quantize_act", "hq_linear",
                     "hq_forward_host",
                     "hq_check_device_error", "hq_debug_set_wait_limit", "hq_debug_inject_fault",
                     "hq_debug_set_gemm_variant", "hq_quantize_act_noalloc", "hq_debug_plan",
            "hq_debug_mma_ceiling", "hq_debug_tmap_cache"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
        return lib


def exported_symbols():
    lib = load_library()
    return {name: hasattr(lib, name) for name in EXPORTED}


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------

def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("tensor must live in CUDA device memory")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _host_ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if t.is_cuda:
        raise ValueError("tensor must live in host memory")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != 0:
        if status == 4:  # HQ_ERR_CUDA: name the code behind it
            code = load_library().hq_debug_last_cuda_error()
            raise HQError(status, f"{where} (CUDA code {code})")
        raise HQError(status, where)


# ---------------------------------------------------------------------------
# C ABI, same names
# ---------------------------------------------------------------------------

def hq_version() -> int:
    return load_library().hq_version()


def hq_status_string(status: int) -> str:
    return load_library().hq_status_string(status).decode()


def hq_calib_act_absmax(desc: LayerDesc, X, absmax, T=None, stream=None):
    T = X.shape[0] if T is None else T
    _check(load_library().hq_calib_act_absmax(ctypes.byref(desc), _ptr(X), T, _ptr(absmax),
                                              _stream(stream)), "hq_calib_act_absmax")


def hq_prepare_weights(desc: LayerDesc, W, bias, act_absmax, alpha, w_codes, w_scale, colsum,
                       sigma_inv, bias_f32, stream=None):
    _check(load_library().hq_prepare_weights(
        ctypes.byref(desc), _ptr(W), _ptr(bias), _ptr(act_absmax), float(alpha), _ptr(w_codes),
        _ptr(w_scale), _ptr(colsum), _ptr(sigma_inv), _ptr(bias_f32), _stream(stream)),
        "hq_prepare_weights")


def hq_quantize_act_workspace_bytes(desc: LayerDesc, T: int) -> int:
    return load_library().hq_quantize_act_workspace_bytes(ctypes.byref(desc), T)


def hq_quantize_act(desc: LayerDesc, X, sigma_inv, a_codes, a_scale, a_mean=None, workspace=None,
                    T=None, stream=None):
    T = X.shape[0] if T is None else T
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().hq_quantize_act(
        ctypes.byref(desc), _ptr(X), T, _ptr(sigma_inv), _ptr(a_codes), _ptr(a_scale),
        _ptr(a_mean), _ptr(workspace), ws_bytes, _stream(stream)), "hq_quantize_act")


def hq_linear(desc: LayerDesc, a_codes, a_scale, a_mean, w_codes, w_scale, colsum, bias_f32, Y,
              acc_debug=None, T=None, stream=None):
    T = a_codes.shape[0] if T is None else T
    _check(load_library().hq_linear(
        ctypes.byref(desc), T, _ptr(a_codes), _ptr(a_scale), _ptr(a_mean), _ptr(w_codes),
        _ptr(w_scale), _ptr(colsum), _ptr(bias_f32), _ptr(Y), _ptr(acc_debug), _stream(stream)),
        "hq_linear")


def hq_forward_host(desc: LayerDesc, X_host, X_dev, sigma_inv, a_codes, a_scale, a_mean,
                    workspace, w_codes, w_scale, colsum, bias_f32, Y_dev, Y_host, chunks=8,
                    T=None, stream=None):
    """The layer end to end on (pinned) host tensors: uploads, kernels and
    downloads of `chunks` row chunks overlapped (see include/hq.h).  X_host
    and Y_host are CPU tensors; X_dev, Y_dev device staging tensors."""
    T = X_host.shape[0] if T is None else T
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().hq_forward_host(
        ctypes.byref(desc), _host_ptr(X_host), T, _ptr(X_dev), _ptr(sigma_inv), _ptr(a_codes),
        _ptr(a_scale), _ptr(a_mean), _ptr(workspace), ws_bytes, _ptr(w_codes), _ptr(w_scale),
        _ptr(colsum), _ptr(bias_f32), _ptr(Y_dev), _host_ptr(Y_host), int(chunks),
        _stream(stream)), "hq_forward_host")


def hq_quantize_act_noalloc(desc: LayerDesc, X, sigma_inv, a_codes, a_scale, a_mean=None,
                            T=None, stream=None):
    """hq_quantize_act for callers that cannot allocate device memory: the
    per-tensor scale's workspace is a fixed 256-byte device array inside the
    library (see include/hq.h).  The first call on a device looks up that
    array's address, so make it before any stream capture; calls that overlap
    on the GPU share the array and race."""
    T = X.shape[0] if T is None else T
    _check(load_library().hq_quantize_act_noalloc(
        ctypes.byref(desc), _ptr(X), T, _ptr(sigma_inv), _ptr(a_codes), _ptr(a_scale),
        _ptr(a_mean), _stream(stream)), "hq_quantize_act_noalloc")


def hq_check_device_error(stream=None) -> int:
    """Synchronizes the stream and returns (and clears) the device error word."""
    return load_library().hq_check_device_error(_stream(stream))


def hq_debug_set_wait_limit(nanoseconds: int):
    _check(load_library().hq_debug_set_wait_limit(int(nanoseconds)), "hq_debug_set_wait_limit")


def hq_debug_inject_fault(kind: int):
    _check(load_library().hq_debug_inject_fault(int(kind)), "hq_debug_inject_fault")


def hq_debug_plan(desc: LayerDesc, T: int, sms: int, pair_clusters: int) -> dict:
    """The launch shapes the library chooses for desc and T tokens on a device
    with `sms` SMs and `pair_clusters` CTA-pair clusters (host only)."""
    out = [ctypes.c_int32(0) for _ in range(4)]
    _check(load_library().hq_debug_plan(ctypes.byref(desc), int(T), int(sms), int(pair_clusters),
                                        *(ctypes.byref(o) for o in out)), "hq_debug_plan")
    return {"quant_rows": out[0].value, "quant_threads": out[1].value,
            "gemm_pair": bool(out[2].value), "gemm_bn": out[3].value}


def hq_debug_mma_ceiling(pair: bool, k_blocks: int, stream=None) -> int:
    """Launches the MMA-only loop (int8 tensor-core ceiling) on the stream;
    returns the number of CTAs launched (ops = ctas * k_blocks * 4 * 2 *
    128 * 256 * 32)."""
    lib = load_library()
    n = ctypes.c_int32(0)
    _check(lib.hq_debug_mma_ceiling(1 if pair else 0, int(k_blocks), ctypes.byref(n),
                                    _stream(stream)), "hq_debug_mma_ceiling")
    return int(n.value)


def hq_debug_tmap_cache() -> dict:
    """Cumulative tensor-map cache hits and misses of the library."""
    h, m = ctypes.c_uint64(0), ctypes.c_uint64(0)
    _check(load_library().hq_debug_tmap_cache(ctypes.byref(h), ctypes.byref(m)),
           "hq_debug_tmap_cache")
    return {"hits": int(h.value), "misses": int(m.value)}


def hq_debug_set_gemm_variant(variant: int):
    """Selects the GEMM kernel of later hq_linear calls (HQ_GEMM_*)."""
    _check(load_library().hq_debug_set_gemm_variant(int(variant)), "hq_debug_set_gemm_variant")


# ---------------------------------------------------------------------------
# group-wise form (include/hq_gw.h), same names
# ---------------------------------------------------------------------------

def hq_debug_last_cuda_error() -> int:
    """The code behind the last HQ_ERR_CUDA (cleared by reading)."""
    return int(load_library().hq_debug_last_cuda_error())


def hq_gw_scale_ld(T: int) -> int:
    """Leading dimension of the [K/64][ld] activation scale array for T tokens."""
    return int(load_library().hq_gw_scale_ld(int(T)))


def hq_gw_sigma_inv(desc: GwDesc, W, act_absmax, alpha, sigma_inv, stream=None):
    _check(load_library().hq_gw_sigma_inv(ctypes.byref(desc), _ptr(W), _ptr(act_absmax),
                                          float(alpha), _ptr(sigma_inv), _stream(stream)),
           "hq_gw_sigma_inv")


def hq_gw_prepare_weights(desc: GwDesc, W, bias, sigma_inv, L1, L2, w_codes, w_scale, l1s, l2b,
                          bias_f32, stream=None):
    _check(load_library().hq_gw_prepare_weights(
        ctypes.byref(desc), _ptr(W), _ptr(bias), _ptr(sigma_inv), _ptr(L1), _ptr(L2),
        _ptr(w_codes), _ptr(w_scale), _ptr(l1s), _ptr(l2b), _ptr(bias_f32), _stream(stream)),
        "hq_gw_prepare_weights")


def hq_gw_quantize_act_workspace_bytes(desc: GwDesc, T: int) -> int:
    return int(load_library().hq_gw_quantize_act_workspace_bytes(ctypes.byref(desc), int(T)))


def hq_gw_quantize_act(desc: GwDesc, X, sigma_inv, l1s, a_codes, a_scale, u, workspace=None,
                       T=None, stream=None):
    T = X.shape[0] if T is None else T
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().hq_gw_quantize_act(
        ctypes.byref(desc), _ptr(X), T, _ptr(sigma_inv), _ptr(l1s), _ptr(a_codes), _ptr(a_scale),
        _ptr(u), _ptr(workspace), ws_bytes, _stream(stream)), "hq_gw_quantize_act")


def hq_gw_linear(desc: GwDesc, a_codes, a_scale, u, w_codes, w_scale, l2b, bias_f32, Y, T=None,
                 stream=None):
    T = a_codes.shape[0] if T is None else T
    _check(load_library().hq_gw_linear(
        ctypes.byref(desc), T, _ptr(a_codes), _ptr(a_scale), _ptr(u), _ptr(w_codes),
        _ptr(w_scale), _ptr(l2b), _ptr(bias_f32), _ptr(Y), _stream(stream)), "hq_gw_linear")


def hq_gw_debug_linear_f32(desc: GwDesc, a_codes, a_scale, u, w_codes, w_scale, l2b, bias_f32,
                           Y32, T=None, stream=None):
    T = a_codes.shape[0] if T is None else T
    _check(load_library().hq_gw_debug_linear_f32(
        ctypes.byref(desc), T, _ptr(a_codes), _ptr(a_scale), _ptr(u), _ptr(w_codes),
        _ptr(w_scale), _ptr(l2b), _ptr(bias_f32), _ptr(Y32), _stream(stream)),
        "hq_gw_debug_linear_f32")


# ---------------------------------------------------------------------------
# one layer's caller-side buffers
# ---------------------------------------------------------------------------

class HadamardQuantLinear:
    """Prepared weights and activation buffers of one Hadamard-domain layer.

    Allocation is the caller's (PyTorch); the library only reads and writes the
    tensors it is given.  `forward(X)` = hq_quantize_act + hq_linear."""

    def __init__(self, desc: LayerDesc, W, bias=None, act_absmax=None, alpha=0.5, device=None,
                 static_scale=None):
        """static_scale: the activation scale s (real units, code = rne(V / s))
        of HQ_PER_TENSOR_STATIC, required in that mode and refused in the
        others; it is written into a_scale[0] of every buffer set."""
        import torch
        self.static_scale = self._check_static_scale(desc, static_scale)
        self.desc = desc
        dev = W.device if device is None else device
        K, N = desc.K, desc.N
        self.w_codes = torch.empty((N, K), dtype=torch.int8, device=dev)
        self.w_scale = torch.empty(N, dtype=torch.float32, device=dev)
        self.colsum = torch.empty(N, dtype=torch.float32, device=dev)
        self.sigma_inv = torch.empty(K, dtype=torch.float32, device=dev)
        self.bias_f32 = torch.empty(N, dtype=torch.float32, device=dev)
        self.use_sigma = act_absmax is not None
        hq_prepare_weights(desc, W, bias, act_absmax, alpha, self.w_codes, self.w_scale,
                           self.colsum, self.sigma_inv, self.bias_f32)
        ws = hq_quantize_act_workspace_bytes(desc, 0)
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev) if ws else None
        self._bufs = {}

    def buffers(self, T: int):
        import torch
        b = self._bufs.get(T)
        if b is None:
            dev = self.w_codes.device
            per_row = self.desc.act_gran == HQ_PER_TOKEN
            if self.desc.code_format == HQ_CODES_I4_PACKED:  # two codes per byte
                codes = torch.empty((T, self.desc.K // 2), dtype=torch.uint8, device=dev)
            else:
                codes = torch.empty((T, self.desc.K), dtype=torch.int8, device=dev)
            b = {"a_codes": codes,
                 "a_scale": torch.empty(T if per_row else 1, dtype=torch.float32, device=dev),
                 "a_mean": torch.empty(T, dtype=torch.float32, device=dev)}
            if self.desc.act_gran == HQ_PER_TENSOR_STATIC:
                # an input of the quantizer and of the GEMM in this mode
                b["a_scale"].fill_(self.static_scale)
            self._bufs[T] = b
        return b

    @staticmethod
    def _check_static_scale(desc, static_scale):
        if desc.act_gran == HQ_PER_TENSOR_STATIC:
            if static_scale is None:
                raise ValueError("HQ_PER_TENSOR_STATIC needs static_scale (the activation scale)")
            v = float(static_scale)
            if not (v > 0.0 and v < float("inf")):
                raise ValueError(f"static_scale must be positive and finite, got {v}")
            return v
        if static_scale is not None:
            raise ValueError("static_scale is only used with HQ_PER_TENSOR_STATIC")
        return None

    def quantize(self, X):
        b = self.buffers(X.shape[0])
        hq_quantize_act(self.desc, X, self.sigma_inv if self.use_sigma else None, b["a_codes"],
                        b["a_scale"], b["a_mean"], self.workspace)
        return b

    def forward(self, X, Y=None, acc_debug=None):
        import torch
        T = X.shape[0]
        if Y is None:
            Y = torch.empty((T, self.desc.N), dtype=torch.bfloat16, device=X.device)
        b = self.quantize(X)
        mean = b["a_mean"] if self.desc.centering != HQ_CENTER_NONE else None
        hq_linear(self.desc, b["a_codes"], b["a_scale"], mean, self.w_codes, self.w_scale,
                  self.colsum, self.bias_f32, Y, acc_debug)
        return Y

    __call__ = forward

    def forward_host(self, X_host, Y_host=None, chunks=8):
        """Y_host = the layer on X_host (pinned CPU bf16 tensors), with the
        uploads, kernels and downloads of `chunks` row chunks overlapped
        (hq_forward_host).  Device staging buffers are kept per token count."""
        import torch
        T = X_host.shape[0]
        b = self.buffers(T)
        dev = self.w_codes.device
        if "X_dev" not in b:
            b["X_dev"] = torch.empty((T, self.desc.K), dtype=torch.bfloat16, device=dev)
            b["Y_dev"] = torch.empty((T, self.desc.N), dtype=torch.bfloat16, device=dev)
        if Y_host is None:
            Y_host = torch.empty((T, self.desc.N), dtype=torch.bfloat16).pin_memory()
        hq_forward_host(self.desc, X_host, b["X_dev"], self.sigma_inv if self.use_sigma else None,
                        b["a_codes"], b["a_scale"], b["a_mean"], self.workspace, self.w_codes,
                        self.w_scale, self.colsum, self.bias_f32, b["Y_dev"], Y_host, chunks)
        return Y_host

    # ------------------------------------------------------------------
    # prepared-weights blob (deployment: skip hq_prepare_weights at load)
    # ------------------------------------------------------------------
    # Little-endian layout:
    #   b"HQPW", u32 version (2), 9 x i32 hq_layer_desc fields in header order,
    #   u32 use_sigma, f64 static_scale (0 when the mode has none; version 2
    #   only -- version 1 blobs, without it, still load), then five sections,
    #   each u64 byte count + payload:
    #   w_codes int8 [N*K], w_scale f32 [N], colsum f32 [N], sigma_inv f32 [K],
    #   bias_f32 f32 [N]; then u32 CRC-32 of everything before it.
    _BLOB_MAGIC = b"HQPW"
    _BLOB_VERSION = 2

    def export_prepared(self) -> bytes:
        """The prepared weights and the layer description as one blob."""
        import struct
        import zlib
        import numpy as np
        d = self.desc
        head = self._BLOB_MAGIC + struct.pack("<I", self._BLOB_VERSION)
        head += struct.pack("<9i", d.K, d.N, d.had_order, d.a_bits, d.w_bits, d.act_gran,
                            d.centering, d.code_format, d.out_order)
        head += struct.pack("<I", 1 if self.use_sigma else 0)
        head += struct.pack("<d", self.static_scale if self.static_scale is not None else 0.0)
        parts = [head]
        for t, dt in ((self.w_codes, np.int8), (self.w_scale, np.float32),
                      (self.colsum, np.float32), (self.sigma_inv, np.float32),
                      (self.bias_f32, np.float32)):
            raw = t.detach().contiguous().cpu().numpy().astype(dt, copy=False).tobytes()
            parts.append(struct.pack("<Q", len(raw)) + raw)
        body = b"".join(parts)
        return body + struct.pack("<I", zlib.crc32(body) & 0xFFFFFFFF)

    @classmethod
    def from_prepared(cls, blob: bytes, device=None) -> "HadamardQuantLinear":
        """A layer from export_prepared()'s blob, without running the weight
        preparation.  Raises ValueError on a malformed or corrupted blob."""
        import struct
        import zlib
        import numpy as np
        import torch
        blob = bytes(blob)
        if len(blob) < 4 + 4 + 36 + 4 + 4 or blob[:4] != cls._BLOB_MAGIC:
            raise ValueError("not a prepared-weights blob")
        body, crc = blob[:-4], struct.unpack("<I", blob[-4:])[0]
        if zlib.crc32(body) & 0xFFFFFFFF != crc:
            raise ValueError("prepared-weights blob: checksum mismatch")
        version = struct.unpack_from("<I", body, 4)[0]
        if version not in (1, cls._BLOB_VERSION):
            raise ValueError(f"prepared-weights blob: unsupported version {version}")
        f = struct.unpack_from("<9i", body, 8)
        desc = LayerDesc(f[0], f[1], f[2], a_bits=f[3], w_bits=f[4], act_gran=f[5],
                         centering=f[6], code_format=f[7], out_order=f[8])
        use_sigma = bool(struct.unpack_from("<I", body, 44)[0])
        K, N = desc.K, desc.N
        off = 48
        static_scale = None
        if version >= 2:
            if len(body) < off + 8:
                raise ValueError("prepared-weights blob: truncated")
            s_val = struct.unpack_from("<d", body, off)[0]
            off += 8
            if desc.act_gran == HQ_PER_TENSOR_STATIC:
                static_scale = s_val
        try:
            static_scale = cls._check_static_scale(desc, static_scale)
        except ValueError as e:
            raise ValueError(f"prepared-weights blob: {e}") from None
        arrays = []
        for dt, count in ((np.int8, N * K), (np.float32, N), (np.float32, N), (np.float32, K),
                          (np.float32, N)):
            if off + 8 > len(body):
                raise ValueError("prepared-weights blob: truncated")
            nbytes = struct.unpack_from("<Q", body, off)[0]
            off += 8
            if nbytes != count * np.dtype(dt).itemsize or off + nbytes > len(body):
                raise ValueError("prepared-weights blob: section size does not match the description")
            arrays.append(np.frombuffer(body, dtype=dt, count=count, offset=off).copy())
            off += nbytes
        if off != len(body):
            raise ValueError("prepared-weights blob: trailing bytes")
        dev = torch.device("cuda") if device is None else torch.device(device)
        self = cls.__new__(cls)
        self.desc = desc
        self.w_codes = torch.from_numpy(arrays[0].reshape(N, K)).to(dev)
        self.w_scale, self.colsum, self.sigma_inv, self.bias_f32 = (
            torch.from_numpy(a).to(dev) for a in arrays[1:])
        self.use_sigma = use_sigma
        self.static_scale = static_scale
        ws = hq_quantize_act_workspace_bytes(desc, 0) if dev.type == "cuda" else 0
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev) if ws else None
        self._bufs = {}
        return self


class GroupWiseQuantLinear:
    """Prepared weights and activation buffers of one group-wise layer
    (include/hq_gw.h): 64-channel groups, each with its own H_64 block and
    scale, and a rank-`rank` 16-bit branch.  `forward(X)` =
    hq_gw_quantize_act + hq_gw_linear.

    The low-rank factors are an input of the weight preparation: `factors` =
    (L1 [rank,K], L2 [N,rank]) of W diag(sigma), or None to take them here
    from a singular value decomposition of W diag(sigma) (torch.linalg.svd in
    fp32 on the device, an offline step; the method fixes only L2 L1)."""

    def __init__(self, desc: GwDesc, W, bias=None, act_absmax=None, alpha=0.5, factors=None,
                 sigma_inv=None):
        """sigma_inv: a given smoothing vector (fp32 [K]) instead of the one
        hq_gw_sigma_inv derives from act_absmax and alpha."""
        import torch
        self.desc = desc
        dev = W.device
        K, N, r = desc.K, desc.N, desc.rank
        if sigma_inv is not None:
            self.sigma_inv = sigma_inv.to(device=dev, dtype=torch.float32).contiguous()
            if tuple(self.sigma_inv.shape) != (K,):
                raise ValueError(f"sigma_inv must have shape ({K},)")
            self.use_sigma = True
        else:
            self.sigma_inv = torch.empty(K, dtype=torch.float32, device=dev)
            hq_gw_sigma_inv(desc, W, act_absmax, alpha, self.sigma_inv)
            self.use_sigma = act_absmax is not None
        if r > 0:
            if factors is None:
                What = W.float() / self.sigma_inv[None, :]
                U, S, Vh = torch.linalg.svd(What, full_matrices=False)
                k = min(r, S.numel())  # beyond min(N, K) the factors are zero
                L1 = torch.zeros((r, K), dtype=torch.float32, device=dev)
                L2 = torch.zeros((N, r), dtype=torch.float32, device=dev)
                L1[:k] = Vh[:k]
                L2[:, :k] = U[:, :k] * S[:k]
                factors = (L1, L2)
            L1, L2 = (f.to(device=dev, dtype=torch.float32).contiguous() for f in factors)
            if tuple(L1.shape) != (r, K) or tuple(L2.shape) != (N, r):
                raise ValueError(f"factors must be L1 [{r},{K}] and L2 [{N},{r}], got "
                                 f"{tuple(L1.shape)} and {tuple(L2.shape)}")
            self.factors = (L1, L2)  # fp32, as given to the weight preparation
            self.l1s = torch.empty((r, K), dtype=torch.bfloat16, device=dev)
            self.l2b = torch.empty((N, r), dtype=torch.bfloat16, device=dev)
        else:
            L1 = L2 = None
            self.factors = None
            self.l1s = self.l2b = None
        self.w_codes = torch.empty((N, K), dtype=torch.float8_e4m3fn, device=dev)
        self.w_scale = torch.empty((K // 64, N), dtype=torch.float32, device=dev)
        self.bias_f32 = torch.empty(N, dtype=torch.float32, device=dev)
        hq_gw_prepare_weights(desc, W, bias, self.sigma_inv if self.use_sigma else None, L1, L2,
                              self.w_codes, self.w_scale, self.l1s, self.l2b, self.bias_f32)
        self._bufs = {}

    def buffers(self, T: int):
        import torch
        b = self._bufs.get(T)
        if b is None:
            dev = self.w_codes.device
            K, r = self.desc.K, self.desc.rank
            ws = hq_gw_quantize_act_workspace_bytes(self.desc, T)
            b = {"a_codes": torch.empty((T, K), dtype=torch.float8_e4m3fn, device=dev),
                 "a_scale": torch.empty((K // 64, hq_gw_scale_ld(T)), dtype=torch.float32,
                                        device=dev),
                 "u": torch.empty((T, r), dtype=torch.bfloat16, device=dev) if r else None,
                 "workspace": torch.empty(ws, dtype=torch.uint8, device=dev) if ws else None}
            self._bufs[T] = b
        return b

    def quantize(self, X):
        b = self.buffers(X.shape[0])
        hq_gw_quantize_act(self.desc, X, self.sigma_inv if self.use_sigma else None, self.l1s,
                           b["a_codes"], b["a_scale"], b["u"], b["workspace"])
        return b

    def forward(self, X, Y=None):
        import torch
        if Y is None:
            Y = torch.empty((X.shape[0], self.desc.N), dtype=torch.bfloat16, device=X.device)
        b = self.quantize(X)
        hq_gw_linear(self.desc, b["a_codes"], b["a_scale"], b["u"], self.w_codes, self.w_scale,
                     self.l2b, self.bias_f32, Y, T=X.shape[0])
        return Y

    __call__ = forward


"""Python binding of libpoetx, the B200 (sm_100a) POET-X layer library.

Argument marshalling only: every function here has the name and the arguments of the C entry
point it wraps (include/poetx.h) and passes device pointers, sizes and the stream through
ctypes.  Array arguments may be torch tensors (their data_ptr() is passed), integers (raw
device addresses) or None (NULL).  A non-OK status raises PoetxError.  There is no fallback:
if libpoetx.so has not been built the first call raises.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "poetx_desc", "PoetxError", "POETX_F32", "POETX_BF16", "POETX_FAST", "POETX_MEM", "STATUS",
    "lib", "library_path", "exported_symbols", "poetx_workspace_size", "poetx_cnp", "poetx_cnp_blocks",
    "poetx_cnp_blocks_workspace_size", "poetx_absorb", "poetx_forward", "poetx_backward",
    "poetx_merge", "poetx_status_string", "poetx_device_status", "poetx_test_gemm",
    "poetx_launch_count", "poetx_profile_enable", "poetx_profile_summary", "KERNEL_CLASSES",
    "poetx_cnp_blocks_noalloc", "poetx_adamw_cfg", "poetx_adamw_step",
    "poetx_adamw_reset", "poetx_wc_saved_size", "poetx_wc_workspace_size", "poetx_wc_forward", "poetx_wc_backward",
    "poetx_xq_quantize", "poetx_xq_dequantize", "poetx_xq_forward", "poetx_xq_backward", "poetx_xq_merge",
    "poetx_check_permutation", "poetx_test_wait_timeout", "poetx_cnp_forward", "poetx_fourperm_workspace_size",
    "poetx_fourperm_forward", "poetx_fourperm_backward",
]

POETX_F32, POETX_BF16 = 0, 1
POETX_FAST, POETX_MEM = 0, 1
STATUS = {
    0: "POETX_OK", 1: "POETX_ERR_INVALID_ARG", 2: "POETX_ERR_UNSUPPORTED_SHAPE", 3: "POETX_ERR_ALIGNMENT",
    4: "POETX_ERR_WORKSPACE", 5: "POETX_ERR_CUDA", 6: "POETX_ERR_DEVICE_TIMEOUT",
}

KERNEL_CLASSES = ["w_gemm", "bd_gemm", "grad_gemm", "cnp_gemm", "merge_gemm", "permute", "elementwise", "test_gemm",
                  "optimizer", "w_gemm_adj", "cnp_adj"]

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(_HERE, "libpoetx.so")


class poetx_desc(ctypes.Structure):
    _fields_ = [("d_in", ctypes.c_int), ("d_out", ctypes.c_int), ("b", ctypes.c_int), ("k", ctypes.c_int),
                ("dtype", ctypes.c_int), ("mode", ctypes.c_int)]

    def __repr__(self):
        return (f"poetx_desc(d_in={self.d_in}, d_out={self.d_out}, b={self.b}, k={self.k}, "
                f"dtype={self.dtype}, mode={self.mode})")


class poetx_adamw_cfg(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("gamma", ctypes.c_float), ("beta1", ctypes.c_float),
                ("beta2", ctypes.c_float), ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float)]


class PoetxError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_LL = ctypes.c_longlong
_D = ctypes.POINTER(poetx_desc)

_SIGNATURES = {
    "poetx_workspace_size": (_SZ, [_D, _I]),
    "poetx_cnp_blocks_workspace_size": (_SZ, [_D, _I]),
    "poetx_cnp": (_I, [_D, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_cnp_blocks": (_I, [_D, _I, _P, _P, _P, _SZ, _P]),
    "poetx_cnp_blocks_noalloc": (_I, [_D, _I, _P, _P, _P]),
    "poetx_absorb": (_I, [_D, _P, _P, _P, _P, _P]),
    "poetx_forward": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_cnp_forward": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_backward": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_merge": (_I, [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_adamw_step": (_I, [ctypes.POINTER(poetx_adamw_cfg), _LL, _I, _P, _P, _P, _P, _P]),
    "poetx_adamw_reset": (_I, [_LL, _P, _P, _P]),
    "poetx_wc_saved_size": (_SZ, [_D]),
    "poetx_wc_workspace_size": (_SZ, [_D]),
    "poetx_wc_forward": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_wc_backward": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_xq_quantize": (_I, [_D, _P, _P, _P, _P]),
    "poetx_xq_dequantize": (_I, [_D, _P, _P, _P, _P]),
    "poetx_xq_forward": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_xq_backward": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_xq_merge": (_I, [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_check_permutation": (_I, [_P, _I]),
    "poetx_fourperm_workspace_size": (_SZ, [_D, _I]),
    "poetx_fourperm_forward": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_fourperm_backward": (_I, [_D, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "poetx_test_wait_timeout": (_I, [_LL, _P, _P]),
    "poetx_status_string": (ctypes.c_char_p, [_I]),
    "poetx_device_status": (_I, [ctypes.POINTER(ctypes.c_int)]),
    "poetx_launch_count": (ctypes.c_ulonglong, []),
    "poetx_profile_enable": (_I, [_I]),
    "poetx_profile_summary": (_I, [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_float)]),
    "poetx_test_gemm": (_I, [_I, _I, _I, _I, _I, _I,
                             _P, _LL, _LL, _LL, _LL, _LL, _I,
                             _P, _LL, _LL, _LL, _LL, _LL, _I,
                             _P, _I, _LL, _LL, _LL, _LL, ctypes.c_float, ctypes.c_float, _P,
                             _LL, _LL, _LL, _I, _P]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Loads libpoetx.so (built in-tree by orthogonal_equivalence_cnp_b200.build)."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m orthogonal_equivalence_cnp_b200.build`")
        handle = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def exported_symbols():
    return sorted(_SIGNATURES)


def _ptr(x):
    """Device address of an array argument: a CUDA tensor (contiguous; checked), a raw device
    address (int, the caller's responsibility) or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not getattr(x, "is_cuda", False):
        raise ValueError("array arguments must be CUDA tensors (or raw device addresses)")
    if not x.is_contiguous():
        raise ValueError("array arguments must be contiguous")
    return x.data_ptr()


def _need(x, name, numel, dtype=None):
    """Checks that tensor x (if it is one) holds at least `numel` elements of `dtype`; the library
    cannot see sizes, so a short buffer would be written past its end."""
    if x is None or isinstance(x, int):
        return
    import torch
    if dtype is not None and x.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {x.dtype}")
    if x.numel() < numel:
        raise ValueError(f"{name}: needs at least {numel} elements, has {x.numel()}")


def _act_dtype(desc):
    import torch
    return torch.bfloat16 if desc.dtype == POETX_BF16 else torch.float32


def _check_layer(desc, n_tokens=0, **arrays):
    """Size and type checks of the layer arrays by name (theta_*, Q_*, X, Y, dY, dX, W0p, perm_*)."""
    import torch
    b, din, dout, dt = desc.b, desc.d_in, desc.d_out, _act_dtype(desc)
    P = b * (b - 1) // 2
    need = {"theta_R": (dout // b * P, torch.float32), "theta_P": (din // b * P, torch.float32),
            "grad_theta_R": (dout // b * P, torch.float32), "grad_theta_P": (din // b * P, torch.float32),
            "Q_R": (dout * b, dt), "Q_P": (din * b, dt), "W0p": (dout * din, dt),
            "X": (n_tokens * din, dt), "dX": (n_tokens * din, dt), "Y": (n_tokens * dout, dt),
            "dY": (n_tokens * dout, dt), "perm_L": (dout, torch.int32), "perm_R": (din, torch.int32)}
    for name, x in arrays.items():
        key = name.replace("_old", "").replace("_new", "")
        if key in need:
            _need(x, name, *need[key])


def _nbytes(x):
    if x is None:
        return 0
    return x.numel() * x.element_size()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, where: str):
    if status != 0:
        raise PoetxError(status, where)


def poetx_status_string(status: int) -> str:
    return lib().poetx_status_string(status).decode()


def poetx_workspace_size(desc: poetx_desc, n_tokens: int) -> int:
    return lib().poetx_workspace_size(ctypes.byref(desc), n_tokens)


def poetx_cnp_blocks_workspace_size(desc: poetx_desc, n_blocks: int) -> int:
    return lib().poetx_cnp_blocks_workspace_size(ctypes.byref(desc), n_blocks)


def poetx_cnp(desc, theta_R, theta_P, Q_R, Q_P, workspace, ws_bytes=None, stream=None):
    _check_layer(desc, theta_R=theta_R, theta_P=theta_P, Q_R=Q_R, Q_P=Q_P)
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_cnp(ctypes.byref(desc), _ptr(theta_R), _ptr(theta_P), _ptr(Q_R), _ptr(Q_P),
                           _ptr(workspace), ws_bytes, _stream(stream)), "poetx_cnp")


def _check_blocks(desc, n_blocks, theta, Q):
    import torch
    b = desc.b
    _need(theta, "theta", n_blocks * b * (b - 1) // 2, torch.float32)
    _need(Q, "Q", n_blocks * b * b, _act_dtype(desc))


def poetx_cnp_blocks(desc, n_blocks, theta, Q, workspace, ws_bytes=None, stream=None):
    _check_blocks(desc, n_blocks, theta, Q)
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_cnp_blocks(ctypes.byref(desc), n_blocks, _ptr(theta), _ptr(Q), _ptr(workspace), ws_bytes,
                                  _stream(stream)), "poetx_cnp_blocks")


def poetx_absorb(desc, W0, perm_L, perm_R, W0p, stream=None):
    _check(lib().poetx_absorb(ctypes.byref(desc), _ptr(W0), _ptr(perm_L), _ptr(perm_R), _ptr(W0p),
                              _stream(stream)), "poetx_absorb")


def poetx_forward(desc, n_tokens, X, W0p, perm_L, perm_R, Q_R, Q_P, Y, saved, workspace, ws_bytes=None,
                  stream=None):
    _check_layer(desc, n_tokens, X=X, W0p=W0p, perm_L=perm_L, perm_R=perm_R, Q_R=Q_R, Q_P=Q_P, Y=Y)
    if saved is not None and not isinstance(saved, int):
        _need(saved, "saved", n_tokens * (desc.d_in + desc.d_out), _act_dtype(desc))
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_forward(ctypes.byref(desc), n_tokens, _ptr(X), _ptr(W0p), _ptr(perm_L), _ptr(perm_R),
                               _ptr(Q_R), _ptr(Q_P), _ptr(Y), _ptr(saved), _ptr(workspace), ws_bytes,
                               _stream(stream)), "poetx_forward")


def poetx_cnp_forward(desc, n_tokens, X, W0p, perm_L, perm_R, theta_R, theta_P, Q_R, Q_P, Y, saved, workspace,
                      ws_bytes=None, stream=None):
    _check_layer(desc, n_tokens, X=X, W0p=W0p, perm_L=perm_L, perm_R=perm_R, theta_R=theta_R, theta_P=theta_P,
                 Q_R=Q_R, Q_P=Q_P, Y=Y)
    if saved is not None and not isinstance(saved, int):
        _need(saved, "saved", n_tokens * (desc.d_in + desc.d_out), _act_dtype(desc))
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_cnp_forward(ctypes.byref(desc), n_tokens, _ptr(X), _ptr(W0p), _ptr(perm_L), _ptr(perm_R),
                                   _ptr(theta_R), _ptr(theta_P), _ptr(Q_R), _ptr(Q_P), _ptr(Y), _ptr(saved),
                                   _ptr(workspace), ws_bytes, _stream(stream)), "poetx_cnp_forward")


def poetx_backward(desc, n_tokens, dY, X, W0p, perm_L, perm_R, Q_R, Q_P, theta_R, theta_P, saved, dX,
                   grad_theta_R, grad_theta_P, workspace, ws_bytes=None, stream=None):
    _check_layer(desc, n_tokens, dY=dY, X=X, W0p=W0p, perm_L=perm_L, perm_R=perm_R, Q_R=Q_R, Q_P=Q_P,
                 theta_R=theta_R, theta_P=theta_P, dX=dX, grad_theta_R=grad_theta_R, grad_theta_P=grad_theta_P)
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_backward(ctypes.byref(desc), n_tokens, _ptr(dY), _ptr(X), _ptr(W0p), _ptr(perm_L),
                                _ptr(perm_R), _ptr(Q_R), _ptr(Q_P), _ptr(theta_R), _ptr(theta_P), _ptr(saved),
                                _ptr(dX), _ptr(grad_theta_R), _ptr(grad_theta_P), _ptr(workspace),
                                ws_bytes, _stream(stream)), "poetx_backward")


def poetx_adamw_step(cfg, n, t, theta, grad, m, v, stream=None):
    _check(lib().poetx_adamw_step(ctypes.byref(cfg), n, t, _ptr(theta), _ptr(grad), _ptr(m), _ptr(v),
                                  _stream(stream)), "poetx_adamw_step")


def poetx_adamw_reset(n, m, v, stream=None):
    _check(lib().poetx_adamw_reset(n, _ptr(m), _ptr(v), _stream(stream)), "poetx_adamw_reset")


def poetx_wc_saved_size(desc) -> int:
    return lib().poetx_wc_saved_size(ctypes.byref(desc))


def poetx_wc_workspace_size(desc) -> int:
    return lib().poetx_wc_workspace_size(ctypes.byref(desc))


def poetx_wc_forward(desc, n_tokens, X, W0p, perm_L, perm_R, Q_R, Q_P, Y, wc_saved, workspace, ws_bytes=None,
                     stream=None):
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_wc_forward(ctypes.byref(desc), n_tokens, _ptr(X), _ptr(W0p), _ptr(perm_L), _ptr(perm_R),
                                  _ptr(Q_R), _ptr(Q_P), _ptr(Y), _ptr(wc_saved), _ptr(workspace), ws_bytes,
                                  _stream(stream)), "poetx_wc_forward")


def poetx_wc_backward(desc, n_tokens, dY, X, W0p, perm_L, perm_R, Q_R, theta_R, theta_P, wc_saved, dX, grad_theta_R,
                      grad_theta_P, workspace, ws_bytes=None, stream=None):
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_wc_backward(ctypes.byref(desc), n_tokens, _ptr(dY), _ptr(X), _ptr(W0p), _ptr(perm_L),
                                   _ptr(perm_R), _ptr(Q_R), _ptr(theta_R), _ptr(theta_P), _ptr(wc_saved), _ptr(dX),
                                   _ptr(grad_theta_R), _ptr(grad_theta_P), _ptr(workspace), ws_bytes,
                                   _stream(stream)), "poetx_wc_backward")


def poetx_merge(desc, W0p, Q_R, Q_P, perm_L_old, perm_R_old, perm_L_new, perm_R_new, theta_R, theta_P, workspace,
                ws_bytes=None, stream=None):
    _check_layer(desc, W0p=W0p, Q_R=Q_R, Q_P=Q_P, perm_L_old=perm_L_old, perm_R_old=perm_R_old,
                 perm_L_new=perm_L_new, perm_R_new=perm_R_new, theta_R=theta_R, theta_P=theta_P)
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_merge(ctypes.byref(desc), _ptr(W0p), _ptr(Q_R), _ptr(Q_P), _ptr(perm_L_old),
                             _ptr(perm_R_old), _ptr(perm_L_new), _ptr(perm_R_new), _ptr(theta_R), _ptr(theta_P),
                             _ptr(workspace), ws_bytes, _stream(stream)), "poetx_merge")


def poetx_xq_quantize(desc, W0p, W0q, W0s, stream=None):
    _check(lib().poetx_xq_quantize(ctypes.byref(desc), _ptr(W0p), _ptr(W0q), _ptr(W0s), _stream(stream)),
           "poetx_xq_quantize")


def poetx_xq_dequantize(desc, W0q, W0s, W0p, stream=None):
    _check(lib().poetx_xq_dequantize(ctypes.byref(desc), _ptr(W0q), _ptr(W0s), _ptr(W0p), _stream(stream)),
           "poetx_xq_dequantize")


def poetx_xq_forward(desc, n_tokens, X, W0q, W0s, perm_L, perm_R, Q_R, Q_P, Y, workspace, ws_bytes=None,
                     stream=None):
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_xq_forward(ctypes.byref(desc), n_tokens, _ptr(X), _ptr(W0q), _ptr(W0s), _ptr(perm_L),
                                  _ptr(perm_R), _ptr(Q_R), _ptr(Q_P), _ptr(Y), _ptr(workspace), ws_bytes,
                                  _stream(stream)), "poetx_xq_forward")


def poetx_xq_backward(desc, n_tokens, dY, X, W0q, W0s, perm_L, perm_R, Q_R, Q_P, theta_R, theta_P, dX,
                      grad_theta_R, grad_theta_P, workspace, ws_bytes=None, stream=None):
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_xq_backward(ctypes.byref(desc), n_tokens, _ptr(dY), _ptr(X), _ptr(W0q), _ptr(W0s),
                                   _ptr(perm_L), _ptr(perm_R), _ptr(Q_R), _ptr(Q_P), _ptr(theta_R), _ptr(theta_P),
                                   _ptr(dX), _ptr(grad_theta_R), _ptr(grad_theta_P), _ptr(workspace), ws_bytes,
                                   _stream(stream)), "poetx_xq_backward")


def poetx_xq_merge(desc, W0q, W0s, Q_R, Q_P, perm_L_old, perm_R_old, perm_L_new, perm_R_new, theta_R, theta_P,
                   workspace, ws_bytes=None, stream=None):
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_xq_merge(ctypes.byref(desc), _ptr(W0q), _ptr(W0s), _ptr(Q_R), _ptr(Q_P), _ptr(perm_L_old),
                                _ptr(perm_R_old), _ptr(perm_L_new), _ptr(perm_R_new), _ptr(theta_R),
                                _ptr(theta_P), _ptr(workspace), ws_bytes, _stream(stream)), "poetx_xq_merge")


def poetx_check_permutation(perm, n=None):
    """perm: a HOST int32 array (numpy or CPU tensor) or a raw host address; raises unless it is a
    bijection of [0, n)."""
    import numpy as np
    if isinstance(perm, int):
        if n is None:
            raise ValueError("a raw host address needs its length n")
        addr = perm
    else:
        arr = np.ascontiguousarray(np.asarray(perm), dtype=np.int32)
        if n is not None and n > arr.size:
            raise ValueError(f"n = {n} exceeds the array's {arr.size} elements")
        perm, addr, n = arr, arr.ctypes.data, arr.size if n is None else n
    _check(lib().poetx_check_permutation(addr, n), "poetx_check_permutation")


def poetx_device_status():
    """Returns (status, detail) after synchronising; status 0 means no device-side timeout."""
    d = ctypes.c_int(0)
    s = lib().poetx_device_status(ctypes.byref(d))
    return s, d.value


def poetx_test_gemm(dtype, M, N, K, batch, splits, a, a_rows, a_cols, a_ld, a_zrow, a_zcol, a_mn,
                    b, b_rows, b_cols, b_ld, b_zrow, b_zcol, b_mn, d, d_dtype, d_ld, d_zrow, d_zcol,
                    d_split_stride, alpha, beta, c, c_ld, c_zrow, c_zcol, diag, stream=None):
    """Test hook of the GEMM core (include/poetx_testing.h)."""
    _check(lib().poetx_test_gemm(dtype, M, N, K, batch, splits, _ptr(a), a_rows, a_cols, a_ld, a_zrow, a_zcol,
                                 a_mn, _ptr(b), b_rows, b_cols, b_ld, b_zrow, b_zcol, b_mn, _ptr(d), d_dtype,
                                 d_ld, d_zrow, d_zcol, d_split_stride, alpha, beta, _ptr(c), c_ld, c_zrow,
                                 c_zcol, diag, _stream(stream)), "poetx_test_gemm")


def poetx_launch_count() -> int:
    return lib().poetx_launch_count()


def poetx_profile_enable(on: bool):
    _check(lib().poetx_profile_enable(1 if on else 0), "poetx_profile_enable")


def poetx_profile_summary():
    """{class name: (launches, total device ms)} of the launches recorded since poetx_profile_enable(True)."""
    n = len(KERNEL_CLASSES)
    counts = (ctypes.c_int * n)()
    ms = (ctypes.c_float * n)()
    _check(lib().poetx_profile_summary(counts, ms), "poetx_profile_summary")
    return {KERNEL_CLASSES[i]: (counts[i], ms[i]) for i in range(n)}


def poetx_cnp_blocks_noalloc(desc, n_blocks, theta, Q, stream=None):
    """CNP forward that takes no workspace (built-in 32 MiB device scratch; see include/poetx.h)."""
    _check_blocks(desc, n_blocks, theta, Q)
    _check(lib().poetx_cnp_blocks_noalloc(ctypes.byref(desc), n_blocks, _ptr(theta), _ptr(Q), _stream(stream)),
           "poetx_cnp_blocks_noalloc")


def poetx_test_wait_timeout(limit_ns, returned, stream=None):
    _check(lib().poetx_test_wait_timeout(int(limit_ns), _ptr(returned), _stream(stream)), "poetx_test_wait_timeout")


def poetx_fourperm_workspace_size(desc, n_tokens):
    return lib().poetx_fourperm_workspace_size(ctypes.byref(desc), n_tokens)


def poetx_fourperm_forward(desc, n_tokens, X, W0, perm_L, perm_R, Q_R, Q_P, Y, saved, workspace, ws_bytes=None,
                           stream=None):
    _check_layer(desc, n_tokens, X=X, W0p=W0, perm_L=perm_L, perm_R=perm_R, Q_R=Q_R, Q_P=Q_P, Y=Y)
    _need(saved, "saved", n_tokens * (desc.d_in + desc.d_out), _act_dtype(desc))
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_fourperm_forward(ctypes.byref(desc), n_tokens, _ptr(X), _ptr(W0), _ptr(perm_L), _ptr(perm_R),
                                        _ptr(Q_R), _ptr(Q_P), _ptr(Y), _ptr(saved), _ptr(workspace), ws_bytes,
                                        _stream(stream)), "poetx_fourperm_forward")


def poetx_fourperm_backward(desc, n_tokens, dY, W0, perm_L, perm_R, Q_R, Q_P, theta_R, theta_P, saved, dX,
                            grad_theta_R, grad_theta_P, workspace, ws_bytes=None, stream=None):
    _check_layer(desc, n_tokens, dY=dY, W0p=W0, perm_L=perm_L, perm_R=perm_R, Q_R=Q_R, Q_P=Q_P, theta_R=theta_R,
                 theta_P=theta_P, dX=dX, grad_theta_R=grad_theta_R, grad_theta_P=grad_theta_P)
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check(lib().poetx_fourperm_backward(ctypes.byref(desc), n_tokens, _ptr(dY), _ptr(W0), _ptr(perm_L), _ptr(perm_R),
                                         _ptr(Q_R), _ptr(Q_P), _ptr(theta_R), _ptr(theta_P), _ptr(saved), _ptr(dX),
                                         _ptr(grad_theta_R), _ptr(grad_theta_P), _ptr(workspace), ws_bytes,
                                         _stream(stream)), "poetx_fourperm_backward")

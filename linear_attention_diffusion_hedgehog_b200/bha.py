"""ctypes binding for libbha (include/bha.h): argument marshalling only.

Every entry point takes torch tensors that already live on a CUDA device, checks their
dtype / shape / contiguity on the host, and passes raw device pointers, sizes and the
current CUDA stream to the C ABI.  All arithmetic runs in the library's CUDA kernels; there
is no CPU fallback, and calling any entry point without the built library raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbha.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "bha.h")

BHA_OK, BHA_ERR_INVALID, BHA_ERR_UNSUPPORTED, BHA_ERR_CUDA, BHA_ERR_TIMEOUT = 0, -1, -2, -3, -4
BHA_BF16, BHA_F32 = 0, 1
_DTYPE_CODE = {torch.bfloat16: BHA_BF16, torch.float32: BHA_F32}


class BhaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class Dims(ctypes.Structure):
    _fields_ = [
        ("num_requests", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("feature_dim", ctypes.c_int32),
        ("max_block", ctypes.c_int32),
        ("total_tokens", ctypes.c_int32),
        ("num_slots", ctypes.c_int32),
        ("act_dtype", ctypes.c_int32),
    ]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_SIGS = {
    "bha_featuremap": (ctypes.c_int, [ctypes.POINTER(Dims), _P, _I32, _P, _P, _I32, _P]),
    "bha_featuremap_checked": (ctypes.c_int, [ctypes.POINTER(Dims), _P, _I32, _P, _P, _I32, _P, _P]),
    "bha_hybrid_attn": (ctypes.c_int, [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                       _P, _P, _P]),
    "bha_commit_block": (ctypes.c_int, [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P, _P,
                                        _P]),
    "bha_hybrid_attn_commit": (ctypes.c_int, [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P,
                                              _P, _P, _P, _P, _P]),
    "bha_full_prefix_attn": (ctypes.c_int, [ctypes.POINTER(Dims), _P, _P, _P, _P, _P,
                                            ctypes.c_int64, _P, _P, ctypes.c_size_t, _P, _P]),
    "bha_full_prefix_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(Dims), ctypes.c_int64]),
    "bha_full_prefix_attn_noalloc": (ctypes.c_int, [ctypes.POINTER(Dims), _P, _P, _P, _P, _P,
                                                    ctypes.c_int64, _P, _P, _P]),
    "bha_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bha_kernel_variant": (ctypes.c_int, [ctypes.POINTER(Dims), _I32]),
    "bha_version": (ctypes.c_int, []),
    "bha_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_int64, _P, _P]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libbha.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libbha.so not found at {LIB_PATH}; build it with "
                "`python -m linear_attention_diffusion_hedgehog_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/bha.h declares."""
    src = open(HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bha_\w+)\s*\(", src)))


def selftest_bounded_wait(limit_cycles, dev_err, stream=None):
    """Runs the library's bounded wait on an mbarrier that never completes; dev_err (a device
    int32 tensor, zeroed by the caller) receives BHA_ERR_TIMEOUT once the wait gives up."""
    _cuda(dev_err, "dev_err", dtype=torch.int32)
    with torch.cuda.device(dev_err.device):  # the library uses the current device
        st = lib().bha_selftest_bounded_wait(int(limit_cycles), _ptr(dev_err),
                                             _stream(dev_err.device, stream))
    _check(st, "bha_selftest_bounded_wait")


def status_string(status: int) -> str:
    return lib().bha_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != BHA_OK:
        raise BhaError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device, stream=None):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _need(cond, msg):
    if not cond:
        raise ValueError(msg)


def _cuda(t, name, dtype=None, ndim=None):
    _need(isinstance(t, torch.Tensor), f"{name} must be a torch.Tensor")
    _need(t.is_cuda, f"{name} must be on a CUDA device")
    _need(t.is_contiguous(), f"{name} must be contiguous")
    if dtype is not None:
        _need(t.dtype == dtype, f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None:
        _need(t.dim() == ndim, f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    return t


def make_dims(R, Hq, Hkv, d, F, max_block, T, num_slots, act_dtype) -> Dims:
    return Dims(int(R), int(Hq), int(Hkv), int(d), int(F), int(max_block), int(T),
                int(num_slots), _DTYPE_CODE[act_dtype] if isinstance(act_dtype, torch.dtype)
                else int(act_dtype))


def kernel_variant(dims: Dims, which: int) -> int:
    return lib().bha_kernel_variant(ctypes.byref(dims), which)


# ----------------------------------------------------------------------- entry points

def featuremap(x, W, out_dtype=torch.float32, out=None, dev_err=None, stream=None):
    """phi(x) = [softmax(xW), softmax(-xW)] per head.  x [T, H, d]; W [Hkv, d, F/2].
    dev_err: optional device int32 tensor of one element that receives BHA_ERR_TIMEOUT if the
    kernel's watchdog gave up (bha_featuremap_checked)."""
    _cuda(x, "x", ndim=3)
    _cuda(W, "W", dtype=x.dtype, ndim=3)
    T, H, d = x.shape
    Hkv, dw, Fh = W.shape
    _need(dw == d, "W must be [Hkv, d, F/2]")
    if out is None:
        out = torch.empty((T, H, 2 * Fh), dtype=out_dtype, device=x.device)
    _cuda(out, "out", dtype=out_dtype, ndim=3)
    _need(tuple(out.shape) == (T, H, 2 * Fh), "out must be [T, H, F]")
    dims = make_dims(0, Hkv, Hkv, d, 2 * Fh, 1, T, 0, x.dtype)  # R, Hq, slots unused here
    with torch.cuda.device(x.device):  # the library uses the current device
        if dev_err is None:
            st = lib().bha_featuremap(ctypes.byref(dims), _ptr(x), H, _ptr(W), _ptr(out),
                                      _DTYPE_CODE[out_dtype], _stream(x.device, stream))
        else:
            _cuda(dev_err, "dev_err", dtype=torch.int32)
            st = lib().bha_featuremap_checked(ctypes.byref(dims), _ptr(x), H, _ptr(W), _ptr(out),
                                              _DTYPE_CODE[out_dtype], _ptr(dev_err),
                                              _stream(x.device, stream))
    _check(st, "bha_featuremap")
    return out


def hybrid_attn(cu_blk, Q, K, V, S, Z, W, *, max_block, alpha=None, state_slot=None, out=None,
                dev_err=None, stream=None):
    """One decode step of a block-hybrid layer.  See include/bha.h for the layout."""
    _cuda(Q, "Q", ndim=3)
    dt = Q.dtype
    _cuda(K, "K", dtype=dt, ndim=3)
    _cuda(V, "V", dtype=dt, ndim=3)
    _cuda(W, "W", dtype=dt, ndim=3)
    _cuda(S, "S", dtype=torch.float32, ndim=4)
    _cuda(Z, "Z", dtype=torch.float32, ndim=3)
    _cuda(cu_blk, "cu_blk", dtype=torch.int32, ndim=1)
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    F = S.shape[2]
    R = cu_blk.shape[0] - 1
    _need(tuple(K.shape) == (T, Hkv, d) and tuple(V.shape) == (T, Hkv, d), "K/V must be [T, Hkv, d]")
    _need(tuple(W.shape) == (Hkv, d, F // 2), "W must be [Hkv, d, F/2]")
    _need(tuple(S.shape[1:]) == (Hkv, F, d) and tuple(Z.shape) == (S.shape[0], Hkv, F),
          "S must be [slots, Hkv, F, d], Z [slots, Hkv, F]")
    if alpha is not None:
        _cuda(alpha, "alpha", dtype=torch.float32, ndim=1)
        _need(alpha.shape[0] == Hq, "alpha must be [Hq]")
    if state_slot is not None:
        _cuda(state_slot, "state_slot", dtype=torch.int32, ndim=1)
        _need(state_slot.shape[0] == R, "state_slot must be [R]")
    if out is None:
        out = torch.empty_like(Q)
    _cuda(out, "out", dtype=dt, ndim=3)
    if dev_err is not None:
        _cuda(dev_err, "dev_err", dtype=torch.int32)
    dims = make_dims(R, Hq, Hkv, d, F, max_block, T, S.shape[0], dt)
    with torch.cuda.device(Q.device):  # the library uses the current device
        st = lib().bha_hybrid_attn(ctypes.byref(dims), _ptr(cu_blk), _ptr(state_slot), _ptr(Q),
                                   _ptr(K), _ptr(V), _ptr(S), _ptr(Z), _ptr(W), _ptr(alpha),
                                   _ptr(out), _ptr(dev_err), _stream(Q.device, stream))
    _check(st, "bha_hybrid_attn")
    return out


def hybrid_attn_commit(cu_blk, Q, K, V, S, Z, W, *, max_block, alpha=None, state_slot=None,
                       out=None, dev_err=None, stream=None):
    """The last denoising step of a block fused with its commit: returns the step's output over
    the states as passed in, and folds each request's block into S and Z in place."""
    _cuda(Q, "Q", ndim=3)
    dt = Q.dtype
    _cuda(K, "K", dtype=dt, ndim=3)
    _cuda(V, "V", dtype=dt, ndim=3)
    _cuda(W, "W", dtype=dt, ndim=3)
    _cuda(S, "S", dtype=torch.float32, ndim=4)
    _cuda(Z, "Z", dtype=torch.float32, ndim=3)
    _cuda(cu_blk, "cu_blk", dtype=torch.int32, ndim=1)
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    F = S.shape[2]
    R = cu_blk.shape[0] - 1
    _need(tuple(K.shape) == (T, Hkv, d) and tuple(V.shape) == (T, Hkv, d), "K/V must be [T, Hkv, d]")
    _need(tuple(W.shape) == (Hkv, d, F // 2), "W must be [Hkv, d, F/2]")
    _need(tuple(S.shape[1:]) == (Hkv, F, d) and tuple(Z.shape) == (S.shape[0], Hkv, F),
          "S must be [slots, Hkv, F, d], Z [slots, Hkv, F]")
    if alpha is not None:
        _cuda(alpha, "alpha", dtype=torch.float32, ndim=1)
        _need(alpha.shape[0] == Hq, "alpha must be [Hq]")
    if state_slot is not None:
        _cuda(state_slot, "state_slot", dtype=torch.int32, ndim=1)
        _need(state_slot.shape[0] == R, "state_slot must be [R]")
    if out is None:
        out = torch.empty_like(Q)
    _cuda(out, "out", dtype=dt, ndim=3)
    if dev_err is not None:
        _cuda(dev_err, "dev_err", dtype=torch.int32)
    dims = make_dims(R, Hq, Hkv, d, F, max_block, T, S.shape[0], dt)
    with torch.cuda.device(Q.device):  # the library uses the current device
        st = lib().bha_hybrid_attn_commit(ctypes.byref(dims), _ptr(cu_blk), _ptr(state_slot),
                                          _ptr(Q), _ptr(K), _ptr(V), _ptr(S), _ptr(Z), _ptr(W),
                                          _ptr(alpha), _ptr(out), _ptr(dev_err),
                                          _stream(Q.device, stream))
    _check(st, "bha_hybrid_attn_commit")
    return out


def commit_block(cu_blk, K, V, W, S, Z, *, max_block, state_slot=None, dev_err=None, stream=None):
    """Fold each request's finished block into its states, in place."""
    _cuda(K, "K", ndim=3)
    dt = K.dtype
    _cuda(V, "V", dtype=dt, ndim=3)
    _cuda(W, "W", dtype=dt, ndim=3)
    _cuda(S, "S", dtype=torch.float32, ndim=4)
    _cuda(Z, "Z", dtype=torch.float32, ndim=3)
    _cuda(cu_blk, "cu_blk", dtype=torch.int32, ndim=1)
    T, Hkv, d = K.shape
    F = S.shape[2]
    R = cu_blk.shape[0] - 1
    _need(tuple(V.shape) == (T, Hkv, d), "V must be [T, Hkv, d]")
    _need(tuple(W.shape) == (Hkv, d, F // 2), "W must be [Hkv, d, F/2]")
    _need(tuple(S.shape[1:]) == (Hkv, F, d) and tuple(Z.shape) == (S.shape[0], Hkv, F),
          "S must be [slots, Hkv, F, d], Z [slots, Hkv, F]")
    if state_slot is not None:
        _cuda(state_slot, "state_slot", dtype=torch.int32, ndim=1)
        _need(state_slot.shape[0] == R, "state_slot must be [R]")
    if dev_err is not None:
        _cuda(dev_err, "dev_err", dtype=torch.int32)
    dims = make_dims(R, Hkv, Hkv, d, F, max_block, T, S.shape[0], dt)
    with torch.cuda.device(K.device):  # the library uses the current device
        st = lib().bha_commit_block(ctypes.byref(dims), _ptr(cu_blk), _ptr(state_slot), _ptr(K),
                                    _ptr(V), _ptr(W), _ptr(S), _ptr(Z), _ptr(dev_err),
                                    _stream(K.device, stream))
    _check(st, "bha_commit_block")
    return S, Z


def full_prefix_workspace_bytes(R, Hq, Hkv, d, max_block, T, kv_capacity, dtype=torch.bfloat16):
    dims = make_dims(R, Hq, Hkv, d, 2, max_block, T, 0, dtype)
    return int(lib().bha_full_prefix_workspace_bytes(ctypes.byref(dims), int(kv_capacity)))


def full_prefix_attn(cu_blk, kv_len, Q, Kc, Vc, *, max_block, workspace=None, out=None,
                     dev_err=None, stream=None):
    """Softmax teacher over each request's whole cache.  Kc/Vc [R, Hkv, capacity, d]."""
    _cuda(Q, "Q", ndim=3)
    dt = Q.dtype
    _cuda(Kc, "Kc", dtype=dt, ndim=4)
    _cuda(Vc, "Vc", dtype=dt, ndim=4)
    _cuda(cu_blk, "cu_blk", dtype=torch.int32, ndim=1)
    _cuda(kv_len, "kv_len", dtype=torch.int32, ndim=1)
    T, Hq, d = Q.shape
    R, Hkv, cap, dk = Kc.shape
    _need(dk == d and tuple(Vc.shape) == tuple(Kc.shape), "Kc/Vc must be [R, Hkv, capacity, d]")
    _need(cu_blk.shape[0] == R + 1 and kv_len.shape[0] == R, "cu_blk [R+1], kv_len [R]")
    need = full_prefix_workspace_bytes(R, Hq, Hkv, d, max_block, T, cap, dt)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    if out is None:
        out = torch.empty_like(Q)
    _cuda(out, "out", dtype=dt, ndim=3)
    if dev_err is not None:
        _cuda(dev_err, "dev_err", dtype=torch.int32)
    dims = make_dims(R, Hq, Hkv, d, 2, max_block, T, 0, dt)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(Q.device):  # the library uses the current device
        st = lib().bha_full_prefix_attn(ctypes.byref(dims), _ptr(cu_blk), _ptr(kv_len), _ptr(Q),
                                        _ptr(Kc), _ptr(Vc), cap, _ptr(out), _ptr(workspace), wbytes,
                                        _ptr(dev_err), _stream(Q.device, stream))
    _check(st, "bha_full_prefix_attn")
    return out


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


def full_prefix_attn_noalloc(cu_blk, kv_len, Q, Kc, Vc, *, max_block, out=None, dev_err=None,
                             stream=None):
    """Softmax teacher without a caller workspace: the split partials use the library's fixed
    device scratch array (shared by every call; concurrent calls must be serialised)."""
    _cuda(Q, "Q", ndim=3)
    dt = Q.dtype
    _cuda(Kc, "Kc", dtype=dt, ndim=4)
    _cuda(Vc, "Vc", dtype=dt, ndim=4)
    _cuda(cu_blk, "cu_blk", dtype=torch.int32, ndim=1)
    _cuda(kv_len, "kv_len", dtype=torch.int32, ndim=1)
    T, Hq, d = Q.shape
    R, Hkv, cap, dk = Kc.shape
    _need(dk == d and tuple(Vc.shape) == tuple(Kc.shape), "Kc/Vc must be [R, Hkv, capacity, d]")
    _need(cu_blk.shape[0] == R + 1 and kv_len.shape[0] == R, "cu_blk [R+1], kv_len [R]")
    if out is None:
        out = torch.empty_like(Q)
    _cuda(out, "out", dtype=dt, ndim=3)
    if dev_err is not None:
        _cuda(dev_err, "dev_err", dtype=torch.int32)
    dims = make_dims(R, Hq, Hkv, d, 2, max_block, T, 0, dt)
    with torch.cuda.device(Q.device):  # the library uses the current device
        st = lib().bha_full_prefix_attn_noalloc(ctypes.byref(dims), _ptr(cu_blk), _ptr(kv_len),
                                                _ptr(Q), _ptr(Kc), _ptr(Vc), cap, _ptr(out),
                                                _ptr(dev_err), _stream(Q.device, stream))
    _check(st, "bha_full_prefix_attn_noalloc")
    return out

"""Python binding of the Lynx C ABI (include/lynx.h).

Argument marshalling only: every step of the layer runs in the CUDA library
``_build/liblynx.so``; torch provides device memory and the current stream.
There is no fallback: if the library is missing or a call fails, an exception
is raised.

The functions carry the C names; tensors are torch tensors on the current CUDA
device, bf16 unless stated, row-major and contiguous.
"""
import ctypes
import os
import re

from . import build as _build

LIB_PATH = _build.LIB

LYNX_OK = 0
LYNX_ERR_INVALID_ARG = 1
LYNX_ERR_UNSUPPORTED_SHAPE = 2
LYNX_ERR_MISALIGNED = 3
LYNX_ERR_WORKSPACE_TOO_SMALL = 4
LYNX_ERR_CUDA = 5
LYNX_ERR_DEVICE_TIMEOUT = 6

LYNX_ACT_NONE = 0
LYNX_ACT_GELU_TANH = 1


class LynxError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__(f"{what}: {lynx_status_string(status)} ({status})")


_lib = None


def library():
    """Load the CUDA library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"Lynx CUDA library not built ({LIB_PATH} missing); run "
                "`python -m activation_sparse_gemm_lynx_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        p, i64, sz, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        sigs = {
            "lynx_status_string": ([i32], ctypes.c_char_p),
            "lynx_version": ([], i32),
            "lynx_lora_rank": ([], i32),
            "lynx_lora_rank_supported": ([i64], i32),
            "lynx_vals_bytes": ([i64, i64], sz),
            "lynx_meta_bytes": ([i64, i64], sz),
            "lynx_workspace_bytes": ([i64, i64, i64, i64], sz),
            "lynx_sparsify_workspace_bytes": ([i64, i64], sz),
            "lynx_sparsify": ([p, i64, i64, p, p, p, p, sz, p], i32),
            "lynx_sparsify_noalloc": ([p, i64, i64, p, p, p, p], i32),
            "lynx_sparsify_noalloc_max_rows": ([], i64),
            "lynx_linear": ([p, p, p, p, p, i64, i64, i64, i64, i32, p, p, sz, p], i32),
            "lynx_linear_act": ([p, p, p, p, p, i64, i64, i64, i64, i32, i32, p, p, sz, p], i32),
            "lynx_linear_begin": ([p, p, p, p, p, i64, i64, i64, i64, i32, i32, p, p, sz, p], i32),
            "lynx_linear_finish": ([p, p, p, p, p, i64, i64, i64, i64, i32, i32, p, p, sz, p], i32),
            "lynx_linear_dense": ([p, p, p, p, p, i64, i64, i64, i64, p, p, sz, p], i32),
            "lynx_linear_fused": ([p, p, p, p, p, i64, i64, i64, i64, i32, p, p, sz, p], i32),
            "lynx_linear_host_workspace_bytes": ([i64, i64, i64, i64], sz),
            "lynx_linear_host": ([p, p, p, p, p, i64, i64, i64, i64, i32, p, p, sz, p], i32),
            "lynx_linear_host_act": ([p, p, p, p, p, i64, i64, i64, i64, i32, i32, p, p, sz, p], i32),
            "lynx_sparse_gemm": ([p, p, p, p, p, p, i64, i64, i64, i64, p, p], i32),
            "lynx_check_error": ([p, p], i32),
            "lynx_meta_hw_to_canonical": ([p, p, i64, i64], i32),
            "lynx_meta_canonical_to_hw": ([p, p, i64, i64], i32),
            "lynx_debug_set_stall": ([i32], i32),
            "lynx_profile_set_split_event": ([p], p),
            "lynx_profile_set_part": ([i32], i32),
        }
        for name, (args, res) in sigs.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
    return _lib


def header_functions():
    """Names of the functions include/lynx.h declares."""
    path = os.path.join(_build.INCLUDE, "lynx.h")
    text = open(path).read()
    return sorted(set(re.findall(r"^\s*LYNX_API\s+(?:const\s+)?\w+\*?\s+\*?(lynx_\w+)\s*\(", text, re.M)))


def lynx_status_string(status):
    return library().lynx_status_string(int(status)).decode()


def lynx_version():
    return library().lynx_version()


def lynx_lora_rank():
    """The LoRA rank the RT-Lynx pages use (64), the default of these bindings."""
    return library().lynx_lora_rank()


def lynx_lora_rank_supported(r):
    """True if the kernels accept LoRA rank r (r % 16 == 0, 16 <= r <= 256)."""
    return bool(library().lynx_lora_rank_supported(int(r)))


def lynx_vals_bytes(M, K):
    return library().lynx_vals_bytes(M, K)


def lynx_meta_bytes(M, K):
    return library().lynx_meta_bytes(M, K)


def lynx_workspace_bytes(M, N, K, r=64):
    return library().lynx_workspace_bytes(M, N, K, r)


def _check(status, what):
    if status != LYNX_OK:
        raise LynxError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype=None, shape=None):
    import torch

    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def lynx_sparsify_workspace_bytes(M, K):
    return library().lynx_sparsify_workspace_bytes(M, K)


def lynx_sparsify(X, vals=None, meta=None, row_scale=None, workspace=None, stream=None,
                  want_scale=True):
    """S(X): returns (vals [M,K/2] bf16, meta uint8 [lynx_meta_bytes], row_scale [M] f32 or None)."""
    import torch

    _need(X, "X", torch.bfloat16)
    M, K = X.shape
    if vals is None:
        vals = torch.empty((M, K // 2), dtype=torch.bfloat16, device=X.device)
    if meta is None:
        meta = torch.empty(lynx_meta_bytes(M, K), dtype=torch.uint8, device=X.device)
    if row_scale is None and want_scale:
        row_scale = torch.empty(M, dtype=torch.float32, device=X.device)
    if workspace is None:
        workspace = torch.empty(lynx_sparsify_workspace_bytes(M, K), dtype=torch.uint8,
                                device=X.device)
    _need(vals, "vals", torch.bfloat16, (M, K // 2))
    _need(meta, "meta", torch.uint8)
    _need(workspace, "workspace", torch.uint8)
    if meta.numel() < lynx_meta_bytes(M, K):
        raise ValueError("meta buffer too small")
    if row_scale is not None:
        _need(row_scale, "row_scale", torch.float32, (M,))
    st = library().lynx_sparsify(_ptr(X), M, K, _ptr(vals), _ptr(meta), _ptr(row_scale),
                                 _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "lynx_sparsify")
    return vals, meta, row_scale


def lynx_sparsify_noalloc_max_rows():
    return library().lynx_sparsify_noalloc_max_rows()


def lynx_sparsify_noalloc(X, vals, meta, row_scale=None, stream=None):
    """S(X) into caller buffers, with the library's fixed scratch instead of a
    workspace; allocates nothing.  Returns (vals, meta, row_scale)."""
    import torch

    _need(X, "X", torch.bfloat16)
    M, K = X.shape
    _need(vals, "vals", torch.bfloat16, (M, K // 2))
    _need(meta, "meta", torch.uint8)
    if meta.numel() < lynx_meta_bytes(M, K):
        raise ValueError("meta buffer too small")
    if row_scale is not None:
        _need(row_scale, "row_scale", torch.float32, (M,))
    st = library().lynx_sparsify_noalloc(_ptr(X), M, K, _ptr(vals), _ptr(meta), _ptr(row_scale),
                                         _stream(stream))
    _check(st, "lynx_sparsify_noalloc")
    return vals, meta, row_scale


def _linear_args(X, W, bias, A, B):
    import torch

    _need(X, "X", torch.bfloat16)
    _need(W, "W", torch.bfloat16)
    M, K = X.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("W must be [N,K]")
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,))
    if (A is None) != (B is None):
        raise ValueError("A and B must both be given or both be None")
    r = 0
    if A is not None:
        r = A.shape[0]
        _need(A, "A", torch.bfloat16, (r, K))
        _need(B, "B", torch.bfloat16, (N, r))
    return M, N, K, r


def _linear_buffers(X, W, bias, A, B, Y, workspace):
    import torch

    M, N, K, r = _linear_args(X, W, bias, A, B)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _need(Y, "Y", torch.bfloat16, (M, N))
    if workspace is None:
        workspace = torch.empty(lynx_workspace_bytes(M, N, K, r or 64), dtype=torch.uint8,
                                device=X.device)
    _need(workspace, "workspace", torch.uint8)
    return M, N, K, r, Y, workspace


def lynx_linear(X, W, bias=None, A=None, B=None, skip_sparsify=False, Y=None, workspace=None,
                stream=None):
    """Y = S(X) W^T + bias + (X A^T) B^T (S(X) = X if skip_sparsify). Returns Y."""
    M, N, K, r, Y, workspace = _linear_buffers(X, W, bias, A, B, Y, workspace)
    st = library().lynx_linear(_ptr(X), _ptr(W), _ptr(bias), _ptr(A), _ptr(B), M, N, K, r,
                               1 if skip_sparsify else 0, _ptr(Y), _ptr(workspace),
                               workspace.numel(), _stream(stream))
    _check(st, "lynx_linear")
    return Y


def lynx_linear_act(X, W, bias=None, A=None, B=None, skip_sparsify=False, act=LYNX_ACT_GELU_TANH,
                    Y=None, workspace=None, stream=None):
    """Y = act(S(X) W^T + bias + (X A^T) B^T), the activation applied in the
    GEMM epilogue (LYNX_ACT_NONE or LYNX_ACT_GELU_TANH). Returns Y."""
    M, N, K, r, Y, workspace = _linear_buffers(X, W, bias, A, B, Y, workspace)
    st = library().lynx_linear_act(_ptr(X), _ptr(W), _ptr(bias), _ptr(A), _ptr(B), M, N, K, r,
                                   1 if skip_sparsify else 0, int(act), _ptr(Y), _ptr(workspace),
                                   workspace.numel(), _stream(stream))
    _check(st, "lynx_linear_act")
    return Y


def _linear_half(name, X, W, bias, A, B, skip_sparsify, act, Y, workspace, stream):
    M, N, K, r, Y, workspace = _linear_buffers(X, W, bias, A, B, Y, workspace)
    st = getattr(library(), name)(_ptr(X), _ptr(W), _ptr(bias), _ptr(A), _ptr(B), M, N, K, r,
                                  1 if skip_sparsify else 0, int(act), _ptr(Y), _ptr(workspace),
                                  workspace.numel(), _stream(stream))
    _check(st, name)
    return Y


def lynx_linear_begin(X, W, bias=None, A=None, B=None, skip_sparsify=False, act=LYNX_ACT_NONE, Y=None,
                      workspace=None, stream=None):
    """First half of lynx_linear_act: the sparsify (or LoRA-down) pass into
    `workspace` (see include/lynx.h).  Returns Y (not yet written)."""
    return _linear_half("lynx_linear_begin", X, W, bias, A, B, skip_sparsify, act, Y, workspace, stream)


def lynx_linear_finish(X, W, bias=None, A=None, B=None, skip_sparsify=False, act=LYNX_ACT_NONE, Y=None,
                       workspace=None, stream=None):
    """Second half of lynx_linear_act: the GEMM from the workspace a completed
    lynx_linear_begin filled.  Returns Y."""
    return _linear_half("lynx_linear_finish", X, W, bias, A, B, skip_sparsify, act, Y, workspace, stream)


def lynx_linear_fused(X, W, bias=None, A=None, B=None, act=LYNX_ACT_NONE, Y=None, workspace=None,
                      stream=None):
    """The fully fused variant: the 2:4 selection and compression inside the
    GEMM, after a slim pass for s and T (see include/lynx.h).  Returns Y."""
    M, N, K, r, Y, workspace = _linear_buffers(X, W, bias, A, B, Y, workspace)
    st = library().lynx_linear_fused(_ptr(X), _ptr(W), _ptr(bias), _ptr(A), _ptr(B), M, N, K, r,
                                     int(act), _ptr(Y), _ptr(workspace), workspace.numel(),
                                     _stream(stream))
    _check(st, "lynx_linear_fused")
    return Y


def lynx_linear_host_workspace_bytes(M, N, K, r=64):
    return library().lynx_linear_host_workspace_bytes(M, N, K, r)


def lynx_linear_host(X_host, W, bias=None, A=None, B=None, skip_sparsify=False, Y_host=None,
                     workspace=None, stream=None):
    """The layer on host activations: X_host [M,K] and Y_host [M,N] are CPU bf16
    tensors (pinned for asynchronous copies); W, bias, A, B are CUDA tensors.
    Returns Y_host, complete once `stream` (default: the current stream) has
    reached this point."""
    return _linear_host(X_host, W, bias, A, B, skip_sparsify, None, Y_host, workspace, stream)


def lynx_linear_host_act(X_host, W, bias=None, A=None, B=None, skip_sparsify=False,
                         act=LYNX_ACT_GELU_TANH, Y_host=None, workspace=None, stream=None):
    """lynx_linear_host with the activation of lynx_linear_act."""
    return _linear_host(X_host, W, bias, A, B, skip_sparsify, int(act), Y_host, workspace, stream)


def _linear_host(X_host, W, bias, A, B, skip_sparsify, act, Y_host, workspace, stream):
    import torch

    if X_host is None or X_host.is_cuda or X_host.dtype != torch.bfloat16 or not X_host.is_contiguous():
        raise ValueError("X_host must be a contiguous bf16 CPU tensor")
    _need(W, "W", torch.bfloat16)
    M, K = X_host.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("W must be [N,K]")
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,))
    if (A is None) != (B is None):
        raise ValueError("A and B must both be given or both be None")
    r = 0
    if A is not None:
        r = A.shape[0]
        _need(A, "A", torch.bfloat16, (r, K))
        _need(B, "B", torch.bfloat16, (N, r))
    if Y_host is None:
        Y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    if Y_host.is_cuda or Y_host.dtype != torch.bfloat16 or tuple(Y_host.shape) != (M, N) or \
            not Y_host.is_contiguous():
        raise ValueError("Y_host must be a contiguous bf16 CPU tensor of shape [M,N]")
    need = lynx_linear_host_workspace_bytes(M, N, K, r if r else 64)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    _need(workspace, "workspace", torch.uint8)
    if act is None:
        st = library().lynx_linear_host(_ptr(X_host), _ptr(W), _ptr(bias), _ptr(A), _ptr(B), M, N, K,
                                        r, 1 if skip_sparsify else 0, _ptr(Y_host), _ptr(workspace),
                                        workspace.numel(), _stream(stream))
        _check(st, "lynx_linear_host")
    else:
        st = library().lynx_linear_host_act(_ptr(X_host), _ptr(W), _ptr(bias), _ptr(A), _ptr(B), M, N,
                                            K, r, 1 if skip_sparsify else 0, act, _ptr(Y_host),
                                            _ptr(workspace), workspace.numel(), _stream(stream))
        _check(st, "lynx_linear_host_act")
    return Y_host


def lynx_linear_dense(X, W, bias=None, A=None, B=None, Y=None, workspace=None, stream=None):
    """Dense path of a skipped layer: Y = X W^T + bias + (X A^T) B^T."""
    import torch

    M, N, K, r = _linear_args(X, W, bias, A, B)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _need(Y, "Y", torch.bfloat16, (M, N))
    if workspace is None:
        workspace = torch.empty(lynx_workspace_bytes(M, N, K, r or 64), dtype=torch.uint8,
                                device=X.device)
    st = library().lynx_linear_dense(_ptr(X), _ptr(W), _ptr(bias), _ptr(A), _ptr(B), M, N, K, r,
                                     _ptr(Y), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "lynx_linear_dense")
    return Y


def lynx_sparse_gemm(vals, meta, W, bias=None, T=None, B=None, Y=None, stream=None):
    """Y = S(X) W^T + bias + T B^T on a precomputed S(X) (vals + hardware metadata)."""
    import torch

    _need(vals, "vals", torch.bfloat16)
    _need(meta, "meta", torch.uint8)
    _need(W, "W", torch.bfloat16)
    M, K2 = vals.shape
    K = 2 * K2
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("W must be [N,K] with K = 2 * vals.shape[1]")
    if meta.numel() < lynx_meta_bytes(M, K):
        raise ValueError("meta buffer too small")
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, (N,))
    if (T is None) != (B is None):
        raise ValueError("T and B must both be given or both be None")
    r = 0
    if T is not None:
        r = T.shape[1]
        _need(T, "T", torch.bfloat16, (M, r))
        _need(B, "B", torch.bfloat16, (N, r))
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=vals.device)
    _need(Y, "Y", torch.bfloat16, (M, N))
    st = library().lynx_sparse_gemm(_ptr(vals), _ptr(meta), _ptr(T), _ptr(W), _ptr(bias),
                                    _ptr(B), M, N, K, r, _ptr(Y), _stream(stream))
    _check(st, "lynx_sparse_gemm")
    return Y


def lynx_check_error(stream=None):
    """Synchronise the stream and return (status, raw device code); clears the code."""
    code = ctypes.c_uint32(0)
    st = library().lynx_check_error(_stream(stream), ctypes.byref(code))
    return st, code.value


def lynx_meta_hw_to_canonical(hw, M, K):
    """numpy uint8 hardware metadata -> numpy uint8 [M, K/8] canonical nibbles."""
    import numpy as np

    hw = np.ascontiguousarray(hw, dtype=np.uint8)
    if hw.size < lynx_meta_bytes(M, K):
        raise ValueError("hardware metadata buffer too small")
    out = np.empty((M, K // 8), dtype=np.uint8)
    st = library().lynx_meta_hw_to_canonical(hw.ctypes.data_as(ctypes.c_void_p),
                                             out.ctypes.data_as(ctypes.c_void_p), M, K)
    _check(st, "lynx_meta_hw_to_canonical")
    return out


def lynx_meta_canonical_to_hw(canonical, M, K):
    """numpy uint8 [M, K/8] canonical nibbles -> numpy uint8 hardware metadata."""
    import numpy as np

    canonical = np.ascontiguousarray(canonical, dtype=np.uint8)
    if canonical.shape != (M, K // 8):
        raise ValueError("canonical metadata must be [M, K/8]")
    out = np.empty(lynx_meta_bytes(M, K), dtype=np.uint8)
    st = library().lynx_meta_canonical_to_hw(canonical.ctypes.data_as(ctypes.c_void_p),
                                             out.ctypes.data_as(ctypes.c_void_p), M, K)
    _check(st, "lynx_meta_canonical_to_hw")
    return out


def lynx_profile_set_split_event(event):
    """Record `event` (a torch.cuda.Event, or None) between the two kernels of
    every later lynx_linear call (see include/lynx.h)."""
    handle = None if event is None else ctypes.c_void_p(event.cuda_event)
    return library().lynx_profile_set_split_event(handle)


def lynx_profile_set_part(part):
    """Profiling hook: 1 = only the sparsify / LoRA-down pass of each later
    lynx_linear call, 2 = only what follows it, 0 = the whole layer (see
    include/lynx.h).  Returns the previous part."""
    return library().lynx_profile_set_part(int(part))


def lynx_debug_set_stall(enable):
    """Test hook: make later launches time out (see include/lynx.h)."""
    return library().lynx_debug_set_stall(1 if enable else 0)

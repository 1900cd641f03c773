"""CPU oracle for the RT-Lynx online 2:4 activation-sparse linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It
shares no code with the CUDA library and never imports it.

All arrays are numpy.  bf16 tensors travel as ``uint16`` arrays holding the
raw bf16 bit patterns.  The arithmetic lives in ``lynx_oracle.c`` (plain C,
fp64 accumulation); this module only marshals arguments.

Functions follow the pages on "RT-Lynx: Putting GEMM Sparsity in the Right
Place for Diffusion Models" (qingkeai.online article, sections 02-03):

* :func:`select_groups` -- Top-2 of 4 by magnitude, ties to the lower index.
* :func:`sparsify` -- S(X): selection, norm compensation s = sum|x|/sum|kept|
  (fp32), compensated kept values rounded to bf16, canonical 2-bit metadata.
* :func:`linear` -- Y = S(X) W^T + bias + (X A^T) B^T in fp64 (S(X) := X for
  a skipped layer).
* :func:`bf16_rne` -- IEEE round-to-nearest-even fp32 -> bf16.
* :func:`gelu_tanh` -- GELU (tanh form) in fp64, the activation the library can
  apply to a layer's output (not part of the pages' method).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.oracle_bf16_rne.argtypes = [p, p, i64]
        lib.oracle_select_groups.argtypes = [p, i64, p, p]
        lib.oracle_sparsify.argtypes = [p, i64, i64, p, p, p, p]
        lib.oracle_linear.argtypes = [p, p, p, p, p, i64, i64, i64, i64, ctypes.c_int, p, p, p]
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_gelu_tanh.argtypes = [p, i64, p]
        for f in (lib.oracle_bf16_rne, lib.oracle_select_groups, lib.oracle_sparsify,
                  lib.oracle_linear, lib.oracle_set_threads, lib.oracle_gelu_tanh):
            f.restype = None
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a, name):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"{name}: expected uint16 bf16 bit patterns, got {a.dtype}")
    return a


def bf16_to_f32(bits):
    """Widen bf16 bit patterns (uint16) to float32 (exact)."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_rne(x):
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_bf16_rne(_ptr(x), _ptr(out), x.size)
    return out


def select_groups(groups):
    """groups: [n,4] bf16 bits -> (lo[n], hi[n]) kept positions, lo < hi."""
    g = _u16(groups, "groups").reshape(-1, 4)
    n = g.shape[0]
    lo = np.empty(n, dtype=np.int32)
    hi = np.empty(n, dtype=np.int32)
    _load().oracle_select_groups(_ptr(g), n, _ptr(lo), _ptr(hi))
    return lo, hi


def sparsify(X):
    """S(X) for X [M,K] (bf16 bits; K % 8 == 0 so metadata rows are whole bytes).

    Returns dict with ``vals`` [M,K/2] uint16, ``meta`` [M,K/8] uint8 (canonical
    nibbles), ``scale`` [M] float32 and ``sums`` [M,4] float64 holding
    (sum|x| fp32, sum|kept| fp32, sum|x| fp64, sum|kept| fp64).
    """
    X = _u16(X, "X")
    M, K = X.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    vals = np.empty((M, K // 2), dtype=np.uint16)
    meta = np.empty((M, K // 8), dtype=np.uint8)
    scale = np.empty(M, dtype=np.float32)
    sums = np.empty((M, 4), dtype=np.float64)
    _load().oracle_sparsify(_ptr(X), M, K, _ptr(vals), _ptr(meta), _ptr(scale), _ptr(sums))
    return {"vals": vals, "meta": meta, "scale": scale, "sums": sums}


def linear(X, W, bias=None, A=None, B=None, skip=False, want_sx=False):
    """Y = S(X) W^T + bias + (X A^T) B^T in fp64.

    X [M,K], W [N,K], bias [N] or None, A [r,K] / B [N,r] (both or neither),
    all bf16 bit patterns.  Returns (Y [M,N] f64, T [M,r] f64 or None,
    SX [M,K] f64 or None).
    """
    X = _u16(X, "X")
    W = _u16(W, "W")
    M, K = X.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("W must be [N,K]")
    if (A is None) != (B is None):
        raise ValueError("A and B must both be given or both be None")
    r = 0
    if A is not None:
        A = _u16(A, "A")
        B = _u16(B, "B")
        r = A.shape[0]
        if A.shape != (r, K) or B.shape != (N, r):
            raise ValueError("A must be [r,K] and B [N,r]")
    if bias is not None:
        bias = _u16(bias, "bias")
        if bias.shape != (N,):
            raise ValueError("bias must be [N]")
    Y = np.empty((M, N), dtype=np.float64)
    T = np.empty((M, r), dtype=np.float64) if r else None
    SX = np.empty((M, K), dtype=np.float64) if want_sx else None
    _load().oracle_linear(_ptr(X), _ptr(W), _ptr(bias), _ptr(A), _ptr(B), M, N, K, r,
                          1 if skip else 0, _ptr(Y), _ptr(T), _ptr(SX))
    return Y, T, SX


def gelu_tanh(v):
    """GELU, tanh form (Hendrycks & Gimpel), elementwise in fp64:
    v/2 (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))).  The activation the library
    can apply to a layer's output; compose as gelu_tanh(linear(...)[0])."""
    a = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty_like(a)
    _load().oracle_gelu_tanh(_ptr(a), a.size, _ptr(out))
    return out


_threads = None


def num_threads():
    """Threads the oracle's OpenMP loops use (set_num_threads, else
    OMP_NUM_THREADS, else all cores)."""
    if _threads is not None:
        return _threads
    env = os.environ.get("OMP_NUM_THREADS")
    return int(env) if env else os.cpu_count()


def set_num_threads(n):
    """Run the oracle's parallel loops on `n` threads from now on (timing only:
    each output element is computed by one thread, in a fixed order)."""
    global _threads
    _load().oracle_set_threads(int(n))
    _threads = int(n)

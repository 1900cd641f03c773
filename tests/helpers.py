"""Test-side helpers: bf16 bit handling, tolerances and an independent reading
of the metadata operand layout (written from its definition in include/lynx.h,
not taken from the library)."""
import numpy as np


def f32(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_ulp_distance(a_bits, b_bits):
    """Number of bf16 steps between two arrays of bf16 bit patterns (+0 == -0)."""
    def key(b):
        b = np.asarray(b, dtype=np.uint16).astype(np.int32)
        mag = b & 0x7FFF
        return np.where(b & 0x8000, -mag, mag)
    return np.abs(key(a_bits) - key(b_bits))


def hw_meta_offsets(M, K, rows=None):
    """(byte offset, bit shift) of the nibble of every (row m < M, group g) in the
    hardware metadata buffer: block (m//128, k//128) of 2048 bytes, lane
    (m%8) + 8*((k//16)%2) + 16*((m%128)//16), 32-bit word (k%128)//32, bit
    (k%16) + 16*((m//8)%2).  `rows` restricts it to those rows."""
    m = (np.arange(M, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64))[:, None]
    k = (4 * np.arange(K // 4, dtype=np.int64))[None, :]
    kblocks = (K + 127) // 128
    mi, ki = m % 128, k % 128
    lane = (mi % 8) + 8 * ((ki // 16) % 2) + 16 * (mi // 16)
    word = ki // 32
    bit = (ki % 16) + 16 * ((mi // 8) % 2)
    byte = ((m // 128) * kblocks + (k // 128)) * 2048 + lane * 16 + word * 4 + bit // 8
    return byte, bit % 8


def canonical_from_hw(hw, M, K, rows=None):
    """Hardware metadata bytes -> canonical [M, K/8] nibble bytes (or only the
    given rows, in their order)."""
    hw = np.asarray(hw, dtype=np.uint8).reshape(-1)
    byte, shift = hw_meta_offsets(M, K, rows)
    nib = (hw[byte] >> shift.astype(np.uint8)) & 0xF          # [rows, K/4]
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def hw_from_canonical(canon, M, K):
    """Canonical [M, K/8] -> hardware bytes (padding rows: pattern of a zero row)."""
    kblocks = (K + 127) // 128
    mpad = (M + 255) // 256 * 256   # 128-row blocks come in pairs
    out = np.zeros(mpad // 128 * kblocks * 2048, dtype=np.uint8)
    full = np.full((mpad, K // 8), 0x44, dtype=np.uint8)
    full[:M] = canon
    nib = np.empty((mpad, K // 4), dtype=np.uint8)
    nib[:, 0::2] = full & 0xF
    nib[:, 1::2] = full >> 4
    byte, shift = hw_meta_offsets(mpad, K)
    np.bitwise_or.at(out, byte.reshape(-1), (nib << shift.astype(np.uint8)).reshape(-1))
    return out


def dense_from_canonical(vals_bits, canon, K):
    """Scatter compressed values back to a dense [M,K] float64 matrix."""
    M = vals_bits.shape[0]
    nib = np.empty((M, K // 4), dtype=np.uint8)
    nib[:, 0::2] = canon & 0xF
    nib[:, 1::2] = canon >> 4
    lo = (nib & 3).astype(np.int64)
    hi = ((nib >> 2) & 3).astype(np.int64)
    v = f32(vals_bits).astype(np.float64).reshape(M, K // 4, 2)
    out = np.zeros((M, K // 4, 4))
    rows = np.arange(M)[:, None]
    grp = np.arange(K // 4)[None, :]
    out[rows, grp, lo] = v[:, :, 0]
    out[rows, grp, hi] = v[:, :, 1]
    return out.reshape(M, K)


def y_tolerance_check(y_gpu, y_ref, sx_rows, w_rows):
    """The layer's numeric bar: elementwise |dY| <= 2e-2 * ||S(X)_m||_2 * ||W_n||_2
    and relative Frobenius error <= 5e-3 (fp32 accumulation, bf16 output)."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    bound = 2e-2 * np.outer(np.linalg.norm(sx_rows, axis=1), np.linalg.norm(w_rows, axis=1))
    err = np.abs(y_gpu - y_ref)
    worst = float((err / np.maximum(bound, 1e-30)).max())
    fro = float(np.linalg.norm(y_gpu - y_ref) / max(np.linalg.norm(y_ref), 1e-30))
    return worst, fro


def kept_from_x(x_bits, canon, K):
    """The uncompensated kept values (bf16 bits, [M, K/2]) at the positions the
    canonical metadata names."""
    M = x_bits.shape[0]
    nib = np.empty((M, K // 4), dtype=np.uint8)
    nib[:, 0::2] = canon & 0xF
    nib[:, 1::2] = canon >> 4
    lo = (nib & 3).astype(np.int64)
    hi = ((nib >> 2) & 3).astype(np.int64)
    g = np.asarray(x_bits, dtype=np.uint16).reshape(M, K // 4, 4)
    rows = np.arange(M)[:, None]
    grp = np.arange(K // 4)[None, :]
    out = np.empty((M, K // 4, 2), dtype=np.uint16)
    out[:, :, 0] = g[rows, grp, lo]
    out[:, :, 1] = g[rows, grp, hi]
    return out.reshape(M, K // 2)


def workspace_views(raw, M, K, r=64):
    """Split a lynx_linear workspace (numpy uint8) into its documented parts:
    kept values [M,K/2] (bf16 bits), metadata bytes, s [M] f32, T/s [M,r] bf16 bits."""
    def a256(x):
        return (x + 255) // 256 * 256
    kblocks = (K + 127) // 128
    meta_bytes = (M + 255) // 256 * 2 * kblocks * 2048
    o_meta = a256(M * K)
    o_scale = a256(o_meta + meta_bytes)
    o_t = a256(o_scale + 4 * M)
    vals = raw[: M * K].view(np.uint16).reshape(M, K // 2)
    meta = raw[o_meta: o_meta + meta_bytes]
    scale = raw[o_scale: o_scale + 4 * M].view(np.float32)
    t = raw[o_t: o_t + 2 * M * r].view(np.uint16).reshape(M, r)
    return vals, meta, scale, t

"""Test-side readers of the library's packed layouts, restated from the
layout comments of include/svdq.h (independent of the library's code).

They turn packed device/host buffers back into the oracle's logical arrays:
codes [rows, K] (0..15), scales [rows, K/16] (ue4m3 patterns), AWQ q [K, N].
"""
import numpy as np


def unpack_codes(packed, K):
    """[rows, K/2] bytes -> [rows, K] codes; element 2j = low nibble of byte j."""
    p = np.asarray(packed, dtype=np.uint8).reshape(-1, K // 2)
    out = np.empty((p.shape[0], K), dtype=np.uint8)
    out[:, 0::2] = p & 0x0F
    out[:, 1::2] = p >> 4
    return out


def scale_index(rows, K):
    """Byte offset of scale (m, kb) for all m < rows, kb < K/16 (tile order)."""
    m = np.arange(rows)[:, None]
    kb = np.arange(K // 16)[None, :]
    return ((m // 128) * (K // 64) + kb // 4) * 512 + (m % 32) * 16 + ((m % 128) // 32) * 4 + kb % 4


def untile_scales(buf, rows, K):
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    return buf[scale_index(rows, K)]


def padding_scales(buf, rows, K):
    """Scales of the rows between `rows` and the next multiple of 128."""
    pad = (rows + 127) // 128 * 128
    if pad == rows:
        return np.zeros((0, K // 16), np.uint8)
    idx = scale_index(pad, K)[rows:]
    return np.asarray(buf, dtype=np.uint8).reshape(-1)[idx]


def awq_unpack(qweight, K, N):
    """Fragment-order words -> q [K, N] (see the AWQ layout in svdq.h)."""
    nb_n, g_n = N // 16, K // 64
    w = np.asarray(qweight, dtype=np.uint32).reshape(nb_n, g_n, 32, 4)
    q = np.empty((K, N), dtype=np.uint8)
    lane = np.arange(32)
    g, t = lane // 4, lane % 4
    for i in range(8):
        nib = ((w >> np.uint32(4 * i)) & np.uint32(15)).astype(np.uint8)
        reg, odd = i % 4, i // 4
        c = g + 8 * (reg % 2)
        kq = 2 * t + odd + 8 * (reg // 2)
        k_idx = (np.arange(g_n)[None, :, None, None] * 64 + np.arange(4)[None, None, None, :] * 16
                 + kq[None, None, :, None])
        n_idx = np.arange(nb_n)[:, None, None, None] * 16 + c[None, None, :, None]
        q[np.broadcast_to(k_idx, nib.shape), np.broadcast_to(n_idx, nib.shape)] = nib
    return q


def bf16_bits_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- writers
# (the inverse direction: oracle arrays -> the library's packed layouts, so a
# kernel can be run on operands that the oracle produced)

def pack_codes(codes):
    """[rows, K] codes -> [rows, K/2] bytes (element 2j in the low nibble)."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def tile_scales(sf, rows, K):
    """[rows, K/16] scales -> tile-order buffer with rows padded to 128 (pad = 0)."""
    pad = (rows + 127) // 128 * 128
    buf = np.zeros(pad * (K // 16), dtype=np.uint8)
    buf[scale_index(rows, K)] = np.asarray(sf, dtype=np.uint8)
    return buf


def awq_pack(q):
    """q [K, N] (0..15) -> fragment-order words (the inverse of awq_unpack)."""
    q = np.asarray(q, dtype=np.uint8)
    K, N = q.shape
    nb_n, g_n = N // 16, K // 64
    w = np.zeros((nb_n, g_n, 32, 4), dtype=np.uint32)
    lane = np.arange(32)
    g, t = lane // 4, lane % 4
    for i in range(8):
        reg, odd = i % 4, i // 4
        c = g + 8 * (reg % 2)
        kq = 2 * t + odd + 8 * (reg // 2)
        k_idx = (np.arange(g_n)[None, :, None, None] * 64 + np.arange(4)[None, None, None, :] * 16
                 + kq[None, None, :, None])
        n_idx = np.arange(nb_n)[:, None, None, None] * 16 + c[None, None, :, None]
        nib = q[np.broadcast_to(k_idx, w.shape), np.broadcast_to(n_idx, w.shape)].astype(np.uint32)
        w |= nib << np.uint32(4 * i)
    return w.reshape(-1)


def bf16_bits(values):
    """bf16 bit patterns of float64 values that are exact bf16 numbers."""
    f = np.asarray(values, dtype=np.float64).astype(np.float32)
    if not np.array_equal(f.astype(np.float64), np.asarray(values, dtype=np.float64)):
        raise ValueError("not bf16 values")
    u = f.view(np.uint32)
    if (u & 0xFFFF).any():
        raise ValueError("not bf16 values")
    return (u >> 16).astype(np.uint16)

"""Test-side readers of the library's packed layouts, restated from the
layout comments of include/svdq.h (independent of the library's code).

They turn packed device/host buffers back into the oracle's logical arrays:
codes [rows, K] (0..15), scales [rows, K/16] (ue4m3 patterns), AWQ q [K, N].
"""
import numpy as np


def _ks(K):
    return (K + 255) // 256


def _replicas(th):
    """Copies of each scale atom: 4 in 256-row (weight) tiles, 1 in 128-row tiles."""
    return 4 if th == 256 else 1


def _tile_bytes(th):
    return th * 128 + (th // 128) * 2048 * _replicas(th)


def bundle_size(rows, K, th):
    return ((rows + th - 1) // th) * _ks(K) * _tile_bytes(th)


def _tile(m, k, K, th):
    return ((m // th) * _ks(K) + k // 256) * _tile_bytes(th)


def code_index(rows, K, th):
    """Byte offsets of the code bytes (elements 2j, 2j+1) of rows x K/2, in bundle order."""
    m = np.arange(rows)[:, None]
    k = np.arange(0, K, 2)[None, :]
    r = m % th
    kb = (k % 256) // 2
    return _tile(m, k, K, th) + r * 128 + ((((kb >> 4) ^ r) & 7) << 4) + (kb & 15)


def scale_index(rows, K, th, rep=0):
    """Byte offsets of the block scales of rows x K/16 (replica rep), in bundle order."""
    m = np.arange(rows)[:, None]
    k = np.arange(0, K, 16)[None, :]
    r = m % th
    j = (k % 256) // 16
    atom = 512 * _replicas(th)
    return (_tile(m, k, K, th) + th * 128 + (j // 4) * (th // 128) * atom + (r // 128) * atom + rep * 512
            + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4)


def scale_replicas_agree(buf, rows, K, th):
    """Every replica of every block scale holds the same byte."""
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    first = buf[scale_index(rows, K, th)]
    return all(np.array_equal(buf[scale_index(rows, K, th, q)], first) for q in range(1, _replicas(th)))


def bundle_unpack(buf, rows, K, th):
    """Bundle bytes -> (codes [rows, K] 0..15, scales [rows, K/16] ue4m3 patterns)."""
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    cb = buf[code_index(rows, K, th)]
    codes = np.empty((rows, K), dtype=np.uint8)
    codes[:, 0::2] = cb & 0x0F
    codes[:, 1::2] = cb >> 4
    return codes, buf[scale_index(rows, K, th)]


def bundle_pack(codes, scales, rows, K, th):
    """(codes [rows, K], scales [rows, K/16]) -> bundle bytes; padding stays zero."""
    buf = np.zeros(bundle_size(rows, K, th), dtype=np.uint8)
    c = np.asarray(codes, dtype=np.uint8)
    buf[code_index(rows, K, th)] = c[:, 0::2] | (c[:, 1::2] << 4)
    for q in range(_replicas(th)):
        buf[scale_index(rows, K, th, q)] = np.asarray(scales, dtype=np.uint8)
    return buf


def bundle_padding_is_zero(buf, rows, K, th):
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    used = np.zeros(buf.size, dtype=bool)
    used[code_index(rows, K, th)] = True
    for q in range(_replicas(th)):
        used[scale_index(rows, K, th, q)] = True
    return not buf[~used].any()


def lowrank_index(rows, th):
    """Byte offsets of element (m, j), j < 64, of a low-rank tile buffer (bf16, 2 bytes)."""
    m = np.arange(rows)[:, None]
    j = np.arange(64)[None, :]
    r = m % th
    return (m // th) * th * 128 + r * 128 + ((((j >> 3) ^ r) & 7) << 4) + (j & 7) * 2


def lowrank_unpack(buf, rows, th):
    """Low-rank tile bytes -> bf16 bit patterns [rows, 64] (uint16)."""
    b = np.asarray(buf, dtype=np.uint8).reshape(-1)
    idx = lowrank_index(rows, th)
    return (b[idx].astype(np.uint16) | (b[idx + 1].astype(np.uint16) << 8))


def lowrank_pack(bits, th):
    """bf16 bit patterns [rows, r<=64] -> low-rank tile bytes (columns r.. zero)."""
    bits = np.asarray(bits, dtype=np.uint16)
    rows, r = bits.shape
    full = np.zeros((rows, 64), dtype=np.uint16)
    full[:, :r] = bits
    buf = np.zeros(((rows + th - 1) // th) * th * 128, dtype=np.uint8)
    idx = lowrank_index(rows, th)
    buf[idx] = (full & 0xFF).astype(np.uint8)
    buf[idx + 1] = (full >> 8).astype(np.uint8)
    return buf


def _awq_positions(K, N):
    """(k index, n index) of every nibble of the qweight array, by word and nibble, written
    from the layout in svdq.h: word (((Q*G + grp)*4 + b)*32 + lane)*4 + j, lane = 4g + t."""
    G = K // 64
    shape = (N // 64, G, 4, 32, 4)            # quad, group, block, lane, word j
    Q, grp, b, lane, j = np.indices(shape)
    g, t = lane // 4, lane % 4
    ks, ns = [], []
    for i in range(8):
        reg, odd = i % 4, i // 4
        c = g + 8 * (reg % 2)
        kq = 2 * t + odd + 8 * (reg // 2)
        ks.append(grp * 64 + j * 16 + kq)
        ns.append(Q * 64 + b * 16 + c)
    return ks, ns


def awq_unpack(qweight, K, N):
    """Fragment-order words -> q [K, N] (see the AWQ layout in svdq.h)."""
    w = np.asarray(qweight, dtype=np.uint32).reshape(N // 64, K // 64, 4, 32, 4)
    q = np.empty((K, N), dtype=np.uint8)
    ks, ns = _awq_positions(K, N)
    for i in range(8):
        q[ks[i], ns[i]] = ((w >> np.uint32(4 * i)) & np.uint32(15)).astype(np.uint8)
    return q


def awq_group_unpack(vals, K, N):
    """Per-group parameters (scales or zeros) in the library layout -> [K/64, N]."""
    v = np.asarray(vals).reshape(N // 64, K // 64, 64)
    return v.transpose(1, 0, 2).reshape(K // 64, N)


def bf16_bits_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- writers
# (the inverse direction: oracle arrays -> the library's packed layouts, so a
# kernel can be run on operands that the oracle produced)

def awq_pack(q):
    """q [K, N] (0..15) -> fragment-order words (the inverse of awq_unpack)."""
    q = np.asarray(q, dtype=np.uint8)
    K, N = q.shape
    w = np.zeros((N // 64, K // 64, 4, 32, 4), dtype=np.uint32)
    ks, ns = _awq_positions(K, N)
    for i in range(8):
        w |= q[ks[i], ns[i]].astype(np.uint32) << np.uint32(4 * i)
    return w.reshape(-1)


def awq_group_pack(vals):
    """[K/64, N] per-group parameters -> the library layout ((n/64)*G + g)*64 + n%64 (flattened)."""
    v = np.asarray(vals)
    g_n, N = v.shape
    return np.ascontiguousarray(v.reshape(g_n, N // 64, 64).transpose(1, 0, 2)).reshape(-1)


def bf16_bits(values):
    """bf16 bit patterns of float64 values that are exact bf16 numbers."""
    f = np.asarray(values, dtype=np.float64).astype(np.float32)
    if not np.array_equal(f.astype(np.float64), np.asarray(values, dtype=np.float64)):
        raise ValueError("not bf16 values")
    u = f.view(np.uint32)
    if (u & 0xFFFF).any():
        raise ValueError("not bf16 values")
    return (u >> 16).astype(np.uint16)


# ---- INT4 W4A4 operands: codes [rows][K/2] (element k in byte k/2, low nibble for even k, two's
# complement), scales [K/64][ld] bf16 (group-major)
def int4_pack(q):
    q = np.asarray(q, dtype=np.int8)
    u = (q.astype(np.int16) & 0xF).astype(np.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


def int4_unpack(codes, rows, K):
    c = np.asarray(codes, dtype=np.uint8).reshape(-1, K // 2)[:rows]
    lo = (c & 0xF).astype(np.int16)
    hi = (c >> 4).astype(np.int16)
    q = np.empty((rows, K), np.int8)
    q[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    q[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    return q


def int4_scales_pack(s, ld):
    """s: float64 [rows, K/64] holding bf16 values -> uint16 [K/64, ld] (columns past rows 0)."""
    rows, groups = s.shape
    out = np.zeros((groups, ld), np.uint16)
    out[:, :rows] = bf16_bits(s.T)
    return out


def int4_scales_unpack(buf, rows, groups, ld):
    b = np.asarray(buf, dtype=np.uint16).reshape(groups, ld)
    return bf16_bits_to_f64(b[:, :rows].T)

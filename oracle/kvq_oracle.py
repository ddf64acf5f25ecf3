"""Plain NumPy oracle: group quantize + nibble pack, dense decode, float64
attention, and the m/z/u block merge.

TEST INFRASTRUCTURE ONLY (see the package docstring): imported by ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs, never by the CUDA
product path.

Precision, as the pages fix it: the stored format is float32 scales and
unsigned byte codes; decoded K/V are float32 arrays; attention arithmetic is
float64 ("Block KV decoding: less workspace, more time", section "Compare
equivalent representations first": all methods do float64 attention, the
float32 refers to storage only).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# Symmetric integer range per bit width.  4-bit codes live in [-7, 7] and are
# stored +7 in [0, 14] (15 unused); 8-bit codes live in [-127, 127] and are
# stored +127 as an unsigned byte.  "KV分组打包：4-bit到底省了多少？", section
# "一个字节里到底装了什么".
QMAX = {4: 7, 8: 127}


@dataclass
class PackedMatrix:
    """One packed N x D matrix, exactly the arrays the pages store.

    codes  -- uint8, 1-D.  4-bit: two codes per byte over the row-major
              flattened padded code matrix; 8-bit: one code per byte.
    scales -- float32.  axis 0 (K): [ceil(N/g), D], one scale per channel per
              group of g tokens.  axis 1 (V): [N, ceil(D/g)], one scale per
              token per group of g features.
    shape  -- int32 [2], the original (N, D), kept so decode can crop.
    """

    codes: np.ndarray
    scales: np.ndarray
    shape: np.ndarray
    bits: int
    group: int
    axis: int

    @property
    def padded_shape(self) -> tuple[int, int]:
        n, d = (int(v) for v in self.shape)
        g = self.group
        if self.axis == 0:
            return (-(-n // g) * g, d)
        return (n, -(-d // g) * g)


# --------------------------------------------------------------------------
# nibble packing
# --------------------------------------------------------------------------

def pair_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two biased 4-bit codes per byte: even-indexed code in the low nibble,
    odd-indexed code in the high nibble ("KV分组打包", section
    "一个字节里到底装了什么": packed = codes[0::2] | codes[1::2] << 4)."""
    c = np.asarray(codes, dtype=np.uint8).ravel()
    if c.size % 2:
        raise ValueError("nibble pairing needs an even number of codes")
    return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)


def split_nibbles(packed: np.ndarray) -> np.ndarray:
    """Inverse of pair_nibbles: low = b & 15, high = b >> 4, interleaved back
    into code order (same section)."""
    b = np.asarray(packed, dtype=np.uint8).ravel()
    out = np.empty(b.size * 2, dtype=np.uint8)
    out[0::2] = b & 15
    out[1::2] = b >> 4
    return out


# --------------------------------------------------------------------------
# quantize / pack
# --------------------------------------------------------------------------

def quantize_groups(xg: np.ndarray, bits: int) -> tuple[np.ndarray, np.ndarray]:
    """Symmetric group quantization over the LAST axis of ``xg``.

    scale = max|x| / qmax per group in float32, with scale = 1 for an all-zero
    group so decode stays zero and nothing divides by zero ("KV分组打包",
    sections "一个字节里到底装了什么" and "小练习与常见错误").  code =
    round(x / scale), round half to even (NumPy's rounding), clipped to
    [-qmax, qmax], then biased by +qmax into an unsigned byte.
    Returns (biased codes uint8 with xg's shape, scales float32 with the last
    axis dropped).
    """
    qmax = QMAX[bits]
    x = np.asarray(xg, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)
    scale = (amax / np.float32(qmax)).astype(np.float32)
    scale = np.where(amax == 0, np.float32(1.0), scale).astype(np.float32)
    q = np.rint(x / scale[..., None]).astype(np.float32)
    q = np.clip(q, -qmax, qmax)
    codes = (q.astype(np.int16) + qmax).astype(np.uint8)
    return codes, scale


def pack_matrix(x: np.ndarray, bits: int, group: int, axis: int) -> PackedMatrix:
    """Pack one N x D matrix.

    axis = 0 is the K layout: groups of ``group`` consecutive tokens within
    each channel.  axis = 1 is the V layout: groups of ``group`` consecutive
    features within each token ("KV分组打包", section
    "为什么分组要同时看方向与长度").  A short last group is zero-padded
    (same section); padded positions quantize to code 0 (stored qmax).
    """
    if bits not in QMAX:
        raise ValueError("bits must be 4 or 8")
    if group < 2 or group % 2:
        raise ValueError("group must be even and >= 2")
    x = np.asarray(x, dtype=np.float32)
    if x.ndim != 2:
        raise ValueError("expected an N x D matrix")
    n, d = x.shape
    g = group
    if axis == 0:
        n_pad = -(-n // g) * g
        xp = np.zeros((n_pad, d), dtype=np.float32)
        xp[:n] = x
        # (groups, g, D) -> put the within-group token axis last
        xg = xp.reshape(n_pad // g, g, d).transpose(0, 2, 1)
        codes_g, scales = quantize_groups(xg, bits)          # [G, D, g], [G, D]
        codes = codes_g.transpose(0, 2, 1).reshape(n_pad, d)
    elif axis == 1:
        d_pad = -(-d // g) * g
        xp = np.zeros((n, d_pad), dtype=np.float32)
        xp[:, :d] = x
        xg = xp.reshape(n, d_pad // g, g)
        codes_g, scales = quantize_groups(xg, bits)          # [N, G, g], [N, G]
        codes = codes_g.reshape(n, d_pad)
    else:
        raise ValueError("axis must be 0 (K) or 1 (V)")
    flat = codes.ravel()                                      # row-major
    packed = pair_nibbles(flat) if bits == 4 else flat.astype(np.uint8).copy()
    return PackedMatrix(packed, scales.astype(np.float32),
                        np.array([n, d], dtype=np.int32), bits, g, axis)


def pack_k(k: np.ndarray, bits: int, group: int) -> PackedMatrix:
    """K is N x D, grouped along tokens within each channel."""
    return pack_matrix(k, bits, group, axis=0)


def pack_v(v: np.ndarray, bits: int, group: int) -> PackedMatrix:
    """V is N x D, grouped along features within each token."""
    return pack_matrix(v, bits, group, axis=1)


def _codes_of(p: PackedMatrix) -> np.ndarray:
    return split_nibbles(p.codes) if p.bits == 4 else np.asarray(p.codes, np.uint8)


def unpack_matrix(p: PackedMatrix) -> np.ndarray:
    """Decode to float32: (code - qmax) * scale, restore the padded shape, then
    crop the padding back to the stored (N, D) ("KV分组打包", section
    "一个字节里到底装了什么": decode keeps the original shape, removes the group
    padding and multiplies by the matching scale; it is not two's-complement
    int4 and not a codebook)."""
    qmax = QMAX[p.bits]
    n, d = (int(v) for v in p.shape)
    pn, pd = p.padded_shape
    codes = _codes_of(p)[: pn * pd].reshape(pn, pd)
    q = codes.astype(np.float32) - np.float32(qmax)
    g = p.group
    if p.axis == 0:
        s = np.repeat(p.scales, g, axis=0)                    # [pn, D]
    else:
        s = np.repeat(p.scales, g, axis=1)                    # [N, pd]
    x = (q * s).astype(np.float32)
    return x[:n, :d]


def unpack_rows(p: PackedMatrix, t0: int, t1: int) -> np.ndarray:
    """Decode only tokens [t0, t1) of a packed matrix, reading only the bytes
    and scales those tokens need -- the per-block decode of the blocked method
    ("Block KV decoding: less workspace, more time", section "Do not average
    independently normalized blocks": decode a block of tokens at a time)."""
    qmax = QMAX[p.bits]
    n, d = (int(v) for v in p.shape)
    t1 = min(t1, n)
    if t1 <= t0:
        return np.zeros((0, d), dtype=np.float32)
    pn, pd = p.padded_shape
    c0, c1 = t0 * pd, t1 * pd                                 # flat code range
    if p.bits == 4:
        b0, b1 = c0 // 2, -(-c1 // 2)
        codes = split_nibbles(p.codes[b0:b1])[c0 - 2 * b0: c0 - 2 * b0 + (c1 - c0)]
    else:
        codes = np.asarray(p.codes[c0:c1], np.uint8)
    q = codes.reshape(t1 - t0, pd).astype(np.float32) - np.float32(qmax)
    g = p.group
    if p.axis == 0:
        rows = np.arange(t0, t1) // g
        s = p.scales[rows]                                     # [rows, D]
    else:
        s = np.repeat(p.scales[t0:t1], g, axis=1)
    x = (q * s).astype(np.float32)
    return x[:, :d]


# --------------------------------------------------------------------------
# ledgers
# --------------------------------------------------------------------------

def payload_bytes(pk: PackedMatrix, pv: PackedMatrix) -> int:
    """Bytes of every array the format keeps: codes + float32 scales + the two
    int32 shape pairs ("KV分组打包", table in section
    "同一输入上的精度与空间交换": e.g. 5,136 B for 4-bit group 32 at N=128,
    D=32)."""
    return int(pk.codes.nbytes + pk.scales.nbytes + pk.shape.nbytes
               + pv.codes.nbytes + pv.scales.nbytes + pv.shape.nbytes)


def fixed_array_bytes(n: int, d: int, n_q: int, block: int) -> dict:
    """Shape x dtype size of the named arrays of the dense and the blocked
    method ("Block KV decoding: less workspace, more time", table in section
    "Which arrays shrink?"): decoded float32 K and V, one float64 score
    matrix."""
    f32, f64 = 4, 8
    return {
        "decoded_kv_dense": 2 * n * d * f32,
        "decoded_kv_block": 2 * block * d * f32,
        "scores_dense": n_q * n * f64,
        "scores_block": n_q * block * f64,
    }


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def attend_dense(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Row-wise softmax(scale * Q K^T) V in float64 ("给长前缀列一张有单位的资源账本",
    section "prefill 与 decode" onward: S = QK^T/sqrt(d_k), softmax, PV; the
    scale is an explicit argument).  The max is subtracted before exp, which
    leaves the result unchanged in exact arithmetic."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    s = float(scale) * (q @ k.T)
    s = s - s.max(axis=1, keepdims=True)
    w = np.exp(s)
    return (w @ v) / w.sum(axis=1, keepdims=True)


def attend_bruteforce(q, k, v, scale: float) -> np.ndarray:
    """Full softmax by explicit Python sums over every key, no matrix
    routines: out_i = sum_j exp(s_ij) v_j / sum_j exp(s_ij)
    ("给长前缀列一张有单位的资源账本", section "FlashAttention为什么不必保存整张热图").
    Only for tiny inputs."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq, d = q.shape
    n = k.shape[0]
    out = np.zeros((nq, v.shape[1]), np.float64)
    for i in range(nq):
        s = []
        for j in range(n):
            acc = 0.0
            for c in range(d):
                acc += float(q[i, c]) * float(k[j, c])
            s.append(float(scale) * acc)
        top = max(s)
        den = 0.0
        num = [0.0] * v.shape[1]
        for j in range(n):
            w = math.exp(s[j] - top)
            den += w
            for c in range(v.shape[1]):
                num[c] += w * float(v[j, c])
        for c in range(v.shape[1]):
            out[i, c] = num[c] / den
    return out


def partial_state(q, k, v, scale: float):
    """(m, z, u) of one block of keys in float64, per query row:
    m = max score, z = sum exp(s - m), u = exp(s - m) @ V.  An empty block
    has m = -inf, z = 0, u = 0 ("Block KV decoding", section "Do not average
    independently normalized blocks": initial m is -inf and z, u are zero)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq = q.shape[0]
    if k.shape[0] == 0:
        return (np.full(nq, -np.inf), np.zeros(nq), np.zeros((nq, v.shape[1])))
    s = float(scale) * (q @ k.T)
    m = s.max(axis=1)
    w = np.exp(s - m[:, None])
    return m, w.sum(axis=1), w @ v


def merge_partials(a, b):
    """Merge two (m, z, u) states with the block rule
    m_new = max(m_a, m_b); each side is rescaled by exp(m_side - m_new)
    ("Block KV decoding", section "Do not average independently normalized
    blocks"; "给长前缀列一张有单位的资源账本", section
    "FlashAttention为什么不必保存整张热图": both the old sum and the old weighted
    sum are rescaled).  A side with z == 0 (no valid key, m = -inf) is skipped
    so -inf - (-inf) is never formed (same section)."""
    ma, za, ua = (np.asarray(t, np.float64) for t in a)
    mb, zb, ub = (np.asarray(t, np.float64) for t in b)
    m = np.maximum(ma, mb)
    fa = np.where(za > 0, np.exp(np.where(za > 0, ma - m, 0.0)), 0.0)
    fb = np.where(zb > 0, np.exp(np.where(zb > 0, mb - m, 0.0)), 0.0)
    return m, fa * za + fb * zb, fa[:, None] * ua + fb[:, None] * ub


def attend_blocked(q, k, v, scale: float, block: int, trace: list | None = None) -> np.ndarray:
    """The m/z/u block merge exactly as the pages print it, in float64
    ("Block KV decoding", section "Do not average independently normalized
    blocks"; "注意力分塊", section "只要保留三個累積量"):

        m_new = max(m_old, max(block_scores))
        a     = exp(m_old - m_new)
        z_new = a*z_old + sum(exp(block_scores - m_new))
        u_new = a*u_old + exp(block_scores - m_new) @ block_V
        output = u / z

    m starts at -inf, z and u at zero; the first block takes over (a = 0).
    If ``trace`` is a list, (m, z, u) after every block is appended to it.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq = q.shape[0]
    m = np.full(nq, -np.inf)
    z = np.zeros(nq)
    u = np.zeros((nq, v.shape[1]))
    for t0 in range(0, k.shape[0], block):
        kb = k[t0:t0 + block]
        vb = v[t0:t0 + block]
        if kb.shape[0] == 0:
            continue
        s = float(scale) * (q @ kb.T)
        m_new = np.maximum(m, s.max(axis=1))
        a = np.where(np.isneginf(m), 0.0, np.exp(np.where(np.isneginf(m), 0.0, m - m_new)))
        p = np.exp(s - m_new[:, None])
        z = a * z + p.sum(axis=1)
        u = a[:, None] * u + p @ vb
        m = m_new
        if trace is not None:
            trace.append((m.copy(), z.copy(), u.copy()))
    return u / z[:, None]


def attend_blocked_packed(q, pk: PackedMatrix, pv: PackedMatrix, scale: float, block: int,
                          sizes: dict | None = None) -> np.ndarray:
    """The pages' "decode and merge blocks" method: decode ``block`` tokens of
    K and V from the packed arrays at a time and fold them into m/z/u, so the
    full decoded K/V and the full score matrix never exist ("Block KV
    decoding", sections "Do not average independently normalized blocks" and
    "Which arrays shrink?").  If ``sizes`` is a dict, the largest decoded K/V
    and score array byte sizes seen are recorded in it."""
    q = np.asarray(q, np.float64)
    n = int(pk.shape[0])
    nq = q.shape[0]
    m = np.full(nq, -np.inf)
    z = np.zeros(nq)
    u = np.zeros((nq, int(pv.shape[1])))
    kv_max = sc_max = 0
    for t0 in range(0, n, block):
        kb = unpack_rows(pk, t0, t0 + block)
        vb = unpack_rows(pv, t0, t0 + block)
        kv_max = max(kv_max, kb.nbytes + vb.nbytes)
        s = float(scale) * (q @ kb.astype(np.float64).T)
        sc_max = max(sc_max, s.nbytes)
        m_new = np.maximum(m, s.max(axis=1))
        a = np.where(np.isneginf(m), 0.0, np.exp(np.where(np.isneginf(m), 0.0, m - m_new)))
        p = np.exp(s - m_new[:, None])
        z = a * z + p.sum(axis=1)
        u = a[:, None] * u + p @ vb.astype(np.float64)
        m = m_new
    if sizes is not None:
        sizes["decoded_kv_block"] = kv_max
        sizes["scores_block"] = sc_max
    return u / z[:, None]


def attend_gqa_heads(q_bh: np.ndarray, k_hat: np.ndarray, v_hat: np.ndarray,
                     length: int, scale: float) -> np.ndarray:
    """One query head's rows against one KV head's decoded cache, keys
    [0, length) only: positions at or beyond the length enter neither the max
    nor the sum ("给长前缀列一张有单位的资源账本", section
    "FlashAttention为什么不必保存整张热图": masked positions take no part).
    Non-causal: every query row reads every valid key ("注意力分塊", opening
    section: the queries read the whole existing context)."""
    if length <= 0:
        raise ValueError("a row with no valid key has no softmax")
    return attend_dense(q_bh, k_hat[:length], v_hat[:length], scale)


def attend_gqa(q: np.ndarray, k_hat: np.ndarray, v_hat: np.ndarray,
               lengths, scale: float) -> np.ndarray:
    """Grouped-query attention over decoded caches.

    q      [B, H_q, Lq, D]
    k_hat  [B, H_kv, N, D] float32 decoded K
    v_hat  [B, H_kv, N, D] float32 decoded V
    Query head h reads KV head h // (H_q / H_kv): each group of H_q/H_kv query
    heads shares one K/V head ("给长前缀列一张有单位的资源账本", section
    "GQA改变共享接口").  Returns float64 [B, H_q, Lq, D].
    """
    b_, hq, lq, d = q.shape
    hkv = k_hat.shape[1]
    if hq % hkv:
        raise ValueError("H_q must be a multiple of H_kv")
    grp = hq // hkv
    out = np.zeros((b_, hq, lq, v_hat.shape[-1]), np.float64)
    for b in range(b_):
        for h in range(hq):
            out[b, h] = attend_gqa_heads(q[b, h], k_hat[b, h // grp], v_hat[b, h // grp],
                                         int(lengths[b]), scale)
    return out


def attend_gqa_window(q: np.ndarray, k_hat: np.ndarray, v_hat: np.ndarray, lengths,
                      k_win: np.ndarray, v_win: np.ndarray, win_lengths, scale: float) -> np.ndarray:
    """Grouped-query attention over a packed cache plus a window of recent
    tokens kept unquantized.

    The pages leave this as the next study: keep the same packed format and
    spend a limited high-precision budget on the most recent tokens
    ("KV分组打包：4-bit到底省了多少？", section "小练习与常见错误", last
    paragraph).  Reading taken here: the keys of sequence b are its decoded
    packed tokens [0, lengths[b]) followed by its window tokens
    [0, win_lengths[b]), stored as given (no quantization), and each query row
    takes one softmax over all of them -- softmax(QK^T/sqrt(d))V over the
    concatenation ("给长前缀列一张有单位的资源账本", section
    "FlashAttention为什么不必保存整张热图": positions past either length take
    no part).  GQA as in ``attend_gqa``.

    q [B, H_q, Lq, D]; k_hat, v_hat [B, H_kv, N, D] decoded; k_win, v_win
    [B, H_kv, W, D]; returns float64 [B, H_q, Lq, D].
    """
    b_, hq, lq, d = q.shape
    hkv = k_hat.shape[1]
    if hq % hkv:
        raise ValueError("H_q must be a multiple of H_kv")
    grp = hq // hkv
    out = np.zeros((b_, hq, lq, v_hat.shape[-1]), np.float64)
    for b in range(b_):
        n, w = int(lengths[b]), int(win_lengths[b])
        if n + w <= 0:
            raise ValueError("a row with no valid key has no softmax")
        for h in range(hq):
            g = h // grp
            k = np.concatenate([np.asarray(k_hat[b, g, :n], np.float64), np.asarray(k_win[b, g, :w], np.float64)])
            v = np.concatenate([np.asarray(v_hat[b, g, :n], np.float64), np.asarray(v_win[b, g, :w], np.float64)])
            out[b, h] = attend_dense(q[b, h], k, v, scale)
    return out


def attend_gqa_causal(q: np.ndarray, k_hat: np.ndarray, v_hat: np.ndarray,
                      lengths, scale: float) -> np.ndarray:
    """Causal multi-query attention over decoded caches: the Lq query rows of
    sequence b are its last Lq positions, L - Lq .. L - 1 (L = lengths[b]),
    and query i reads keys [0, L - Lq + i] only.  Keys after a query's own
    position are masked: they enter neither the max nor the sum
    ("给长前缀列一张有单位的资源账本", section "FlashAttention为什么不必保存整张
    热图").  The pages' own studies are non-causal ("注意力分塊", opening
    section, which names causal training prefill as something its method
    does not replace); this is the masked form their rule gives.  GQA as in
    ``attend_gqa``.  Returns float64 [B, H_q, Lq, D]; a row with no visible
    key (L < Lq) raises.
    """
    b_, hq, lq, d = q.shape
    hkv = k_hat.shape[1]
    if hq % hkv:
        raise ValueError("H_q must be a multiple of H_kv")
    grp = hq // hkv
    out = np.zeros((b_, hq, lq, v_hat.shape[-1]), np.float64)
    for b in range(b_):
        n = int(lengths[b])
        for h in range(hq):
            for i in range(lq):
                visible = n - lq + i + 1
                if visible <= 0:
                    raise ValueError("a row with no valid key has no softmax")
                out[b, h, i] = attend_dense(q[b, h, i:i + 1], k_hat[b, h // grp, :visible],
                                            v_hat[b, h // grp, :visible], scale)[0]
    return out


def rel_l2_error(out: np.ndarray, ref: np.ndarray) -> float:
    """||out - ref||_2 / ||ref||_2 over the whole output ("KV分组打包", section
    "同一输入上的精度与空间交换": relative L2 output error per input, then the
    mean over inputs)."""
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(out - ref) / np.linalg.norm(ref))


"""Pins for the CPU oracle: each check compares the oracle with something
other than itself -- values the pages print, closed forms, brute force on tiny
inputs, or the quantizer's own error bound.  Each raises AssertionError when
the oracle breaks the pinned fact.  ``tests/test_oracle_pins.py`` runs them,
and also plants plausible mistakes in the oracle to show that each mistake
trips at least one of them.
"""

from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

import oracle.kvq_oracle as O
import workloads as W
from tests.conftest import read_golden


def _num(tok: str) -> float:
    if tok == "ln2":
        return math.log(2.0)
    if tok == "ln3":
        return math.log(3.0)
    return float(Fraction(tok))


# --------------------------------------------------------------------------
# format pins
# --------------------------------------------------------------------------

def pin_nibble_example():
    kv, _ = read_golden("nibble_example.txt")
    codes = np.array([int(c) for c in kv["codes_biased"].split()], np.uint8)
    packed = O.pair_nibbles(codes)
    assert packed.tolist() == [int(kv["packed_hex"], 16)], packed
    back = O.split_nibbles(packed)
    assert back.tolist() == [int(kv["low_nibble"]), int(kv["high_nibble"])]
    signed = back.astype(int) - O.QMAX[4]
    assert signed.tolist() == [int(c) for c in kv["codes_signed"].split()]
    # the same byte out of a full pack: one V token [-5, 6, 7, 0], group 4:
    # max|x| = 7 so scale = 1 and the codes are x + 7 -> 2, 13, 14, 7.
    p = O.pack_v(np.array([[-5.0, 6.0, 7.0, 0.0]], np.float32), 4, 4)
    assert p.codes.tolist() == [0xD2, 0x7E], p.codes
    assert p.scales.tolist() == [[1.0]]
    assert O.unpack_matrix(p).tolist() == [[-5.0, 6.0, 7.0, 0.0]]


def pin_all_zero():
    """All-zero input: scale falls back to 1, codes are the bias, decode is
    zero, and nothing divides by zero."""
    for bits in (4, 8):
        for axis in (0, 1):
            with np.errstate(divide="raise", invalid="raise"):
                p = O.pack_matrix(np.zeros((35, 13), np.float32), bits, 8, axis)
                x = O.unpack_matrix(p)
            assert np.all(p.scales == 1.0)
            codes = O.split_nibbles(p.codes) if bits == 4 else p.codes
            assert np.all(codes == O.QMAX[bits])
            assert x.shape == (35, 13) and np.all(x == 0.0)


def pin_round_half_even():
    """Ties round to even.  A V token [0.5, 1.5, 2.5, 7] in one group of 4 has
    scale exactly 1, so the codes are rint(x) + 7 = 7, 9, 9, 14."""
    p = O.pack_v(np.array([[0.5, 1.5, 2.5, 7.0]], np.float32), 4, 4)
    assert O.split_nibbles(p.codes).tolist() == [7, 9, 9, 14]
    q = O.pack_v(np.array([[-0.5, -1.5, -2.5, -7.0]], np.float32), 4, 4)
    assert O.split_nibbles(q.codes).tolist() == [7, 5, 5, 0]


def pin_extreme_code():
    """The element of largest magnitude in a non-zero group maps to code
    +-qmax: scale = max|x| / qmax, so max|x| / scale = qmax up to one
    rounding."""
    rng = np.random.default_rng(7)
    for bits in (4, 8):
        x = rng.standard_normal((64, 32)).astype(np.float32)
        p = O.pack_matrix(x, bits, 8, axis=1)
        codes = (O.split_nibbles(p.codes) if bits == 4 else p.codes).reshape(64, 32).astype(int)
        g = codes.reshape(64, 4, 8) - O.QMAX[bits]
        xa = np.abs(x.reshape(64, 4, 8))
        arg = xa.argmax(axis=2)
        top = np.take_along_axis(g, arg[..., None], axis=2)[..., 0]
        assert np.all(np.abs(top) == O.QMAX[bits])
        assert codes.max() <= 2 * O.QMAX[bits] and codes.min() >= 0


def pin_error_bound():
    """Round-to-nearest: every decoded element lies within half a step
    (scale / 2) of its input, up to float32 rounding.  Checked for both
    layouts, both widths, both group sizes, on the 35 x 13 boundary case."""
    _, k, v = W.edge_35x13(0)
    for bits in (4, 8):
        for g in (8, 32):
            for axis, x in ((0, k), (1, v)):
                p = O.pack_matrix(x, bits, g, axis)
                y = O.unpack_matrix(p)
                assert y.shape == x.shape
                if axis == 0:
                    s = np.repeat(p.scales, g, axis=0)[: x.shape[0]]
                else:
                    s = np.repeat(p.scales, g, axis=1)[:, : x.shape[1]]
                err = np.abs(y.astype(np.float64) - x.astype(np.float64))
                assert np.all(err <= 0.5 * s * (1 + 1e-5) + 1e-7), float((err / s).max())


def pin_grouping_axes():
    """K is grouped along tokens within each channel; V along features within
    each token.  Scaling one K channel by 100 changes only that channel's
    scales; scaling one V token by 100 changes only that token's scales."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 32)).astype(np.float32)
    pk = O.pack_k(x, 4, 8)
    assert pk.scales.shape == (8, 32)
    y = x.copy()
    y[:, 5] *= 100
    pk2 = O.pack_k(y, 4, 8)
    changed = np.argwhere(pk2.scales != pk.scales)
    assert set(changed[:, 1].tolist()) == {5}
    pv = O.pack_v(x, 4, 8)
    assert pv.scales.shape == (64, 4)
    z = x.copy()
    z[9, :] *= 100
    pv2 = O.pack_v(z, 4, 8)
    changed = np.argwhere(pv2.scales != pv.scales)
    assert set(changed[:, 0].tolist()) == {9}
    # K scale of (group gi, channel c) is max over tokens gi*8 .. gi*8+7
    expect = (np.abs(x).reshape(8, 8, 32).max(axis=1) / np.float32(7)).astype(np.float32)
    assert np.array_equal(pk.scales, expect)


def pin_flat_pairing_odd_width():
    """Pairs are taken over the row-major flattened padded code matrix, so
    with an odd width a byte straddles two rows.  K 2 x 3, group 2, values
    chosen so every scale is 1 and codes are x + 7."""
    k = np.array([[1.0, -2.0, 7.0], [7.0, 7.0, -3.0]], np.float32)
    p = O.pack_k(k, 4, 2)
    # flattened codes: 8 5 14 14 14 4 -> bytes 8|5<<4, 14|14<<4, 14|4<<4
    assert p.codes.tolist() == [8 | 5 << 4, 14 | 14 << 4, 14 | 4 << 4]
    assert np.array_equal(O.unpack_matrix(p), k)


def pin_crop_35x13():
    """The 35 x 13 case round-trips to exactly (35, 13): padding never
    survives decode, for K (35 -> 40 or 64 tokens padded) and V (13 -> 16 or
    32 features padded)."""
    _, k, v = W.edge_35x13(0)
    for g, kpad, vpad in ((8, 40, 16), (32, 64, 32)):
        pk, pv = O.pack_k(k, 4, g), O.pack_v(v, 4, g)
        assert pk.padded_shape == (kpad, 13) and pv.padded_shape == (35, vpad)
        assert pk.codes.size == kpad * 13 // 2 and pv.codes.size == 35 * vpad // 2
        assert O.unpack_matrix(pk).shape == (35, 13)
        assert O.unpack_matrix(pv).shape == (35, 13)
        # per-row decode agrees with the whole-matrix decode
        for t0 in range(0, 35, 7):
            assert np.array_equal(O.unpack_rows(pk, t0, t0 + 7), O.unpack_matrix(pk)[t0:t0 + 7])
            assert np.array_equal(O.unpack_rows(pv, t0, t0 + 7), O.unpack_matrix(pv)[t0:t0 + 7])


def pin_eight_bit():
    """8-bit: codes in [-127, 127] stored +127, one per byte."""
    x = np.array([[-127.0, 0.0, 1.0, 127.0]], np.float32)
    p = O.pack_v(x, 8, 4)
    assert p.codes.tolist() == [0, 127, 128, 254]
    assert np.array_equal(O.unpack_matrix(p), x)


def pin_ledger():
    kv, rows = read_golden("ledger_n128_d32.txt")
    q, k, v = W.single_head(128, 32, 4, 0, "clean")
    for g, bits, want in rows:
        pk, pv = O.pack_k(k, int(bits), int(g)), O.pack_v(v, int(bits), int(g))
        assert O.payload_bytes(pk, pv) == int(want), (g, bits)
    assert k.nbytes + v.nbytes == int(kv["float32_kv_bytes"])
    pk, pv = O.pack_k(k, 4, 32), O.pack_v(v, 4, 32)
    saving = 100 * (1 - O.payload_bytes(pk, pv) / (k.nbytes + v.nbytes))
    assert round(saving, 1) == float(kv["saving_pct_g32_4bit"])


def pin_workspace_sizes():
    kv, _ = read_golden("workspace_n512_d32_q4.txt")
    sizes = O.fixed_array_bytes(512, 32, 4, 32)
    for key in ("decoded_kv_dense", "decoded_kv_block", "scores_dense", "scores_block"):
        assert sizes[key] == int(kv[key]), key
    # and the blocked method really only ever holds one block
    q, k, v = W.single_head(512, 32, 4, 0, "clean")
    seen: dict = {}
    O.attend_blocked_packed(q, O.pack_k(k, 4, 32), O.pack_v(v, 4, 32), 1 / math.sqrt(32), 32, seen)
    assert seen["decoded_kv_block"] == int(kv["decoded_kv_block"])
    assert seen["scores_block"] == int(kv["scores_block"])


# --------------------------------------------------------------------------
# attention pins
# --------------------------------------------------------------------------

def pin_17_over_3():
    kv, _ = read_golden("online_softmax_17_3.txt")
    s = [_num(t) for t in kv["scores"].split()]
    vals = [_num(t) for t in kv["values"].split()]
    # D = 1, Q = [[1]], K = scores, scale 1 -> the scores are exactly s
    q = np.array([[1.0]])
    k = np.array(s)[:, None]
    v = np.array(vals)[:, None]
    trace: list = []
    out = O.attend_blocked(q, k, v, 1.0, block=2, trace=trace)
    assert len(trace) == 2
    for i, stop in enumerate(("stop1", "stop2")):
        m, z, u = trace[i]
        assert abs(m[0] - _num(kv[stop + "_m"])) < 1e-15
        assert abs(z[0] - _num(kv[stop + "_z"])) < 1e-14
        assert abs(u[0, 0] - _num(kv[stop + "_u"])) < 1e-13
        assert abs(u[0, 0] / z[0] - _num(kv[stop + "_out"])) < 1e-14
    assert abs(out[0, 0] - 17 / 3) < 1e-14
    assert abs(O.attend_dense(q, k, v, 1.0)[0, 0] - 17 / 3) < 1e-14


def pin_17_over_3_window_and_causal():
    """The pages' worked example through the two later paths.  Window: the
    first two keys packed (decoded values given as they are), the third in
    the window -- one softmax over all three gives 17/3.  Causal: three query
    rows at positions 0, 1, 2 read one, two and three keys, giving the value
    2, the first stop's 10/3 and the final 17/3."""
    kv, _ = read_golden("online_softmax_17_3.txt")
    s = [_num(t) for t in kv["scores"].split()]
    vals = [_num(t) for t in kv["values"].split()]
    k = np.array(s)[None, None, :, None]            # [B, H, N, D] with D = 1
    v = np.array(vals)[None, None, :, None]
    q1 = np.ones((1, 1, 1, 1))
    win = O.attend_gqa_window(q1, k[:, :, :2], v[:, :, :2], [2], k[:, :, 2:], v[:, :, 2:], [1], 1.0)
    assert abs(win[0, 0, 0, 0] - _num(kv["stop2_out"])) < 1e-14
    q3 = np.ones((1, 1, 3, 1))
    rows = O.attend_gqa_causal(q3, k, v, [3], 1.0)[0, 0, :, 0]
    assert abs(rows[0] - vals[0]) < 1e-15
    assert abs(rows[1] - _num(kv["stop1_out"])) < 1e-14
    assert abs(rows[2] - _num(kv["stop2_out"])) < 1e-14


def block_average(q, k, v, scale, block):
    """The wrong baseline the pages warn about: softmax each block on its own,
    then average the block outputs with equal weight."""
    outs = []
    for t0 in range(0, k.shape[0], block):
        outs.append(O.attend_dense(q, k[t0:t0 + block], v[t0:t0 + block], scale))
    return np.mean(outs, axis=0)


def pin_negative_example():
    """Scores 0, 10, 20 with values 1, 3, 5, blocks {0, 10} and {20}: the full
    softmax is (1 + 3e^10 + 5e^20) / (1 + e^10 + e^20) ~= 4.99991 while the
    block average is ~= 3.99995 ("注意力分塊", section
    "為什麼每塊單獨歸一化再平均不對")."""
    q = np.array([[1.0]])
    k = np.array([[0.0], [10.0], [20.0]])
    v = np.array([[1.0], [3.0], [5.0]])
    e10, e20 = math.exp(10), math.exp(20)
    exact = (1 + 3 * e10 + 5 * e20) / (1 + e10 + e20)
    for out in (O.attend_dense(q, k, v, 1.0), O.attend_blocked(q, k, v, 1.0, 2),
                O.attend_bruteforce(q, k, v, 1.0)):
        assert abs(out[0, 0] - exact) < 1e-12
    avg = block_average(q, k, v, 1.0, 2)[0, 0]
    assert abs(exact - 4.99991) < 1e-5 and abs(avg - 3.99995) < 1e-5
    assert abs(avg - exact) > 0.5


def pin_dense_vs_blocked():
    """The 18 inputs (3 seeds x 2 lengths x 3 distributions), 4-bit group 32:
    dense decode and block decode + merge agree within 1e-10, at block 32 and
    at block 7 ("Block KV decoding", section "Compare equivalent
    representations first"; "注意力分塊", section "練習與排錯")."""
    for n, seed, dist in W.SINGLE_HEAD_GRID:
        q, k, v = W.single_head(n, 32, 4, seed, dist)
        pk, pv = O.pack_k(k, 4, 32), O.pack_v(v, 4, 32)
        dense = O.attend_dense(q, O.unpack_matrix(pk), O.unpack_matrix(pv), 1 / math.sqrt(32))
        for block in (32, 7):
            blk = O.attend_blocked_packed(q, pk, pv, 1 / math.sqrt(32), block)
            assert np.max(np.abs(blk - dense)) < 1e-10, (n, seed, dist, block)


def pin_bruteforce():
    """Tiny inputs: explicit-sum softmax, the dense path and the blocked path
    agree to 1e-12; a one-token cache returns its value row exactly."""
    rng = np.random.default_rng(11)
    for n in range(1, 9):
        q = rng.standard_normal((3, 5))
        k = rng.standard_normal((n, 5))
        v = rng.standard_normal((n, 4))
        bf = O.attend_bruteforce(q, k, v, 0.7)
        assert np.max(np.abs(O.attend_dense(q, k, v, 0.7) - bf)) < 1e-12
        for block in (1, 2, 3, 7):
            assert np.max(np.abs(O.attend_blocked(q, k, v, 0.7, block) - bf)) < 1e-12
    v1 = rng.standard_normal((1, 6))
    out = O.attend_dense(rng.standard_normal((2, 3)), rng.standard_normal((1, 3)), v1, 1.0)
    assert np.max(np.abs(out - v1)) < 1e-15


def pin_large_scores_stay_finite():
    """Scores near 1000 overflow a plain exp; the max shift keeps the result
    finite and equal to the closed form ("注意力分塊", section "練習與排錯")."""
    q = np.array([[1.0]])
    k = np.array([[1000.0], [999.0], [998.0]])
    v = np.array([[1.0], [2.0], [4.0]])
    w = np.array([1.0, math.exp(-1), math.exp(-2)])
    exact = float(w @ v[:, 0] / w.sum())
    for out in (O.attend_dense(q, k, v, 1.0), O.attend_blocked(q, k, v, 1.0, 1)):
        assert np.isfinite(out).all() and abs(out[0, 0] - exact) < 1e-12


def pin_merge_partials():
    """Split-KV: partial (m, z, u) states over any split of the keys, merged
    in any bracketing, give the dense result; empty partials are skipped."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal((4, 8))
    k = rng.standard_normal((50, 8)) * 3
    v = rng.standard_normal((50, 8))
    dense = O.attend_dense(q, k, v, 0.5)
    cuts = [0, 0, 13, 13, 31, 50]          # includes two empty pieces
    parts = [O.partial_state(q, k[a:b], v[a:b], 0.5) for a, b in zip(cuts[:-1], cuts[1:])]
    left = parts[0]
    for p in parts[1:]:
        left = O.merge_partials(left, p)
    right = parts[-1]
    for p in reversed(parts[:-1]):
        right = O.merge_partials(p, right)
    for m, z, u in (left, right):
        assert np.isfinite(m).all()
        assert np.max(np.abs(u / z[:, None] - dense)) < 1e-12


def pin_gqa_and_lengths():
    """Query head h reads KV head h // (H_q / H_kv); keys at or beyond a
    sequence's length are ignored.  Checked against brute force per head."""
    rng = np.random.default_rng(9)
    b_, hq, hkv, lq, n, d = 2, 4, 2, 3, 9, 5
    q = rng.standard_normal((b_, hq, lq, d))
    k = rng.standard_normal((b_, hkv, n, d))
    v = rng.standard_normal((b_, hkv, n, d))
    lens = [9, 4]
    out = O.attend_gqa(q, k, v, lens, 0.9)
    for b in range(b_):
        for h in range(hq):
            hk = h // (hq // hkv)
            bf = O.attend_bruteforce(q[b, h], k[b, hk, :lens[b]], v[b, hk, :lens[b]], 0.9)
            assert np.max(np.abs(out[b, h] - bf)) < 1e-12


def pin_window():
    """Packed cache plus an unquantized recent window: brute force over the
    concatenated keys of each (b, head), window positions past each
    sequence's window length ignored (filled with huge values here so that
    reading them would show), a packed part of length 0, and the two-part
    block merge of the packed and window states giving the same rows."""
    rng = np.random.default_rng(21)
    b_, hq, hkv, lq, n, w_cap, d = 3, 4, 2, 2, 7, 5, 6
    q = rng.standard_normal((b_, hq, lq, d))
    k = rng.standard_normal((b_, hkv, n, d))
    v = rng.standard_normal((b_, hkv, n, d))
    kw = rng.standard_normal((b_, hkv, w_cap, d))
    vw = rng.standard_normal((b_, hkv, w_cap, d))
    lens, wl = [7, 0, 3], [2, 5, 0]
    for b in range(b_):
        kw[b, :, wl[b]:] = 1e6
        vw[b, :, wl[b]:] = -1e6
    out = O.attend_gqa_window(q, k, v, lens, kw, vw, wl, 0.7)
    for b in range(b_):
        for h in range(hq):
            hk = h // (hq // hkv)
            kk = np.concatenate([k[b, hk, :lens[b]], kw[b, hk, :wl[b]]])
            vv = np.concatenate([v[b, hk, :lens[b]], vw[b, hk, :wl[b]]])
            bf = O.attend_bruteforce(q[b, h], kk, vv, 0.7)
            assert np.max(np.abs(out[b, h] - bf)) < 1e-12
            if lens[b] and wl[b]:
                st = O.merge_partials(O.partial_state(q[b, h], k[b, hk, :lens[b]], v[b, hk, :lens[b]], 0.7),
                                      O.partial_state(q[b, h], kw[b, hk, :wl[b]], vw[b, hk, :wl[b]], 0.7))
                assert np.max(np.abs(st[2] / st[1][:, None] - out[b, h])) < 1e-12
    # no window at all is the plain cache
    assert np.max(np.abs(O.attend_gqa_window(q, k, v, [7, 4, 3], kw, vw, [0, 0, 0], 0.7)
                         - O.attend_gqa(q, k, v, [7, 4, 3], 0.7))) < 1e-12


def pin_causal():
    """Causal rows: brute force over each query's visible keys [0, L - Lq + i]
    (keys past it filled with huge values so that reading them would show);
    one query row is the plain cache; the last row of a chunk sees every
    key, the first row L - Lq + 1 of them."""
    rng = np.random.default_rng(23)
    b_, hq, hkv, lq, n, d = 2, 4, 2, 3, 9, 5
    q = rng.standard_normal((b_, hq, lq, d))
    k = rng.standard_normal((b_, hkv, n, d))
    v = rng.standard_normal((b_, hkv, n, d))
    lens = [9, 5]
    k[1, :, 5:] = 1e6
    v[1, :, 5:] = -1e6
    out = O.attend_gqa_causal(q, k, v, lens, 0.8)
    for b in range(b_):
        for h in range(hq):
            hk = h // (hq // hkv)
            for i in range(lq):
                vis = lens[b] - lq + i + 1
                bf = O.attend_bruteforce(q[b, h, i:i + 1], k[b, hk, :vis], v[b, hk, :vis], 0.8)
                assert np.max(np.abs(out[b, h, i] - bf[0])) < 1e-12
    full = O.attend_gqa(q, k, v, lens, 0.8)
    assert np.max(np.abs(out[:, :, -1] - full[:, :, -1])) < 1e-12
    assert np.max(np.abs(out[:, :, 0] - full[:, :, 0])) > 1e-3      # the first row sees fewer keys
    one = O.attend_gqa_causal(q[:, :, :1], k, v, lens, 0.8)
    assert np.max(np.abs(one - O.attend_gqa(q[:, :, :1], k, v, lens, 0.8))) < 1e-12


def pin_rel_l2_definition():
    """The error measure itself, by closed forms: zero for identical arrays,
    1 for twice the reference, |e| / |x| for an error orthogonal to the
    reference (here 3-4-5: |e| = 5 against |x| = 10), taken over the whole
    array, not per row."""
    x = np.array([[6.0, 0.0], [0.0, 8.0]])
    assert O.rel_l2_error(x, x) == 0.0
    assert abs(O.rel_l2_error(2 * x, x) - 1.0) < 1e-15
    e = np.array([[0.0, 3.0], [4.0, 0.0]])
    assert abs(O.rel_l2_error(x + e, x) - 0.5) < 1e-15
    # whole-array norm: a per-row mean would give (3/6 + 4/8) / 2 = 0.5 too, so
    # use rows of different scale to tell them apart
    y = np.array([[1.0, 0.0], [0.0, 100.0]])
    f = np.array([[0.0, 1.0], [0.0, 0.0]])
    assert abs(O.rel_l2_error(y + f, y) - 1.0 / math.sqrt(10001.0)) < 1e-15


def pin_rel_l2_band():
    """Soft check (parity unpinned at the value level): the mean relative L2
    output error on the six clean inputs lands near the pages' table, and the
    4-bit / 8-bit ratio is near 127 / 7.  Band: within 25% of each printed
    value."""
    _, rows = read_golden("rel_l2_clean.txt")
    got = {}
    for g, bits, pct in rows:
        errs = []
        for n in (128, 512):
            for seed in (0, 1, 2):
                q, k, v = W.single_head(n, 32, 4, seed, "clean")
                ref = O.attend_dense(q, k, v, 1 / math.sqrt(32))
                pk, pv = O.pack_k(k, int(bits), int(g)), O.pack_v(v, int(bits), int(g))
                out = O.attend_dense(q, O.unpack_matrix(pk), O.unpack_matrix(pv), 1 / math.sqrt(32))
                errs.append(O.rel_l2_error(out, ref))
        got[(g, bits)] = 100 * float(np.mean(errs))
        assert abs(got[(g, bits)] / float(pct) - 1) < 0.25, (g, bits, got[(g, bits)], pct)
    ratio = got[("32", "4")] / got[("32", "8")]
    assert 10 < ratio < 30, ratio


ALL_PINS = [
    pin_nibble_example, pin_all_zero, pin_round_half_even, pin_extreme_code,
    pin_error_bound, pin_grouping_axes, pin_flat_pairing_odd_width, pin_crop_35x13,
    pin_eight_bit, pin_ledger, pin_workspace_sizes, pin_17_over_3,
    pin_negative_example, pin_dense_vs_blocked, pin_bruteforce,
    pin_large_scores_stay_finite, pin_merge_partials, pin_gqa_and_lengths, pin_window,
    pin_causal, pin_17_over_3_window_and_causal, pin_rel_l2_definition,
]

"""CPU tests: the oracle against its pins, and mutation tests that plant a
plausible mistake in the oracle and check that some pin catches it."""

from __future__ import annotations

import numpy as np
import pytest

import oracle.kvq_oracle as O
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_rel_l2_soft_band():
    P.pin_rel_l2_band()


def _fails_some_pin(pins=None):
    failed = []
    for pin in pins or P.ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, FloatingPointError, ValueError, IndexError):
            failed.append(pin.__name__)
    return failed


# ---- planted mistakes ------------------------------------------------------

def _swapped_pair(codes):
    c = np.asarray(codes, np.uint8).ravel()
    return (c[1::2] | (c[0::2] << 4)).astype(np.uint8)


def _swapped_split(packed):
    b = np.asarray(packed, np.uint8).ravel()
    out = np.empty(b.size * 2, np.uint8)
    out[0::2] = b >> 4
    out[1::2] = b & 15
    return out


def _round_half_up(xg, bits):
    qmax = O.QMAX[bits]
    x = np.asarray(xg, np.float32)
    amax = np.max(np.abs(x), axis=-1)
    scale = np.where(amax == 0, np.float32(1), (amax / np.float32(qmax))).astype(np.float32)
    q = np.clip(np.floor(x / scale[..., None] + np.float32(0.5)), -qmax, qmax)
    return (q.astype(np.int16) + qmax).astype(np.uint8), scale


def _scale_off_by_one(xg, bits):
    qmax = O.QMAX[bits]
    x = np.asarray(xg, np.float32)
    amax = np.max(np.abs(x), axis=-1)
    scale = np.where(amax == 0, np.float32(1), (amax / np.float32(qmax + 1))).astype(np.float32)
    q = np.clip(np.rint(x / scale[..., None]), -qmax, qmax)
    return (q.astype(np.int16) + qmax).astype(np.uint8), scale


def _no_zero_fallback(xg, bits):
    qmax = O.QMAX[bits]
    x = np.asarray(xg, np.float32)
    scale = (np.max(np.abs(x), axis=-1) / np.float32(qmax)).astype(np.float32)
    q = np.clip(np.rint(x / scale[..., None]), -qmax, qmax)
    return (np.nan_to_num(q).astype(np.int16) + qmax).astype(np.uint8), scale


def _k_on_wrong_axis(k, bits, group):
    return O.pack_matrix(k, bits, group, axis=1)


def _blocked_without_rescale_u(q, k, v, scale, block, trace=None):
    q, k, v = (np.asarray(t, np.float64) for t in (q, k, v))
    m = np.full(q.shape[0], -np.inf)
    z = np.zeros(q.shape[0])
    u = np.zeros((q.shape[0], v.shape[1]))
    for t0 in range(0, k.shape[0], block):
        s = scale * (q @ k[t0:t0 + block].T)
        m_new = np.maximum(m, s.max(axis=1))
        a = np.where(np.isneginf(m), 0.0, np.exp(np.where(np.isneginf(m), 0.0, m - m_new)))
        p = np.exp(s - m_new[:, None])
        z = a * z + p.sum(axis=1)
        u = u + p @ v[t0:t0 + block]             # the a*u_old rescale dropped
        m = m_new
        if trace is not None:
            trace.append((m.copy(), z.copy(), u.copy()))
    return u / z[:, None]


def _blocked_packed_without_rescale_u(q, pk, pv, scale, block, sizes=None):
    q = np.asarray(q, np.float64)
    m = np.full(q.shape[0], -np.inf)
    z = np.zeros(q.shape[0])
    u = np.zeros((q.shape[0], int(pv.shape[1])))
    for t0 in range(0, int(pk.shape[0]), block):
        kb = O.unpack_rows(pk, t0, t0 + block).astype(np.float64)
        vb = O.unpack_rows(pv, t0, t0 + block).astype(np.float64)
        if sizes is not None:
            sizes["decoded_kv_block"] = max(sizes.get("decoded_kv_block", 0), 4 * (kb.size + vb.size))
            sizes["scores_block"] = max(sizes.get("scores_block", 0), 8 * q.shape[0] * kb.shape[0])
        s = scale * (q @ kb.T)
        m_new = np.maximum(m, s.max(axis=1))
        a = np.where(np.isneginf(m), 0.0, np.exp(np.where(np.isneginf(m), 0.0, m - m_new)))
        p = np.exp(s - m_new[:, None])
        z = a * z + p.sum(axis=1)
        u = u + p @ vb                             # the a*u_old rescale dropped
        m = m_new
    return u / z[:, None]


def _merge_without_rescale(a, b):
    ma, za, ua = a
    mb, zb, ub = b
    return np.maximum(ma, mb), za + zb, ua + ub


def _gqa_modulo(q, k_hat, v_hat, lengths, scale):
    b_, hq = q.shape[:2]
    hkv = k_hat.shape[1]
    out = np.zeros(q.shape[:3] + (v_hat.shape[-1],))
    for b in range(b_):
        for h in range(hq):
            out[b, h] = O.attend_gqa_heads(q[b, h], k_hat[b, h % hkv], v_hat[b, h % hkv],
                                           int(lengths[b]), scale)
    return out


def _heads_ignore_length(q_bh, k_hat, v_hat, length, scale):
    return O.attend_dense(q_bh, k_hat, v_hat, scale)


def _unpack_no_crop(p):
    qmax = O.QMAX[p.bits]
    pn, pd = p.padded_shape
    codes = O._codes_of(p)[: pn * pd].reshape(pn, pd).astype(np.float32) - qmax
    s = np.repeat(p.scales, p.group, axis=0 if p.axis == 0 else 1)
    return codes * s


def _dense_without_scale(q, k, v, scale):
    q, k, v = (np.asarray(t, np.float64) for t in (q, k, v))
    s = q @ k.T
    w = np.exp(s - s.max(axis=1, keepdims=True))
    return (w @ v) / w.sum(axis=1, keepdims=True)


def _window_scale_dropped(q, k_hat, v_hat, lengths, k_win, v_win, win_lengths, scale):
    out = _ORIG_WINDOW(q, k_hat, v_hat, lengths, k_win, v_win, win_lengths, 1.0)
    return out


def _window_length_ignored(q, k_hat, v_hat, lengths, k_win, v_win, win_lengths, scale):
    full = [k_win.shape[2]] * len(win_lengths)
    return _ORIG_WINDOW(q, k_hat, v_hat, lengths, k_win, v_win, full, scale)


def _window_before_packed_length(q, k_hat, v_hat, lengths, k_win, v_win, win_lengths, scale):
    # the window replaces the packed tail instead of following it
    cut = [max(0, int(n) - int(w)) for n, w in zip(lengths, win_lengths)]
    return _ORIG_WINDOW(q, k_hat, v_hat, cut, k_win, v_win, win_lengths, scale)


def _rel_l2_per_row(out, ref):
    out = np.atleast_2d(np.asarray(out, np.float64))
    ref = np.atleast_2d(np.asarray(ref, np.float64))
    return float(np.mean(np.linalg.norm(out - ref, axis=-1) / np.linalg.norm(ref, axis=-1)))


def _rel_l1(out, ref):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(out - ref).sum() / np.abs(ref).sum())


_ORIG_WINDOW = O.attend_gqa_window
_ORIG_CAUSAL = O.attend_gqa_causal


def _causal_off_by_one(q, k_hat, v_hat, lengths, scale):
    # each query also sees the next position
    longer = [min(int(n) + 1, k_hat.shape[2]) for n in lengths]
    return _ORIG_CAUSAL(q, k_hat, v_hat, longer, scale)


def _causal_rows_reversed(q, k_hat, v_hat, lengths, scale):
    # query i takes the limit of query Lq - 1 - i
    return _ORIG_CAUSAL(q[:, :, ::-1], k_hat, v_hat, lengths, scale)[:, :, ::-1]


MUTATIONS = {
    "nibble_order_swapped": [("pair_nibbles", _swapped_pair), ("split_nibbles", _swapped_split)],
    "round_half_up": [("quantize_groups", _round_half_up)],
    "scale_divides_by_qmax_plus_1": [("quantize_groups", _scale_off_by_one)],
    "no_all_zero_fallback": [("quantize_groups", _no_zero_fallback)],
    "k_grouped_along_features": [("pack_k", _k_on_wrong_axis)],
    "blocked_drops_a_u_old": [("attend_blocked", _blocked_without_rescale_u)],
    "packed_blocked_drops_a_u_old": [("attend_blocked_packed", _blocked_packed_without_rescale_u)],
    "merge_without_rescale": [("merge_partials", _merge_without_rescale)],
    "gqa_head_modulo": [("attend_gqa", _gqa_modulo)],
    "length_mask_ignored": [("attend_gqa_heads", _heads_ignore_length)],
    "decode_keeps_padding": [("unpack_matrix", _unpack_no_crop)],
    "score_scale_dropped": [("attend_dense", _dense_without_scale)],
    "eight_bit_bias_128": [("QMAX", {4: 7, 8: 128})],
    "window_scale_dropped": [("attend_gqa_window", _window_scale_dropped)],
    "window_length_ignored": [("attend_gqa_window", _window_length_ignored)],
    "window_replaces_packed_tail": [("attend_gqa_window", _window_before_packed_length)],
    "causal_sees_one_more_key": [("attend_gqa_causal", _causal_off_by_one)],
    "causal_rows_reversed": [("attend_gqa_causal", _causal_rows_reversed)],
    "rel_l2_per_row_mean": [("rel_l2_error", _rel_l2_per_row)],
    "rel_l1_instead_of_l2": [("rel_l2_error", _rel_l1)],
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    for attr, repl in MUTATIONS[name]:
        monkeypatch.setattr(O, attr, repl)
    failed = _fails_some_pin()
    assert failed, f"planted mistake {name!r} passed every pin"

"""GPU parity: kvq_pack bit-exact against the oracle, kvq_attend within
2e-3 * max|V_hat| of the float64 oracle on the same decoded cache, on every
workload shape -- the single-head grid, the 35 x 13 edge case, ragged GQA
cases spanning several blocks and a tail, and the full-size decode,
long-context and chunk workloads (every head)."""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from tests.gpu_util import (DEV, assert_head_packed_equal, bf16_values, check_rows, check_rows_rounded,
                            oracle_rows, pack_gpu, single_head_scale, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sm_b200
    return sm_b200


# ---------------------------------------------------------------------------
# pack
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits,group", W.FORMATS)
def test_pack_single_head_grid(sm, bits, group):
    for n, seed, dist in W.SINGLE_HEAD_GRID:
        q, k, v = W.single_head(n, 32, 4, seed, dist)
        cache = pack_gpu(sm, k[None, None], v[None, None], bits, group)
        assert_head_packed_equal(cache, 0, 0, O.pack_k(k, bits, group), O.pack_v(v, bits, group))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("group", [8, 32])
@pytest.mark.parametrize("in_dtype", [torch.float32, torch.bfloat16])
def test_pack_35x13(sm, bits, group, in_dtype):
    _, k, v = W.edge_35x13(0)
    if in_dtype == torch.bfloat16:
        k, v = bf16_values(k), bf16_values(v)
    cache = pack_gpu(sm, k[None, None], v[None, None], bits, group, in_dtype)
    assert_head_packed_equal(cache, 0, 0, O.pack_k(k, bits, group), O.pack_v(v, bits, group))


def test_pack_all_zero_and_ties(sm):
    z = np.zeros((1, 1, 35, 13), np.float32)
    cache = pack_gpu(sm, z, z, 4, 8)
    assert_head_packed_equal(cache, 0, 0, O.pack_k(z[0, 0], 4, 8), O.pack_v(z[0, 0], 4, 8))
    ties = np.array([[0.5, 1.5, 2.5, 7.0, -0.5, -1.5, -2.5, -7.0]] * 4, np.float32)
    cache = pack_gpu(sm, ties[None, None], ties[None, None], 4, 8)
    assert_head_packed_equal(cache, 0, 0, O.pack_k(ties, 4, 8), O.pack_v(ties, 4, 8))


def test_pack_ties_d128(sm):
    """Width 128, group 32 (the warp-per-row V kernel): every group holds +-7
    (scale exactly 1) and half-integers, so the quotient lands on rounding
    ties and must round half to even; also a few random rows."""
    rng = np.random.default_rng(12)
    x = rng.integers(-14, 15, size=(1, 2, 64, 128)).astype(np.float32) / 2
    x[..., ::32] = 7.0
    x[..., 1, :] = rng.standard_normal(128).astype(np.float32)
    cache = pack_gpu(sm, x, x, 4, 32)
    for h in range(2):
        assert_head_packed_equal(cache, 0, h, O.pack_k(x[0, h], 4, 32), O.pack_v(x[0, h], 4, 32))
    cache8 = pack_gpu(sm, x * 127 / 7, x * 127 / 7, 8, 32)
    for h in range(2):
        y = (x[0, h] * 127 / 7).astype(np.float32)
        assert_head_packed_equal(cache8, 0, h, O.pack_k(y, 8, 32), O.pack_v(y, 8, 32))


def test_pack_halves_separately(sm):
    """K alone over a group-aligned range, then V alone over one token (the
    decode-step append), equals packing both together."""
    rng = np.random.default_rng(13)
    k = rng.standard_normal((2, 3, 64, 128)).astype(np.float32)
    v = rng.standard_normal((2, 3, 64, 128)).astype(np.float32)
    both = pack_gpu(sm, k, v, 4, 32)
    sep = sm.PackedCache(2, 3, 64, 128, 4, 32, DEV)
    sm.pack(to_dev(k), None, sep)
    for t in range(64):
        sm.pack(None, to_dev(v[:, :, t:t + 1]), sep, t0=t)
    for a, b in ((both.k_codes, sep.k_codes), (both.v_codes, sep.v_codes),
                 (both.k_scales, sep.k_scales), (both.v_scales, sep.v_scales)):
        assert torch.equal(a, b)


def test_pack_append_matches_whole(sm):
    """Packing [0, 64) then [64, 100) then re-packing the tail group from its
    start, [96, 130), gives the bytes of a whole [0, 130) pack."""
    rng = np.random.default_rng(4)
    k = rng.standard_normal((2, 3, 130, 40)).astype(np.float32)
    v = rng.standard_normal((2, 3, 130, 40)).astype(np.float32)
    whole = pack_gpu(sm, k, v, 4, 32)
    part = sm.PackedCache(2, 3, 130, 40, 4, 32, DEV)
    sm.pack(to_dev(k[:, :, 0:64]), to_dev(v[:, :, 0:64]), part, t0=0)
    sm.pack(to_dev(k[:, :, 64:100]), to_dev(v[:, :, 64:100]), part, t0=64)
    sm.pack(to_dev(k[:, :, 96:130]), to_dev(v[:, :, 96:130]), part, t0=96)
    for a, b in ((whole.k_codes, part.k_codes), (whole.v_codes, part.v_codes),
                 (whole.k_scales, part.k_scales), (whole.v_scales, part.v_scales)):
        assert torch.equal(a, b)
    for b_ in range(2):
        for h in range(3):
            assert_head_packed_equal(whole, b_, h, O.pack_k(k[b_, h], 4, 32), O.pack_v(v[b_, h], 4, 32))


# ---------------------------------------------------------------------------
# attend: single-head grid (72 comparisons) and the 35 x 13 case
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits,group", W.FORMATS)
def test_attend_single_head_grid(sm, bits, group):
    worst = 0.0
    for n, seed, dist in W.SINGLE_HEAD_GRID:
        q, k, v = W.single_head(n, 32, 4, seed, dist)
        cache = pack_gpu(sm, k[None, None], v[None, None], bits, group)
        lens = torch.tensor([n], dtype=torch.int32, device=DEV)
        out = sm.attend(to_dev(q[None, None]), cache, lens, single_head_scale(32))
        want, pk, pv, vh = oracle_rows(q, k, v, bits, group, n, single_head_scale(32))
        worst = max(worst, check_rows(out[0, 0].cpu().numpy(), want, vh, f"{n}/{seed}/{dist}"))
    sm.check()


@pytest.mark.parametrize("bits,group", W.FORMATS)
def test_attend_35x13(sm, bits, group):
    q, k, v = W.edge_35x13(0)
    cache = pack_gpu(sm, k[None, None], v[None, None], bits, group)
    lens = torch.tensor([35], dtype=torch.int32, device=DEV)
    out = sm.attend(to_dev(q[None, None]), cache, lens, single_head_scale(13))
    want, *_, vh = oracle_rows(q, k, v, bits, group, 35, single_head_scale(13))
    check_rows(out[0, 0].cpu().numpy(), want, vh, "35x13")
    # also against the pages' block-7 decode-and-merge path
    blk = O.attend_blocked_packed(q, O.pack_k(k, bits, group), O.pack_v(v, bits, group),
                                  single_head_scale(13), 7)
    check_rows(out[0, 0].cpu().numpy(), blk, vh, "35x13 vs block 7")


# ---------------------------------------------------------------------------
# attend: ragged GQA cases, split invariance, dtype, lengths
# ---------------------------------------------------------------------------

def _gqa_case(b_, hq, hkv, n_cap, d, lens, lq=1, seed=0, bits=4, group=32, outliers=False):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((b_, hkv, n_cap, d)).astype(np.float32)
    v = rng.standard_normal((b_, hkv, n_cap, d)).astype(np.float32)
    if outliers:
        k[:, :, :, ::37] *= 8
        v[:, :, :, 5::41] *= 8
    q = (rng.standard_normal((b_, hq, lq, d)) / math.sqrt(d)).astype(np.float32)
    return q, k, v, np.asarray(lens, np.int32)


def _check_gqa(sm, q, k, v, lens, bits, group, scale, q_dtype=torch.bfloat16, splits=0,
               heads=None, out_dtype_check=True):
    b_, hq, lq, d = q.shape
    hkv = k.shape[1]
    grp = hq // hkv
    cache = pack_gpu(sm, k, v, bits, group)
    qd = to_dev(q, q_dtype)
    qv = qd.float().cpu().numpy()
    out = sm.attend(qd, cache, to_dev(lens, torch.int32), scale, splits=splits)
    sm.check()
    assert out.dtype == q_dtype
    o = out.float().cpu().numpy()
    sel = heads if heads is not None else [(b, h) for b in range(b_) for h in range(hkv)]
    for b, h in sel:
        rows = qv[b, h * grp:(h + 1) * grp].reshape(grp * lq, d)
        want, pk, pv, vh = oracle_rows(rows, k[b, h], v[b, h], bits, group, int(lens[b]), scale)
        assert_head_packed_equal(cache, b, h, pk, pv)
        got = o[b, h * grp:(h + 1) * grp].reshape(grp * lq, d)
        if q_dtype == torch.bfloat16:
            check_rows_rounded(got, want, 2e-3 * float(np.abs(vh).max()), f"b{b} h{h}")
        else:
            check_rows(got, want, vh, f"b{b} h{h}")
    return o


@pytest.mark.parametrize("splits", [0, 1, 2, 7, 1000])
def test_gqa_ragged_split_invariance(sm, splits):
    # lengths not multiples of 32 or 128, one of a single token, capacity 300
    q, k, v, lens = _gqa_case(3, 8, 2, 300, 128, [300, 157, 1])
    _check_gqa(sm, q, k, v, lens, 4, 32, 1.0, splits=splits)


@pytest.mark.parametrize("bits,group", W.FORMATS)
def test_gqa_formats_fp32_q(sm, bits, group):
    q, k, v, lens = _gqa_case(2, 4, 1, 200, 64, [200, 77], seed=3)
    _check_gqa(sm, q, k, v, lens, bits, group, 1.0, q_dtype=torch.float32)


def test_gqa_multi_query_rows(sm):
    q, k, v, lens = _gqa_case(2, 8, 2, 260, 128, [260, 129], lq=5, seed=5, outliers=True)
    _check_gqa(sm, q, k, v, lens, 4, 32, 1.0)


@pytest.mark.parametrize("sign", [1.0, -1.0])
@pytest.mark.parametrize("lq", [32, 64])
def test_chunk_reference_moves_inside_block(sm, sign, lq):
    """Score spikes placed so that a row's running reference must move in
    the second, third and fourth 32-column quarter of a 128-token block (and
    in the first block, after its first quarter), each by more than the lazy
    threshold: the p already written for the block is rescaled, and O and z
    of the earlier blocks too.  Both signs of the scale (a negative scale
    turns the row maximum into a minimum of the raw scores)."""
    rng = np.random.default_rng(77)
    b_, hq, hkv, n, d = 2, 8, 2, 520, 128
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    q = (u[None, None, None, :] + 0.05 * rng.standard_normal((b_, hq, lq, d))).astype(np.float32)
    k = rng.standard_normal((b_, hkv, n, d)).astype(np.float32)
    v = rng.standard_normal((b_, hkv, n, d)).astype(np.float32)
    # (token, natural-log score): block 0 quarter 2, block 1 quarter 1,
    # block 2 quarter 2, block 3 quarter 3; each about 11 log2 units above the last
    for t, c in ((80, 10.0), (168, 18.0), (326, 26.0), (484, 34.0)):
        k[:, :, t, :] = sign * c * u
    lens = np.asarray([520, 300], np.int32)
    cache = pack_gpu(sm, k, v, 4, 32)
    assert sm.kernel_name(cache, hq, lq).startswith("chunk")
    for splits in (0, 1, 3):
        _check_gqa(sm, q, k, v, lens, 4, 32, sign, splits=splits)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("lq", [32, 64])
def test_chunk_tensor_core_ragged(sm, bits, lq):
    """The tcgen05 chunk kernel (128 or 256 query rows per KV head): ragged
    lengths that end inside a 128-token block and inside a K group, a
    sequence shorter than one block, and several splits."""
    q, k, v, lens = _gqa_case(3, 8, 2, 700, 128, [700, 300, 77], lq=lq, seed=21 + bits, bits=bits)
    cache = pack_gpu(sm, k, v, bits, 32)
    assert sm.kernel_name(cache, 8, lq).startswith("chunk")
    for splits in (0, 1, 5):
        _check_gqa(sm, q, k, v, lens, bits, 32, 1.0, splits=splits)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("hq,hkv,lq", [(8, 2, 1), (4, 2, 1), (2, 2, 1), (2, 2, 3), (4, 2, 2)])
def test_decode_rows(sm, bits, hq, hkv, lq):
    """One to four query rows per KV head at D = 128, g = 32: lengths that end
    inside a block and inside a K group, one a power of two, one shorter
    than a K group, and several splits."""
    q, k, v, lens = _gqa_case(4, hq, hkv, 700, 128, [700, 300, 128, 29], lq=lq, seed=31 + bits + hq + lq,
                              bits=bits, outliers=True)
    for splits in (0, 1, 5):
        _check_gqa(sm, q, k, v, lens, bits, 32, 1.0, splits=splits)


@pytest.mark.parametrize("bits", [4, 8])
def test_decode_fp32_q_sharp(sm, bits):
    """f32 Q and a large score scale: the running maximum moves by far more
    than any rescale threshold from block to block, and the softmax is far
    from uniform."""
    q, k, v, lens = _gqa_case(2, 8, 2, 1000, 128, [1000, 517], seed=40 + bits, bits=bits)
    for j, f in enumerate([1.0, 2.0, 3.5, 5.0]):
        k[:, :, 250 * j:250 * (j + 1), :] *= f      # keys grow along the sequence
    k[:, :, ::128, :] *= 2.0                        # and one strong key per block
    _check_gqa(sm, q, k, v, lens, bits, 32, 3.0, q_dtype=torch.float32, splits=3)


def test_decode_bad_lengths(sm):
    q, k, v, _ = _gqa_case(3, 8, 2, 256, 128, [256, 256, 256], seed=9)
    cache = pack_gpu(sm, k, v, 4, 32)
    assert sm.kernel_name(cache, 8, 1).startswith("decode_gqa4")
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device=DEV)
    lens = torch.tensor([256, 0, 200], dtype=torch.int32, device=DEV)
    sm.attend(to_dev(q, torch.bfloat16), cache, lens, 1.0, out=out, splits=4)
    with pytest.raises(sm.KVQError) as e:
        sm.check()
    assert e.value.name == "KVQ_ERR_LENGTH"
    assert torch.all(out[1] == 0)
    assert torch.isfinite(out.float()).all()
    sm.check()


@pytest.mark.parametrize("hq,lq,bits", [(8, 1, 4), (8, 1, 8), (8, 32, 4), (8, 32, 8), (2, 1, 4)])
@pytest.mark.parametrize("zero_k", [True, False])
def test_zero_values_give_exact_zero(sm, hq, lq, bits, zero_k):
    """A zero V cache (every group's scale 1, every code qmax) decodes to
    exact zeros, so every output row is exactly zero: the tolerance
    2e-3 * max|V| is 0 here.  With K zero too every score is 0; with K random
    the softmax is not uniform.  Decode (4/8-bit), chunk and generic kernels."""
    q, k, v, lens = _gqa_case(2, hq, 2, 300, 128, [300, 157], lq=lq, seed=50 + bits, bits=bits)
    v[:] = 0.0
    if zero_k:
        k[:] = 0.0
    o = _check_gqa(sm, q, k, v, lens, bits, 32, 1.0)
    assert np.all(o == 0.0)


def test_repeat_is_bit_identical(sm):
    q, k, v, lens = _gqa_case(2, 8, 2, 300, 128, [300, 200], seed=6)
    cache = pack_gpu(sm, k, v, 4, 32)
    qd, ld = to_dev(q, torch.bfloat16), to_dev(lens, torch.int32)
    a = sm.attend(qd, cache, ld, 1.0, splits=5)
    b = sm.attend(qd, cache, ld, 1.0, splits=5)
    assert torch.equal(a, b)


def test_every_output_written(sm):
    q, k, v, lens = _gqa_case(2, 8, 2, 300, 128, [300, 33], seed=7)
    cache = pack_gpu(sm, k, v, 4, 32)
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device=DEV)
    sm.attend(to_dev(q, torch.bfloat16), cache, to_dev(lens, torch.int32), 1.0, out=out, splits=3)
    assert torch.isfinite(out.float()).all()


def test_bad_lengths_reported(sm):
    q, k, v, _ = _gqa_case(3, 4, 2, 64, 32, [64, 64, 64], seed=8)
    cache = pack_gpu(sm, k, v, 4, 32)
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device=DEV)
    lens = torch.tensor([64, 0, 64], dtype=torch.int32, device=DEV)
    sm.attend(to_dev(q, torch.bfloat16), cache, lens, 1.0, out=out)
    with pytest.raises(sm.KVQError) as e:
        sm.check()
    assert e.value.name == "KVQ_ERR_LENGTH"
    assert torch.all(out[1] == 0)
    assert torch.isfinite(out.float()).all()
    sm.check()                     # the error word was cleared
    lens = torch.tensor([64, 65, 64], dtype=torch.int32, device=DEV)
    sm.attend(to_dev(q, torch.bfloat16), cache, lens, 1.0, out=out)
    with pytest.raises(sm.KVQError):
        sm.check()


# ---------------------------------------------------------------------------
# full-size workloads, every head against the oracle
# ---------------------------------------------------------------------------

def _full_case(sm, name, seed=0, bits=4, group=None, splits=0):
    """The named workload at its full size, in the launch configuration the
    bench times (automatic splits): every (b, h_kv) head's cache bytes and
    output rows against the oracle.  Different heads take different paths
    through the work plan (whole-segment output or partials and the merge,
    worker boundaries at different blocks), so none is left out."""
    q, k, v, lens, meta = W.gqa_case(name, seed)
    q = bf16_values(q)
    _check_gqa(sm, q, k, v, lens, bits, group or meta["group"], 1.0, splits=splits)


def test_decode_gqa_full(sm):
    _full_case(sm, "decode_gqa")


@pytest.mark.parametrize("bits,group", [(8, 32), (4, 8), (8, 8)])
def test_decode_gqa_full_formats(sm, bits, group):
    """The decode workload in the other code widths and group sizes of the
    tuned decode kernel."""
    small = sm.PackedCache(1, 8, 64, 128, bits, group, DEV)
    assert sm.kernel_name(small, 32, 1).startswith("decode_gqa4")
    _full_case(sm, "decode_gqa", bits=bits, group=group)


def test_long_context_full(sm):
    _full_case(sm, "long_context")


@pytest.mark.parametrize("bits", [4, 8])
def test_chunk_full(sm, bits):
    _full_case(sm, "chunk", bits=bits)


# ---------------------------------------------------------------------------
# attend with a recent-token window kept unquantized (kvq_attend_window)
# ---------------------------------------------------------------------------

def _check_window(sm, q, k, v, lens, kw, vw, wl, bits, group, scale, q_dtype=torch.bfloat16,
                  win_dtype=torch.float32, splits=0):
    """kvq_attend_window against the oracle's softmax over the decoded packed
    tokens followed by the window tokens (as stored, bf16-rounded where the
    window is bf16), within 2e-3 * max|V| over the values attended."""
    b_, hq, lq, d = q.shape
    hkv = k.shape[1]
    cache = pack_gpu(sm, k, v, bits, group)
    qd = to_dev(q, q_dtype)
    kwd, vwd = to_dev(kw, win_dtype), to_dev(vw, win_dtype)
    out = sm.attend_window(qd, cache, to_dev(lens, torch.int32), kwd, vwd, to_dev(wl, torch.int32), scale,
                           splits=splits)
    sm.check()
    assert out.dtype == q_dtype
    o = out.float().cpu().numpy()
    k_hat, v_hat = np.zeros_like(k), np.zeros_like(v)
    for b in range(b_):
        for h in range(hkv):
            k_hat[b, h] = O.unpack_matrix(O.pack_k(k[b, h], bits, group))
            v_hat[b, h] = O.unpack_matrix(O.pack_v(v[b, h], bits, group))
    kwv, vwv = kwd.float().cpu().numpy(), vwd.float().cpu().numpy()
    want = O.attend_gqa_window(qd.float().cpu().numpy(), k_hat, v_hat, lens, kwv, vwv, wl, scale)
    for b in range(b_):
        vals = np.concatenate([v_hat[b, :, :lens[b]].ravel(), vwv[b, :, :wl[b]].ravel()])
        tol = 2e-3 * float(np.abs(vals).max())
        # a row that follows one window key can sit near max|V| itself, where
        # one bf16 rounding of the output alone exceeds the tolerance: a bf16
        # output is checked through its rounding interval
        if q_dtype == torch.bfloat16:
            check_rows_rounded(o[b], want[b], tol, f"b{b}")
        else:
            check_rows(o[b], want[b], vals, f"b{b}")
    return o


def _window(b_, hkv, w_cap, d, wl, seed):
    rng = np.random.default_rng(seed)
    kw = rng.standard_normal((b_, hkv, w_cap, d)).astype(np.float32)
    vw = rng.standard_normal((b_, hkv, w_cap, d)).astype(np.float32)
    wl = np.asarray(wl, np.int32)
    for b in range(b_):
        kw[b, :, wl[b]:] = 1e4          # past a window's length: must not be read
        vw[b, :, wl[b]:] = -1e4
    return kw, vw, wl


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("win_dtype", [torch.float32, torch.bfloat16])
def test_window_decode(sm, bits, win_dtype):
    """Tuned decode kernel (four heads per KV head, D 128, g 32) plus a
    window: packed lengths ending inside a block, one sequence with no packed
    token (window only), one with an empty window, several splits."""
    q, k, v, lens = _gqa_case(4, 8, 2, 700, 128, [700, 0, 300, 29], seed=60 + bits, bits=bits, outliers=True)
    cache = pack_gpu(sm, k, v, bits, 32)
    assert sm.kernel_name(cache, 8, 1).startswith("decode_gqa4")
    kw, vw, wl = _window(4, 2, 32, 128, [31, 5, 0, 32], seed=61)
    for splits in (0, 1, 5):
        _check_window(sm, q, k, v, lens, kw, vw, wl, bits, 32, 1.0, win_dtype=win_dtype, splits=splits)


def test_window_decode_long(sm):
    """A long sequence split over many workers (the part-parallel merge) plus
    a window whose keys dominate some rows (large scores)."""
    q, k, v, lens = _gqa_case(1, 8, 2, 20000, 128, [19999], seed=62)
    kw, vw, wl = _window(1, 2, 64, 128, [40], seed=63)
    kw[:, :, :8] *= 4.0
    _check_window(sm, q, k, v, lens, kw, vw, wl, 4, 32, 1.0)


@pytest.mark.parametrize("lq", [32, 64])
def test_window_chunk(sm, lq):
    """Tensor-core chunk kernel (feature-major partials) plus a window."""
    q, k, v, lens = _gqa_case(3, 8, 2, 700, 128, [700, 300, 0], lq=lq, seed=64)
    cache = pack_gpu(sm, k, v, 4, 32)
    assert sm.kernel_name(cache, 8, lq).startswith("chunk")
    kw, vw, wl = _window(3, 2, 48, 128, [48, 0, 7], seed=65)
    for splits in (0, 1):
        _check_window(sm, q, k, v, lens, kw, vw, wl, 4, 32, 1.0, splits=splits)


@pytest.mark.parametrize("bits,group", [(4, 8), (8, 32)])
def test_window_generic(sm, bits, group):
    """Generic kernel (D 64, several query rows) plus a window, f32 Q."""
    q, k, v, lens = _gqa_case(3, 4, 2, 200, 64, [200, 1, 0], lq=3, seed=66, bits=bits, group=group)
    kw, vw, wl = _window(3, 2, 20, 64, [3, 20, 1], seed=67)
    _check_window(sm, q, k, v, lens, kw, vw, wl, bits, group, 0.125, q_dtype=torch.float32)


@pytest.mark.parametrize("d", [50, 72])
def test_window_many_rows(sm, d):
    """A window pass of more than eight query rows that is not a multiple of
    four (fourteen: two heads per KV head, seven queries), a head dimension
    that is not a multiple of 32 (and, at 50, not of 4), two window tiles."""
    q, k, v, lens = _gqa_case(2, 4, 2, 200, d, [200, 61], lq=7, seed=90 + d)
    kw, vw, wl = _window(2, 2, 40, d, [40, 9], seed=91 + d)
    _check_window(sm, q, k, v, lens, kw, vw, wl, 4, 32, 0.125, win_dtype=torch.bfloat16)


def test_window_bad_lengths(sm):
    """No key at all (both lengths 0) or a window length past its capacity is
    reported; the keyless sequence's rows are zeros, the others stay finite."""
    q, k, v, _ = _gqa_case(3, 8, 2, 256, 128, [256, 256, 256], seed=68)
    cache = pack_gpu(sm, k, v, 4, 32)
    kw, vw, _ = _window(3, 2, 16, 128, [16, 16, 16], seed=69)
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device=DEV)
    lens = torch.tensor([256, 0, 100], dtype=torch.int32, device=DEV)
    wl = torch.tensor([3, 0, 16], dtype=torch.int32, device=DEV)
    sm.attend_window(to_dev(q, torch.bfloat16), cache, lens, to_dev(kw), to_dev(vw), wl, 1.0, out=out)
    with pytest.raises(sm.KVQError) as e:
        sm.check()
    assert e.value.name == "KVQ_ERR_LENGTH"
    assert torch.all(out[1] == 0)
    assert torch.isfinite(out.float()).all()
    sm.check()
    wl = torch.tensor([3, 17, 16], dtype=torch.int32, device=DEV)
    lens = torch.tensor([256, 10, 100], dtype=torch.int32, device=DEV)
    sm.attend_window(to_dev(q, torch.bfloat16), cache, lens, to_dev(kw), to_dev(vw), wl, 1.0, out=out)
    with pytest.raises(sm.KVQError):
        sm.check()
    sm.check()


# ---------------------------------------------------------------------------
# tuned decode at group size 8
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [4, 8])
def test_decode_g8(sm, bits):
    """The tuned decode kernel at g = 8 (four K scale rows per 32-token block,
    sixteen V scales per token): lengths ending inside a K group of 8 and
    inside a block, one shorter than a group, outlier channels, splits."""
    q, k, v, lens = _gqa_case(4, 8, 2, 700, 128, [700, 301, 128, 5], seed=70 + bits, bits=bits, outliers=True)
    cache = pack_gpu(sm, k, v, bits, 8)
    assert sm.kernel_name(cache, 8, 1).startswith("decode_gqa4")
    for splits in (0, 1, 5):
        _check_gqa(sm, q, k, v, lens, bits, 8, 1.0, splits=splits)


@pytest.mark.parametrize("bits", [4, 8])
def test_decode_g8_zero_and_window(sm, bits):
    """g = 8: a zero V cache gives exact zeros; and a window on top."""
    q, k, v, lens = _gqa_case(2, 8, 2, 300, 128, [300, 157], seed=72 + bits)
    v0 = np.zeros_like(v)
    o = _check_gqa(sm, q, k, v0, lens, bits, 8, 1.0)
    assert np.all(o == 0.0)
    kw, vw, wl = _window(2, 2, 16, 128, [9, 16], seed=73)
    _check_window(sm, q, k, v, lens, kw, vw, wl, bits, 8, 1.0)


# ---------------------------------------------------------------------------
# causal multi-query attention (kvq_attend_causal)
# ---------------------------------------------------------------------------

def _check_causal(sm, q, k, v, lens, bits, group, scale, q_dtype=torch.bfloat16, splits=0):
    """kvq_attend_causal against the oracle's causal rows on the decoded cache,
    within 2e-3 * max|V_hat| of the head; a bf16 output through its rounding
    interval (a row near the start of a sequence reads few keys, so |O| can
    approach max|V_hat|, where one bf16 rounding alone exceeds the
    tolerance)."""
    b_, hq, lq, d = q.shape
    hkv = k.shape[1]
    cache = pack_gpu(sm, k, v, bits, group)
    qd = to_dev(q, q_dtype)
    out = sm.attend(qd, cache, to_dev(lens, torch.int32), scale, splits=splits, causal=True)
    sm.check()
    o = out.float().cpu().numpy()
    k_hat, v_hat = np.zeros_like(k), np.zeros_like(v)
    for b in range(b_):
        for h in range(hkv):
            k_hat[b, h] = O.unpack_matrix(O.pack_k(k[b, h], bits, group))
            v_hat[b, h] = O.unpack_matrix(O.pack_v(v[b, h], bits, group))
    want = O.attend_gqa_causal(qd.float().cpu().numpy(), k_hat, v_hat, lens, scale)
    grp = hq // hkv
    for b in range(b_):
        for h in range(hq):
            vh = v_hat[b, h // grp, :lens[b]]
            if q_dtype == torch.bfloat16:
                check_rows_rounded(o[b, h], want[b, h], 2e-3 * float(np.abs(vh).max()), f"b{b} h{h}")
            else:
                check_rows(o[b, h], want[b, h], vh, f"b{b} h{h}")
    return o


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("lq", [32, 64])
def test_causal_chunk(sm, bits, lq):
    """Tensor-core chunk kernel with the causal mask: the last rows of a
    block see part of it, some rows see no key of a split's first blocks,
    lengths ending inside a block, one barely longer than the chunk."""
    q, k, v, lens = _gqa_case(3, 8, 2, 700, 128, [700, 300, lq + 13], lq=lq, seed=80 + bits + lq, bits=bits)
    cache = pack_gpu(sm, k, v, bits, 32)
    assert sm.kernel_name(cache, 8, lq).startswith("chunk")
    for splits in (0, 1, 5):
        _check_causal(sm, q, k, v, lens, bits, 32, 1.0, splits=splits)


@pytest.mark.parametrize("bits,group", [(4, 32), (8, 8)])
def test_causal_generic(sm, bits, group):
    """Generic kernel (D 64, five query rows, f32 Q) with the causal mask;
    one sequence exactly Lq long (its first row reads one key)."""
    q, k, v, lens = _gqa_case(3, 4, 2, 200, 64, [200, 37, 5], lq=5, seed=82, bits=bits)
    for splits in (0, 3):
        _check_causal(sm, q, k, v, lens, bits, group, 0.125, q_dtype=torch.float32, splits=splits)


def test_causal_one_row_is_plain(sm):
    """One query row at the last position sees every key: the causal call
    equals the plain one bit for bit."""
    q, k, v, lens = _gqa_case(2, 8, 2, 300, 128, [300, 157], seed=84)
    cache = pack_gpu(sm, k, v, 4, 32)
    qd, ld = to_dev(q, torch.bfloat16), to_dev(lens, torch.int32)
    a = sm.attend(qd, cache, ld, 1.0)
    b = sm.attend(qd, cache, ld, 1.0, causal=True)
    sm.check()
    assert torch.equal(a, b)


def test_causal_short_length(sm):
    """A sequence shorter than the chunk: reported, its rows without a
    visible key are zeros, every other row finite and correct."""
    q, k, v, _ = _gqa_case(2, 4, 2, 64, 64, [64, 64], lq=6, seed=85)
    cache = pack_gpu(sm, k, v, 4, 32)
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device=DEV)
    lens = torch.tensor([64, 3], dtype=torch.int32, device=DEV)
    sm.attend(to_dev(q), cache, lens, 0.125, out=out, causal=True)
    with pytest.raises(sm.KVQError) as e:
        sm.check()
    assert e.value.name == "KVQ_ERR_LENGTH"
    o = out.cpu().numpy()
    assert np.isfinite(o).all()
    assert np.all(o[1, :, :3] == 0)            # rows 0..2 of sequence 1 see no key
    sm.check()

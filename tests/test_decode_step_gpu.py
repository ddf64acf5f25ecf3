"""GPU parity of the decode step (kvq_decode_step): append each sequence's new
token, then attend.  Many successive steps on one cache, with ragged lengths
that cross K-group and 32-token block boundaries at different steps; after
every step the cache bytes of every valid token and every output row are
compared with the oracle's whole-cache pack of the same tokens and its float64
attention ("Block KV decoding: less workspace, more time", section "Use the
failure to choose the next question": the complete generation path)."""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import DEV, assert_head_packed_equal, check_rows, check_rows_rounded, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sm_b200
    return sm_b200


def _run_steps(sm, b_, hq, hkv, n_cap, d, start, steps, bits, group, in_dtype=torch.float32,
               q_dtype=torch.bfloat16, seed=0, splits=0):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((b_, hkv, n_cap, d)).astype(np.float32)
    v = rng.standard_normal((b_, hkv, n_cap, d)).astype(np.float32)
    k[:, :, :, ::37] *= 8.0                          # a few outlier channels
    if in_dtype == torch.bfloat16:
        k = torch.from_numpy(k).to(torch.bfloat16).float().numpy()
        v = torch.from_numpy(v).to(torch.bfloat16).float().numpy()
    lens = np.asarray(start, np.int32)
    assert lens.max() + steps <= n_cap
    # the prefix: every sequence's tokens before its first step (later tokens
    # of the cache's rows are written as the steps reach them)
    cache = sm.PackedCache(b_, hkv, n_cap, d, bits, group, DEV)
    prefix = np.zeros_like(k), np.zeros_like(v)
    for b in range(b_):
        prefix[0][b, :, :lens[b] - 1] = k[b, :, :lens[b] - 1]
        prefix[1][b, :, :lens[b] - 1] = v[b, :, :lens[b] - 1]
    sm.pack(to_dev(prefix[0], in_dtype), to_dev(prefix[1], in_dtype), cache)
    grp = hq // hkv
    out = torch.empty((b_, hq, 1, d), dtype=q_dtype, device=DEV)
    ws = torch.empty(max(sm.workspace_size(cache, hq, 1, splits), 16), dtype=torch.uint8, device=DEV)
    crossed = set()
    for s in range(steps):
        # lengths[b] counts the new token t = lengths[b] - 1
        k_tail = np.full((b_, hkv, group, d), 1e4, np.float32)       # rows past t % g: never read
        v_new = np.zeros((b_, hkv, d), np.float32)
        for b in range(b_):
            t = int(lens[b]) - 1
            g0 = t // group * group
            k_tail[b, :, :t - g0 + 1] = k[b, :, g0:t + 1]
            v_new[b] = v[b, :, t]
            if t % group == 0:
                crossed.add(("group", t))
            if t % 32 == 0:
                crossed.add(("block", t))
        q = (rng.standard_normal((b_, hq, 1, d)) / math.sqrt(d)).astype(np.float32)
        qd = to_dev(q, q_dtype)
        ld = torch.from_numpy(lens.copy()).to(DEV)
        sm.decode_step(qd, cache, ld, to_dev(k_tail, in_dtype), to_dev(v_new, in_dtype), 1.0, out=out,
                       workspace=ws, splits=splits)
        sm.check()
        o = out.float().cpu().numpy()
        qv = qd.float().cpu().numpy()
        for b in range(b_):
            n = int(lens[b])
            for h in range(hkv):
                pk, pv = O.pack_k(k[b, h, :n], bits, group), O.pack_v(v[b, h, :n], bits, group)
                assert_head_packed_equal(cache, b, h, pk, pv)
                kh, vh = O.unpack_matrix(pk), O.unpack_matrix(pv)
                want = O.attend_gqa_heads(qv[b, h * grp:(h + 1) * grp, 0], kh, vh, n, 1.0)
                got, what = o[b, h * grp:(h + 1) * grp, 0], f"step {s} b{b} h{h} len {n}"
                if q_dtype == torch.bfloat16:
                    # a short sequence's row can sit near max|V| (one key: the
                    # row is that key's value), where the bf16 output's own
                    # rounding exceeds the tolerance: check the rounding interval
                    check_rows_rounded(got, want, 2e-3 * float(np.abs(vh[:n]).max()), what)
                else:
                    check_rows(got, want, vh[:n], what)
        lens = lens + 1
    return crossed


def test_decode_step_many_steps(sm):
    """48 steps of the tuned decode kernel's shape (four query heads per KV
    head, D 128, 4-bit g32): sequences start at 1, 30, 95 and 200 tokens, so
    each crosses a K-group / block boundary at a different step."""
    crossed = _run_steps(sm, 4, 16, 4, 300, 128, [1, 30, 95, 200], 48, 4, 32, seed=1)
    assert sum(1 for c in crossed if c[0] == "group") >= 4


@pytest.mark.parametrize("bits,group", [(8, 32), (4, 8), (8, 8)])
def test_decode_step_formats(sm, bits, group):
    _run_steps(sm, 3, 8, 2, 200, 128, [7, 31, 64], 40, bits, group, seed=2 + bits + group, splits=3)


def test_decode_step_bf16_rows_generic(sm):
    """bf16 input rows, f32 Q (the generic kernel: D 64, two query heads per KV
    head) and a group of 16."""
    _run_steps(sm, 2, 4, 2, 120, 64, [1, 47], 40, 4, 16, in_dtype=torch.bfloat16, q_dtype=torch.float32,
               seed=5)


def test_decode_step_bad_length(sm):
    """A length of 0 is reported and leaves that sequence's cache untouched."""
    cache = sm.PackedCache(2, 2, 64, 128, 4, 32, DEV)
    before = [t.clone() for t in (cache.k_codes, cache.k_scales, cache.v_codes, cache.v_scales)]
    q = torch.zeros((2, 8, 1, 128), dtype=torch.bfloat16, device=DEV)
    kt = torch.ones((2, 2, 32, 128), device=DEV)
    vn = torch.ones((2, 2, 128), device=DEV)
    lens = torch.tensor([0, 0], dtype=torch.int32, device=DEV)
    out = sm.decode_step(q, cache, lens, kt, vn, 1.0)
    with pytest.raises(sm.KVQError) as e:
        sm.check()
    assert e.value.name == "KVQ_ERR_LENGTH"
    for a, b_ in zip(before, (cache.k_codes, cache.k_scales, cache.v_codes, cache.v_scales)):
        assert torch.equal(a, b_)
    assert torch.all(out == 0)
    sm.check()


@pytest.mark.parametrize("bits,steps", [(4, 2), (8, 1)])
def test_decode_step_full_size(sm, bits, steps):
    """The decode workload's shape at full size (B 32, H_q 32, H_kv 8, D 128,
    about 4,096 tokens) in the launch configuration the bench times (automatic
    splits), every head compared.  With 4-bit codes the split has room to count
    each appending head's append as one more plan slot (the workers that
    append cover one block fewer, and some worker ranges start at such a
    slot); with 8-bit codes it has not, and the plan is the plain one."""
    start = [4094 - 3 * (b % 4) for b in range(32)]
    _run_steps(sm, 32, 32, 8, 4096, 128, start, steps, bits, 32, seed=40 + bits)

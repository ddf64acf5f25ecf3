"""kvq_attend_noalloc: attention for callers that cannot allocate device
memory at call time (an engine that reserved all of its device memory at
start-up, or a loop where a cudaMalloc would synchronize the device).  Its
split scratch is a fixed array inside the library.

Checked through the C ABI: two calls in a row on one cache, with different Q
and lengths, each equal bit for bit to kvq_attend with a caller workspace and
each within the attention tolerance the parity tests use (2e-3 * max|V_hat|)
of the float64 oracle; and a request larger than the fixed array is refused.
This file sorts last so that a failure here stops a -x run only after every
other test has run; it also passes alone in a fresh process."""

from __future__ import annotations

import ctypes
import math

import numpy as np
import pytest
import torch

from tests.gpu_util import bf16_rounding_gap

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def sm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sm_b200
    return sm_b200


def _case(sm, seed, b_, hkv, n, d):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((b_, hkv, n, d)).astype(np.float32)
    v = rng.standard_normal((b_, hkv, n, d)).astype(np.float32)
    cache = sm.PackedCache(b_, hkv, n, d, 4, 32, DEV)
    sm.pack(torch.from_numpy(k).to(DEV), torch.from_numpy(v).to(DEV), cache)
    return cache, k, v


def _q(seed, b_, hq, d):
    rng = np.random.default_rng(seed)
    q = (rng.standard_normal((b_, hq, 1, d)) / math.sqrt(d)).astype(np.float32)
    return torch.from_numpy(q).to(DEV).to(torch.bfloat16)


def _noalloc(sm, cache, qd, ld, out, splits=0):
    c = cache.struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return sm.lib.kvq_attend_noalloc(qd.data_ptr(), 1, ctypes.byref(c), ld.data_ptr(),
                                     qd.shape[1], qd.shape[2], 1.0, out.data_ptr(), splits, stream)


def _oracle_check(cache_k, cache_v, qd, lens, got, heads):
    """The noalloc output of the sampled heads against the float64 oracle,
    within 2e-3 * max|V_hat| of the head (beyond the bf16 output's rounding)."""
    import oracle as O
    q = qd.float().cpu().numpy()
    o = got.float().cpu().numpy()
    hq, hkv = q.shape[1], cache_k.shape[1]
    grp = hq // hkv
    for b, h in heads:
        n = int(lens[b])
        pk, pv = O.pack_k(cache_k[b, h], 4, 32), O.pack_v(cache_v[b, h], 4, 32)
        kh, vh = O.unpack_matrix(pk), O.unpack_matrix(pv)
        want = O.attend_gqa_heads(q[b, h * grp:(h + 1) * grp, 0], kh, vh, n, 1.0)
        # the bf16 output through its rounding interval: a one-token
        # sequence's row is that token's value, near max|V|, where the
        # output's own rounding exceeds the tolerance
        gap = float(bf16_rounding_gap(o[b, h * grp:(h + 1) * grp, 0], want).max())
        tol = 2e-3 * float(np.abs(vh[:n]).max())
        assert gap <= tol, (b, h, gap, tol)


def test_noalloc_two_calls_match_attend(sm):
    """Two noalloc calls back to back on one cache, with different Q and
    different lengths (so the split layout, and which scratch slots hold
    partials, changes between them): each equals kvq_attend with a caller
    workspace bit for bit (same kernels, same plan), and each matches the
    oracle.  Leftover scratch contents of the first call must not reach the
    second."""
    b_, hq, hkv, n, d = 6, 8, 2, 2000, 128
    cache, k, v = _case(sm, 11, b_, hkv, n, d)
    calls = [(_q(21, b_, hq, d), [2000, 157, 1, 999, 1500, 64]),
             (_q(22, b_, hq, d), [33, 2000, 1024, 700, 5, 1999])]
    assert sm.workspace_size(cache, hq, 1) <= sm.lib.kvq_noalloc_scratch_bytes()
    for i, (qd, lens) in enumerate(calls):
        ld = torch.tensor(lens, dtype=torch.int32, device=DEV)
        want = sm.attend(qd, cache, ld, 1.0)
        got = torch.full_like(qd, float("nan"))
        assert _noalloc(sm, cache, qd, ld, got) == 0
        sm.check()
        assert torch.equal(got, want), f"call {i}: differs from kvq_attend"
        _oracle_check(k, v, qd, lens, got, [(b, h) for b in range(b_) for h in range(hkv)])


def test_noalloc_full_size(sm):
    """The decode workload's shape (batch 32, H_q 32, H_kv 8, context 4096):
    two calls in a row with different Q, each equal to kvq_attend."""
    cache, k, v = _case(sm, 12, 32, 8, 4096, 128)
    ld = torch.full((32,), 4096, dtype=torch.int32, device=DEV)
    assert sm.workspace_size(cache, 32, 1) <= sm.lib.kvq_noalloc_scratch_bytes()
    for seed in (31, 32):
        qd = _q(seed, 32, 32, 128)
        want = sm.attend(qd, cache, ld, 1.0)
        got = torch.full_like(qd, float("nan"))
        assert _noalloc(sm, cache, qd, ld, got) == 0
        sm.check()
        assert torch.equal(got, want)
    _oracle_check(k, v, qd, [4096] * 32, got, [(0, 0), (13, 5), (31, 7)])


def test_noalloc_refuses_oversize(sm):
    cache, _, _ = _case(sm, 13, 32, 8, 4096, 128)
    qd = _q(33, 32, 32, 128)
    ld = torch.full((32,), 4096, dtype=torch.int32, device=DEV)
    splits = 5000
    assert sm.workspace_size(cache, 32, 1, splits) > sm.lib.kvq_noalloc_scratch_bytes()
    out = torch.zeros_like(qd)
    assert _noalloc(sm, cache, qd, ld, out, splits=splits) == 4       # KVQ_ERR_WORKSPACE
    assert torch.count_nonzero(out) == 0                              # nothing launched

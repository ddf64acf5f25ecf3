"""kvq_attend_noalloc: attention for callers that cannot allocate device
memory at call time (an engine that reserved all of its device memory at
start-up, or a loop where a cudaMalloc would synchronize the device).  Its
split scratch is a fixed array inside the library.

Checked through the C ABI: two calls in a row, each against kvq_attend with a
caller workspace, within the attention tolerance the parity tests use
(2e-3 * max|V_hat|); and a request larger than the fixed array is refused.
This file sorts last so that a failure here stops a -x run only after every
other test has run; it also passes alone in a fresh process."""

from __future__ import annotations

import ctypes
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def sm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sm_b200
    return sm_b200


def _case(sm, seed, b_, hq, hkv, n, d, lens):
    import oracle as O
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((b_, hkv, n, d)).astype(np.float32)
    v = rng.standard_normal((b_, hkv, n, d)).astype(np.float32)
    q = (rng.standard_normal((b_, hq, 1, d)) / math.sqrt(d)).astype(np.float32)
    cache = sm.PackedCache(b_, hkv, n, d, 4, 32, DEV)
    sm.pack(torch.from_numpy(k).to(DEV), torch.from_numpy(v).to(DEV), cache)
    vmax = max(float(np.abs(O.unpack_matrix(O.pack_v(v[b, h], 4, 32))).max())
               for b in range(b_) for h in range(hkv))
    qd = torch.from_numpy(q).to(DEV).to(torch.bfloat16)
    ld = torch.tensor(lens, dtype=torch.int32, device=DEV)
    return cache, qd, ld, vmax


def _noalloc(sm, cache, qd, ld, out, splits=0):
    c = cache.struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return sm.lib.kvq_attend_noalloc(qd.data_ptr(), 1, ctypes.byref(c), ld.data_ptr(),
                                     qd.shape[1], qd.shape[2], 1.0, out.data_ptr(), splits, stream)


def test_noalloc_two_calls_match_attend(sm):
    cases = [(11, 3, 8, 2, 300, 128, [300, 157, 1]),
             (12, 32, 32, 8, 4096, 128, [4096] * 32)]
    for seed, b_, hq, hkv, n, d, lens in cases:
        cache, qd, ld, vmax = _case(sm, seed, b_, hq, hkv, n, d, lens)
        assert sm.workspace_size(cache, hq, 1) <= sm.lib.kvq_noalloc_scratch_bytes()
        want = sm.attend(qd, cache, ld, 1.0)
        got = torch.full_like(qd, float("nan"))
        assert _noalloc(sm, cache, qd, ld, got) == 0
        sm.check()
        err = float((got.float() - want.float()).abs().max())
        assert torch.isfinite(got.float()).all()
        assert err <= 2e-3 * vmax, (seed, err)


def test_noalloc_refuses_oversize(sm):
    cache, qd, ld, _ = _case(sm, 13, 32, 32, 8, 4096, 128, [4096] * 32)
    splits = 5000
    assert sm.workspace_size(cache, 32, 1, splits) > sm.lib.kvq_noalloc_scratch_bytes()
    out = torch.zeros_like(qd)
    assert _noalloc(sm, cache, qd, ld, out, splits=splits) == 4       # KVQ_ERR_WORKSPACE
    assert torch.count_nonzero(out) == 0                              # nothing launched

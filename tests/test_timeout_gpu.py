"""The tuned decode kernel's bounded waits, made to run out on purpose
without any fault (kvq_selftest_timeout): one completion is armed for 16
bytes no copy brings, so one worker's wait runs out after a short limit.
The call must end with KVQ_ERR_TIMEOUT within the limit plus the bounded
drain, every other worker must finish, and the device must stay usable: a
normal call right after it matches the oracle."""

from __future__ import annotations

import ctypes
import math
import time

import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_util import DEV, check_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sm_b200
    return sm_b200


@pytest.mark.parametrize("bits,group", [(4, 32), (8, 32)])
def test_lost_completion_ends_with_timeout(sm, bits, group):
    rng = np.random.default_rng(90 + bits)
    b_, hq, hkv, n, d = 2, 8, 2, 512, 128
    k = rng.standard_normal((b_, hkv, n, d)).astype(np.float32)
    v = rng.standard_normal((b_, hkv, n, d)).astype(np.float32)
    q = (rng.standard_normal((b_, hq, 1, d)) / math.sqrt(d)).astype(np.float32)
    cache = sm.PackedCache(b_, hkv, n, d, bits, group, DEV)
    sm.pack(to_dev(k), to_dev(v), cache)
    assert sm.kernel_name(cache, hq, 1).startswith("decode_gqa4")
    qd = to_dev(q, torch.bfloat16)
    lens = torch.tensor([n, 300], dtype=torch.int32, device=DEV)
    out = torch.zeros_like(qd)
    splits = 2                        # 2 CTAs: every worker gets several blocks
    ws = torch.empty(max(sm.workspace_size(cache, hq, 1, splits), 16), dtype=torch.uint8, device=DEV)
    sm.check()
    c = cache.struct()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    t0 = time.monotonic()
    st = sm.lib.kvq_selftest_timeout(qd.data_ptr(), 1, ctypes.byref(c), lens.data_ptr(), hq, 1.0, out.data_ptr(),
                                     ws.data_ptr(), ws.numel(), splits, 1, 100, stream)
    assert st == 0
    with pytest.raises(sm.KVQError) as e:
        sm.check()
    elapsed = time.monotonic() - t0
    assert e.value.name == "KVQ_ERR_TIMEOUT"
    assert elapsed < 10.0, elapsed
    sm.check()                        # cleared; the device answers
    # a normal call afterwards is correct
    got = sm.attend(qd, cache, lens, 1.0, splits=splits)
    sm.check()
    o = got.float().cpu().numpy()
    qv = qd.float().cpu().numpy()
    grp = hq // hkv
    for b in range(b_):
        for h in range(hkv):
            pk, pv = O.pack_k(k[b, h], bits, group), O.pack_v(v[b, h], bits, group)
            kh, vh = O.unpack_matrix(pk), O.unpack_matrix(pv)
            want = O.attend_gqa_heads(qv[b, h * grp:(h + 1) * grp, 0], kh, vh, int(lens[b]), 1.0)
            check_rows(o[b, h * grp:(h + 1) * grp, 0], want, vh[:int(lens[b])], f"b{b} h{h}")


def test_selftest_argument_rules(sm):
    cache = sm.PackedCache(1, 1, 64, 64, 4, 32, DEV)       # D 64: not the tuned decode kernel
    q = torch.zeros((1, 4, 1, 64), dtype=torch.bfloat16, device=DEV)
    lens = torch.tensor([64], dtype=torch.int32, device=DEV)
    out = torch.zeros_like(q)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=DEV)
    c = cache.struct()
    call = lambda lb, ms: sm.lib.kvq_selftest_timeout(q.data_ptr(), 1, ctypes.byref(c), lens.data_ptr(), 4, 1.0,
                                                      out.data_ptr(), ws.data_ptr(), ws.numel(), 0, lb, ms, None)
    assert call(1, 100) == 8          # KVQ_ERR_UNSUPPORTED: another kernel
    cache2 = sm.PackedCache(1, 1, 64, 128, 4, 32, DEV)
    c2 = cache2.struct()
    q2 = torch.zeros((1, 4, 1, 128), dtype=torch.bfloat16, device=DEV)
    out2 = torch.zeros_like(q2)
    call2 = lambda lb, ms: sm.lib.kvq_selftest_timeout(q2.data_ptr(), 1, ctypes.byref(c2), lens.data_ptr(), 4, 1.0,
                                                       out2.data_ptr(), ws.data_ptr(), ws.numel(), 0, lb, ms, None)
    assert call2(-1, 100) == 1 and call2(0, 0) == 1 and call2(0, 20000) == 1

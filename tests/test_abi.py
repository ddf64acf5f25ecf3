"""CPU tests of the C ABI: the library loads, exports every function
include/kvq.h declares, sizes its arrays like the oracle's, and rejects bad
arguments on the host before any launch (fake pointers are never touched)."""

from __future__ import annotations

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle as O
import sm_b200 as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    return re.findall(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", text)


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert len(names) >= 8
    out = subprocess.run(["nm", "-D", "--defined-only", K.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, n
        assert hasattr(K.lib, n)
    # nothing but the C ABI leaks out
    assert {e for e in exported if e.startswith("kvq")} == set(names)


def test_strerror_covers_every_status():
    for code, name in K.STATUS.items():
        text = K.lib.kvq_strerror(code).decode()
        assert text and text != "unknown status", name
    assert K.lib.kvq_strerror(99).decode() == "unknown status"


@pytest.mark.parametrize("bits,group,n,d", [(4, 32, 128, 32), (4, 8, 35, 13), (8, 8, 35, 13),
                                            (8, 32, 512, 32), (4, 32, 4096, 128)])
def test_cache_sizes_match_oracle_arrays(bits, group, n, d):
    x = np.zeros((n, d), np.float32)
    pk, pv = O.pack_k(x, bits, group), O.pack_v(x, bits, group)
    heads = 3 * 2
    kc, ks, vc, vs = K.cache_sizes(3, 2, n, d, bits, group)
    assert kc == heads * pk.codes.nbytes
    assert ks == heads * pk.scales.nbytes
    assert vc == heads * pv.codes.nbytes
    assert vs == heads * pv.scales.nbytes


def _cache(bits=4, group=32, B=2, H=2, N=64, D=32, ptr=0x10000):
    return K._Cache(bits, group, B, H, N, D, ptr, ptr + 0x100000, ptr + 0x200000, ptr + 0x300000)


@pytest.mark.parametrize("bad", [dict(bits=5), dict(bits=2), dict(group=7), dict(group=0),
                                 dict(B=0), dict(H=0), dict(N=0), dict(D=0)])
def test_bad_cache_rejected(bad):
    c = _cache(**bad)
    st = K.lib.kvq_pack(0x1000, 0x2000, K.KVQ_F32, 0, 8, ctypes.byref(c), None)
    assert st == 1
    st = K.lib.kvq_attend(0x1000, K.KVQ_BF16, ctypes.byref(c), 0x3000, 4, 1, 1.0, 0x4000,
                          0x5000, 1 << 30, 0, None)
    assert st == 1
    assert K.lib.kvq_workspace_size(ctypes.byref(c), 4, 1, 0) == 0


def test_pack_range_rules():
    c = _cache(group=32, N=64)
    call = lambda t0, t1, dt=K.KVQ_F32, kp=0x1000: K.lib.kvq_pack(kp, 0x2000, dt, t0, t1,
                                                                 ctypes.byref(c), None)
    assert call(8, 40) == 1          # t0 not a group start
    assert call(0, 0) == 1           # empty range
    assert call(32, 16) == 1         # reversed
    assert call(0, 65) == 1          # beyond capacity
    assert call(-32, 8) == 1
    assert call(0, 8, dt=7) == 1     # unknown dtype
    assert K.lib.kvq_pack(None, None, K.KVQ_F32, 0, 8, ctypes.byref(c), None) == 1  # both NULL
    assert call(0, 8, kp=0x1002) == 3  # misaligned float32 input


def test_attend_argument_rules():
    c = _cache()
    ws = 1 << 30

    def call(q=0x1000, dt=K.KVQ_BF16, cache=c, lens=0x3000, hq=4, lq=1, o=0x4000, w=0x5000,
             wsb=ws, splits=0):
        return K.lib.kvq_attend(q, dt, ctypes.byref(cache), lens, hq, lq, 1.0, o, w, wsb, splits,
                                None)

    assert call(hq=3) == 1                       # H_q not a multiple of H_kv
    assert call(hq=0) == 1
    assert call(lq=0) == 1
    assert call(dt=3) == 1
    assert call(splits=-1) == 1
    assert call(q=0) == 1 and call(o=0) == 1 and call(lens=0) == 1
    assert call(cache=_cache(ptr=0x10008)) == 3  # cache arrays not 16-byte aligned
    assert call(q=0x1001) == 3                   # bf16 Q misaligned
    # Q and O must be 16-byte aligned whatever their dtype: a bf16 Q two bytes
    # off would otherwise change which kernel runs after kvq_workspace_size
    # sized the workspace for another
    assert call(q=0x1002) == 3
    assert call(q=0x1008, dt=K.KVQ_F32) == 3
    assert call(o=0x4002) == 3
    assert call(lens=0x3002) == 3
    assert call(cache=_cache(D=300)) == 8        # unsupported width
    assert call(w=0) == 4                        # no workspace
    assert call(wsb=16) == 4                     # too small
    assert call(w=0x5008) == 3                   # misaligned workspace


def test_cache_bytes_is_the_sum_of_the_array_sizes():
    for shape in [(4, 32, 3, 2, 128, 32), (4, 8, 1, 1, 35, 13), (8, 32, 32, 8, 4096, 128)]:
        bits, group, B, H, N, D = shape
        c = K._Cache(bits, group, B, H, N, D, 0, 0, 0, 0)
        assert K.lib.kvq_cache_bytes(ctypes.byref(c)) == sum(K.cache_sizes(B, H, N, D, bits, group))
    assert K.lib.kvq_cache_bytes(ctypes.byref(_cache(bits=5))) == 0
    assert K.lib.kvq_cache_bytes(None) == 0
    # the decode workload's cache: 168 MB, as the byte accounting says
    c = K._Cache(4, 32, 32, 8, 4096, 128, 0, 0, 0, 0)
    assert K.lib.kvq_cache_bytes(ctypes.byref(c)) == 32 * 8 * (4096 * 64 * 2 + 128 * 128 * 4 + 4096 * 4 * 4)


def test_workspace_size_grows_with_splits():
    c = _cache(B=4, H=2, N=4096, D=128)
    a = K.lib.kvq_workspace_size(ctypes.byref(c), 8, 1, 8)
    b = K.lib.kvq_workspace_size(ctypes.byref(c), 8, 1, 64)
    assert 0 < a < b


def test_window_argument_rules():
    """kvq_attend_window rejects bad window arguments on the host (every call
    here fails before a launch), and its workspace holds one more slot per
    (b, h) than kvq_attend's."""
    c = _cache()
    plain = K.lib.kvq_workspace_size(ctypes.byref(c), 4, 1, 0)
    need = K.lib.kvq_workspace_size_window(ctypes.byref(c), 4, 1, 0)
    assert need > plain > 0

    def call(kw=0x6000, vw=0x7000, wdt=K.KVQ_BF16, wl=0x8000, wcap=16, w=0x5000, wsb=need, lens=0x3000, hq=4):
        return K.lib.kvq_attend_window(0x1000, K.KVQ_BF16, ctypes.byref(c), lens, kw, vw, wdt, wl, wcap, hq, 1,
                                       1.0, 0x4000, w, wsb, 0, None)

    assert call(wdt=3) == 1                      # window dtype
    assert call(wcap=0) == 1                     # no window capacity
    assert call(kw=0) == 1 and call(vw=0) == 1 and call(wl=0) == 1
    assert call(hq=3) == 1
    assert call(kw=0x6001) == 3                  # bf16 window misaligned
    assert call(vw=0x7001, wdt=K.KVQ_F32) == 3
    assert call(wl=0x8002) == 3
    assert call(wsb=plain) == 4                  # the plain workspace is too small
    assert call(w=0) == 4
    assert call(w=0x5008) == 3


def test_causal_argument_rules():
    """kvq_attend_causal takes kvq_attend's arguments and rules."""
    c = _cache()

    def call(hq=4, lq=4, lens=0x3000, w=0x5000, wsb=1 << 30, dt=K.KVQ_BF16):
        return K.lib.kvq_attend_causal(0x1000, dt, ctypes.byref(c), lens, hq, lq, 1.0, 0x4000, w, wsb, 0, None)

    assert call(hq=3) == 1
    assert call(lq=0) == 1
    assert call(dt=3) == 1
    assert call(lens=0) == 1
    assert call(lens=0x3002) == 3
    assert call(w=0) == 4
    assert call(wsb=16) == 4


def test_decode_step_argument_rules():
    """kvq_decode_step takes kvq_attend's rules with Lq = 1, plus its two
    input rows; every call here fails on the host before any launch."""
    c = _cache()

    def call(q=0x1000, lens=0x3000, kt=0x6000, vn=0x7000, dt=K.KVQ_F32, hq=4, w=0x5000, wsb=1 << 30, o=0x4000):
        return K.lib.kvq_decode_step(q, K.KVQ_BF16, ctypes.byref(c), lens, kt, vn, dt, hq, 1.0, o, w, wsb, 0,
                                     None)

    assert call(hq=3) == 1
    assert call(kt=0) == 1 and call(vn=0) == 1
    assert call(dt=5) == 1
    assert call(kt=0x6002) == 3                 # float32 rows misaligned
    assert call(vn=0x7001, dt=K.KVQ_BF16) == 3
    assert call(q=0x1002) == 3 and call(o=0x4008) == 3
    assert call(lens=0x3002) == 3
    assert call(w=0) == 4
    assert call(wsb=16) == 4
    assert K.lib.kvq_decode_step(0x1000, K.KVQ_BF16, ctypes.byref(_cache(bits=3)), 0x3000, 0x6000, 0x7000,
                                 K.KVQ_F32, 4, 1.0, 0x4000, 0x5000, 1 << 30, 0, None) == 1


def test_selftest_argument_rules_host():
    """kvq_selftest_timeout checks its arguments on the host (no launch)."""
    c = _cache(B=2, H=2, N=512, D=128)

    def call(lb=1, ms=100, hq=8, w=0x5000, wsb=1 << 30):
        return K.lib.kvq_selftest_timeout(0x1000, K.KVQ_BF16, ctypes.byref(c), 0x3000, hq, 1.0, 0x4000, w, wsb, 0,
                                          lb, ms, None)

    assert call(lb=-1) == 1
    assert call(ms=0) == 1 and call(ms=10001) == 1
    assert call(hq=3) == 1
    assert call(w=0) == 4
    c64 = _cache(B=2, H=2, N=512, D=64)            # not the tuned decode kernel
    assert K.lib.kvq_selftest_timeout(0x1000, K.KVQ_BF16, ctypes.byref(c64), 0x3000, 8, 1.0, 0x4000, 0x5000,
                                      1 << 30, 0, 1, 100, None) == 8

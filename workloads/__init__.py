"""Seeded synthetic inputs for packed-KV attention.

This module only draws random numbers and arranges them into arrays; it holds
none of the method's arithmetic (no quantization, packing or attention), so
both the CUDA path's tests/bench and the CPU oracle can take their inputs from
it.  Every array is a deterministic function of its seed and the indices that
name it, so any (b, h) matrix of a large cache can be regenerated alone.

Workloads (shapes and value distributions as the pages describe them; the
pages use no dataset):

* ``single_head`` -- one head, N keys, D = 32, 4 queries, float32 N(0,1); the
  "clean", "early" and "late" distributions add 3 * q_mean / ||q_mean|| to
  keys 0..15 or to the last 16 keys ("KV分组打包：4-bit到底省了多少？", section
  "同一输入上的精度与空间交换": inputs biased toward the earliest or latest 16
  tokens).
* ``decode_gqa`` -- batch 32, H_q 32, H_kv 8, d_h 128, one query per
  sequence, context 4096.
* ``long_context`` -- batch 8, same heads, lengths uniform in [1000, 32768],
  1% of K and of V channels scaled x8.
* ``chunk`` -- batch 4, 64 queries per sequence, same heads, cache 16384.
"""

from __future__ import annotations

import numpy as np

_K, _V, _Q, _OUT = 1, 2, 3, 4


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(k) for k in key]))


# --------------------------------------------------------------------------
# single-head correctness grid
# --------------------------------------------------------------------------

def single_head(n: int, d: int = 32, n_q: int = 4, seed: int = 0, dist: str = "clean"):
    """Q [n_q, d], K [n, d], V [n, d] float32, i.i.d. N(0,1) from ``seed``,
    drawn in the order Q, K, V from one generator."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n_q, d)).astype(np.float32)
    k = rng.standard_normal((n, d)).astype(np.float32)
    v = rng.standard_normal((n, d)).astype(np.float32)
    if dist != "clean":
        qm = q.astype(np.float64).mean(axis=0)
        bias = (3.0 * qm / np.linalg.norm(qm)).astype(np.float32)
        rows = slice(0, min(16, n)) if dist == "early" else slice(max(0, n - 16), n)
        if dist not in ("early", "late"):
            raise ValueError(dist)
        k[rows] += bias
    return q, k, v


SINGLE_HEAD_GRID = [
    (n, seed, dist)
    for n in (128, 512)
    for seed in (0, 1, 2)
    for dist in ("clean", "early", "late")
]
FORMATS = [(4, 8), (4, 32), (8, 8), (8, 32)]          # (bits, group)


def edge_35x13(seed: int = 0):
    """The 35 x 13 non-divisible boundary case (K and V), float32 N(0,1), with
    4 queries of width 13."""
    rng = np.random.default_rng(1000 + seed)
    q = rng.standard_normal((4, 13)).astype(np.float32)
    k = rng.standard_normal((35, 13)).astype(np.float32)
    v = rng.standard_normal((35, 13)).astype(np.float32)
    return q, k, v


# --------------------------------------------------------------------------
# multi-head caches, generated per (b, h) so samples can be regenerated alone
# --------------------------------------------------------------------------

def kv_head(seed: int, b: int, h: int, n: int, d: int, which: str,
            outlier_channels=None, length: int | None = None) -> np.ndarray:
    """K or V of one (b, h) pair: [n, d] float32 N(0,1).  Tokens at or beyond
    ``length`` are zero (capacity that holds no key).  ``outlier_channels`` is
    a set of channel indices of this head whose values are multiplied by 8."""
    tag = _K if which == "k" else _V
    rng = _rng(seed, tag, b, h)
    n_valid = n if length is None else min(int(length), n)
    x = np.zeros((n, d), dtype=np.float32)
    x[:n_valid] = rng.standard_normal((n_valid, d), dtype=np.float32)
    if outlier_channels:
        idx = np.fromiter(outlier_channels, dtype=np.int64)
        x[:, idx] *= np.float32(8.0)
    return x


def q_heads(seed: int, b_: int, hq: int, lq: int, d: int, prescale: float) -> np.ndarray:
    """Q [B, H_q, Lq, d] float32 N(0,1) times ``prescale`` (1/sqrt(d) in the
    GQA workloads).  The caller rounds it to bf16 where the workload says so."""
    rng = _rng(seed, _Q)
    return (rng.standard_normal((b_, hq, lq, d), dtype=np.float32) * np.float32(prescale)).astype(np.float32)


def outlier_channels(seed: int, h_kv: int, d: int, which: str, frac: float = 0.01) -> dict:
    """1% of the H_kv * d_h channels (10 of 1024 at 8 x 128), chosen by the
    generator separately for K and V.  Returns {h: set(channels)}."""
    tag = _K if which == "k" else _V
    rng = _rng(seed, _OUT, tag)
    total = h_kv * d
    count = max(1, int(round(frac * total)))
    flat = rng.choice(total, size=count, replace=False)
    out: dict = {}
    for f in flat:
        out.setdefault(int(f) // d, set()).add(int(f) % d)
    return out


def long_context_lengths(seed: int, b_: int = 8, lo: int = 1000, hi: int = 32768) -> np.ndarray:
    """Per-sequence lengths uniform in [lo, hi] inclusive."""
    return _rng(seed, 99).integers(lo, hi, size=b_, endpoint=True).astype(np.int32)


# Workload table: the shapes the parity tests and the bench use.
WORKLOADS = {
    "decode_gqa": dict(B=32, H_q=32, H_kv=8, D=128, Lq=1, N=4096, bits=4, group=32,
                       lengths="all N", outliers=False),
    "long_context": dict(B=8, H_q=32, H_kv=8, D=128, Lq=1, N=32768, bits=4, group=32,
                         lengths="uniform [1000, 32768]", outliers=True),
    "chunk": dict(B=4, H_q=32, H_kv=8, D=128, Lq=64, N=16384, bits=(4, 8), group=32,
                  lengths="all N", outliers=False),
}


def gqa_case(name: str, seed: int = 0, b_override: int | None = None, n_override: int | None = None,
             heads=None):
    """Generate (Q, K, V, lengths, meta) for a named workload.

    ``heads`` optionally restricts generation to a list of (b, h_kv) pairs
    (the others are left zero) so samples at full size stay cheap.
    ``b_override`` / ``n_override`` shrink the batch / capacity for small
    parity cases with the same structure."""
    w = dict(WORKLOADS[name])
    b_ = b_override or w["B"]
    n = n_override or w["N"]
    hq, hkv, d, lq = w["H_q"], w["H_kv"], w["D"], w["Lq"]
    if name == "long_context":
        lens = long_context_lengths(seed, b_, lo=min(1000, n), hi=n)
    else:
        lens = np.full(b_, n, dtype=np.int32)
    ko = outlier_channels(seed, hkv, d, "k") if w["outliers"] else {}
    vo = outlier_channels(seed, hkv, d, "v") if w["outliers"] else {}
    k = np.zeros((b_, hkv, n, d), np.float32)
    v = np.zeros((b_, hkv, n, d), np.float32)
    sel = heads if heads is not None else [(b, h) for b in range(b_) for h in range(hkv)]
    for (b, h) in sel:
        k[b, h] = kv_head(seed, b, h, n, d, "k", ko.get(h), int(lens[b]))
        v[b, h] = kv_head(seed, b, h, n, d, "v", vo.get(h), int(lens[b]))
    q = q_heads(seed, b_, hq, lq, d, 1.0 / np.sqrt(d))
    meta = dict(w, B=b_, N=n)
    return q, k, v, lens, meta

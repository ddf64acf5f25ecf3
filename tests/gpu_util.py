"""Helpers shared by the GPU parity tests: move seeded inputs to the device,
run the library through the binding, and compare with the oracle.  Every
expected value comes from the oracle run on the same seeded inputs; nothing
the CUDA path produced is ever fed back to the oracle."""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O

DEV = "cuda:0"
ATTN_TOL = 2e-3          # max|err| <= ATTN_TOL * max|V_hat| of the KV head


def to_dev(x: np.ndarray, dtype=torch.float32) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV).to(dtype).contiguous()


def bf16_values(x: np.ndarray) -> np.ndarray:
    """The float32 values of x rounded to bf16 (round to nearest even), as
    torch rounds a tensor it casts; both sides then see the same Q."""
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def pack_gpu(sm, k: np.ndarray, v: np.ndarray, bits: int, group: int, in_dtype=torch.float32,
             n_cap: int | None = None):
    b_, h_, n, d = k.shape
    cache = sm.PackedCache(b_, h_, n_cap or n, d, bits, group, DEV)
    sm.pack(to_dev(k, in_dtype), to_dev(v, in_dtype), cache)
    return cache


def assert_head_packed_equal(cache, b: int, h: int, pk: O.PackedMatrix, pv: O.PackedMatrix):
    """Codes byte for byte and scales bit for bit."""
    kc = cache.head_k_codes(b, h).cpu().numpy()
    vc = cache.head_v_codes(b, h).cpu().numpy()
    np.testing.assert_array_equal(kc[: pk.codes.size], pk.codes)
    np.testing.assert_array_equal(vc[: pv.codes.size], pv.codes)
    ks = cache.head_k_scales(b, h).cpu().numpy()
    vs = cache.head_v_scales(b, h).cpu().numpy()
    np.testing.assert_array_equal(ks[: pk.scales.shape[0]].view(np.int32), pk.scales.view(np.int32))
    np.testing.assert_array_equal(vs[: pv.scales.shape[0]].view(np.int32), pv.scales.view(np.int32))


def check_rows(out_rows: np.ndarray, want_rows: np.ndarray, v_hat: np.ndarray, what: str):
    tol = ATTN_TOL * float(np.abs(v_hat).max())
    err = float(np.max(np.abs(out_rows.astype(np.float64) - want_rows)))
    assert np.isfinite(out_rows).all(), f"{what}: non-finite output"
    assert err <= tol, f"{what}: max|err| {err:.3e} > {tol:.3e}"
    return err


def oracle_rows(q_vals: np.ndarray, k: np.ndarray, v: np.ndarray, bits: int, group: int,
                length: int, scale: float):
    """Oracle output rows of one (b, h_kv): pack the head, decode it, attend.
    q_vals [rows, D] float32 values (already bf16-rounded where Q is bf16)."""
    pk, pv = O.pack_k(k, bits, group), O.pack_v(v, bits, group)
    kh, vh = O.unpack_matrix(pk), O.unpack_matrix(pv)
    want = O.attend_gqa_heads(q_vals, kh, vh, length, scale)
    return want, pk, pv, vh[:length]


def bf16_rounding_gap(out_bf16: np.ndarray, want: np.ndarray) -> np.ndarray:
    """Distance from each oracle value to the set of reals that round (to
    nearest, ties to even) to the kernel's bf16 output.  The kernel computes
    in float32 and rounds once when it stores O; this is the smallest error
    its float32 result can have had, so ``gap <= tol`` is exactly "some
    float32 result within tol of the oracle gives this output" -- the output
    rounding is allowed for, and nothing more.

    out_bf16: the output's values as float32 (each exactly a bf16 value)."""
    o = np.asarray(out_bf16, np.float32)
    w = np.asarray(want, np.float64)
    a = np.abs(o)
    bits = a.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0), "not bf16 values"
    up = (bits + 0x10000).view(np.float32).astype(np.float64) - a        # spacing above |o|
    down_bits = np.where(bits >= 0x10000, bits - 0x10000, 0).astype(np.uint32)
    down = a.astype(np.float64) - down_bits.view(np.float32).astype(np.float64)
    down = np.where(bits == 0, up, down)                                 # +-0: symmetric
    # half the spacing on the side of the oracle value, mirrored for o < 0
    away = (w - o) * np.where(o < 0, -1.0, 1.0) > 0                     # oracle beyond |o|
    half = np.where(away, up, down) / 2.0
    return np.maximum(0.0, np.abs(w - o) - half)


def check_rows_rounded(out_bf16: np.ndarray, want: np.ndarray, tol: float, what: str) -> float:
    """A bf16 output against the float64 oracle: the oracle value must lie
    within ``tol`` of the output's rounding interval (bf16_rounding_gap)."""
    assert np.isfinite(out_bf16).all(), f"{what}: non-finite output"
    worst = float(bf16_rounding_gap(out_bf16, want).max())
    assert worst <= tol, f"{what}: max|err| beyond the output rounding {worst:.3e} > {tol:.3e}"
    return worst


def single_head_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)

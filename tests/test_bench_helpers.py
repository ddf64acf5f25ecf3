"""CPU tests of bench.py's accounting: the algorithmic byte counts behind
`value` and the roofline, and the profile records it reads `traffic` from."""

import os

import bench


def test_attend_bytes_closed_form():
    """4-bit, g32, D = 128, one sequence of 33 tokens, one KV head, four query
    heads: codes 64 + 64 B per token, V scales 16 B per token, K scales one
    512 B row per started group of 32 (two here), plus bf16 Q and O."""
    got = bench.attend_bytes(1, 4, 1, 128, [33], bits=4, group=32)
    want = 33 * (64 + 64 + 16) + 2 * 512 + 4 * 128 * (2 + 2)
    assert got == want
    # 8-bit doubles the code bytes; g8 quadruples both scale densities
    assert bench.attend_bytes(1, 4, 1, 128, [32], bits=8) == 32 * (128 + 128 + 16) + 512 + 4 * 128 * 4
    assert bench.attend_bytes(1, 4, 1, 128, [32], group=8) == 32 * (64 + 64 + 64) + 4 * 512 + 4 * 128 * 4


def test_append_bytes_closed_form():
    """The decode-step append: a 32-token K group re-packed from float32 and
    one V row packed, per (b, h)."""
    k = 32 * 128 * 4 + 32 * 128 // 2 + 128 * 4
    v = 128 * 4 + 64 + 16
    assert bench.append_bytes(2, 3, 128, 32, 1) == 2 * 3 * (k + v)


def test_profile_records_exist_and_parse():
    """Every profile bench.py may read exists and carries the two lines it
    parses; traffic comes back only while the source hash matches."""
    for name in bench.PROFILE_FOR.values():
        path = os.path.join(bench.ROOT, "profiles", name)
        text = open(path, encoding="utf-8").read()
        assert "kernel_source_sha256_16:" in text and "dram_bytes_per_launch:" in text
    assert bench.recorded_traffic(__file__, "decode_gqa", 4, 32) is None        # hash mismatch
    assert bench.recorded_traffic(__file__, "no_such_workload", 4, 32) is None
    assert bench.recorded_traffic(__file__, "decode_gqa", 4, 32, window=31) is None


@__import__("pytest").mark.gpu
def test_copy_rows_h2d_matches_slice_copy():
    """The e2e loop's pitched copy of pinned host rows into the last rows of
    each (b, h) window lands exactly where a slice assignment puts them and
    leaves the other rows alone."""
    import pytest
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    g = torch.Generator().manual_seed(3)
    for L in (1, 5):
        win = torch.randn(3, 4, 32, 128, generator=g).to(dev)
        want = win.clone()
        rows = torch.randn(3, 4, L, 128, generator=g).pin_memory()
        want[:, :, -L:] = rows.to(dev)
        s = torch.cuda.Stream(dev)
        bench.copy_rows_h2d(win[:, :, -L:], rows, s)
        s.synchronize()
        assert torch.equal(win, want)

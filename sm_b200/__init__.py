"""sm_b200 -- packed-KV online-softmax attention on B200 (sm_100a).

A thin ctypes binding over ``libkvq.so`` (the C ABI in ``include/kvq.h``).
It only marshals arguments: torch tensors supply device pointers, the current
CUDA stream and device memory; every step of quantize/pack and attention runs
in the library's kernels.  If ``libkvq.so`` is missing the import fails: there
is no fallback of any kind.

    cache = sm_b200.PackedCache(B, H_kv, N_cap, D, bits=4, group=32)
    sm_b200.pack(K, V, cache)                     # K, V [B, H_kv, T, D] fp32/bf16
    O = sm_b200.attend(Q, cache, lengths, scale)  # Q [B, H_q, Lq, D] fp32/bf16
    O = sm_b200.attend(Q, cache, lengths, scale, causal=True)   # rows = last Lq positions
    O = sm_b200.attend_window(Q, cache, lengths, K_win, V_win, win_lengths, scale)
                                                  # packed tokens, then an unquantized window
    O = sm_b200.decode_step(Q, cache, lengths, K_tail, V_new, scale)
                                                  # append each sequence's new token, then attend
"""

from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "KVQError", "PackedCache", "pack", "attend", "workspace_size", "check",
    "launch_count", "kernel_name", "cache_sizes", "lib", "LIB_PATH", "attend_noalloc",
    "attend_window", "workspace_size_window", "decode_step",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkvq.so")

KVQ_F32, KVQ_BF16 = 0, 1
STATUS = {
    0: "KVQ_OK", 1: "KVQ_ERR_ARG", 2: "KVQ_ERR_LENGTH", 3: "KVQ_ERR_ALIGN",
    4: "KVQ_ERR_WORKSPACE", 5: "KVQ_ERR_CUDA", 6: "KVQ_ERR_DEVICE", 7: "KVQ_ERR_TIMEOUT",
    8: "KVQ_ERR_UNSUPPORTED",
}


class KVQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        self.name = STATUS.get(self.status, str(status))
        super().__init__(f"{where}: {self.name} ({lib.kvq_strerror(self.status).decode()})")


class _Cache(ctypes.Structure):
    _fields_ = [
        ("bits", ctypes.c_int32), ("group", ctypes.c_int32),
        ("B", ctypes.c_int32), ("H_kv", ctypes.c_int32),
        ("N_cap", ctypes.c_int32), ("D", ctypes.c_int32),
        ("k_codes", ctypes.c_void_p), ("k_scales", ctypes.c_void_p),
        ("v_codes", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkvq.so not built: run `python sm_b200/build.py` ({LIB_PATH})")
    L = ctypes.CDLL(LIB_PATH)
    i32, vp, sz = ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t
    L.kvq_cache_sizes.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(sz)]
    L.kvq_cache_sizes.restype = ctypes.c_int
    L.kvq_cache_bytes.argtypes = [ctypes.POINTER(_Cache)]
    L.kvq_cache_bytes.restype = sz
    L.kvq_pack.argtypes = [vp, vp, ctypes.c_int, i32, i32, ctypes.POINTER(_Cache), vp]
    L.kvq_pack.restype = ctypes.c_int
    L.kvq_attend.argtypes = [vp, ctypes.c_int, ctypes.POINTER(_Cache), vp, i32, i32,
                             ctypes.c_float, vp, vp, sz, i32, vp]
    L.kvq_attend.restype = ctypes.c_int
    L.kvq_workspace_size.argtypes = [ctypes.POINTER(_Cache), i32, i32, i32]
    L.kvq_workspace_size.restype = sz
    L.kvq_check.argtypes = [vp]
    L.kvq_check.restype = ctypes.c_int
    L.kvq_strerror.argtypes = [ctypes.c_int]
    L.kvq_strerror.restype = ctypes.c_char_p
    L.kvq_launch_count.argtypes = []
    L.kvq_launch_count.restype = ctypes.c_uint64
    L.kvq_attend_kernel_name.argtypes = [ctypes.POINTER(_Cache), i32, i32]
    L.kvq_attend_kernel_name.restype = ctypes.c_char_p
    L.kvq_attend_noalloc.argtypes = [vp, ctypes.c_int, ctypes.POINTER(_Cache), vp, i32, i32,
                                     ctypes.c_float, vp, i32, vp]
    L.kvq_attend_noalloc.restype = ctypes.c_int
    L.kvq_noalloc_scratch_bytes.argtypes = []
    L.kvq_noalloc_scratch_bytes.restype = sz
    L.kvq_attend_causal.argtypes = [vp, ctypes.c_int, ctypes.POINTER(_Cache), vp, i32, i32,
                                    ctypes.c_float, vp, vp, sz, i32, vp]
    L.kvq_attend_causal.restype = ctypes.c_int
    L.kvq_attend_window.argtypes = [vp, ctypes.c_int, ctypes.POINTER(_Cache), vp, vp, vp, ctypes.c_int,
                                    vp, i32, i32, i32, ctypes.c_float, vp, vp, sz, i32, vp]
    L.kvq_attend_window.restype = ctypes.c_int
    L.kvq_workspace_size_window.argtypes = [ctypes.POINTER(_Cache), i32, i32, i32]
    L.kvq_workspace_size_window.restype = sz
    L.kvq_decode_step.argtypes = [vp, ctypes.c_int, ctypes.POINTER(_Cache), vp, vp, vp, ctypes.c_int, i32,
                                  ctypes.c_float, vp, vp, sz, i32, vp]
    L.kvq_decode_step.restype = ctypes.c_int
    L.kvq_selftest_timeout.argtypes = [vp, ctypes.c_int, ctypes.POINTER(_Cache), vp, i32, ctypes.c_float, vp, vp,
                                       sz, i32, i32, ctypes.c_uint32, vp]
    L.kvq_selftest_timeout.restype = ctypes.c_int
    return L


lib = _load()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return KVQ_F32
    if t.dtype == torch.bfloat16:
        return KVQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: float32 or bfloat16")


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ok(status: int, where: str) -> None:
    if status != 0:
        raise KVQError(status, where)


def cache_sizes(B: int, H_kv: int, N_cap: int, D: int, bits: int = 4, group: int = 32):
    """Byte sizes of (k_codes, k_scales, v_codes, v_scales)."""
    out = (ctypes.c_size_t * 4)()
    _ok(lib.kvq_cache_sizes(bits, group, B, H_kv, N_cap, D, out), "kvq_cache_sizes")
    return tuple(int(v) for v in out)


class PackedCache:
    """Device memory of one packed cache, allocated through torch.

    k_codes / v_codes are uint8, k_scales / v_scales float32, each flat and
    laid out as ``include/kvq.h`` describes.  Write into them in place if
    needed, but do not rebind them: the C struct the calls pass is built
    once from their addresses."""

    def __init__(self, B: int, H_kv: int, N_cap: int, D: int, bits: int = 4, group: int = 32,
                 device="cuda"):
        self.B, self.H_kv, self.N_cap, self.D = int(B), int(H_kv), int(N_cap), int(D)
        self.bits, self.group = int(bits), int(group)
        kc, ks, vc, vs = cache_sizes(B, H_kv, N_cap, D, bits, group)
        dev = torch.device(device)
        self.k_codes = torch.zeros(kc, dtype=torch.uint8, device=dev)
        self.k_scales = torch.zeros(ks // 4, dtype=torch.float32, device=dev)
        self.v_codes = torch.zeros(vc, dtype=torch.uint8, device=dev)
        self.v_scales = torch.zeros(vs // 4, dtype=torch.float32, device=dev)
        self.device = dev
        # the four buffers never move, so the C struct is built once
        self._struct = _Cache(self.bits, self.group, self.B, self.H_kv, self.N_cap, self.D,
                              self.k_codes.data_ptr(), self.k_scales.data_ptr(),
                              self.v_codes.data_ptr(), self.v_scales.data_ptr())
        self._ws = {}                      # (H_q, Lq, splits, window) -> workspace bytes

    @property
    def Np(self) -> int:
        return -(-self.N_cap // self.group) * self.group

    @property
    def Dp(self) -> int:
        return -(-self.D // self.group) * self.group

    def nbytes(self) -> int:
        return int(lib.kvq_cache_bytes(ctypes.byref(self._struct)))

    def struct(self) -> _Cache:
        return self._struct

    def _workspace_bytes(self, H_q: int, Lq: int, splits: int, window: bool) -> int:
        key = (H_q, Lq, splits, window)
        n = self._ws.get(key)
        if n is None:
            f = lib.kvq_workspace_size_window if window else lib.kvq_workspace_size
            n = int(f(ctypes.byref(self._struct), int(H_q), int(Lq), int(splits)))
            self._ws[key] = n
        return n

    # per-(b, h) views, for tests and inspection
    def head_k_codes(self, b: int, h: int) -> torch.Tensor:
        n = self.k_codes.numel() // (self.B * self.H_kv)
        i = b * self.H_kv + h
        return self.k_codes[i * n:(i + 1) * n]

    def head_v_codes(self, b: int, h: int) -> torch.Tensor:
        n = self.v_codes.numel() // (self.B * self.H_kv)
        i = b * self.H_kv + h
        return self.v_codes[i * n:(i + 1) * n]

    def head_k_scales(self, b: int, h: int) -> torch.Tensor:
        return self.k_scales.view(self.B, self.H_kv, self.Np // self.group, self.D)[b, h]

    def head_v_scales(self, b: int, h: int) -> torch.Tensor:
        return self.v_scales.view(self.B, self.H_kv, self.N_cap, self.Dp // self.group)[b, h]


def _check_cuda(t: torch.Tensor, name: str, dev: torch.device) -> None:
    if not t.is_cuda or t.device != dev:
        raise ValueError(f"{name} must be on {dev}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def pack(K: torch.Tensor | None, V: torch.Tensor | None, cache: PackedCache, t0: int = 0) -> None:
    """Quantize and pack K, V [B, H_kv, T, D] into cache tokens [t0, t0 + T).
    Either may be None to pack only the other half (with K, t0 must be a
    multiple of the group)."""
    if K is None and V is None:
        raise ValueError("K and V are both None")
    ref = K if K is not None else V
    for name, X in (("K", K), ("V", V)):
        if X is not None:
            _check_cuda(X, name, cache.device)
            if X.shape != ref.shape or X.dtype != ref.dtype or X.dim() != 4:
                raise ValueError("K and V must be [B, H_kv, T, D] of one dtype")
    B, H, T, D = ref.shape
    if (B, H, D) != (cache.B, cache.H_kv, cache.D):
        raise ValueError("K/V shape does not match the cache")
    c = cache.struct()
    _ok(lib.kvq_pack(K.data_ptr() if K is not None else None,
                     V.data_ptr() if V is not None else None, _dtype_code(ref), int(t0),
                     int(t0 + T), ctypes.byref(c), _stream(cache.device)), "kvq_pack")


def workspace_size(cache: PackedCache, H_q: int, Lq: int, splits: int = 0) -> int:
    return cache._workspace_bytes(int(H_q), int(Lq), int(splits), False)


def kernel_name(cache: PackedCache, H_q: int, Lq: int) -> str:
    c = cache.struct()
    return lib.kvq_attend_kernel_name(ctypes.byref(c), int(H_q), int(Lq)).decode()


def attend(Q: torch.Tensor, cache: PackedCache, lengths: torch.Tensor, scale: float,
           out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
           splits: int = 0, causal: bool = False) -> torch.Tensor:
    """O = softmax(scale * Q K^T) V over the packed cache, per sequence up to
    its length.  Q [B, H_q, Lq, D] fp32/bf16; lengths int32 [B] on the device;
    returns O like Q (written into ``out`` if given).  causal: the Lq rows are
    the sequence's last Lq positions and row i reads keys [0, L - Lq + i]."""
    _check_cuda(Q, "Q", cache.device)
    _check_cuda(lengths, "lengths", cache.device)
    if lengths.dtype != torch.int32 or lengths.numel() != cache.B:
        raise ValueError("lengths must be int32 [B]")
    if Q.dim() != 4 or Q.shape[0] != cache.B or Q.shape[3] != cache.D:
        raise ValueError("Q must be [B, H_q, Lq, D]")
    H_q, Lq = int(Q.shape[1]), int(Q.shape[2])
    if out is None:
        out = torch.empty_like(Q)
    else:
        _check_cuda(out, "out", cache.device)
        if out.shape != Q.shape or out.dtype != Q.dtype:
            raise ValueError("out must match Q")
    need = workspace_size(cache, H_q, Lq, splits)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=cache.device)
    c = cache.struct()
    fn = lib.kvq_attend_causal if causal else lib.kvq_attend
    _ok(fn(Q.data_ptr(), _dtype_code(Q), ctypes.byref(c), lengths.data_ptr(), H_q, Lq,
           float(scale), out.data_ptr(), workspace.data_ptr(),
           workspace.numel() * workspace.element_size(), int(splits),
           _stream(cache.device)), "kvq_attend_causal" if causal else "kvq_attend")
    return out


def attend_noalloc(Q: torch.Tensor, cache: PackedCache, lengths: torch.Tensor, scale: float,
                   out: torch.Tensor | None = None, splits: int = 0) -> torch.Tensor:
    """attend() for callers that cannot allocate device memory when they call
    (an engine that reserved all of its memory at start-up, or a loop where a
    cudaMalloc would stall other streams): the split scratch is a fixed array
    inside the library, shared by every call on the device, so calls that may
    run at the same time on one device must be ordered.  ``out`` must then be
    preallocated by the caller; this wrapper only creates it when omitted."""
    _check_cuda(Q, "Q", cache.device)
    _check_cuda(lengths, "lengths", cache.device)
    if lengths.dtype != torch.int32 or lengths.numel() != cache.B:
        raise ValueError("lengths must be int32 [B]")
    if Q.dim() != 4 or Q.shape[0] != cache.B or Q.shape[3] != cache.D:
        raise ValueError("Q must be [B, H_q, Lq, D]")
    if out is None:
        out = torch.empty_like(Q)
    c = cache.struct()
    _ok(lib.kvq_attend_noalloc(Q.data_ptr(), _dtype_code(Q), ctypes.byref(c), lengths.data_ptr(),
                               int(Q.shape[1]), int(Q.shape[2]), float(scale), out.data_ptr(),
                               int(splits), _stream(cache.device)), "kvq_attend_noalloc")
    return out


def decode_step(Q: torch.Tensor, cache: PackedCache, lengths: torch.Tensor, K_tail: torch.Tensor,
                V_new: torch.Tensor, scale: float, out: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, splits: int = 0) -> torch.Tensor:
    """One decode step: append each sequence's new token (position
    lengths[b] - 1) to the packed cache and attend over it.  K_tail
    [B, H_kv, g, D] holds the K rows of each sequence's last group from its
    start through the new token (later rows are not read); V_new
    [B, H_kv, D] (or [B, H_kv, 1, D]) the new token's V.  Q [B, H_q, 1, D];
    lengths int32 [B] on the device, counting the new token.  Returns O like Q."""
    _check_cuda(Q, "Q", cache.device)
    _check_cuda(lengths, "lengths", cache.device)
    if lengths.dtype != torch.int32 or lengths.numel() != cache.B:
        raise ValueError("lengths must be int32 [B]")
    if Q.dim() != 4 or Q.shape[0] != cache.B or Q.shape[2] != 1 or Q.shape[3] != cache.D:
        raise ValueError("Q must be [B, H_q, 1, D]")
    _check_cuda(K_tail, "K_tail", cache.device)
    _check_cuda(V_new, "V_new", cache.device)
    if tuple(K_tail.shape) != (cache.B, cache.H_kv, cache.group, cache.D):
        raise ValueError("K_tail must be [B, H_kv, group, D]")
    if V_new.numel() != cache.B * cache.H_kv * cache.D or V_new.shape[0] != cache.B:
        raise ValueError("V_new must be [B, H_kv, D]")
    if K_tail.dtype != V_new.dtype:
        raise ValueError("K_tail and V_new must have one dtype")
    H_q = int(Q.shape[1])
    if out is None:
        out = torch.empty_like(Q)
    else:
        _check_cuda(out, "out", cache.device)
        if out.shape != Q.shape or out.dtype != Q.dtype:
            raise ValueError("out must match Q")
    need = workspace_size(cache, H_q, 1, splits)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=cache.device)
    c = cache.struct()
    _ok(lib.kvq_decode_step(Q.data_ptr(), _dtype_code(Q), ctypes.byref(c), lengths.data_ptr(),
                            K_tail.data_ptr(), V_new.data_ptr(), _dtype_code(K_tail), H_q, float(scale),
                            out.data_ptr(), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                            int(splits), _stream(cache.device)), "kvq_decode_step")
    return out


def workspace_size_window(cache: PackedCache, H_q: int, Lq: int, splits: int = 0) -> int:
    return cache._workspace_bytes(int(H_q), int(Lq), int(splits), True)


def attend_window(Q: torch.Tensor, cache: PackedCache, lengths: torch.Tensor, K_win: torch.Tensor,
                  V_win: torch.Tensor, win_lengths: torch.Tensor, scale: float,
                  out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                  splits: int = 0) -> torch.Tensor:
    """Attention over the packed cache followed by a window of recent tokens
    kept unquantized: sequence b's keys are its packed tokens [0, lengths[b])
    then its window tokens [0, win_lengths[b]).  K_win, V_win
    [B, H_kv, W_cap, D] fp32/bf16 (contiguous); lengths, win_lengths int32 [B]
    on the device; returns O like Q."""
    _check_cuda(Q, "Q", cache.device)
    for t, n in ((lengths, "lengths"), (win_lengths, "win_lengths")):
        _check_cuda(t, n, cache.device)
        if t.dtype != torch.int32 or t.numel() != cache.B:
            raise ValueError(f"{n} must be int32 [B]")
    if Q.dim() != 4 or Q.shape[0] != cache.B or Q.shape[3] != cache.D:
        raise ValueError("Q must be [B, H_q, Lq, D]")
    for t, n in ((K_win, "K_win"), (V_win, "V_win")):
        _check_cuda(t, n, cache.device)
        if t.dim() != 4 or t.shape[0] != cache.B or t.shape[1] != cache.H_kv or t.shape[3] != cache.D:
            raise ValueError(f"{n} must be [B, H_kv, W_cap, D]")
    if K_win.shape != V_win.shape or K_win.dtype != V_win.dtype:
        raise ValueError("K_win and V_win must match")
    H_q, Lq, W_cap = int(Q.shape[1]), int(Q.shape[2]), int(K_win.shape[2])
    if out is None:
        out = torch.empty_like(Q)
    else:
        _check_cuda(out, "out", cache.device)
        if out.shape != Q.shape or out.dtype != Q.dtype:
            raise ValueError("out must match Q")
    need = workspace_size_window(cache, H_q, Lq, splits)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=cache.device)
    c = cache.struct()
    _ok(lib.kvq_attend_window(Q.data_ptr(), _dtype_code(Q), ctypes.byref(c), lengths.data_ptr(),
                              K_win.data_ptr(), V_win.data_ptr(), _dtype_code(K_win), win_lengths.data_ptr(),
                              W_cap, H_q, Lq, float(scale), out.data_ptr(), workspace.data_ptr(),
                              workspace.numel() * workspace.element_size(), int(splits),
                              _stream(cache.device)), "kvq_attend_window")
    return out


def check(device=None) -> None:
    """Wait for the current stream and raise if a kernel recorded an error."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    _ok(lib.kvq_check(_stream(dev)), "kvq_check")


def launch_count() -> int:
    return int(lib.kvq_launch_count())

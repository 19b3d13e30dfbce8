"""ctypes binding of libhga.so (argument marshalling only).

Every step of the routed-attention path runs in the library's CUDA kernels;
this module only turns torch tensors into pointers and sizes, picks the
current CUDA stream and maps status codes to exceptions.  There is no Python
or CPU fallback: if libhga.so cannot be loaded, importing this module fails.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import time
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhga.so")

HGA_OK, HGA_ERR_INVALID_ARG, HGA_ERR_UNSUPPORTED = 0, 1, 2
HGA_ERR_CUDA, HGA_ERR_DEVICE_CHECK, HGA_ERR_TIMEOUT = 3, 4, 5
HGA_ERR_IO, HGA_ERR_CAPACITY = 6, 7
HGA_STORE_CREATE, HGA_STORE_DIRECT = 1, 2
HGA_BF16, HGA_FP32 = 0, 1

EXPORTED = ("hga_build_summaries", "hga_route_chunks", "hga_route_groups",
            "hga_attend", "hga_forward", "hga_index_capacity",
            "hga_validate_params", "hga_check", "hga_status_string",
            "hga_launch_count", "hga_last_cuda_error",
            "hga_set_kernel_variant", "hga_selftest_exp2", "hga_fetch_group_summaries",
            "hga_gather_history", "hga_install_group_cache",
            "hga_gather_history_noalloc", "hga_convert_v", "hga_route", "hga_commit",
            "hga_attend_backward", "hga_decode_step", "hga_store_open", "hga_store_close",
            "hga_store_attach_cache", "hga_store_append", "hga_store_set_length",
            "hga_store_length", "hga_store_page_bytes", "hga_store_pages_per_head",
            "hga_store_read", "hga_store_prepare", "hga_gather_store", "hga_forward_causal",
            "hga_set_wait_limit_ns", "hga_selftest_wait", "hga_debug_stall_next_attend")


class HgaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)}")


class CParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "n_q_heads", "n_kv_heads", "head_dim", "chunk", "group", "qblock",
        "sink", "local", "top_chunks", "top_groups", "dtype", "v_f16", "q_ready")]


@dataclasses.dataclass(frozen=True)
class Params:
    """Mirror of the C struct hga_params."""
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    chunk: int = 64
    group: int = 8
    qblock: int = 64
    sink: int = 64
    local: int = 128
    top_chunks: int = 4
    top_groups: int = 8
    dtype: str = "bf16"
    v_f16: bool = False          # v holds fp16 values (see convert_v)
    q_ready: bool = False        # q complete before the previous kernel can let this one start

    def c(self) -> CParams:
        return CParams(self.n_q_heads, self.n_kv_heads, self.head_dim,
                       self.chunk, self.group, self.qblock, self.sink,
                       self.local, self.top_chunks, self.top_groups,
                       HGA_BF16 if self.dtype == "bf16" else HGA_FP32,
                       int(self.v_f16), int(self.q_ready))

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @staticmethod
    def from_workload(w) -> "Params":
        return Params(w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.group,
                      w.qblock, w.sink, w.local, w.top_chunks, w.top_groups,
                      w.dtype)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m long_context_hga_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(CParams)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    sig = {
        "hga_build_summaries": [P, vp, i64, i64, i64, vp, vp, vp],
        "hga_route_chunks": [P, vp, i64, i64, vp, i64, vp, vp, vp],
        "hga_route_groups": [P, vp, i64, i64, vp, i64, vp, vp, vp, vp, vp],
        "hga_attend": [P, vp, i64, i64, vp, vp, i64, vp, vp, vp, vp, vp],
        "hga_forward": [P, vp, i64, i64, vp, vp, i64, vp, vp, vp, vp, vp, vp,
                        vp, vp, vp],
        "hga_index_capacity": [P, i64, i32],
        "hga_validate_params": [P],
        "hga_check": [vp],
        "hga_status_string": [ctypes.c_int],
        "hga_launch_count": [],
        "hga_last_cuda_error": [],
        "hga_set_kernel_variant": [i32],
        "hga_selftest_exp2": [vp, vp, i64, vp],
        "hga_set_wait_limit_ns": [ctypes.c_uint64],
        "hga_selftest_wait": [vp, vp],
        "hga_debug_stall_next_attend": [i64],
        "hga_convert_v": [P, vp, i64, i64, i64, vp, vp],
        "hga_route": [P, vp, i64, i64, vp, vp, i64, vp, vp, vp, vp, vp],
        "hga_commit": [P, vp, vp, i64, i64, i64, vp, vp, vp, vp],
        "hga_attend_backward": [P, vp, i64, i64, vp, vp, i64, vp, vp, vp, vp, vp, vp, vp,
                                vp, vp],
        "hga_decode_step": [P, vp, i64, vp, vp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "hga_forward_causal": [P, vp, i64, i64, vp, vp, i64, vp, vp, vp, vp, vp, vp,
                               vp, vp, vp],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.hga_index_capacity.restype = ctypes.c_int64
    lib.hga_launch_count.restype = ctypes.c_int64
    lib.hga_status_string.restype = ctypes.c_char_p
    lib.hga_last_cuda_error.restype = ctypes.c_char_p
    return lib


LIB = _load()


def status_string(code: int) -> str:
    return LIB.hga_status_string(code).decode()


def _ok(code: int, what: str):
    if code == HGA_ERR_CUDA:
        raise HgaError(code, f"{what} ({LIB.hga_last_cuda_error().decode()})")
    if code != HGA_OK:
        raise HgaError(code, what)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libhga must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def validate_params(p: Params) -> int:
    return LIB.hga_validate_params(ctypes.byref(p.c()))


def index_capacity(p: Params, t_cap: int, which: int) -> int:
    return LIB.hga_index_capacity(ctypes.byref(p.c()), t_cap, which)


def launch_count() -> int:
    return LIB.hga_launch_count()


def check(stream=None) -> int:
    """Synchronise and return (and clear) the device status word."""
    return LIB.hga_check(_stream(stream))


def build_summaries(p: Params, k, t_begin: int, t_end: int, chunk_sum,
                    group_sum, stream=None):
    t_cap = k.shape[1]
    _ok(LIB.hga_build_summaries(ctypes.byref(p.c()), _ptr(k), t_cap, t_begin,
                                t_end, _ptr(chunk_sum), _ptr(group_sum),
                                _stream(stream)), "hga_build_summaries")


def route_chunks(p: Params, q, q_start: int, chunk_sum, t_cap: int,
                 chunk_idx, chunk_cnt, stream=None):
    _ok(LIB.hga_route_chunks(ctypes.byref(p.c()), _ptr(q), q_start, q.shape[0],
                             _ptr(chunk_sum), t_cap, _ptr(chunk_idx),
                             _ptr(chunk_cnt), _stream(stream)),
        "hga_route_chunks")


def route_groups(p: Params, q, q_start: int, group_sum, t_cap: int, chunk_idx,
                 chunk_cnt, group_idx, group_cnt, stream=None):
    _ok(LIB.hga_route_groups(ctypes.byref(p.c()), _ptr(q), q_start, q.shape[0],
                             _ptr(group_sum), t_cap, _ptr(chunk_idx),
                             _ptr(chunk_cnt), _ptr(group_idx), _ptr(group_cnt),
                             _stream(stream)), "hga_route_groups")


def route(p: Params, q, q_start: int, chunk_sum, group_sum, t_cap: int, chunk_idx, chunk_cnt,
          group_idx, group_cnt, stream=None):
    """Chunk then group routing in one call (same outputs as route_chunks +
    route_groups)."""
    _ok(LIB.hga_route(ctypes.byref(p.c()), _ptr(q), q_start, q.shape[0], _ptr(chunk_sum),
                      _ptr(group_sum), t_cap, _ptr(chunk_idx), _ptr(chunk_cnt),
                      _ptr(group_idx), _ptr(group_cnt), _stream(stream)), "hga_route")


def attend(p: Params, q, q_start: int, k, v, group_idx, group_cnt, o,
           lse=None, stream=None):
    _ok(LIB.hga_attend(ctypes.byref(p.c()), _ptr(q), q_start, q.shape[0],
                       _ptr(k), _ptr(v), k.shape[1], _ptr(group_idx),
                       _ptr(group_cnt), _ptr(o), _ptr(lse), _stream(stream)),
        "hga_attend")


def attend_backward(p: Params, q, q_start: int, k, v, group_idx, group_cnt, o, lse, d_o,
                    d_q, d_k, d_v, stream=None):
    """Gradients of the routed attention with the routing held fixed: d_q
    [n_q][Hq][d], d_k and d_v [Hkv][t_cap][d] (fp32; d_k/d_v zeroed on the
    context's tokens, then accumulated)."""
    _ok(LIB.hga_attend_backward(ctypes.byref(p.c()), _ptr(q), q_start, q.shape[0], _ptr(k),
                                _ptr(v), k.shape[1], _ptr(group_idx), _ptr(group_cnt),
                                _ptr(o), _ptr(lse), _ptr(d_o), _ptr(d_q), _ptr(d_k),
                                _ptr(d_v), _stream(stream)), "hga_attend_backward")


def convert_v(p: Params, v, t_begin: int, t_end: int, v_f16, stream=None):
    """v_f16[:, t_begin:t_end] = fp16(v[:, t_begin:t_end]) (layout [Hkv][t_cap][d])."""
    _ok(LIB.hga_convert_v(ctypes.byref(p.c()), _ptr(v), v.shape[1], t_begin, t_end,
                          _ptr(v_f16), _stream(stream)), "hga_convert_v")


def commit(p: Params, k, v, t_begin: int, t_end: int, chunk_sum, group_sum, v_f16=None,
           stream=None):
    """Summaries of the tokens [t_begin, t_end) (as build_summaries) and, when
    v_f16 is given, their V in fp16 (as convert_v), in one launch."""
    _ok(LIB.hga_commit(ctypes.byref(p.c()), _ptr(k), _ptr(v), k.shape[1], t_begin, t_end,
                       _ptr(chunk_sum), _ptr(group_sum), _ptr(v_f16), _stream(stream)),
        "hga_commit")


def forward(p: Params, q, q_start: int, k, v, bufs: "Buffers", stream=None):
    _ok(LIB.hga_forward(ctypes.byref(p.c()), _ptr(q), q_start, q.shape[0],
                        _ptr(k), _ptr(v), k.shape[1], _ptr(bufs.chunk_sum),
                        _ptr(bufs.group_sum), _ptr(bufs.chunk_idx),
                        _ptr(bufs.chunk_cnt), _ptr(bufs.group_idx),
                        _ptr(bufs.group_cnt), _ptr(bufs.o), _ptr(bufs.lse),
                        _stream(stream)), "hga_forward")


def forward_causal(p: Params, q_ext, q_start: int, k, v, bufs: "Buffers", stream=None):
    """Strictly causal routing variant: q_ext = the qblock queries before
    q_start followed by the segment's queries; block b is routed on the block
    before it, attention uses the segment's own queries."""
    n_q = q_ext.shape[0] - p.qblock
    if n_q < 0:
        raise HgaError(HGA_ERR_INVALID_ARG, "forward_causal: q_ext shorter than one block")
    _ok(LIB.hga_forward_causal(ctypes.byref(p.c()), _ptr(q_ext), q_start, n_q,
                               _ptr(k), _ptr(v), k.shape[1], _ptr(bufs.chunk_sum),
                               _ptr(bufs.group_sum), _ptr(bufs.chunk_idx),
                               _ptr(bufs.chunk_cnt), _ptr(bufs.group_idx),
                               _ptr(bufs.group_cnt), _ptr(bufs.o), _ptr(bufs.lse),
                               _stream(stream)), "hga_forward_causal")


def decode_step(p: Params, q_block, pos: int, k, v, bufs: "Buffers", v_f16=None,
                stream=None):
    """One generation step of one request (hga_decode_step): commits the
    token at `pos`, routes its query block on the queries present in q_block
    (positions b0 .. pos) and attends; returns the token's output row
    [Hq][d], a view into bufs.o.  bufs: allocate(p, t_cap, p.qblock), its
    summaries holding the committed history; v_f16 (optional) receives the
    token's V in fp16 and is what the attention reads."""
    b0 = pos - pos % p.qblock
    n = pos - b0 + 1
    _ok(LIB.hga_decode_step(ctypes.byref(p.c()), _ptr(q_block[:n]), pos, _ptr(k), _ptr(v),
                            k.shape[1], _ptr(bufs.chunk_sum), _ptr(bufs.group_sum),
                            _ptr(bufs.chunk_idx), _ptr(bufs.chunk_cnt), _ptr(bufs.group_idx),
                            _ptr(bufs.group_cnt), _ptr(v_f16), _ptr(bufs.o[:n]),
                            None if bufs.lse is None else _ptr(bufs.lse[:n]),
                            _stream(stream)), "hga_decode_step")
    return bufs.o[n - 1]


@dataclasses.dataclass
class Buffers:
    """Device buffers of one routed-attention problem (allocated by torch)."""
    chunk_sum: torch.Tensor
    group_sum: torch.Tensor
    chunk_idx: torch.Tensor
    chunk_cnt: torch.Tensor
    group_idx: torch.Tensor
    group_cnt: torch.Tensor
    o: torch.Tensor
    lse: Optional[torch.Tensor]


def allocate(p: Params, t_cap: int, n_q: int, device="cuda",
             with_lse: bool = True) -> Buffers:
    d, Hkv = p.head_dim, p.n_kv_heads
    nb = (n_q + p.qblock - 1) // p.qblock
    cc, cg = index_capacity(p, t_cap, 0), index_capacity(p, t_cap, 1)
    if cc < 0 or cg < 0:
        raise HgaError(HGA_ERR_INVALID_ARG, "index_capacity")
    dt = p.torch_dtype
    i32 = torch.int32
    return Buffers(
        chunk_sum=torch.zeros(Hkv, t_cap // p.chunk, d, dtype=dt, device=device),
        group_sum=torch.zeros(Hkv, t_cap // p.group, d, dtype=dt, device=device),
        chunk_idx=torch.empty(Hkv, nb, max(cc, 1), dtype=i32, device=device),
        chunk_cnt=torch.empty(Hkv, nb, dtype=i32, device=device),
        group_idx=torch.empty(Hkv, nb, max(cg, 1), dtype=i32, device=device),
        group_cnt=torch.empty(Hkv, nb, dtype=i32, device=device),
        o=torch.empty(n_q, p.n_q_heads, d, dtype=dt, device=device),
        lse=torch.empty(n_q, p.n_q_heads, dtype=torch.float32, device=device)
        if with_lse else None,
    )


def set_kernel_variant(variant: int):
    """0 = automatic (tcgen05 kernel when eligible), 1 = portable mma.sync."""
    _ok(LIB.hga_set_kernel_variant(variant), "hga_set_kernel_variant")


def selftest_exp2(x: torch.Tensor, stream=None) -> torch.Tensor:
    """The attention kernel's software 2^x applied to a float32 device tensor."""
    y = torch.empty_like(x)
    _ok(LIB.hga_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream(stream)),
        "hga_selftest_exp2")
    return y


def set_wait_limit_ns(ns: int):
    """Limit of every bounded wait of the tensor-core kernels on the current
    device (default 2e9 ns)."""
    _ok(LIB.hga_set_wait_limit_ns(int(ns)), "hga_set_wait_limit_ns")


def selftest_wait(stream=None) -> torch.Tensor:
    """Runs the bounded-wait self test (a wait that nothing completes); returns
    a device tensor holding how long it waited, in ns.  hga_check reports
    HGA_ERR_TIMEOUT afterwards."""
    out = torch.zeros(1, dtype=torch.int64, device="cuda")
    _ok(LIB.hga_selftest_wait(_ptr(out), _stream(stream)), "hga_selftest_wait")
    return out


def debug_stall_next_attend(load_index: int):
    """One-shot test hook: the next tensor-core attention launch stops its K/V
    loads at this ring load, so its waits run into the limit (-1 clears)."""
    _ok(LIB.hga_debug_stall_next_attend(int(load_index)), "hga_debug_stall_next_attend")


# ---------------------------------------------------------------- host tier

class CGroupCache(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("tags", ctypes.c_void_p),
                ("claims", ctypes.c_void_p), ("cap", ctypes.c_int64),
                ("stats", ctypes.c_void_p)]


def _sig_tier():
    P = ctypes.POINTER(CParams)
    vp, i64, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32
    C = ctypes.POINTER(CGroupCache)
    LIB.hga_fetch_group_summaries.argtypes = [P, i64, i64, i64, i64, vp, vp, vp, C, vp, vp]
    LIB.hga_gather_history.argtypes = [P, i64, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, u32,
                                       vp, vp]
    LIB.hga_install_group_cache.argtypes = [P, i64, vp, C, vp]
    LIB.hga_gather_history_noalloc.argtypes = [P, i64, i64, i64, i64, vp, vp, vp, vp, vp, vp,
                                               vp, vp]
    for n in ("hga_fetch_group_summaries", "hga_gather_history", "hga_install_group_cache",
              "hga_gather_history_noalloc"):
        getattr(LIB, n).restype = ctypes.c_int


_sig_tier()


@dataclasses.dataclass
class HostTier:
    """History K/V and group summaries in pinned host memory, an HBM cache of
    group summaries (direct mapped), and device mirrors that routing and
    attention read."""
    t_hist: int
    k_host: torch.Tensor
    v_host: torch.Tensor
    gsum_host: torch.Tensor
    cache_data: torch.Tensor
    tags: torch.Tensor
    claims: torch.Tensor
    stats: torch.Tensor          # int64 [2]: hits, misses
    gen: torch.Tensor            # int32 [Hkv][t_cap/group] generation stamps
    bytes: torch.Tensor          # int64 [1]: history bytes gathered
    step: int = 0

    def c_cache(self) -> CGroupCache:
        return CGroupCache(self.cache_data.data_ptr(), self.tags.data_ptr(),
                           self.claims.data_ptr(), self.tags.shape[1],
                           self.stats.data_ptr())


def make_host_tier(p: Params, k_host: Optional[torch.Tensor], v_host: Optional[torch.Tensor],
                   gsum_host: torch.Tensor, t_hist: int, cache_fraction: float = 0.25,
                   device="cuda") -> HostTier:
    """k_host/v_host/gsum_host: pinned CPU tensors in the all-HBM layouts.
    k_host/v_host may be None when the history K/V lives in a KVStore (the
    tier then serves the group summaries only)."""
    for t in (k_host, v_host, gsum_host):
        if t is not None and not t.is_pinned():
            raise ValueError("host tier tensors must be pinned")
    Hkv, n_groups = gsum_host.shape[0], gsum_host.shape[1]
    cap = max(1, int(-(-cache_fraction * Hkv * n_groups // Hkv)))
    return HostTier(
        t_hist=t_hist, k_host=k_host, v_host=v_host, gsum_host=gsum_host,
        cache_data=torch.zeros(Hkv, cap, p.head_dim, dtype=p.torch_dtype, device=device),
        tags=torch.full((Hkv, cap), -1, dtype=torch.int32, device=device),
        claims=torch.full((Hkv, cap), -1, dtype=torch.int32, device=device),
        stats=torch.zeros(2, dtype=torch.int64, device=device),
        gen=torch.zeros(Hkv, n_groups, dtype=torch.int32, device=device),
        bytes=torch.zeros(1, dtype=torch.int64, device=device))


def fetch_group_summaries(p: Params, q_start: int, n_q: int, t_cap: int,
                          tier: HostTier, chunk_idx, chunk_cnt, group_sum_dev,
                          stream=None):
    c = tier.c_cache()
    _ok(LIB.hga_fetch_group_summaries(
        ctypes.byref(p.c()), q_start, n_q, t_cap, tier.t_hist, _ptr(chunk_idx),
        _ptr(chunk_cnt), _ptr(tier.gsum_host), ctypes.byref(c), _ptr(group_sum_dev),
        _stream(stream)), "hga_fetch_group_summaries")


def gather_history(p: Params, q_start: int, n_q: int, t_cap: int, tier: HostTier,
                   group_idx, group_cnt, k_dev, v_dev, stream=None):
    tier.step += 1
    _ok(LIB.hga_gather_history(
        ctypes.byref(p.c()), q_start, n_q, t_cap, tier.t_hist, _ptr(group_idx),
        _ptr(group_cnt), _ptr(tier.k_host), _ptr(tier.v_host), _ptr(k_dev), _ptr(v_dev),
        _ptr(tier.gen), ctypes.c_uint32(tier.step), _ptr(tier.bytes), _stream(stream)),
        "hga_gather_history")


def gather_history_noalloc(p: Params, q_start: int, n_q: int, t_cap: int, tier: HostTier,
                           group_idx, group_cnt, k_dev, v_dev, stream=None):
    """gather_history with the generation stamps held inside the library
    (no device buffer for them from the caller); tier.gen and tier.step are
    not used."""
    _ok(LIB.hga_gather_history_noalloc(
        ctypes.byref(p.c()), q_start, n_q, t_cap, tier.t_hist, _ptr(group_idx),
        _ptr(group_cnt), _ptr(tier.k_host), _ptr(tier.v_host), _ptr(k_dev), _ptr(v_dev),
        _ptr(tier.bytes), _stream(stream)), "hga_gather_history_noalloc")


def install_group_cache(p: Params, t_cap: int, tier: HostTier, stream=None):
    c = tier.c_cache()
    _ok(LIB.hga_install_group_cache(ctypes.byref(p.c()), t_cap, _ptr(tier.gsum_host),
                                    ctypes.byref(c), _stream(stream)),
        "hga_install_group_cache")


def tiered_step(p: Params, q, q_start: int, tier: HostTier, k_dev, v_dev, bufs: "Buffers",
                side_stream=None):
    """One query segment through the tier: segment summaries, chunk routing,
    summary fetch (cache / host), group routing, history gather on a side
    stream, attention, cache install.  k_dev/v_dev hold the segment's own K/V
    at [q_start, q_start + n_q); bufs.group_sum is the device summary mirror."""
    main = torch.cuda.current_stream()
    side = side_stream or torch.cuda.Stream()
    n_q, t_cap = q.shape[0], k_dev.shape[1]
    build_summaries(p, k_dev, q_start, q_start + n_q, bufs.chunk_sum, bufs.group_sum)
    route_chunks(p, q, q_start, bufs.chunk_sum, t_cap, bufs.chunk_idx, bufs.chunk_cnt)
    fetch_group_summaries(p, q_start, n_q, t_cap, tier, bufs.chunk_idx, bufs.chunk_cnt,
                          bufs.group_sum)
    route_groups(p, q, q_start, bufs.group_sum, t_cap, bufs.chunk_idx, bufs.chunk_cnt,
                 bufs.group_idx, bufs.group_cnt)
    side.wait_stream(main)
    gather_history(p, q_start, n_q, t_cap, tier, bufs.group_idx, bufs.group_cnt, k_dev,
                   v_dev, stream=side)
    main.wait_stream(side)
    attend(p, q, q_start, k_dev, v_dev, bufs.group_idx, bufs.group_cnt, bufs.o, bufs.lse)
    install_group_cache(p, t_cap, tier)


# ---------------------------------------------------------------- file-backed store

class CStoreStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "pages_needed", "hits", "misses", "evictions", "bytes_read")]


def _sig_store():
    P = ctypes.POINTER(CParams)
    vp, i64, i32, u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32
    sig = {
        "hga_store_open": [ctypes.c_char_p, P, i64, i64, i32, ctypes.POINTER(vp)],
        "hga_store_close": [vp],
        "hga_store_attach_cache": [vp, vp, i64, vp],
        "hga_store_append": [vp, vp, vp, i64],
        "hga_store_set_length": [vp, i64],
        "hga_store_read": [vp, i64, i64, vp, vp],
        "hga_store_prepare": [vp, P, i64, i64, i64, vp, vp, i32, ctypes.POINTER(CStoreStats)],
        "hga_gather_store": [P, vp, i64, i64, i64, vp, vp, vp, vp, vp, u32, vp, vp],
    }
    for name, args in sig.items():
        fn = getattr(LIB, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    for name in ("hga_store_length", "hga_store_page_bytes", "hga_store_pages_per_head"):
        getattr(LIB, name).argtypes = [vp]
        getattr(LIB, name).restype = ctypes.c_int64


_sig_store()


def _aligned_bytes(n: int, align: int, pin: bool) -> torch.Tensor:
    raw = torch.empty(n + align, dtype=torch.uint8, pin_memory=pin)
    off = (-raw.data_ptr()) % align
    return raw[off:off + n]


class KVStore:
    """History K/V in one file, read through a bounded page cache in host
    memory (pinned when a kernel gathers from it).  A page is page_tokens
    tokens of one KV head, K then V; the page table [Hkv][n_pages] maps a
    page to its cache slot (-1 absent).  Wraps the hga_store_* calls.

    The cache and page table are tensors of this object that kernels read
    in place: keep the object alive (and do not call reset_cache or
    prepare) until every gather from it has completed on its stream."""

    def __init__(self, p: Params, path: str, t_cap: int, page_tokens: int, cache_pages: int,
                 create: bool = True, direct: bool = False, pin: bool = True):
        self.p, self.path, self.t_cap = p, path, t_cap
        h = ctypes.c_void_p()
        flags = (HGA_STORE_CREATE if create else 0) | (HGA_STORE_DIRECT if direct else 0)
        _ok(LIB.hga_store_open(path.encode(), ctypes.byref(p.c()), t_cap, page_tokens, flags,
                               ctypes.byref(h)), "hga_store_open")
        self.handle = h
        self.page_tokens = page_tokens
        self.page_bytes = int(LIB.hga_store_page_bytes(h))
        self.n_pages = int(LIB.hga_store_pages_per_head(h))
        self.cache_pages = cache_pages
        self.cache = _aligned_bytes(cache_pages * self.page_bytes, 4096, pin)
        self.page_table = _aligned_bytes(p.n_kv_heads * self.n_pages * 4, 64, pin).view(
            torch.int32).view(p.n_kv_heads, self.n_pages)
        _ok(LIB.hga_store_attach_cache(h, _ptr(self.cache), cache_pages, _ptr(self.page_table)),
            "hga_store_attach_cache")
        self._host_idx = None

    @property
    def length(self) -> int:
        return int(LIB.hga_store_length(self.handle))

    def set_length(self, n: int):
        _ok(LIB.hga_store_set_length(self.handle, n), "hga_store_set_length")

    def append(self, k: torch.Tensor, v: torch.Tensor):
        """k, v: CPU [Hkv][n][d] in the store's dtype."""
        k, v = k.contiguous(), v.contiguous()
        if k.device.type != "cpu" or v.device.type != "cpu" or k.shape != v.shape:
            raise ValueError("append takes two CPU tensors of one shape [Hkv][n][d]")
        _ok(LIB.hga_store_append(self.handle, _ptr(k), _ptr(v), k.shape[1]), "hga_store_append")

    def read(self, t_begin: int, t_end: int):
        """Tokens [t_begin, t_end) from the file: CPU K, V [Hkv][n][d]."""
        shape = (self.p.n_kv_heads, t_end - t_begin, self.p.head_dim)
        k = torch.empty(shape, dtype=self.p.torch_dtype)
        v = torch.empty(shape, dtype=self.p.torch_dtype)
        _ok(LIB.hga_store_read(self.handle, t_begin, t_end, _ptr(k), _ptr(v)), "hga_store_read")
        return k, v

    def prepare(self, p: Params, q_start: int, n_q: int, t_hist: int, group_idx_host,
                group_cnt_host, io_threads: int = 8) -> dict:
        st = CStoreStats()
        code = LIB.hga_store_prepare(self.handle, ctypes.byref(p.c()), q_start, n_q, t_hist,
                                     _ptr(group_idx_host), _ptr(group_cnt_host), io_threads,
                                     ctypes.byref(st))
        stats = {n: getattr(st, n) for n, _ in CStoreStats._fields_}
        _ok(code, "hga_store_prepare")
        return stats

    def reset_cache(self, cache_pages: Optional[int] = None):
        """Drops every cached page (the slots and the page table restart
        empty); cache_pages, at most the allocated count, bounds the cache
        from now on."""
        n = self.cache_pages if cache_pages is None else cache_pages
        if not 0 < n <= self.cache.numel() // self.page_bytes:
            raise ValueError("cache_pages exceeds the allocated cache")
        _ok(LIB.hga_store_attach_cache(self.handle, _ptr(self.cache), n,
                                       _ptr(self.page_table)), "hga_store_attach_cache")
        self.cache_pages = n

    def host_index_buffers(self, bufs: "Buffers"):
        """Pinned host copies' storage for a step's group_idx / group_cnt."""
        if (self._host_idx is None or self._host_idx[0].shape != bufs.group_idx.shape
                or self._host_idx[1].shape != bufs.group_cnt.shape):
            self._host_idx = (torch.empty(bufs.group_idx.shape, dtype=torch.int32,
                                          pin_memory=True),
                              torch.empty(bufs.group_cnt.shape, dtype=torch.int32,
                                          pin_memory=True))
        return self._host_idx

    def close(self):
        if self.handle:
            code = LIB.hga_store_close(self.handle)
            self.handle = None
            _ok(code, "hga_store_close")

    def __del__(self):
        try:
            if getattr(self, "handle", None):
                LIB.hga_store_close(self.handle)
                self.handle = None
        except Exception:
            pass


def gather_store(p: Params, store: KVStore, q_start: int, n_q: int, t_hist: int, group_idx,
                 group_cnt, k_dev, v_dev, gen, step: int, nbytes=None, stream=None):
    """k_dev/v_dev: device [Hkv][store.t_cap][d]; group_idx/group_cnt laid out
    for store.t_cap."""
    if k_dev.shape[1] != store.t_cap or v_dev.shape[1] != store.t_cap:
        raise HgaError(HGA_ERR_INVALID_ARG, "gather_store: k_dev/v_dev must span the store's t_cap")
    _ok(LIB.hga_gather_store(ctypes.byref(p.c()), store.handle, q_start, n_q, t_hist,
                             _ptr(group_idx), _ptr(group_cnt), _ptr(k_dev), _ptr(v_dev),
                             _ptr(gen), ctypes.c_uint32(step), _ptr(nbytes), _stream(stream)),
        "hga_gather_store")


def store_step(p: Params, q, q_start: int, tier: HostTier, store: KVStore, k_dev, v_dev,
               bufs: "Buffers", io_threads: int = 8) -> dict:
    """One query segment with the history K/V in a file-backed store: segment
    summaries, chunk routing, group-summary fetch (HBM cache / pinned RAM),
    group routing, the routed indices to the host, the store's page cache
    filled from the file, history gathered from the cache, attention, cache
    install.  Everything runs on the current stream; the host waits once,
    for the indices.  Returns the store's counts for the step, with the
    host's wait for the routing (host_wait_s) and the time the cache took to
    fill (prepare_s)."""
    main = torch.cuda.current_stream()
    n_q, t_cap = q.shape[0], k_dev.shape[1]
    if t_cap != store.t_cap or v_dev.shape[1] != store.t_cap:
        raise HgaError(HGA_ERR_INVALID_ARG, "store_step: k_dev/v_dev must span the store's t_cap")
    build_summaries(p, k_dev, q_start, q_start + n_q, bufs.chunk_sum, bufs.group_sum)
    route_chunks(p, q, q_start, bufs.chunk_sum, t_cap, bufs.chunk_idx, bufs.chunk_cnt)
    fetch_group_summaries(p, q_start, n_q, t_cap, tier, bufs.chunk_idx, bufs.chunk_cnt,
                          bufs.group_sum)
    route_groups(p, q, q_start, bufs.group_sum, t_cap, bufs.chunk_idx, bufs.chunk_cnt,
                 bufs.group_idx, bufs.group_cnt)
    gi_h, gc_h = store.host_index_buffers(bufs)
    gi_h.copy_(bufs.group_idx, non_blocking=True)
    gc_h.copy_(bufs.group_cnt, non_blocking=True)
    t0 = time.perf_counter()
    main.synchronize()                  # also ends the previous step's gather
    t1 = time.perf_counter()
    stats = store.prepare(p, q_start, n_q, tier.t_hist, gi_h, gc_h, io_threads)
    stats["host_wait_s"] = t1 - t0
    stats["prepare_s"] = time.perf_counter() - t1
    tier.step += 1
    gather_store(p, store, q_start, n_q, tier.t_hist, bufs.group_idx, bufs.group_cnt, k_dev,
                 v_dev, tier.gen, tier.step, tier.bytes)
    attend(p, q, q_start, k_dev, v_dev, bufs.group_idx, bufs.group_cnt, bufs.o, bufs.lse)
    install_group_cache(p, t_cap, tier)
    return stats

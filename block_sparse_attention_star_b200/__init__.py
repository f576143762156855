"""Python binding of libstar.so, the Star Attention hot path for NVIDIA B200.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Functions carry the C names of ``include/star.h`` and take torch
tensors (device memory and streams come from PyTorch).  There is no CPU
fallback: if ``libstar.so`` is missing or a call fails, an exception is raised.

Typical use::

    import block_sparse_attention_star_b200 as star
    shape = star.StarShape.make(B=1, Hq=32, Hkv=8, d=128, L=131072, b=32768, T_max=128)
    cache = star.PagedKVCache(shape, device="cuda")
    star.star_phase1_encode(shape, cache, q, k, v, pos_ctx, out)
    o_part, lse_part = star.alloc_partials(shape, T)
    ws = star.workspace(shape, star.STAR_OP_PHASE2, T)
    star.star_phase2_partial(shape, cache, q_query, k_query, v_query, pos_query, T, o_part, lse_part, ws)
    star.star_lse_merge(shape.n, B * T * Hq, d, o_part, lse_part, out_query, lse_query)
"""

from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libstar.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "star.h")

STAR_OK = 0
STAR_ERR_INVALID_ARG = -1
STAR_ERR_UNSUPPORTED_SHAPE = -2
STAR_ERR_ALIGNMENT = -3
STAR_ERR_CAPACITY = -4
STAR_ERR_CUDA = -5
STAR_ERR_TIMEOUT = -6
STAR_ERR_CALLBACK = -7
STAR_LAYER_QKV, STAR_LAYER_OUT = 0, 1
STAR_OP_PHASE1, STAR_OP_PHASE2, STAR_OP_DECODE, STAR_OP_PHASE1_ANCHOR, STAR_OP_PHASE2_PUSH = 1, 2, 3, 4, 5
STAR_DEBUG_SKIP_FIRST_LOAD = 1


class StarError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"star error {code}: {msg}")
        self.code = code


class StarShape(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32),
        ("L", ctypes.c_int32), ("b", ctypes.c_int32), ("n", ctypes.c_int32), ("T_max", ctypes.c_int32),
        ("page_tokens", ctypes.c_int32), ("rope_theta", ctypes.c_double), ("anchor", ctypes.c_int32),
        ("seq_len", ctypes.POINTER(ctypes.c_int32)),
    ]

    @classmethod
    def make(cls, B, Hq, Hkv, d, L, b, T_max, page_tokens=256, rope_theta=500000.0, anchor=0,
             seq_len=None) -> "StarShape":
        """anchor: the anchor size a (the first a tokens of block 1); 0 means b.
        seq_len: per-sequence context lengths (B ints, each in [1, L]) or None; L is then the
        capacity and each sequence's tail starts at its own length."""
        sh = cls(B, Hq, Hkv, d, L, b, L // b if b else 0, T_max, page_tokens, rope_theta, anchor)
        if seq_len is not None:
            lens = [int(x) for x in seq_len]
            if len(lens) != B:
                raise ValueError(f"seq_len has {len(lens)} entries for B = {B}")
            sh._seq_len_buf = (ctypes.c_int32 * B)(*lens)   # kept alive with the shape
            sh.seq_len = ctypes.cast(sh._seq_len_buf, ctypes.POINTER(ctypes.c_int32))
        return sh


class StarShard(ctypes.Structure):
    """Blocks [block_begin, block_end) of every sequence, owned by one GPU (star.h star_shard)."""
    _fields_ = [("block_begin", ctypes.c_int32), ("block_end", ctypes.c_int32)]


class StarExchange(ctypes.Structure):
    """One rank's view of the peer-memory exchange (star.h star_exchange)."""
    _fields_ = [("world", ctypes.c_int32), ("rank", ctypes.c_int32), ("slots", ctypes.c_int32),
                ("peers", ctypes.c_void_p * 8)]


class StarCache(ctypes.Structure):
    _fields_ = [
        ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p), ("page_table", ctypes.c_void_p),
        ("max_pages", ctypes.c_int32), ("num_pages", ctypes.c_int32),
    ]


_lib = None

# int fn(int32 layer, int32 stage, void* in, void* out0, void* out1, void* out2, void* user, stream)
LAYER_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p)


def lib() -> ctypes.CDLL:
    """The loaded libstar.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m block_sparse_attention_star_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ, V = ctypes.POINTER, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p
        sig = {
            "star_version": ([], ctypes.c_char_p),
            "star_last_error": ([], ctypes.c_char_p),
            "star_pages_needed": ([P(StarShape), P(I32)], ctypes.c_int),
            "star_page_table_fill": ([P(StarShape), V, I32, I32], ctypes.c_int),
            "star_workspace_size": ([P(StarShape), ctypes.c_int, I32, P(SZ)], ctypes.c_int),
            "star_build_positions": ([P(StarShape), P(StarCache), V, V, V, V], ctypes.c_int),
            "star_kv_append": ([P(StarShape), P(StarCache), V, V, V, I32, I32, V], ctypes.c_int),
            "star_phase1_encode": ([P(StarShape), P(StarCache), V, V, V, V, V, V, SZ, V], ctypes.c_int),
            "star_phase1_encode_anchored": ([P(StarShape), P(StarCache), V, V, V, V, V, V, V, SZ, V], ctypes.c_int),
            "star_phase2_partial": ([P(StarShape), P(StarCache), V, V, V, V, I32, V, V, V, SZ, V], ctypes.c_int),
            "star_lse_merge": ([I32, I64, I32, V, V, V, V, V], ctypes.c_int),
            "star_decode_step": ([P(StarShape), P(StarCache), V, V, V, V, I32, V, V, V, SZ, V], ctypes.c_int),
            "star_device_status": ([V, P(I32)], ctypes.c_int),
            "star_set_trace_events": ([V, V], ctypes.c_int),
            "star_decode_step_noalloc": ([P(StarShape), P(StarCache), V, V, V, V, I32, V, V, V], ctypes.c_int),
            "star_encode_layers": ([P(StarShape), I32, P(StarCache), V, V, V, V, V, V, LAYER_FN, V, V], ctypes.c_int),
            "star_debug_set": ([ctypes.c_uint64, I32], ctypes.c_int),
            "star_phase1_encode_shard": ([P(StarShape), P(StarCache), P(StarShard), V, V, V, V, V, V, V, V, V],
                                         ctypes.c_int),
            "star_phase2_partial_shard": ([P(StarShape), P(StarCache), P(StarShard), V, V, V, V, I32, V, V, V, SZ, V],
                                          ctypes.c_int),
            "star_decode_partial_shard": ([P(StarShape), P(StarCache), P(StarShard), V, V, V, V, I32, V, V, V, SZ, V],
                                          ctypes.c_int),
            "star_exchange_size": ([I32, I32, I64, I32, P(SZ)], ctypes.c_int),
            "star_phase2_partial_shard_push": ([P(StarShape), P(StarCache), P(StarShard), V, V, V, V, I32,
                                                P(StarExchange), ctypes.c_uint64, V, SZ, V], ctypes.c_int),
            "star_decode_partial_shard_push": ([P(StarShape), P(StarCache), P(StarShard), V, V, V, V, I32,
                                                P(StarExchange), ctypes.c_uint64, V, SZ, V], ctypes.c_int),
            "star_exchange_merge": ([P(StarExchange), I64, I32, ctypes.c_uint64, V, V, V], ctypes.c_int),
            "star_ipc_export": ([V, V, P(ctypes.c_uint64)], ctypes.c_int),
            "star_ipc_open": ([V, ctypes.c_uint64, P(V)], ctypes.c_int),
            "star_ipc_close": ([V, ctypes.c_uint64], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def header_symbols() -> list[str]:
    """Every function the public header declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(star_\w+)\s*\(", text, re.M)))


def _check(rc: int) -> None:
    if rc != STAR_OK:
        raise StarError(rc, lib().star_last_error().decode())


def _ptr(t: torch.Tensor | None, name: str, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def star_version() -> str:
    return lib().star_version().decode()


def star_pages_needed(shape: StarShape) -> int:
    out = ctypes.c_int32()
    _check(lib().star_pages_needed(ctypes.byref(shape), ctypes.byref(out)))
    return out.value


def star_page_table_fill(shape: StarShape, max_pages: int, first_page: int = 0) -> torch.Tensor:
    tab = torch.empty((shape.B, max_pages), dtype=torch.int32)
    _check(lib().star_page_table_fill(ctypes.byref(shape), ctypes.c_void_p(tab.data_ptr()), max_pages, first_page))
    return tab


def star_workspace_size(shape: StarShape, op: int, T: int = 0) -> int:
    out = ctypes.c_size_t()
    _check(lib().star_workspace_size(ctypes.byref(shape), op, T, ctypes.byref(out)))
    return out.value


class PagedKVCache:
    """Device K/V page pools plus the page table, allocated with torch.

    Pools are bf16 [num_pages][Hkv][page_tokens][d]; the page table is the
    block-contiguous assignment of ``star_page_table_fill`` unless given.
    """

    def __init__(self, shape: StarShape, device="cuda", page_table: torch.Tensor | None = None,
                 num_pages: int | None = None):
        self.shape = shape
        self.max_pages = star_pages_needed(shape)
        if page_table is None:
            page_table = star_page_table_fill(shape, self.max_pages)
            num_pages = shape.B * self.max_pages
        elif num_pages is None:
            num_pages = int(page_table.max().item()) + 1
        self.num_pages = int(num_pages)
        P, d = shape.page_tokens, shape.d
        self.k_pool = torch.zeros((self.num_pages, shape.Hkv, P, d), dtype=torch.bfloat16, device=device)
        self.v_pool = torch.zeros_like(self.k_pool)
        self.page_table = page_table.to(device=device, dtype=torch.int32).contiguous()
        self.c = StarCache(self.k_pool.data_ptr(), self.v_pool.data_ptr(), self.page_table.data_ptr(),
                           page_table.shape[1], self.num_pages)

    def gather(self, seq: int, start: int, end: int) -> tuple[torch.Tensor, torch.Tensor]:
        """Cache slots [start, end) of sequence ``seq`` as [tokens, Hkv, d] (a copy)."""
        P = self.shape.page_tokens
        t = torch.arange(start, end, device=self.k_pool.device)
        pages = self.page_table[seq, t // P].long()
        slot = t % P
        k = self.k_pool[pages, :, slot, :]
        v = self.v_pool[pages, :, slot, :]
        return k, v


def star_build_positions(shape, cache: PagedKVCache, pos_ctx, aug_pos, block_map, stream=None):
    _check(lib().star_build_positions(ctypes.byref(shape), ctypes.byref(cache.c), _ptr(pos_ctx, "pos_ctx", torch.int32),
                                      _ptr(aug_pos, "aug_pos", torch.int32), _ptr(block_map, "block_map", torch.int32),
                                      _stream(stream)))


def star_kv_append(shape, cache: PagedKVCache, k, v, pos, start: int, ntok: int, stream=None):
    _check(lib().star_kv_append(ctypes.byref(shape), ctypes.byref(cache.c), _ptr(k, "k", torch.bfloat16),
                                _ptr(v, "v", torch.bfloat16), _ptr(pos, "pos", torch.int32), start, ntok,
                                _stream(stream)))


def star_phase1_encode(shape, cache: PagedKVCache, q, k, v, pos_ctx, out, ws=None, stream=None):
    _check(lib().star_phase1_encode(ctypes.byref(shape), ctypes.byref(cache.c), _ptr(q, "q", torch.bfloat16),
                                    _ptr(k, "k", torch.bfloat16), _ptr(v, "v", torch.bfloat16),
                                    _ptr(pos_ctx, "pos_ctx", torch.int32), _ptr(out, "out", torch.bfloat16),
                                    _ptr(ws, "ws"), 0 if ws is None else ws.numel() * ws.element_size(),
                                    _stream(stream)))


def star_phase1_encode_anchored(shape, cache: PagedKVCache, q, k, v, pos_ctx, anchor_pos, out, ws=None, stream=None):
    """Phase 1 with the anchor's position ids per block (int32 [B][n-1][a], or None for the default)."""
    _check(lib().star_phase1_encode_anchored(ctypes.byref(shape), ctypes.byref(cache.c), _ptr(q, "q", torch.bfloat16),
                                             _ptr(k, "k", torch.bfloat16), _ptr(v, "v", torch.bfloat16),
                                             _ptr(pos_ctx, "pos_ctx", torch.int32),
                                             _ptr(anchor_pos, "anchor_pos", torch.int32),
                                             _ptr(out, "out", torch.bfloat16), _ptr(ws, "ws"),
                                             0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def star_phase2_partial(shape, cache: PagedKVCache, q, k, v, q_pos, T: int, o_part, lse_part, ws, stream=None):
    _check(lib().star_phase2_partial(ctypes.byref(shape), ctypes.byref(cache.c), _ptr(q, "q", torch.bfloat16),
                                     _ptr(k, "k", torch.bfloat16), _ptr(v, "v", torch.bfloat16),
                                     _ptr(q_pos, "q_pos", torch.int32), T, _ptr(o_part, "o_part", torch.float32),
                                     _ptr(lse_part, "lse_part", torch.float32), _ptr(ws, "ws"),
                                     0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def star_lse_merge(n_parts: int, rows: int, d: int, o_part, lse_part, out, lse_out=None, stream=None):
    _check(lib().star_lse_merge(n_parts, rows, d, _ptr(o_part, "o_part", torch.float32),
                                _ptr(lse_part, "lse_part", torch.float32), _ptr(out, "out", torch.bfloat16),
                                _ptr(lse_out, "lse_out", torch.float32), _stream(stream)))


def star_decode_step(shape, cache: PagedKVCache, q, k, v, pos, cur_len: int, out, lse_out, ws, stream=None):
    _check(lib().star_decode_step(ctypes.byref(shape), ctypes.byref(cache.c), _ptr(q, "q", torch.bfloat16),
                                  _ptr(k, "k", torch.bfloat16), _ptr(v, "v", torch.bfloat16),
                                  _ptr(pos, "pos", torch.int32), cur_len, _ptr(out, "out", torch.bfloat16),
                                  _ptr(lse_out, "lse_out", torch.float32), _ptr(ws, "ws"),
                                  ws.numel() * ws.element_size(), _stream(stream)))


def star_set_trace_events(start=None, stop=None) -> None:
    """Record torch.cuda.Event ``start``/``stop`` around each later call's main kernel (None, None: off)."""
    def handle(ev):
        return None if ev is None else ctypes.c_void_p(ev.cuda_event)
    _check(lib().star_set_trace_events(handle(start), handle(stop)))


def star_decode_step_noalloc(shape, cache: PagedKVCache, q, k, v, pos, cur_len: int, out, lse_out, stream=None):
    """star_decode_step with the library's built-in scratch instead of a caller workspace."""
    _check(lib().star_decode_step_noalloc(ctypes.byref(shape), ctypes.byref(cache.c), _ptr(q, "q", torch.bfloat16),
                                          _ptr(k, "k", torch.bfloat16), _ptr(v, "v", torch.bfloat16),
                                          _ptr(pos, "pos", torch.int32), cur_len, _ptr(out, "out", torch.bfloat16),
                                          _ptr(lse_out, "lse_out", torch.float32), _stream(stream)))


def star_encode_layers(shape, caches, pos_ctx, x, q, k, v, o, fn, stream=None):
    """Multi-layer context encoding (star_encode_layers in star.h).

    fn(layer, stage, x, q, k, v, o) enqueues the caller's work on the current stream:
    stage STAR_LAYER_QKV writes q, k, v from x; stage STAR_LAYER_OUT updates x in place
    from the attention output o.  caches: one PagedKVCache per layer.  An exception in
    fn stops the call and is raised again here.
    """
    if isinstance(caches, PagedKVCache):
        raise TypeError("caches must be a sequence of PagedKVCache, one per layer")
    arr = (StarCache * len(caches))(*[c.c for c in caches])
    raised = []

    def trampoline(layer, stage, _in, _o0, _o1, _o2, _user, _stream_handle):
        try:
            fn(int(layer), int(stage), x, q, k, v, o)
            return 0
        except BaseException as e:  # re-raised after the C call returns
            raised.append(e)
            return 1

    cb = LAYER_FN(trampoline)
    rc = lib().star_encode_layers(ctypes.byref(shape), len(caches), arr, _ptr(pos_ctx, "pos_ctx", torch.int32),
                                  _ptr(x, "x"), _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                  _ptr(v, "v", torch.bfloat16), _ptr(o, "o", torch.bfloat16), cb, None,
                                  _stream(stream))
    if raised:
        raise raised[0]
    _check(rc)


def star_device_status(stream=None) -> int:
    code = ctypes.c_int32()
    rc = lib().star_device_status(_stream(stream), ctypes.byref(code))
    _check(rc)
    return code.value


def star_phase1_encode_shard(shape, cache: PagedKVCache, shard: StarShard, q, k, v, pos, k_anchor, v_anchor,
                             pos_anchor, out, stream=None):
    _check(lib().star_phase1_encode_shard(ctypes.byref(shape), ctypes.byref(cache.c), ctypes.byref(shard),
                                          _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                          _ptr(v, "v", torch.bfloat16), _ptr(pos, "pos", torch.int32),
                                          _ptr(k_anchor, "k_anchor", torch.bfloat16),
                                          _ptr(v_anchor, "v_anchor", torch.bfloat16),
                                          _ptr(pos_anchor, "pos_anchor", torch.int32),
                                          _ptr(out, "out", torch.bfloat16), _stream(stream)))


def star_phase2_partial_shard(shape, cache: PagedKVCache, shard: StarShard, q, k, v, q_pos, T: int, o_part, lse_part,
                              ws, stream=None):
    _check(lib().star_phase2_partial_shard(ctypes.byref(shape), ctypes.byref(cache.c), ctypes.byref(shard),
                                           _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                           _ptr(v, "v", torch.bfloat16), _ptr(q_pos, "q_pos", torch.int32), T,
                                           _ptr(o_part, "o_part", torch.float32),
                                           _ptr(lse_part, "lse_part", torch.float32), _ptr(ws, "ws"),
                                           ws.numel() * ws.element_size(), _stream(stream)))


def star_decode_partial_shard(shape, cache: PagedKVCache, shard: StarShard, q, k, v, pos, cur_len: int, o_part,
                              lse_part, ws, stream=None):
    _check(lib().star_decode_partial_shard(ctypes.byref(shape), ctypes.byref(cache.c), ctypes.byref(shard),
                                           _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                           _ptr(v, "v", torch.bfloat16), _ptr(pos, "pos", torch.int32), cur_len,
                                           _ptr(o_part, "o_part", torch.float32),
                                           _ptr(lse_part, "lse_part", torch.float32), _ptr(ws, "ws"),
                                           ws.numel() * ws.element_size(), _stream(stream)))


def star_exchange_size(world: int, slots: int, rows: int, d: int) -> int:
    out = ctypes.c_size_t()
    _check(lib().star_exchange_size(world, slots, rows, d, ctypes.byref(out)))
    return out.value


def star_phase2_partial_shard_push(shape, cache: PagedKVCache, shard: StarShard, q, k, v, q_pos, T: int,
                                   ex: StarExchange, epoch: int, ws, stream=None):
    _check(lib().star_phase2_partial_shard_push(ctypes.byref(shape), ctypes.byref(cache.c), ctypes.byref(shard),
                                                _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                                _ptr(v, "v", torch.bfloat16), _ptr(q_pos, "q_pos", torch.int32), T,
                                                ctypes.byref(ex), epoch, _ptr(ws, "ws"),
                                                ws.numel() * ws.element_size(), _stream(stream)))


def star_decode_partial_shard_push(shape, cache: PagedKVCache, shard: StarShard, q, k, v, pos, cur_len: int,
                                   ex: StarExchange, epoch: int, ws, stream=None):
    _check(lib().star_decode_partial_shard_push(ctypes.byref(shape), ctypes.byref(cache.c), ctypes.byref(shard),
                                                _ptr(q, "q", torch.bfloat16), _ptr(k, "k", torch.bfloat16),
                                                _ptr(v, "v", torch.bfloat16), _ptr(pos, "pos", torch.int32), cur_len,
                                                ctypes.byref(ex), epoch, _ptr(ws, "ws"),
                                                ws.numel() * ws.element_size(), _stream(stream)))


def star_exchange_merge(ex: StarExchange, rows: int, d: int, epoch: int, out, lse_out=None, stream=None):
    _check(lib().star_exchange_merge(ctypes.byref(ex), rows, d, epoch, _ptr(out, "out", torch.bfloat16),
                                     _ptr(lse_out, "lse_out", torch.float32), _stream(stream)))


def star_ipc_export(t: torch.Tensor) -> tuple[bytes, int]:
    """(64-byte IPC handle, offset) of a device tensor's memory, for another process to open."""
    h = (ctypes.c_ubyte * 64)()
    off = ctypes.c_uint64()
    _check(lib().star_ipc_export(ctypes.c_void_p(t.data_ptr()), h, ctypes.byref(off)))
    return bytes(h), off.value


def star_ipc_open(handle: bytes, offset: int) -> int:
    """Device address, valid in this process, of memory another process exported."""
    h = (ctypes.c_ubyte * 64).from_buffer_copy(handle)
    ptr = ctypes.c_void_p()
    _check(lib().star_ipc_open(h, offset, ctypes.byref(ptr)))
    return ptr.value


def star_ipc_close(ptr: int, offset: int) -> None:
    _check(lib().star_ipc_close(ctypes.c_void_p(ptr), offset))


def star_debug_set(wait_limit_ns: int = 0, flags: int = 0) -> None:
    """Failure-detection test hook: the bounded waits' limit (0 = the default 2 s) and
    debug flags (STAR_DEBUG_SKIP_FIRST_LOAD) for later attention and decode launches."""
    _check(lib().star_debug_set(int(wait_limit_ns), int(flags)))


def workspace(shape: StarShape, op: int, T: int = 0, device="cuda") -> torch.Tensor:
    """A uint8 device buffer of star_workspace_size bytes (at least 256)."""
    n = max(256, star_workspace_size(shape, op, T))
    return torch.empty(n, dtype=torch.uint8, device=device)


def alloc_partials(shape: StarShape, T: int, device="cuda") -> tuple[torch.Tensor, torch.Tensor]:
    o = torch.empty((shape.n, shape.B, T, shape.Hq, shape.d), dtype=torch.float32, device=device)
    lse = torch.empty((shape.n, shape.B, T, shape.Hq), dtype=torch.float32, device=device)
    return o, lse

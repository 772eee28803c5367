"""ctypes binding of libusp (the C ABI declared in include/usp.h).

Argument marshalling only: every step of the block runs in the library's CUDA
kernels. PyTorch provides device memory (tensors) and streams. Each virtual
rank's tensor is a separate CUDA tensor; per-rank arguments are lists indexed
by rank. The names follow the API page "mstar.model.components.distributed.
sequence_parallel" (sp_seq_split, scatter_sequence, gather_sequence,
sp_head_slice, sp_head_gather, ulysses_attention) and the ragged transport
page (seq_to_heads / heads_to_seq, here ulysses_seq_to_head /
ulysses_head_to_seq).

Loading fails loudly (OSError) if libusp.so has not been built:
``python -m ulysses_sequence_attention_sp_b200.build``.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libusp.so"

USP_OK = 0
USP_ERR_INVALID_ARG = 1
USP_ERR_SHAPE = 2
USP_ERR_DTYPE = 3
USP_ERR_ALIGN = 4
USP_ERR_CUDA = 5
USP_ERR_TIMEOUT = 6
USP_ERR_UNSUPPORTED = 7
USP_ERR_NO_DEVICE = 8
USP_ERR_BOUNDS = 9

USP_BF16, USP_FP32, USP_FP16 = 0, 1, 2
MAX_WORLD = 32
MAX_HEADS = 256

_DTYPES = {torch.bfloat16: USP_BF16, torch.float32: USP_FP32, torch.float16: USP_FP16}
_NAMES = {"bf16": USP_BF16, "fp32": USP_FP32, "fp16": USP_FP16}
_TORCH = {USP_BF16: torch.bfloat16, USP_FP32: torch.float32, USP_FP16: torch.float16}

_c_i64p = ctypes.POINTER(ctypes.c_int64)
_c_i32p = ctypes.POINTER(ctypes.c_int32)
_c_vpp = ctypes.POINTER(ctypes.c_void_p)

# name -> (restype, argtypes)
_SIGNATURES = {
    "usp_last_error_message": (ctypes.c_char_p, []),
    "usp_version": (ctypes.c_int, []),
    "usp_balanced_ranges": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int32, _c_i64p, _c_i64p]),
    "usp_seq_split": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int32, _c_i64p]),
    "usp_head_chunk_ranges": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, _c_i32p, _c_i32p, _c_i32p]),
    "usp_plan_create": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32]),
    "usp_plan_create_gqa": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_int32, ctypes.c_int32]),
    "usp_plan_query_kv": (ctypes.c_int, [ctypes.c_void_p, _c_i32p, _c_i32p, _c_i32p]),
    "usp_ulysses_seq_to_head_kv": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, _c_vpp, _c_vpp,
                                                  ctypes.c_void_p]),
    "usp_all_gather_rows": (ctypes.c_int, [ctypes.c_void_p, _c_vpp, _c_vpp, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_void_p]),
    "usp_reduce_scatter_rows": (ctypes.c_int, [ctypes.c_void_p, _c_vpp, _c_vpp, ctypes.c_int64, ctypes.c_int64,
                                               ctypes.c_void_p]),
    "usp_plan_create_hybrid": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int64, ctypes.c_int64,
                                              ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                              ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]),
    "usp_plan_query_hybrid": (ctypes.c_int, [ctypes.c_void_p, _c_i32p, _c_i32p]),
    "usp_ulysses_attention_lse": (ctypes.c_int, [ctypes.c_void_p, _c_vpp, _c_vpp, _c_vpp, _c_vpp, ctypes.c_void_p,
                                                 ctypes.c_float, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t,
                                                 ctypes.c_void_p]),
    "usp_plan_set_pack_mode": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32]),
    "usp_plan_set_attention_ctas": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32]),
    "usp_plan_set_attention_kernel": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32]),
    "usp_ulysses_attention_graph_create": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_void_p, _c_vpp,
                                                          _c_vpp, _c_vpp, _c_vpp, ctypes.c_float, ctypes.c_int32,
                                                          ctypes.c_void_p, ctypes.c_size_t]),
    "usp_graph_launch": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "usp_graph_destroy": (ctypes.c_int, [ctypes.c_void_p]),
    "usp_plan_destroy": (ctypes.c_int, [ctypes.c_void_p]),
    "usp_plan_query": (ctypes.c_int, [ctypes.c_void_p, _c_i64p, _c_i64p, _c_i32p, _c_i32p]),
    "usp_scatter_sequence": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, _c_vpp, ctypes.c_int64,
                                            ctypes.c_int64, ctypes.c_void_p]),
    "usp_gather_sequence": (ctypes.c_int, [ctypes.c_void_p, _c_vpp, ctypes.c_void_p, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_void_p]),
    "usp_sp_head_slice": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, _c_vpp, ctypes.c_int64,
                                         ctypes.c_void_p]),
    "usp_sp_head_gather": (ctypes.c_int, [ctypes.c_void_p, _c_vpp, ctypes.c_void_p, ctypes.c_int64,
                                          ctypes.c_void_p]),
    "usp_ulysses_seq_to_head": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, _c_vpp, _c_vpp, ctypes.c_void_p]),
    "usp_ulysses_head_to_seq": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, _c_vpp, _c_vpp, ctypes.c_void_p]),
    "usp_head_attention": (ctypes.c_int, [ctypes.c_void_p, _c_vpp, _c_vpp, _c_vpp, _c_vpp, ctypes.c_float,
                                          ctypes.c_void_p]),
    "usp_ulysses_attention_workspace_size": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32,
                                                            ctypes.POINTER(ctypes.c_size_t)]),
    "usp_ulysses_attention": (ctypes.c_int, [ctypes.c_void_p, _c_vpp, _c_vpp, _c_vpp, _c_vpp, ctypes.c_float,
                                             ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "usp_ulysses_attention_noalloc": (ctypes.c_int, [ctypes.c_void_p, _c_vpp, _c_vpp, _c_vpp, _c_vpp, ctypes.c_float,
                                                     ctypes.c_int32, ctypes.c_void_p]),
    "usp_plan_set_timing_events": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "usp_dist_exchange_counts": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                                ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                _c_i64p, _c_i64p, _c_i64p, _c_i64p]),
    "usp_dist_pack": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32, _c_vpp, ctypes.c_void_p, ctypes.c_void_p]),
    "usp_dist_unpack": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, _c_vpp, ctypes.c_void_p]),
    "usp_dist_workspace_size": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]),
    "usp_dist_attention": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                          ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "usp_kernel_launches": (ctypes.c_uint64, []),
    "usp_device_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32]),
    "usp_debug_wait_timeout": (ctypes.c_int, [ctypes.c_uint32, ctypes.c_void_p]),
}

EXPORTED = tuple(_SIGNATURES)


def library_path() -> str:
    """The in-tree libusp.so, or the build named by $USP_LIBRARY (a variant
    built with extra flags, e.g. the pipeline-trace build)."""
    return os.environ.get("USP_LIBRARY") or os.path.join(_HERE, _LIB_NAME)


def _load():
    path = library_path()
    if not os.path.exists(path):
        raise OSError(f"{path} is missing: build it with `python -m ulysses_sequence_attention_sp_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


class UspError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"[usp error {code}] {message}")
        self.code = code


def _check(rc: int) -> None:
    if rc != USP_OK:
        raise UspError(rc, _lib.usp_last_error_message().decode())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptrs(tensors) -> ctypes.Array:
    return (ctypes.c_void_p * len(tensors))(*[t.data_ptr() for t in tensors])


def version() -> int:
    return _lib.usp_version()


# ------------------------------------------------------------- partition
def balanced_ranges(total: int, parts: int) -> tuple[tuple[int, int], ...]:
    n = max(int(parts), 1)
    starts, lengths = (ctypes.c_int64 * n)(), (ctypes.c_int64 * n)()
    _check(_lib.usp_balanced_ranges(total, parts, starts, lengths))
    return tuple((starts[i], starts[i] + lengths[i]) for i in range(parts))


def sp_seq_split(total: int, world_size: int) -> list[int]:
    n = max(int(world_size), 1)
    counts = (ctypes.c_int64 * n)()
    _check(_lib.usp_seq_split(total, world_size, counts))
    return [counts[i] for i in range(world_size)]


def head_chunk_ranges(group_heads: int, num_chunks: int) -> list[tuple[int, int]]:
    cap = max(int(group_heads), 1)
    n = ctypes.c_int32()
    lo, hi = (ctypes.c_int32 * cap)(), (ctypes.c_int32 * cap)()
    _check(_lib.usp_head_chunk_ranges(group_heads, num_chunks, ctypes.byref(n), lo, hi))
    return [(lo[i], hi[i]) for i in range(n.value)]


# ------------------------------------------------------------------ plan
class Plan:
    """Token and head ownership of `world` virtual ranks on the current device.

    `kv_heads` (default: `heads`) gives k/v fewer heads than q (grouped-query
    attention); query head h then uses kv head h // (heads // kv_heads).
    `ring_size` > 1 makes a Ulysses + Ring hybrid: the `world` ranks form
    ring_size Ulysses groups of world // ring_size consecutive ranks; heads are
    split inside a group and k/v blocks travel around the ring of ranks that
    hold the same heads."""

    def __init__(self, batch: int, seq_len: int, heads: int, head_dim: int, world: int,
                 dtype="bf16", prefix: int = 0, kv_heads: int | None = None, ring_size: int = 1):
        code = _NAMES[dtype] if isinstance(dtype, str) else _DTYPES.get(dtype, dtype)
        handle = ctypes.c_void_p()
        kv_heads = heads if kv_heads is None else kv_heads
        if ring_size < 1 or world % ring_size != 0:
            raise UspError(USP_ERR_INVALID_ARG, f"ring_size {ring_size} must divide world {world}")
        _check(_lib.usp_plan_create_hybrid(ctypes.byref(handle), batch, seq_len, heads, kv_heads, head_dim,
                                           world // ring_size, ring_size, code, prefix))
        self._h = handle
        self.kv_heads = kv_heads
        self.ulysses_size = world // ring_size
        self.ring_size = ring_size
        self.pack_mode = "tma"
        self.batch, self.seq_len, self.heads, self.head_dim = batch, seq_len, heads, head_dim
        self.world, self.dtype_code, self.prefix = world, code, prefix
        self.torch_dtype = _TORCH[code]
        ts, tl = (ctypes.c_int64 * world)(), (ctypes.c_int64 * world)()
        hs, hl = (ctypes.c_int32 * world)(), (ctypes.c_int32 * world)()
        _check(_lib.usp_plan_query(self._h, ts, tl, hs, hl))
        self.token_ranges = tuple((ts[i], ts[i] + tl[i]) for i in range(world))
        self.head_ranges = tuple((hs[i], hs[i] + hl[i]) for i in range(world))
        ks, kl = (ctypes.c_int32 * world)(), (ctypes.c_int32 * world)()
        _check(_lib.usp_plan_query_kv(self._h, None, ks, kl))
        self.kv_head_ranges = tuple((ks[i], ks[i] + kl[i]) for i in range(world))

    @property
    def handle(self):
        if self._h is None:
            raise UspError(USP_ERR_INVALID_ARG, "plan is closed")
        return self._h

    @property
    def tokens(self) -> int:
        return self.prefix + self.seq_len

    def full_shape(self):
        return (self.batch, self.tokens, self.heads, self.head_dim)

    def seq_shard_shape(self, r: int):
        t0, t1 = self.token_ranges[r]
        return (self.batch, self.prefix + t1 - t0, self.heads, self.head_dim)

    def head_shard_shape(self, r: int):
        h0, h1 = self.head_ranges[r]
        return (self.batch, self.tokens, h1 - h0, self.head_dim)

    def kv_full_shape(self):
        return (self.batch, self.tokens, self.kv_heads, self.head_dim)

    def kv_seq_shard_shape(self, r: int):
        t0, t1 = self.token_ranges[r]
        return (self.batch, self.prefix + t1 - t0, self.kv_heads, self.head_dim)

    def kv_head_shard_shape(self, r: int):
        k0, k1 = self.kv_head_ranges[r]
        return (self.batch, self.tokens, k1 - k0, self.head_dim)

    def empty_kv_seq_shards(self, dtype=None, fill=None):
        return [self._empty(self.kv_seq_shard_shape(r), dtype, fill) for r in range(self.world)]

    def empty_seq_shards(self, dtype=None, fill=None):
        return [self._empty(self.seq_shard_shape(r), dtype, fill) for r in range(self.world)]

    def empty_head_shards(self, dtype=None, fill=None):
        return [self._empty(self.head_shard_shape(r), dtype, fill) for r in range(self.world)]

    def _empty(self, shape, dtype, fill):
        t = torch.empty(shape, dtype=dtype or self.torch_dtype, device="cuda")
        if fill is not None:
            t.fill_(fill)
        return t

    def set_pack_mode(self, mode: str) -> None:
        """'tma' (default) or 'vector': how sequence -> head moves run (same bytes)."""
        codes = {"vector": 0, "tma": 1}
        if mode not in codes:
            raise UspError(USP_ERR_INVALID_ARG, f"pack mode must be one of {sorted(codes)}")
        _check(_lib.usp_plan_set_pack_mode(self.handle, codes[mode]))
        self.pack_mode = mode

    def set_attention_ctas(self, max_ctas: int) -> None:
        """Caps the tensor-core attention kernel's CTAs (0: automatic); with
        fewer CTAs than (query tile, batch, head) items each CTA walks several."""
        _check(_lib.usp_plan_set_attention_ctas(self.handle, int(max_ctas)))
        self.attention_ctas = int(max_ctas)

    def set_attention_kernel(self, kernel: str) -> None:
        """'auto' (default), 'one_tile', 'two_tile' or 'two_cta': which
        tensor-core attention kernel runs (same function; see include/usp.h)."""
        codes = {"auto": 0, "one_tile": 1, "two_tile": 2, "two_cta": 3}
        if kernel not in codes:
            raise UspError(USP_ERR_INVALID_ARG, f"attention kernel must be one of {sorted(codes)}")
        _check(_lib.usp_plan_set_attention_kernel(self.handle, codes[kernel]))
        self.attention_kernel = kernel

    def workspace_bytes(self, num_chunks: int = 1) -> int:
        n = ctypes.c_size_t()
        _check(_lib.usp_ulysses_attention_workspace_size(self.handle, num_chunks, ctypes.byref(n)))
        return n.value

    def set_timing_events(self, start=None, stop=None) -> None:
        """Profiling hook: record torch.cuda.Event `start`/`stop` around the
        attention kernels of each ulysses_attention call (None, None: off)."""
        if start is None:
            _check(_lib.usp_plan_set_timing_events(self.handle, None, None))
            return
        _check(_lib.usp_plan_set_timing_events(self.handle, ctypes.c_void_p(start.cuda_event),
                                               ctypes.c_void_p(stop.cuda_event)))

    def close(self) -> None:
        if getattr(self, "_h", None) is not None:
            _lib.usp_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def _check_tensors(plan: Plan, tensors, shapes, what: str) -> None:
    if len(tensors) != len(shapes):
        raise UspError(USP_ERR_INVALID_ARG, f"{what}: expected {len(shapes)} tensors, got {len(tensors)}")
    elem = torch.empty((), dtype=plan.torch_dtype).element_size()
    for i, (t, shape) in enumerate(zip(tensors, shapes)):
        if not t.is_cuda or not t.is_contiguous():
            raise UspError(USP_ERR_INVALID_ARG, f"{what}[{i}] must be a contiguous CUDA tensor")
        if t.element_size() != elem:
            raise UspError(USP_ERR_DTYPE, f"{what}[{i}] has {t.element_size()}-byte elements, plan has {elem}")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise UspError(USP_ERR_SHAPE, f"{what}[{i}] has shape {tuple(t.shape)}, expected {tuple(shape)}")


# --------------------------------------------------------- layout operations
def _shard_shapes(plan: Plan, row_shape):
    return [(plan.batch, plan.prefix + t1 - t0, *row_shape) for t0, t1 in plan.token_ranges]


def scatter_sequence(plan: Plan, x_full, out=None, stream=None):
    """API page, scatter_sequence: per-rank token windows of a replicated tensor
    [B, T', ...] (any row shape: q with H heads, k/v with Hkv heads, a hidden state)."""
    row = tuple(x_full.shape[2:])
    shapes = _shard_shapes(plan, row)
    out = out if out is not None else [torch.empty(sh, dtype=x_full.dtype, device=x_full.device) for sh in shapes]
    _check_tensors(plan, [x_full], [(plan.batch, plan.tokens, *row)], "x_full")
    _check_tensors(plan, out, shapes, "x_shards")
    row_bytes = x_full[0, 0].numel() * x_full.element_size()
    _check(_lib.usp_scatter_sequence(plan.handle, x_full.data_ptr(), _ptrs(out), 0, row_bytes, _stream(stream)))
    return out


def gather_sequence(plan: Plan, shards, out=None, stream=None):
    """API page, gather_sequence: the full tensor from the shards, in rank order."""
    row = tuple(shards[0].shape[2:])
    if out is None:
        out = torch.empty((plan.batch, plan.tokens, *row), dtype=shards[0].dtype, device=shards[0].device)
    _check_tensors(plan, shards, _shard_shapes(plan, row), "x_shards")
    _check_tensors(plan, [out], [(plan.batch, plan.tokens, *row)], "x_full")
    row_bytes = shards[0][0, 0].numel() * shards[0].element_size()
    _check(_lib.usp_gather_sequence(plan.handle, _ptrs(shards), out.data_ptr(), 0, row_bytes, _stream(stream)))
    return out


def sp_head_slice(plan: Plan, x_full, out=None, stream=None):
    """API page, sp_head_slice: each rank's contiguous head group of [B, T', H, D]."""
    out = out if out is not None else [torch.empty(plan.head_shard_shape(r), dtype=x_full.dtype, device=x_full.device)
                                       for r in range(plan.world)]
    _check_tensors(plan, [x_full], [plan.full_shape()], "x_full")
    _check_tensors(plan, out, [plan.head_shard_shape(r) for r in range(plan.world)], "x_head_shards")
    _check(_lib.usp_sp_head_slice(plan.handle, x_full.data_ptr(), _ptrs(out), 0, _stream(stream)))
    return out


def sp_head_gather(plan: Plan, head_shards, out=None, stream=None):
    """API page, sp_head_gather: inverse of sp_head_slice."""
    out = out if out is not None else torch.empty(plan.full_shape(), dtype=head_shards[0].dtype,
                                                  device=head_shards[0].device)
    _check_tensors(plan, head_shards, [plan.head_shard_shape(r) for r in range(plan.world)], "x_head_shards")
    _check_tensors(plan, [out], [plan.full_shape()], "x_full")
    _check(_lib.usp_sp_head_gather(plan.handle, _ptrs(head_shards), out.data_ptr(), 0, _stream(stream)))
    return out


def ulysses_seq_to_head(plan: Plan, tensors, out=None, stream=None, kv: bool = False):
    """Ragged transport page, seq_to_heads: `tensors` is a list of 1..3 lists of
    per-rank sequence shards (q, k, v); returns the matching per-rank head shards.
    kv=True moves k/v tensors over the plan's kv head split (grouped-query attention)."""
    n = len(tensors)
    seq_shape = plan.kv_seq_shard_shape if kv else plan.seq_shard_shape
    head_shape = plan.kv_head_shard_shape if kv else plan.head_shard_shape
    if out is None:
        out = [[torch.empty(head_shape(r), dtype=tensors[0][0].dtype, device=tensors[0][0].device)
                for r in range(plan.world)] for _ in range(n)]
    flat_in = [t for group in tensors for t in group]
    flat_out = [t for group in out for t in group]
    _check_tensors(plan, flat_in, [seq_shape(r) for _ in range(n) for r in range(plan.world)], "in")
    _check_tensors(plan, flat_out, [head_shape(r) for _ in range(n) for r in range(plan.world)], "out")
    fn = _lib.usp_ulysses_seq_to_head_kv if kv else _lib.usp_ulysses_seq_to_head
    _check(fn(plan.handle, n, _ptrs(flat_in), _ptrs(flat_out), _stream(stream)))
    return out


def ulysses_head_to_seq(plan: Plan, tensors, out=None, stream=None):
    """Ragged transport page, heads_to_seq: per-rank head shards back to sequence shards."""
    n = len(tensors)
    if out is None:
        out = [[torch.empty(plan.seq_shard_shape(r), dtype=tensors[0][0].dtype, device=tensors[0][0].device)
                for r in range(plan.world)] for _ in range(n)]
    flat_in = [t for group in tensors for t in group]
    flat_out = [t for group in out for t in group]
    _check_tensors(plan, flat_in, [plan.head_shard_shape(r) for _ in range(n) for r in range(plan.world)], "in")
    _check_tensors(plan, flat_out, [plan.seq_shard_shape(r) for _ in range(n) for r in range(plan.world)], "out")
    _check(_lib.usp_ulysses_head_to_seq(plan.handle, n, _ptrs(flat_in), _ptrs(flat_out), _stream(stream)))
    return out


# ------------------------------------------------------- row collectives
def _row_shapes(plan: Plan, row_shape, full: bool):
    if full:
        return [(plan.batch, plan.seq_len, *row_shape)] * plan.world
    return [(plan.batch, t1 - t0, *row_shape) for t0, t1 in plan.token_ranges]


def all_gather_rows(plan: Plan, local_rows, out=None, stream=None):
    """Ragged transport page, all_gather_rows: rank r's rows [B, T_r, ...] ->
    every rank's full [B, T, ...] (T = the split tokens; no prefix rows)."""
    row = tuple(local_rows[0].shape[2:])
    if out is None:
        out = [torch.empty(sh, dtype=local_rows[0].dtype, device=local_rows[0].device)
               for sh in _row_shapes(plan, row, True)]
    _check_tensors(plan, local_rows, _row_shapes(plan, row, False), "local_rows")
    _check_tensors(plan, out, _row_shapes(plan, row, True), "full_rows")
    row_bytes = local_rows[0][0, 0].numel() * local_rows[0].element_size()
    _check(_lib.usp_all_gather_rows(plan.handle, _ptrs(local_rows), _ptrs(out), plan.batch, row_bytes,
                                    _stream(stream)))
    return out


def reduce_scatter_rows(plan: Plan, partial_full_rows, out=None, stream=None):
    """Ragged transport page, reduce_scatter_rows: every rank's partial
    [B, T, ...] -> rank r's [B, T_r, ...] sum over ranks (fp32 accumulation)."""
    row = tuple(partial_full_rows[0].shape[2:])
    for t in partial_full_rows:
        if t.dtype != plan.torch_dtype:
            raise UspError(USP_ERR_DTYPE, f"partials are {t.dtype}, the plan sums {plan.torch_dtype}")
    if out is None:
        out = [torch.empty(sh, dtype=partial_full_rows[0].dtype, device=partial_full_rows[0].device)
               for sh in _row_shapes(plan, row, False)]
    _check_tensors(plan, partial_full_rows, _row_shapes(plan, row, True), "partial_full_rows")
    _check_tensors(plan, out, _row_shapes(plan, row, False), "local_rows")
    row_bytes = partial_full_rows[0][0, 0].numel() * partial_full_rows[0].element_size()
    _check(_lib.usp_reduce_scatter_rows(plan.handle, _ptrs(partial_full_rows), _ptrs(out), plan.batch, row_bytes,
                                        _stream(stream)))
    return out


# ------------------------------------------------------------- attention
def head_attention(plan: Plan, q_heads, k_heads, v_heads, out=None, scale: float = 0.0, stream=None):
    """run_attention on every rank's head shard (non-causal softmax attention)."""
    shapes = [plan.head_shard_shape(r) for r in range(plan.world)]
    kv_shapes = [plan.kv_head_shard_shape(r) for r in range(plan.world)]
    out = out if out is not None else [torch.empty(s, dtype=plan.torch_dtype, device="cuda") for s in shapes]
    for name, ts, sh in (("q_heads", q_heads, shapes), ("k_heads", k_heads, kv_shapes),
                         ("v_heads", v_heads, kv_shapes), ("o_heads", out, shapes)):
        _check_tensors(plan, ts, sh, name)
    _check(_lib.usp_head_attention(plan.handle, _ptrs(q_heads), _ptrs(k_heads), _ptrs(v_heads), _ptrs(out),
                                   float(scale), _stream(stream)))
    return out


def ulysses_attention(plan: Plan, q, k, v, out=None, scale: float = 0.0, num_chunks: int = 1,
                      workspace=None, stream=None, lse=None):
    """API page, ulysses_attention (with head-chunked passes): per-rank sequence
    shards of q, k, v in; per-rank sequence shards of the attention output out.
    A Ulysses + Ring plan runs the hybrid block. `lse` (a float32 CUDA tensor
    [H, B, T']) also receives every row's log-sum-exp."""
    shapes = [plan.seq_shard_shape(r) for r in range(plan.world)]
    kv_shapes = [plan.kv_seq_shard_shape(r) for r in range(plan.world)]
    out = out if out is not None else [torch.empty(s, dtype=plan.torch_dtype, device="cuda") for s in shapes]
    for name, ts, sh in (("q", q, shapes), ("k", k, kv_shapes), ("v", v, kv_shapes), ("out", out, shapes)):
        _check_tensors(plan, ts, sh, name)
    need = plan.workspace_bytes(num_chunks)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    if workspace.numel() * workspace.element_size() < need:
        raise UspError(USP_ERR_SHAPE, f"workspace needs {need} bytes")
    nbytes = workspace.numel() * workspace.element_size()
    if lse is None:
        _check(_lib.usp_ulysses_attention(plan.handle, _ptrs(q), _ptrs(k), _ptrs(v), _ptrs(out), float(scale),
                                          num_chunks, workspace.data_ptr(), nbytes, _stream(stream)))
        return out
    if (not lse.is_cuda or lse.dtype != torch.float32 or not lse.is_contiguous()
            or tuple(lse.shape) != (plan.heads, plan.batch, plan.tokens)):
        raise UspError(USP_ERR_SHAPE, f"lse must be a contiguous float32 CUDA tensor of shape "
                                      f"{(plan.heads, plan.batch, plan.tokens)}")
    _check(_lib.usp_ulysses_attention_lse(plan.handle, _ptrs(q), _ptrs(k), _ptrs(v), _ptrs(out), lse.data_ptr(),
                                          float(scale), num_chunks, workspace.data_ptr(), nbytes, _stream(stream)))
    return out


class AttentionGraph:
    """One ulysses_attention call captured into a CUDA graph owned by the
    library; launch() replays it (one launch per block). The tensors' addresses
    are fixed in the graph: refresh the inputs by writing into the same q/k/v
    shards. Keeps references to every tensor it uses."""

    def __init__(self, plan: Plan, q, k, v, out=None, scale: float = 0.0, num_chunks: int = 1, workspace=None):
        shapes = [plan.seq_shard_shape(r) for r in range(plan.world)]
        kv_shapes = [plan.kv_seq_shard_shape(r) for r in range(plan.world)]
        out = out if out is not None else [torch.empty(s, dtype=plan.torch_dtype, device="cuda") for s in shapes]
        for name, ts, sh in (("q", q, shapes), ("k", k, kv_shapes), ("v", v, kv_shapes), ("out", out, shapes)):
            _check_tensors(plan, ts, sh, name)
        need = plan.workspace_bytes(num_chunks)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
        if workspace.numel() * workspace.element_size() < need:
            raise UspError(USP_ERR_SHAPE, f"workspace needs {need} bytes")
        handle = ctypes.c_void_p()
        _check(_lib.usp_ulysses_attention_graph_create(ctypes.byref(handle), plan.handle, _ptrs(q), _ptrs(k), _ptrs(v),
                                                       _ptrs(out), float(scale), num_chunks, workspace.data_ptr(),
                                                       workspace.numel() * workspace.element_size()))
        self._h = handle
        self._keep = (plan, list(q), list(k), list(v), workspace)
        self.out = out

    def launch(self, stream=None):
        _check(_lib.usp_graph_launch(self._h, _stream(stream)))
        return self.out

    def close(self) -> None:
        if self._h:
            _lib.usp_graph_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def ulysses_attention_noalloc(plan: Plan, q, k, v, out=None, scale: float = 0.0, num_chunks: int = 1,
                              stream=None):
    """ulysses_attention for callers that cannot allocate device memory: the
    scratch is a fixed array inside the library (NOALLOC_SCRATCH_BYTES, shared by
    all calls; calls that overlap on the GPU race). `out` must be given by such
    a caller; when it is None this helper allocates it with torch for convenience."""
    shapes = [plan.seq_shard_shape(r) for r in range(plan.world)]
    kv_shapes = [plan.kv_seq_shard_shape(r) for r in range(plan.world)]
    out = out if out is not None else [torch.empty(s, dtype=plan.torch_dtype, device="cuda") for s in shapes]
    for name, ts, sh in (("q", q, shapes), ("k", k, kv_shapes), ("v", v, kv_shapes), ("out", out, shapes)):
        _check_tensors(plan, ts, sh, name)
    _check(_lib.usp_ulysses_attention_noalloc(plan.handle, _ptrs(q), _ptrs(k), _ptrs(v), _ptrs(out), float(scale),
                                              num_chunks, _stream(stream)))
    return out


# ------------------------------------------- rank-local (multi-process) steps
# One process per GPU and per sequence-parallel rank: the library packs,
# unpacks and computes; the exchange itself is the caller's collective (the
# `dist` module runs it over torch.distributed). Wire format: include/usp.h.
DIST_SEQ_TO_HEAD, DIST_HEAD_TO_SEQ, DIST_GATHER_SEQ, DIST_GATHER_HEADS = 0, 1, 2, 3


def dist_exchange_counts(batch: int, seq_len: int, heads: int, head_dim: int, world: int, rank: int, exchange: int,
                         ntensors: int = 1, num_chunks: int = 1, chunk: int = 0, prefix: int = 0,
                         kv_heads: int | None = None):
    """Transport page, seq_to_heads' split lists for one exchange of `rank`, in
    elements: (send_counts, send_displs, recv_counts, recv_displs). Needs no
    device."""
    arrs = [(ctypes.c_int64 * max(int(world), 1))() for _ in range(4)]
    _check(_lib.usp_dist_exchange_counts(batch, seq_len, heads, heads if kv_heads is None else kv_heads, head_dim,
                                         world, prefix, rank, exchange, ntensors, num_chunks, chunk, *arrs))
    return tuple([a[i] for i in range(world)] for a in arrs)


def dist_counts(plan: Plan, rank: int, exchange: int, ntensors: int = 1, num_chunks: int = 1, chunk: int = 0):
    """dist_exchange_counts for a plan's sizes."""
    return dist_exchange_counts(plan.batch, plan.seq_len, plan.heads, plan.head_dim, plan.world, rank, exchange,
                                ntensors, num_chunks, chunk, plan.prefix, plan.kv_heads)


def _flat_buffer(t, plan: Plan, what: str):
    if not t.is_cuda or not t.is_contiguous():
        raise UspError(USP_ERR_INVALID_ARG, f"{what} must be a contiguous CUDA tensor")
    return t.data_ptr()


def dist_pack(plan: Plan, rank: int, exchange: int, tensors, send, num_chunks: int = 1, chunk: int = 0,
              stream=None):
    """Fills the flat `send` buffer of one exchange from this rank's tensors
    (sequence shards of q[, k, v], or its head shard o)."""
    n = len(tensors)
    _check_tensors(plan, list(tensors), [None] * n, "in")
    _check(_lib.usp_dist_pack(plan.handle, rank, exchange, n, num_chunks, chunk, _ptrs(tensors),
                              _flat_buffer(send, plan, "send"), _stream(stream)))
    return send


def dist_unpack(plan: Plan, rank: int, exchange: int, recv, out, num_chunks: int = 1, chunk: int = 0,
                stream=None):
    """Reads the flat `recv` buffer of one exchange into this rank's tensors
    (head shards of q[, k, v], or its sequence shard)."""
    n = len(out)
    _check_tensors(plan, list(out), [None] * n, "out")
    _check(_lib.usp_dist_unpack(plan.handle, rank, exchange, n, num_chunks, chunk, _flat_buffer(recv, plan, "recv"),
                                _ptrs(out), _stream(stream)))
    return out


def dist_workspace_bytes(plan: Plan, rank: int) -> int:
    n = ctypes.c_size_t()
    _check(_lib.usp_dist_workspace_size(plan.handle, rank, ctypes.byref(n)))
    return n.value


def dist_attention(plan: Plan, rank: int, exchange: int, recv, send_o, workspace, num_chunks: int = 1,
                   chunk: int = 0, scale: float = 0.0, stream=None):
    """Attention of one head chunk on this rank: received q/k/v (`exchange`
    SEQ_TO_HEAD or GATHER_SEQ) in, the output written into `send_o` in the
    layout of the way back (HEAD_TO_SEQ or GATHER_HEADS)."""
    _check(_lib.usp_dist_attention(plan.handle, rank, exchange, num_chunks, chunk, _flat_buffer(recv, plan, "recv"),
                                   _flat_buffer(send_o, plan, "send_o"), float(scale),
                                   _flat_buffer(workspace, plan, "workspace"),
                                   workspace.numel() * workspace.element_size(), _stream(stream)))
    return send_o


def kernel_launches() -> int:
    """Kernels this library has launched in this process."""
    return int(_lib.usp_kernel_launches())


def device_status(reset: bool = True) -> int:
    """Synchronises the device and returns the library's device-side error word:
    0, a wait's site (a wait ran out) or, in a bounds-checking build, the site
    of a skipped out-of-range access."""
    code = ctypes.c_uint32()
    rc = _lib.usp_device_status(ctypes.byref(code), 1 if reset else 0)
    if rc not in (USP_OK, USP_ERR_TIMEOUT, USP_ERR_BOUNDS):
        _check(rc)
    return code.value


def debug_wait_timeout(limit_us: int, stream=None) -> None:
    _check(_lib.usp_debug_wait_timeout(limit_us, _stream(stream)))

"""Python binding of the paged KV-cache library for B200 (sm_100a).

Argument marshalling only: every operation runs in the CUDA kernels of
``lib/libpa_b200.so`` (or, for the pools, its C++ host code) through its C ABI
(``include/pa.h``); functions keep the C names. PyTorch supplies device memory
and streams. There is no CPU or library fallback: if the shared library is
missing, the first call raises.

Calls: slot write (pa_reshape_and_cache), decode (pa_decode; and
pa_decode_withhold_stage, which tests its bounded waits), the slot write
of each sequence's newest token with decode in one launch (pa_decode_append),
split-K decode and reduce (pa_decode_splitk, pa_splitk_reduce,
pa_decode_splitk_static),
copy-on-write block copy (pa_copy_blocks, pa_copy_blocks_counted), paged
prefill (pa_prefill), the int8 cache (pa_*_q8), the host block pool and
prefix cache (BlockPool, PrefixCache), and the device pool with its beam step
(DevicePool, pa_beam_step).

Layouts (contiguous): k_cache/v_cache [num_blocks, num_kv_heads, block_size,
head_dim]; query/out [num_seqs, num_heads, head_dim]; key/value
[num_tokens, num_kv_heads, head_dim]; block_tables [num_seqs,
max_blocks_per_seq] int32; context_lens [num_seqs] int32; slot_mapping
[num_tokens] int32; src_dst_pairs [n, 2] int64; int8 caches add
k_scale/v_scale [num_blocks, num_kv_heads, block_size] float32.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libpa_b200.so")

PA_F32, PA_F16, PA_BF16 = 0, 1, 2
_DT = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}

PA_DEVERR_BLOCK_ID = 0x1
PA_DEVERR_SLOT = 0x2
PA_DEVERR_CONTEXT = 0x4
PA_DEVERR_TIMEOUT = 0x8
PA_DEVERR_PAIR = 0x10
PA_DEVERR_POOL = 0x20
PA_DPOOL_HEADER_WORDS = 8
PA_DPOOL_TAIL_WORDS = 1024

PA_POOL_LIFO, PA_POOL_FIFO = 0, 1

EXPORTED = (
    "pa_status_string", "pa_read_device_errors", "pa_reshape_and_cache", "pa_decode",
    "pa_splitk_workspace_bytes", "pa_splitk_acc_offset", "pa_decode_splitk", "pa_splitk_reduce",
    "pa_choose_partition", "pa_copy_blocks", "pa_pool_create", "pa_pool_destroy", "pa_pool_num_free",
    "pa_pool_ref_count", "pa_pool_allocate", "pa_pool_share", "pa_pool_free", "pa_pool_append",
    "pa_pool_fork", "pa_pool_release", "pa_decode_splitk_static", "pa_prefill",
    "pa_prefix_cache_create", "pa_prefix_cache_destroy", "pa_prefix_num_entries", "pa_prefix_get_or_create",
    "pa_prefix_release", "pa_prefix_ref_count", "pa_copy_blocks_counted", "pa_dpool_state_bytes", "pa_dpool_init",
    "pa_beam_step", "pa_pool_export", "pa_dpool_load", "pa_reshape_and_cache_q8", "pa_decode_q8",
    "pa_decode_splitk_q8", "pa_copy_blocks_q8", "pa_decode_append", "pa_decode_withhold_stage",
    "pa_prefill_withhold_tile", "pa_beam_step_withhold_arrival",
)

PA_STATIC_SCRATCH_BYTES = 32 * 1024 * 1024


class PagedAttentionError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m paged_kv_cache_340_b200._build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    i32p = ctypes.POINTER(ctypes.c_int32)
    i64p = ctypes.POINTER(ctypes.c_int64)
    sig = {
        "pa_status_string": (ctypes.c_char_p, [i32]),
        "pa_read_device_errors": (i32, [ctypes.POINTER(ctypes.c_uint32), vp]),
        "pa_reshape_and_cache": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]),
        "pa_decode": (i32, [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, f32, i32, i32, i32, i32, vp, vp]),
        "pa_decode_append": (i32, [vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, f32, i32, i32, i32, i32,
                                   vp, vp]),
        "pa_decode_withhold_stage": (i32, [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, f32, i32, i32, i32, i32,
                                           vp, i32, i32, i32, ctypes.c_ulonglong, vp]),
        "pa_splitk_workspace_bytes": (sz, [i32, i32, i32, i32, i32]),
        "pa_splitk_acc_offset": (sz, [i32, i32, i32, i32]),
        "pa_decode_splitk": (i32, [vp, sz, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, f32, i32, i32, i32, i32,
                                   i32, vp, vp]),
        "pa_splitk_reduce": (i32, [vp, vp, sz, vp, i32, i32, i32, i32, i32, i32, vp]),
        "pa_choose_partition": (i32, [i32, i32, i32, i32, i32, i32]),
        "pa_copy_blocks": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]),
        "pa_pool_create": (vp, [i32, i32, i32, i32p]),
        "pa_pool_destroy": (None, [vp]),
        "pa_pool_num_free": (i32, [vp]),
        "pa_pool_ref_count": (i32, [vp, i32]),
        "pa_pool_allocate": (i32, [vp, i32p]),
        "pa_pool_share": (i32, [vp, i32]),
        "pa_pool_free": (i32, [vp, i32]),
        "pa_pool_append": (i32, [vp, i32p, i32, i32p, i32, i32p, i64p, i32, ctypes.POINTER(ctypes.c_int)]),
        "pa_pool_fork": (i32, [vp, i32p, i32, i32p, i32]),
        "pa_pool_release": (i32, [vp, i32p, i32]),
        "pa_decode_splitk_static": (i32, [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, f32, i32, i32, i32, i32,
                                          i32, i32, vp]),
        "pa_prefill_withhold_tile": (i32, [vp, vp, vp, i32, i32, vp, vp, vp, i32, vp, i32, i32, i32, i32, f32, i32, i32,
                                           i32, i32, i32, i32, i32, i32, ctypes.c_ulonglong, vp]),
        "pa_prefill": (i32, [vp, vp, vp, i32, i32, vp, vp, vp, i32, vp, i32, i32, i32, i32, f32, i32, i32, i32, i32,
                             vp]),
        "pa_prefix_cache_create": (vp, [vp, i32]),
        "pa_prefix_cache_destroy": (None, [vp]),
        "pa_prefix_num_entries": (i32, [vp]),
        "pa_prefix_get_or_create": (i32, [vp, i32p, i32, i32p, i32, ctypes.POINTER(ctypes.c_int),
                                          ctypes.POINTER(ctypes.c_int)]),
        "pa_prefix_release": (i32, [vp, i32p, i32]),
        "pa_prefix_ref_count": (i32, [vp, i32p, i32]),
        "pa_copy_blocks_counted": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]),
        "pa_dpool_state_bytes": (sz, [i32]),
        "pa_dpool_init": (i32, [vp, i32, i32, i32, vp, vp]),
        "pa_beam_step": (i32, [vp, i32, i32, vp, vp, i32, vp, i32, vp, vp, i32, vp, vp, vp, vp]),
        "pa_beam_step_withhold_arrival": (i32, [vp, i32, i32, vp, vp, i32, vp, i32, vp, vp, i32, vp, vp, vp, i32,
                                                ctypes.c_ulonglong, vp]),
        "pa_pool_export": (i32, [vp, i32p, i32p, ctypes.POINTER(ctypes.c_int)]),
        "pa_dpool_load": (i32, [vp, i32, i32, i32, vp, vp, i32, vp]),
        "pa_reshape_and_cache_q8": (i32, [vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]),
        "pa_decode_q8": (i32, [vp, vp, i32, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, f32, i32, i32, i32, vp,
                               vp]),
        "pa_decode_splitk_q8": (i32, [vp, sz, vp, i32, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, f32, i32, i32,
                                      i32, i32, vp, vp]),
        "pa_copy_blocks_q8": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


class _Library:
    """The shared library, loaded on first use (so that ``_build`` can be
    imported, and run, before the library exists). Any call without the built
    library raises ImportError: there is no fallback."""
    _cdll = None

    def __getattr__(self, name):
        if _Library._cdll is None:
            _Library._cdll = _load()
        return getattr(_Library._cdll, name)


_lib = _Library()


def status_string(status: int) -> str:
    return _lib.pa_status_string(int(status)).decode()


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise PagedAttentionError(what, rc)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return _DT[t.dtype]


# ------------------------------------------------------------------ device

def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None) -> None:
    NB, Hkv, bs, D = k_cache.shape
    rc = _lib.pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping),
                                   slot_mapping.shape[0], NB, Hkv, D, bs, _dtype(k_cache), _stream(stream))
    _check(rc, "pa_reshape_and_cache")


def pa_decode(out, query, k_cache, v_cache, block_tables, context_lens, scale, seq_order=None,
              stream=None) -> None:
    S, Hq, D = query.shape
    NB, Hkv, bs, _ = k_cache.shape
    rc = _lib.pa_decode(_ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                        block_tables.shape[1], _ptr(context_lens), S, Hq, Hkv, D, float(scale), bs, NB,
                        _dtype(k_cache), _dtype(out), _ptr(seq_order), _stream(stream))
    _check(rc, "pa_decode")


def pa_decode_withhold_stage(out, query, k_cache, v_cache, block_tables, context_lens, scale, seq, kv_head, stage,
                             wait_limit_ns, seq_order=None, stream=None) -> None:
    """pa_decode with the copy of one 16-token stage of one (sequence, kv
    head) withheld, so that its bounded wait runs out (a test of the timeout
    path; that head group's output is undefined)."""
    S, Hq, D = query.shape
    NB, Hkv, bs, _ = k_cache.shape
    rc = _lib.pa_decode_withhold_stage(_ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                       block_tables.shape[1], _ptr(context_lens), S, Hq, Hkv, D, float(scale), bs, NB,
                                       _dtype(k_cache), _dtype(out), _ptr(seq_order), int(seq), int(kv_head),
                                       int(stage), int(wait_limit_ns), _stream(stream))
    _check(rc, "pa_decode_withhold_stage")


def pa_decode_append(out, query, new_key, new_value, k_cache, v_cache, block_tables, context_lens, scale,
                     seq_order=None, stream=None) -> None:
    """Writes new_key / new_value [S, Hkv, D] as token context_lens[s] - 1 of
    each sequence (into the slot its table gives), then decodes: one launch."""
    S, Hq, D = query.shape
    NB, Hkv, bs, _ = k_cache.shape
    rc = _lib.pa_decode_append(_ptr(out), _ptr(query), _ptr(new_key), _ptr(new_value), _ptr(k_cache),
                               _ptr(v_cache), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S, Hq,
                               Hkv, D, float(scale), bs, NB, _dtype(k_cache), _dtype(out), _ptr(seq_order),
                               _stream(stream))
    _check(rc, "pa_decode_append")


def pa_splitk_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len, partition_size) -> int:
    return int(_lib.pa_splitk_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len, partition_size))


def pa_splitk_acc_offset(num_seqs, num_heads, max_context_len, partition_size) -> int:
    return int(_lib.pa_splitk_acc_offset(num_seqs, num_heads, max_context_len, partition_size))


def pa_decode_splitk(workspace, query, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
                     partition_size, seq_order=None, stream=None) -> None:
    S, Hq, D = query.shape
    NB, Hkv, bs, _ = k_cache.shape
    rc = _lib.pa_decode_splitk(_ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(query),
                               _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1],
                               _ptr(context_lens), S, Hq, Hkv, D, float(scale), bs, NB, int(max_context_len),
                               int(partition_size), _dtype(k_cache), _ptr(seq_order), _stream(stream))
    _check(rc, "pa_decode_splitk")


# ------------------------------------------------------------ int8 caches
# k_cache/v_cache int8 [NB, Hkv, bs, D]; k_scale/v_scale float32 [NB, Hkv, bs].

def pa_reshape_and_cache_q8(key, value, k_cache, v_cache, k_scale, v_scale, slot_mapping, stream=None) -> None:
    NB, Hkv, bs, D = k_cache.shape
    assert k_cache.dtype == torch.int8 and k_scale.dtype == torch.float32
    rc = _lib.pa_reshape_and_cache_q8(_ptr(key), _ptr(value), _dtype(key), _ptr(k_cache), _ptr(v_cache),
                                      _ptr(k_scale), _ptr(v_scale), _ptr(slot_mapping), slot_mapping.shape[0], NB,
                                      Hkv, D, bs, _stream(stream))
    _check(rc, "pa_reshape_and_cache_q8")


def pa_decode_q8(out, query, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale, seq_order=None,
                 stream=None) -> None:
    S, Hq, D = query.shape
    NB, Hkv, bs, _ = k_cache.shape
    assert k_cache.dtype == torch.int8 and k_scale.dtype == torch.float32
    rc = _lib.pa_decode_q8(_ptr(out), _ptr(query), _dtype(query), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale),
                           _ptr(v_scale), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S, Hq, Hkv,
                           D, float(scale), bs, NB, _dtype(out), _ptr(seq_order), _stream(stream))
    _check(rc, "pa_decode_q8")


def pa_decode_splitk_q8(workspace, query, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale,
                        max_context_len, partition_size, seq_order=None, stream=None) -> None:
    S, Hq, D = query.shape
    NB, Hkv, bs, _ = k_cache.shape
    assert k_cache.dtype == torch.int8 and k_scale.dtype == torch.float32
    rc = _lib.pa_decode_splitk_q8(_ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(query),
                                  _dtype(query), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
                                  _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S, Hq, Hkv, D,
                                  float(scale), bs, NB, int(max_context_len), int(partition_size), _ptr(seq_order),
                                  _stream(stream))
    _check(rc, "pa_decode_splitk_q8")


def pa_copy_blocks_q8(k_cache, v_cache, k_scale, v_scale, src_dst_pairs, stream=None) -> None:
    NB, Hkv, bs, D = k_cache.shape
    n = src_dst_pairs.shape[0] if src_dst_pairs is not None else 0
    rc = _lib.pa_copy_blocks_q8(_ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
                                _ptr(src_dst_pairs) if n else None, n, NB, Hkv, D, bs, _stream(stream))
    _check(rc, "pa_copy_blocks_q8")


def pa_splitk_reduce(out, workspace, context_lens, max_context_len, partition_size, stream=None) -> None:
    S, Hq, D = out.shape
    rc = _lib.pa_splitk_reduce(_ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _ptr(context_lens), S, Hq, D, int(max_context_len), int(partition_size),
                               _dtype(out), _stream(stream))
    _check(rc, "pa_splitk_reduce")


def pa_decode_splitk_static(out, query, k_cache, v_cache, block_tables, context_lens, scale, max_context_len,
                            partition_size, stream=None) -> None:
    """Split-K decode plus reduce with the library's fixed scratch array
    instead of a caller workspace (for callers that cannot allocate; calls on
    one device must not overlap)."""
    S, Hq, D = query.shape
    NB, Hkv, bs, _ = k_cache.shape
    rc = _lib.pa_decode_splitk_static(_ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                      block_tables.shape[1], _ptr(context_lens), S, Hq, Hkv, D, float(scale), bs,
                                      NB, int(max_context_len), int(partition_size), _dtype(k_cache), _dtype(out),
                                      _stream(stream))
    _check(rc, "pa_decode_splitk_static")


def pa_prefill(out, query, q_start, max_q_len, k_cache, v_cache, block_tables, context_lens, scale,
               stream=None) -> None:
    """Causal attention of each sequence's new query tokens (rows q_start[s] ..
    q_start[s+1]-1 of query [T, Hq, D]) over its paged cache."""
    T, Hq, D = query.shape
    NB, Hkv, bs, _ = k_cache.shape
    S = context_lens.shape[0]
    rc = _lib.pa_prefill(_ptr(out), _ptr(query), _ptr(q_start), T, int(max_q_len), _ptr(k_cache), _ptr(v_cache),
                         _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S, Hq, Hkv, D, float(scale),
                         bs, NB, _dtype(k_cache), _dtype(out), _stream(stream))
    _check(rc, "pa_prefill")


def pa_prefill_withhold_tile(out, query, q_start, max_q_len, k_cache, v_cache, block_tables, context_lens, scale,
                             seq, kv_head, query_tile, tile, wait_limit_ns, stream=None) -> None:
    """pa_prefill with the copy of one 64-token K tile of one (sequence, kv
    head, query tile) withheld, so that its bounded wait runs out (a test of
    the timeout path; that CTA's output rows are undefined)."""
    T, Hq, D = query.shape
    NB, Hkv, bs, _ = k_cache.shape
    S = context_lens.shape[0]
    rc = _lib.pa_prefill_withhold_tile(_ptr(out), _ptr(query), _ptr(q_start), T, int(max_q_len), _ptr(k_cache),
                                       _ptr(v_cache), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S,
                                       Hq, Hkv, D, float(scale), bs, NB, _dtype(k_cache), _dtype(out), int(seq),
                                       int(kv_head), int(query_tile), int(tile), int(wait_limit_ns), _stream(stream))
    _check(rc, "pa_prefill_withhold_tile")


def pa_choose_partition(num_seqs, num_kv_heads, max_context_len, block_size, head_dim, kv_dtype) -> int:
    return int(_lib.pa_choose_partition(num_seqs, num_kv_heads, max_context_len, block_size, head_dim,
                                        _DT[kv_dtype] if isinstance(kv_dtype, torch.dtype) else int(kv_dtype)))


def pa_copy_blocks(k_cache, v_cache, src_dst_pairs, stream=None) -> None:
    NB, Hkv, bs, D = k_cache.shape
    n = src_dst_pairs.shape[0] if src_dst_pairs is not None else 0
    rc = _lib.pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(src_dst_pairs) if n else None, n, NB, Hkv, D,
                             bs, _dtype(k_cache), _stream(stream))
    _check(rc, "pa_copy_blocks")


def pa_copy_blocks_counted(k_cache, v_cache, src_dst_pairs, num_pairs, stream=None) -> None:
    """pa_copy_blocks over the first num_pairs[0] (a device int32, read by the
    kernel) rows of src_dst_pairs [max_pairs, 2] int64."""
    NB, Hkv, bs, D = k_cache.shape
    m = src_dst_pairs.shape[0]
    rc = _lib.pa_copy_blocks_counted(_ptr(k_cache), _ptr(v_cache), _ptr(src_dst_pairs) if m else None,
                                     _ptr(num_pairs) if m else None, m, NB, Hkv, D, bs, _dtype(k_cache),
                                     _stream(stream))
    _check(rc, "pa_copy_blocks_counted")


class DevicePool:
    """Device block pool (pa_dpool_* calls): the state lives in a device int32
    tensor; ``ref`` and ``ring`` are views of its reference counts and free-list
    ring, ``header`` of [num_blocks, block_size, policy, head, count, marker]."""

    def __init__(self, num_blocks: int, block_size: int, policy: int = PA_POOL_LIFO, free_order=None,
                 device="cuda", stream=None, host_pool: "Optional[BlockPool]" = None):
        """A fresh pool (free list free_order, else 0..num_blocks-1), or, with
        host_pool, a copy of that host pool's counts and free list."""
        self.num_blocks, self.block_size, self.policy = num_blocks, block_size, policy
        nbytes = int(_lib.pa_dpool_state_bytes(num_blocks))
        if nbytes == 0:
            raise PagedAttentionError("pa_dpool_state_bytes", -3)
        self.state = torch.empty(nbytes // 4, dtype=torch.int32, device=device)
        if host_pool is not None:
            assert host_pool.num_blocks == num_blocks and host_pool.block_size == block_size
            ref, fl = host_pool.export()
            self._keep = (torch.from_numpy(ref).to(device), torch.from_numpy(fl).to(device))
            _check(_lib.pa_dpool_load(_ptr(self.state), num_blocks, block_size, policy, _ptr(self._keep[0]),
                                      _ptr(self._keep[1]) if fl.shape[0] else None, fl.shape[0], _stream(stream)),
                   "pa_dpool_load")
        else:
            fo = None
            if free_order is not None:
                fo = torch.as_tensor(np.asarray(free_order, dtype=np.int32)).to(device)
            _check(_lib.pa_dpool_init(_ptr(self.state), num_blocks, block_size, policy, _ptr(fo), _stream(stream)),
                   "pa_dpool_init")
            self._keep = fo
        h = PA_DPOOL_HEADER_WORDS
        self.header = self.state[:6]
        self.ref = self.state[h:h + num_blocks]
        self.ring = self.state[h + num_blocks:h + 2 * num_blocks]

    def free_list(self) -> list:
        """The free list, front first (synchronises)."""
        hdr = self.header.cpu().tolist()
        ring = self.ring.cpu().tolist()
        return [ring[(hdr[3] + k) % self.num_blocks] for k in range(hdr[4])]


def pa_beam_step(pool: DevicePool, old_tables, old_context_lens, parents, new_tables, new_context_lens,
                 slot_mapping, cow_pairs, num_cow, stream=None) -> None:
    """One beam-search step on the device: new beam i continues old beam
    parents[i] and writes one token (all tensors on the device; see pa.h)."""
    num_old = old_context_lens.shape[0]
    num_new = parents.shape[0]
    mb = new_tables.shape[1] if new_tables.dim() == 2 else old_tables.shape[1]
    rc = _lib.pa_beam_step(_ptr(pool.state), pool.num_blocks, pool.block_size,
                           _ptr(old_tables) if num_old else None, _ptr(old_context_lens) if num_old else None,
                           num_old, _ptr(parents) if num_new else None, num_new,
                           _ptr(new_tables) if num_new else None, _ptr(new_context_lens) if num_new else None, mb,
                           _ptr(slot_mapping) if num_new else None, _ptr(cow_pairs) if num_new else None,
                           _ptr(num_cow), _stream(stream))
    _check(rc, "pa_beam_step")


def pa_beam_step_withhold_arrival(pool: DevicePool, old_tables, old_context_lens, parents, new_tables,
                                  new_context_lens, slot_mapping, cow_pairs, num_cow, cta, wait_limit_ns,
                                  stream=None) -> None:
    """pa_beam_step with one CTA's arrival at the first grid barrier withheld,
    so that the barrier's bounded wait runs out (a test of the timeout path:
    the step applies nothing and the state is marked unusable)."""
    num_old = old_context_lens.shape[0]
    num_new = parents.shape[0]
    mb = new_tables.shape[1] if new_tables.dim() == 2 else old_tables.shape[1]
    rc = _lib.pa_beam_step_withhold_arrival(
        _ptr(pool.state), pool.num_blocks, pool.block_size, _ptr(old_tables) if num_old else None,
        _ptr(old_context_lens) if num_old else None, num_old, _ptr(parents) if num_new else None, num_new,
        _ptr(new_tables) if num_new else None, _ptr(new_context_lens) if num_new else None, mb,
        _ptr(slot_mapping) if num_new else None, _ptr(cow_pairs) if num_new else None, _ptr(num_cow), int(cta),
        int(wait_limit_ns), _stream(stream))
    _check(rc, "pa_beam_step_withhold_arrival")


def pa_read_device_errors(stream=None) -> int:
    flags = ctypes.c_uint32(0)
    _check(_lib.pa_read_device_errors(ctypes.byref(flags), _stream(stream)), "pa_read_device_errors")
    return int(flags.value)


def splitk_views(workspace: torch.Tensor, num_seqs, num_heads, head_dim, max_context_len, partition_size):
    """(ml, acc) float32 views of a split-K workspace, as laid out by pa_decode_splitk:
    ml [S, Hq, max_parts, 2], acc [S, Hq, max_parts, head_dim]."""
    mp = -(-max_context_len // partition_size)
    off = pa_splitk_acc_offset(num_seqs, num_heads, max_context_len, partition_size)
    flat = workspace.view(torch.uint8)
    ml = flat[: num_seqs * num_heads * mp * 8].view(torch.float32).view(num_seqs, num_heads, mp, 2)
    acc = flat[off: off + num_seqs * num_heads * mp * head_dim * 4].view(torch.float32)
    return ml, acc.view(num_seqs, num_heads, mp, head_dim)


# -------------------------------------------------------------- host pool

def _i32p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


class BlockPool:
    """Host block pool (pa_pool_* calls): free list, reference counts and the
    copy-on-write decision. Tables are numpy int32 rows owned by the caller."""

    def __init__(self, num_blocks: int, block_size: int, policy: int = PA_POOL_LIFO, free_order=None):
        self.block_size = block_size
        self.num_blocks = num_blocks
        order = None
        if free_order is not None:
            self._order = np.ascontiguousarray(np.asarray(free_order, dtype=np.int32))
            order = _i32p(self._order)
        h = _lib.pa_pool_create(num_blocks, block_size, policy, order)
        if not h:
            raise PagedAttentionError("pa_pool_create", -3)
        self._h = ctypes.c_void_p(h)
        self._destroy = _lib.pa_pool_destroy  # still callable at interpreter exit, when _lib may be gone

    def __del__(self):
        h, destroy = getattr(self, "_h", None), getattr(self, "_destroy", None)
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self._h = None

    def num_free(self) -> int:
        return int(_lib.pa_pool_num_free(self._h))

    def ref_count(self, block: int) -> int:
        rc = int(_lib.pa_pool_ref_count(self._h, int(block)))
        if rc < 0:
            raise PagedAttentionError("pa_pool_ref_count", rc)
        return rc

    def allocate(self) -> int:
        b = ctypes.c_int32(-1)
        _check(_lib.pa_pool_allocate(self._h, ctypes.byref(b)), "pa_pool_allocate")
        return int(b.value)

    def share(self, block: int) -> None:
        _check(_lib.pa_pool_share(self._h, int(block)), "pa_pool_share")

    def free(self, block: int) -> None:
        _check(_lib.pa_pool_free(self._h, int(block)), "pa_pool_free")

    def append(self, table: np.ndarray, num_tokens: int, n_new: int, want_slots: bool = True,
               cow_capacity: int = 64) -> Tuple[int, Optional[np.ndarray], np.ndarray]:
        """Appends n_new tokens to the sequence (table row, num_tokens).
        Returns (new num_tokens, slots int32 [n_new] or None, cow pairs int64 [k, 2])."""
        assert table.dtype == np.int32 and table.flags["C_CONTIGUOUS"]
        nt = ctypes.c_int32(num_tokens)
        slots = np.empty(n_new, np.int32) if want_slots else None
        cow = np.empty((cow_capacity, 2), np.int64)
        ncow = ctypes.c_int(0)
        rc = _lib.pa_pool_append(self._h, _i32p(table), table.shape[0], ctypes.byref(nt), int(n_new),
                                 _i32p(slots) if slots is not None else None,
                                 cow.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), cow_capacity,
                                 ctypes.byref(ncow))
        _check(rc, "pa_pool_append")
        return int(nt.value), slots, cow[: ncow.value].copy()

    def fork(self, table: np.ndarray, num_tokens: int, dst: np.ndarray) -> None:
        _check(_lib.pa_pool_fork(self._h, _i32p(table), int(num_tokens), _i32p(dst), dst.shape[0]), "pa_pool_fork")

    def release(self, table: np.ndarray, num_tokens: int) -> None:
        _check(_lib.pa_pool_release(self._h, _i32p(table), int(num_tokens)), "pa_pool_release")

    def export(self) -> Tuple[np.ndarray, np.ndarray]:
        """(reference counts [num_blocks], free list front first)."""
        ref = np.empty(self.num_blocks, np.int32)
        fl = np.empty(max(1, self.num_blocks), np.int32)
        n = ctypes.c_int(0)
        _check(_lib.pa_pool_export(self._h, _i32p(ref), _i32p(fl), ctypes.byref(n)), "pa_pool_export")
        return ref, fl[: n.value].copy()


class PrefixCache:
    """Prefix cache (pa_prefix_* calls) over a BlockPool: a token list's
    blocks are taken once and reused while any request holds the prefix."""

    def __init__(self, pool: BlockPool, hash_bits: int = 0):
        self.pool = pool  # keeps the pool alive
        h = _lib.pa_prefix_cache_create(pool._h, int(hash_bits))
        if not h:
            raise PagedAttentionError("pa_prefix_cache_create", -3)
        self._h = ctypes.c_void_p(h)
        self._destroy = _lib.pa_prefix_cache_destroy  # still callable at interpreter exit

    def __del__(self):
        h, destroy = getattr(self, "_h", None), getattr(self, "_destroy", None)
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self._h = None

    @staticmethod
    def _tokens(tokens) -> np.ndarray:
        return np.ascontiguousarray(np.asarray(tokens, dtype=np.int32).reshape(-1))

    def get_or_create(self, tokens) -> Tuple[list, bool]:
        """Returns (block ids, hit)."""
        t = self._tokens(tokens)
        cap = (t.shape[0] + self.pool.block_size - 1) // self.pool.block_size
        ids = np.empty(max(1, cap), np.int32)
        n, hit = ctypes.c_int(0), ctypes.c_int(0)
        _check(_lib.pa_prefix_get_or_create(self._h, _i32p(t), t.shape[0], _i32p(ids), cap, ctypes.byref(n),
                                            ctypes.byref(hit)), "pa_prefix_get_or_create")
        return ids[: n.value].tolist(), bool(hit.value)

    def release(self, tokens) -> None:
        t = self._tokens(tokens)
        _check(_lib.pa_prefix_release(self._h, _i32p(t), t.shape[0]), "pa_prefix_release")

    def ref_count(self, tokens) -> int:
        t = self._tokens(tokens)
        rc = int(_lib.pa_prefix_ref_count(self._h, _i32p(t), t.shape[0]))
        if rc < 0:
            raise PagedAttentionError("pa_prefix_ref_count", rc)
        return rc

    def num_entries(self) -> int:
        return int(_lib.pa_prefix_num_entries(self._h))

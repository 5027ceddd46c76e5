"""CPU oracle for paged KV-cache decode attention.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg and reference arm (``--impl reference``) of ``bench.py`` may
import this package. The CUDA library and
its Python binding never import it, and the two share no code: this package
wraps ``pa_oracle.c`` (plain single-threaded C in double precision) through
ctypes, plus the host block pool in ``block_pool.py``.

Every function takes numpy arrays. Floating-point inputs are the values after
rounding to their storage dtype, widened to float64 by the caller.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .block_pool import BlockPool, Sequence, append_tokens, fork, release  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compiles pa_oracle.c into liboracle.so (plain gcc, no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
        ci, cd = ctypes.c_int, ctypes.c_double
        lib.oracle_blocks_needed.argtypes = [ci, ci]
        lib.oracle_paged_decode.argtypes = [f64p, f64p, f64p, f64p, i32p, ci, i32p, ci, ci, ci, ci, ci, ci, cd]
        lib.oracle_splitk_partials.argtypes = [f64p, f64p, f64p, f64p, f64p, f64p, i32p, ci, i32p,
                                               ci, ci, ci, ci, ci, ci, cd, ci, ci]
        lib.oracle_splitk_merge.argtypes = [f64p, f64p, f64p, f64p, i32p, ci, ci, ci, ci, ci]
        lib.oracle_reshape_and_cache.argtypes = [u8p, u8p, u8p, u8p, i32p, ci, ci, ci, ci, ci, ci]
        lib.oracle_copy_blocks.argtypes = [u8p, u8p, i64p, ci, ci, ctypes.c_int64]
        lib.oracle_paged_prefill.argtypes = [f64p, f64p, i32p, f64p, f64p, i32p, ci, i32p, ci, ci, ci, ci, ci, ci,
                                             cd]
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        i8p = np.ctypeslib.ndpointer(np.int8, flags="C_CONTIGUOUS")
        lib.oracle_quantize_rows.argtypes = [f32p, ci, ci, i8p, f32p]
        lib.oracle_reshape_and_cache_q8.argtypes = [i8p, i8p, f32p, f32p, f32p, f32p, i32p, ci, ci, ci, ci, ci]
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str) -> None:
    if rc != 0:
        names = {-1: "bad argument", -2: "block table too short", -3: "block id out of range",
                 -4: "slot out of range", -5: "out of memory"}
        raise OracleError(f"{what}: {names.get(rc, rc)}")


def blocks_needed(num_tokens: int, block_size: int) -> int:
    """ceil(num_tokens / block_size), the block count of a sequence."""
    n = _load().oracle_blocks_needed(int(num_tokens), int(block_size))
    _check(0 if n >= 0 else n, "blocks_needed")
    return n


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def paged_decode(query, k_cache, v_cache, block_tables, context_lens, scale, block_size) -> np.ndarray:
    """out[s, h] = softmax(scale * q[s, h] . K_s^T) V_s over context_lens[s]
    tokens gathered through block_tables[s]; shapes as in pa_oracle.c."""
    q, kc, vc = _f64(query), _f64(k_cache), _f64(v_cache)
    bt, cl = _i32(block_tables), _i32(context_lens)
    S, Hq, D = q.shape
    NB, Hkv, bs, D2 = kc.shape
    assert D2 == D and bs == block_size and vc.shape == kc.shape and bt.shape[0] == S
    out = np.zeros_like(q)
    rc = _load().oracle_paged_decode(out, q, kc, vc, bt, bt.shape[1], cl, S, Hq, Hkv, D, bs, NB, float(scale))
    _check(rc, "paged_decode")
    return out


def splitk_partials(query, k_cache, v_cache, block_tables, context_lens, scale, block_size,
                    partition_size, max_parts):
    """Per-partition (m, l, acc) in double: m/l [S, Hq, max_parts], acc [S, Hq, max_parts, D].
    Entries of empty partitions stay NaN."""
    q, kc, vc = _f64(query), _f64(k_cache), _f64(v_cache)
    bt, cl = _i32(block_tables), _i32(context_lens)
    S, Hq, D = q.shape
    NB, Hkv, bs, _ = kc.shape
    m = np.full((S, Hq, max_parts), np.nan)
    l = np.full((S, Hq, max_parts), np.nan)
    acc = np.full((S, Hq, max_parts, D), np.nan)
    rc = _load().oracle_splitk_partials(m, l, acc, q, kc, vc, bt, bt.shape[1], cl, S, Hq, Hkv, D, bs, NB,
                                        float(scale), int(partition_size), int(max_parts))
    _check(rc, "splitk_partials")
    return m, l, acc


def splitk_merge(part_m, part_l, part_acc, context_lens, partition_size) -> np.ndarray:
    """Closed-form log-sum-exp merge of split-K partials -> out [S, Hq, D]."""
    m, l, acc = _f64(part_m), _f64(part_l), _f64(part_acc)
    cl = _i32(context_lens)
    S, Hq, P, D = acc.shape
    out = np.zeros((S, Hq, D))
    rc = _load().oracle_splitk_merge(out, m, l, acc, cl, S, Hq, D, int(partition_size), P)
    _check(rc, "splitk_merge")
    return out


def _bytes_view(a: np.ndarray) -> np.ndarray:
    assert a.flags["C_CONTIGUOUS"]
    return a.reshape(-1).view(np.uint8)


def reshape_and_cache(k_cache: np.ndarray, v_cache: np.ndarray, key: np.ndarray, value: np.ndarray,
                      slot_mapping) -> None:
    """In place: writes key/value [T, Hkv, D] rows into the pools through
    slot_mapping (raw bytes; any element type)."""
    NB, Hkv, bs, D = k_cache.shape
    assert key.dtype == k_cache.dtype == v_cache.dtype == value.dtype
    sm = _i32(slot_mapping)
    T = sm.shape[0]
    assert key.shape == (T, Hkv, D) and value.shape == (T, Hkv, D)
    rc = _load().oracle_reshape_and_cache(_bytes_view(k_cache), _bytes_view(v_cache),
                                          _bytes_view(np.ascontiguousarray(key)),
                                          _bytes_view(np.ascontiguousarray(value)),
                                          sm, T, NB, Hkv, D, bs, k_cache.itemsize)
    _check(rc, "reshape_and_cache")


def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, src_dst_pairs) -> None:
    """In place: whole-block byte copies for each (src, dst) pair, in order."""
    NB = k_cache.shape[0]
    pairs = np.ascontiguousarray(np.asarray(src_dst_pairs, dtype=np.int64).reshape(-1, 2))
    block_bytes = k_cache.nbytes // NB
    rc = _load().oracle_copy_blocks(_bytes_view(k_cache), _bytes_view(v_cache), pairs, pairs.shape[0],
                                    NB, block_bytes)
    _check(rc, "copy_blocks")


def paged_prefill(query, q_start, k_cache, v_cache, block_tables, context_lens, scale, block_size) -> np.ndarray:
    """Causal attention of each sequence's new query tokens (rows q_start[s] ..
    q_start[s+1]-1 of query [T, Hq, D]) over its cache; token i of sequence s
    sits at position context_lens[s] - q_len + i."""
    q, kc, vc = _f64(query), _f64(k_cache), _f64(v_cache)
    qs, bt, cl = _i32(q_start), _i32(block_tables), _i32(context_lens)
    T, Hq, D = q.shape
    NB, Hkv, bs, _ = kc.shape
    S = cl.shape[0]
    assert qs.shape[0] == S + 1 and bs == block_size
    out = np.zeros_like(q)
    rc = _load().oracle_paged_prefill(out, q, qs, kc, vc, bt, bt.shape[1], cl, S, Hq, Hkv, D, bs, NB, float(scale))
    _check(rc, "paged_prefill")
    return out


# ------------------------------------------------------------ int8 KV cache

def quantize_rows(x):
    """Symmetric int8 codes and fp32 scales of each row (last axis) of x,
    computed in fp32 as pa_oracle.c states: returns (codes int8, scales f32)."""
    x32 = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    n = x32.shape[-1]
    rows = x32.size // n
    q = np.empty(x32.shape, np.int8)
    s = np.empty(x32.shape[:-1], np.float32)
    _check(_load().oracle_quantize_rows(x32.reshape(-1), rows, n, q.reshape(-1), s.reshape(-1)), "quantize_rows")
    return q, s


def reshape_and_cache_q8(k_cache, v_cache, k_scale, v_scale, key, value, slot_mapping) -> None:
    """In place: quantizes key/value [T, Hkv, D] (fp32 values) row by row into
    the int8 pools [NB, Hkv, bs, D] and scale pools [NB, Hkv, bs]."""
    NB, Hkv, bs, D = k_cache.shape
    assert k_cache.dtype == v_cache.dtype == np.int8 and k_scale.dtype == v_scale.dtype == np.float32
    for a in (k_cache, v_cache, k_scale, v_scale):
        assert a.flags["C_CONTIGUOUS"]
    sm = _i32(slot_mapping)
    T = sm.shape[0]
    kf = np.ascontiguousarray(np.asarray(key, dtype=np.float32))
    vf = np.ascontiguousarray(np.asarray(value, dtype=np.float32))
    assert kf.shape == (T, Hkv, D) and vf.shape == (T, Hkv, D)
    rc = _load().oracle_reshape_and_cache_q8(k_cache.reshape(-1), v_cache.reshape(-1), k_scale.reshape(-1),
                                             v_scale.reshape(-1), kf.reshape(-1), vf.reshape(-1), sm, T, NB, Hkv, D,
                                             bs)
    _check(rc, "reshape_and_cache_q8")


def dequantize(codes, scales) -> np.ndarray:
    """K = q * scale in double (exact: an 8-bit code times an fp32 scale)."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scales, dtype=np.float64)[..., None]


def paged_decode_q8(query, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale, block_size):
    """Paged decode over an int8 cache: attention over the dequantized K/V."""
    return paged_decode(query, dequantize(k_cache, k_scale), dequantize(v_cache, v_scale), block_tables,
                        context_lens, scale, block_size)

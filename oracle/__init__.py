"""CPU oracle (fp64) for paged decode attention and the decode-step KV append.

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` leg may import it; the product package never does.
The arithmetic lives in ``oracle.c`` (plain C, double precision, one output
element at a time); this module compiles it with gcc and marshals numpy
arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

DT = {"f32": 0, "bf16": 1, "e4m3": 2, "e5m2": 3, "int8": 4}
NP_DT = {"f32": np.float32, "bf16": np.uint16, "e4m3": np.uint8, "e5m2": np.uint8, "int8": np.int8}

_lib = None


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile the oracle into a shared object (no fast-math, no FP contraction)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= max(
            os.path.getmtime(src), os.path.getmtime(os.path.join(HERE, "oracle.h"))):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
           "-I", HERE, src, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def _bind(lib):
    P = ctypes.c_void_p
    i32, i64, f32, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
    lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3_value.restype = f64
    lib.orc_e4m3_encode.argtypes = [f32]
    lib.orc_e4m3_encode.restype = ctypes.c_uint8
    lib.orc_e4m3_encode_array.argtypes = [P, P, i64]
    lib.orc_e4m3_encode_array.restype = None
    lib.orc_int8_encode.argtypes = [f32]
    lib.orc_int8_encode.restype = ctypes.c_int8
    lib.orc_e5m2_value.argtypes = [ctypes.c_uint8]
    lib.orc_e5m2_value.restype = f64
    lib.orc_e5m2_encode_array.argtypes = [P, P, i64]
    lib.orc_e5m2_encode_array.restype = None
    lib.orc_paged_decode.argtypes = [P, P, i32, P, P, i32, P, P, i32, i32, i32, i32, i32, i32, i32,
                                     f64, f64, f64, P, i32, i32, P, P]
    lib.orc_paged_decode.restype = i32
    lib.orc_paged_decode_lse.argtypes = [P, P, P, i32, P, P, i32, P, P, i32, i32, i32, i32, i32, i32, i32,
                                         f64, f64, f64, P, i32, i32, P, P]
    lib.orc_paged_decode_lse.restype = i32
    lib.orc_reshape_and_cache.argtypes = [P, P, i32, P, P, i32, P, P, i64, i32, i32, i32, i32, i32, f32, f32, P, P]
    lib.orc_reshape_and_cache.restype = i32
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle library; ``path`` loads another build of it."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class OracleError(RuntimeError):
    pass


def e4m3_value(code: int, lib=None) -> float:
    return (lib or load()).orc_e4m3_value(int(code))


def e4m3_encode(x, lib=None) -> np.ndarray:
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    out = np.empty(x.size, dtype=np.uint8)
    lib.orc_e4m3_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def e5m2_value(code: int, lib=None) -> float:
    return (lib or load()).orc_e5m2_value(int(code))


def e5m2_encode(x, lib=None) -> np.ndarray:
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    out = np.empty(x.size, dtype=np.uint8)
    lib.orc_e5m2_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def paged_decode(q, q_dtype, k_cache, v_cache, kv_dtype, block_tables, seq_lens,
                 num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                 scale, k_scale=1.0, v_scale=1.0, seqs=None, lib=None, q_len=1, k_head_scales=None,
                 v_head_scales=None, return_lse=False):
    """fp64 attention output [len(seqs) or num_seqs, num_heads, head_dim]; with q_len > 1,
    q is [num_seqs, q_len, num_heads, head_dim] (query j at position seq_len - q_len + j,
    causal) and the output [rows, q_len, num_heads, head_dim]. With ``return_lse`` also the
    natural log of every row's softmax denominator (shape of the output without head_dim)."""
    lib = lib or load()
    q = np.ascontiguousarray(q, dtype=NP_DT[q_dtype])
    k_cache = np.ascontiguousarray(k_cache, dtype=NP_DT[kv_dtype])
    v_cache = np.ascontiguousarray(v_cache, dtype=NP_DT[kv_dtype])
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    S = sl.shape[0]
    MB = bt.shape[1] if bt.ndim == 2 else 0
    sub = None if seqs is None else np.ascontiguousarray(seqs, dtype=np.int32)
    khs = None if k_head_scales is None else np.ascontiguousarray(k_head_scales, dtype=np.float32)
    vhs = None if v_head_scales is None else np.ascontiguousarray(v_head_scales, dtype=np.float32)
    rows = S if sub is None else sub.size
    out = np.zeros((rows, num_heads, head_dim) if q_len == 1 else (rows, q_len, num_heads, head_dim),
                   dtype=np.float64)
    lse = np.zeros(out.shape[:-1], dtype=np.float64) if return_lse else None
    st = lib.orc_paged_decode_lse(_ptr(out), _ptr(lse), _ptr(q), DT[q_dtype], _ptr(k_cache), _ptr(v_cache),
                                  DT[kv_dtype], _ptr(bt), _ptr(sl), S, num_heads, num_kv_heads, head_dim,
                                  block_size, MB, num_blocks, float(scale), float(k_scale), float(v_scale),
                                  _ptr(sub), 0 if sub is None else int(sub.size), int(q_len), _ptr(khs), _ptr(vhs))
    if st != 0:
        raise OracleError(f"orc_paged_decode status {st}")
    return (out, lse) if return_lse else out


def reshape_and_cache(k, v, in_dtype, k_cache, v_cache, kv_dtype, slot_mapping,
                      num_kv_heads, head_dim, block_size, num_blocks,
                      k_scale=1.0, v_scale=1.0, rows=None, lib=None, k_head_scales=None,
                      v_head_scales=None) -> None:
    """Write rows of k/v ([T, Hkv, d]) into the numpy caches in place (FP8: per-tensor scales, or
    one per KV head when k_head_scales / v_head_scales are given)."""
    lib = lib or load()
    k = np.ascontiguousarray(k, dtype=NP_DT[in_dtype])
    v = np.ascontiguousarray(v, dtype=NP_DT[in_dtype])
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert k_cache.dtype == NP_DT[kv_dtype] and v_cache.dtype == NP_DT[kv_dtype]
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    khs = None if k_head_scales is None else np.ascontiguousarray(k_head_scales, dtype=np.float32)
    vhs = None if v_head_scales is None else np.ascontiguousarray(v_head_scales, dtype=np.float32)
    st = lib.orc_reshape_and_cache(_ptr(k), _ptr(v), DT[in_dtype], _ptr(k_cache), _ptr(v_cache), DT[kv_dtype],
                                   _ptr(sm), _ptr(r), 0 if r is None else int(r.size), int(sm.size),
                                   num_kv_heads, head_dim, block_size, num_blocks,
                                   float(np.float32(k_scale)), float(np.float32(v_scale)), _ptr(khs), _ptr(vhs))
    if st != 0:
        raise OracleError(f"orc_reshape_and_cache status {st}")


def empty_cache(num_blocks, num_kv_heads, block_size, head_dim, kv_dtype):
    return np.zeros((num_blocks, num_kv_heads, block_size, head_dim), dtype=NP_DT[kv_dtype])


def run_step(batch, seqs=None, lib=None):
    """The whole decode step on the CPU: history fill, append, attention.

    Returns (out fp64, k_cache, v_cache). With ``seqs`` only the blocks those
    sequences reference are filled and only their outputs are computed.
    """
    sp = batch.spec
    kc = empty_cache(batch.num_blocks, sp.num_kv_heads, sp.block_size, sp.head_dim, sp.kv_dtype)
    vc = empty_cache(batch.num_blocks, sp.num_kv_heads, sp.block_size, sp.head_dim, sp.kv_dtype)
    rows = None
    new_rows = None
    if seqs is not None:
        from workloads import subset_tokens
        rows = subset_tokens(batch, seqs)
        new_rows = np.asarray(seqs, dtype=np.int64)
    reshape_and_cache(batch.hist_k, batch.hist_v, sp.in_dtype, kc, vc, sp.kv_dtype, batch.hist_slots,
                      sp.num_kv_heads, sp.head_dim, sp.block_size, batch.num_blocks,
                      batch.k_scale, batch.v_scale, rows=rows, lib=lib)
    reshape_and_cache(batch.new_k, batch.new_v, sp.in_dtype, kc, vc, sp.kv_dtype, batch.new_slots,
                      sp.num_kv_heads, sp.head_dim, sp.block_size, batch.num_blocks,
                      batch.k_scale, batch.v_scale, rows=new_rows, lib=lib)
    out = paged_decode(batch.q, sp.q_dtype, kc, vc, sp.kv_dtype, batch.block_tables, batch.seq_lens,
                       sp.num_heads, sp.num_kv_heads, sp.head_dim, sp.block_size, batch.num_blocks,
                       batch.scale, batch.k_scale, batch.v_scale, seqs=seqs, lib=lib)
    return out, kc, vc

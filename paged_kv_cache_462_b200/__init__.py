"""Paged KV-cache decode attention for NVIDIA B200 (sm_100a).

A thin ctypes binding of ``libpagedkv.so`` (C ABI declared in ``include/pkv.h``).
Functions here only check and marshal torch tensors (device pointers, sizes,
dtypes, the current CUDA stream); every step of the computation runs in the
library's CUDA kernels. There is no CPU fallback: without the built library
(``python -m paged_kv_cache_462_b200.build``) every call raises.

Entry points (same names as the C ABI):

* ``reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, ...)`` — append
  the decode step's new K/V rows into their cache slots.
* ``paged_attention_decode(out, q, k_cache, v_cache, block_tables, seq_lens,
  scale, ...)`` — single-query grouped attention for every sequence, reading
  K/V block by block through the block table.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpagedkv.so")

F32, BF16, FP8_E4M3, FP8_E5M2, INT8 = 0, 1, 2, 3, 4
DEVERR_BLOCK_ID, DEVERR_SEQ_LEN, DEVERR_SLOT, DEVERR_TIMEOUT, DEVERR_PLAN = 1, 2, 4, 8, 16

# uint8 caches hold E4M3 codes; E5M2 caches are passed as torch.float8_e5m2 tensors
_TORCH_DTYPE = {torch.float32: F32, torch.bfloat16: BF16, torch.uint8: FP8_E4M3, torch.float8_e4m3fn: FP8_E4M3,
                torch.float8_e5m2: FP8_E5M2, torch.int8: INT8}

_lib = None


class PkvError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: status {status} ({status_string(status)})")


def load_library():
    """Load libpagedkv.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_462_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.paged_attention_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    lib.paged_attention_workspace_size.restype = sz
    lib.pkv_workspace_init.argtypes = [P, sz, P]
    lib.pkv_workspace_init.restype = i32
    lib.paged_attention_decode.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, f32, i32, i32, i32, i32,
                                           f32, f32, i32, P, sz, P]
    lib.paged_attention_decode.restype = i32
    lib.paged_decode_step.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, f32, i32, i32, i32, i32,
                                      f32, f32, i32, P, sz, P, P, P, i32, P]
    lib.paged_decode_step.restype = i32
    lib.reshape_and_cache_head_scales.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, P, P, P, P]
    lib.reshape_and_cache_head_scales.restype = i32
    lib.paged_attention_decode_head_scales.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, f32, i32, i32,
                                                       i32, i32, P, P, i32, P, sz, P]
    lib.paged_attention_decode_head_scales.restype = i32
    lib.paged_attention_decode_mq.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, i32, f32, i32, i32, i32,
                                              i32, f32, f32, i32, P, sz, P]
    lib.paged_attention_decode_mq.restype = i32
    lib.pkv_test_decode_timeout.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, f32, i32, i32, i32, i32,
                                            f32, f32, i32, P, sz, i32, P]
    lib.pkv_test_decode_timeout.restype = i32
    lib.reshape_and_cache.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, f32, f32, P, P]
    lib.reshape_and_cache.restype = i32
    lib.pkv_read_device_error.argtypes = [P, sz, ctypes.POINTER(ctypes.c_int32), i32, P]
    lib.pkv_read_device_error.restype = i32
    lib.pkv_default_partitions.argtypes = [i32, i32, i32, i32, i32]
    lib.pkv_default_partitions.restype = i32
    lib.pkv_set_fp8_kernel.argtypes = [i32]
    lib.pkv_set_fp8_kernel.restype = i32
    lib.paged_attention_shared_prefix_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
    lib.paged_attention_shared_prefix_workspace_size.restype = sz
    lib.paged_attention_decode_shared_prefix.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, f32, i32, i32,
                                                         i32, i32, f32, f32, P, P, P, P, P, i32, i32, i32, P, sz,
                                                         P]
    lib.paged_attention_decode_shared_prefix.restype = i32
    lib.paged_decode_step_shared_prefix.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, f32, i32, i32, i32,
                                                    i32, f32, f32, P, P, P, P, P, i32, i32, i32, P, sz, P, P, P,
                                                    i32, P]
    lib.paged_decode_step_shared_prefix.restype = i32
    lib.pkv_validate_tables.argtypes = [P, P, i32, i32, i32, i32, P, ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(ctypes.c_int32)]
    lib.pkv_validate_tables.restype = i32
    lib.pkv_status_string.argtypes = [i32]
    lib.pkv_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().pkv_status_string(int(status)).decode()


def _check(fn, status):
    if status != 0:
        raise PkvError(fn, status)


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _TORCH_DTYPE[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def _launch_device(name, t) -> int:
    """The current CUDA device (where the library launches), once `t` is known to be a CUDA tensor."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return torch.cuda.current_device()


def _cuda(name, t: torch.Tensor, dev: int | None = None):
    """Device pointer of a contiguous CUDA tensor on device `dev` (the current device, where the
    library launches; a tensor elsewhere would be read through a pointer this device cannot use)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dev is not None and t.device.index != dev:
        raise ValueError(f"{name} is on {t.device}, the current CUDA device is cuda:{dev}")
    return ctypes.c_void_p(t.data_ptr())


def workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, num_partitions=0) -> int:
    n = load_library().paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, num_partitions)
    if n == 0:
        raise PkvError("paged_attention_workspace_size", 2)
    return int(n)


def new_workspace(num_seqs, num_heads, num_kv_heads, head_dim, num_partitions=0, device=None) -> torch.Tensor:
    """A zeroed (i.e. initialised) workspace tensor for paged_attention_decode."""
    n = workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, num_partitions)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check("pkv_workspace_init",
           load_library().pkv_workspace_init(_cuda("workspace", workspace), workspace.numel(), _stream_handle(stream)))


FP8_KERNEL_MMA = 0        # warp-level tensor cores on codes widened to f16 (the default)
FP8_KERNEL_TCGEN05 = 1    # fifth-generation tensor cores reading the 8-bit tiles (tcgen05.mma)


def set_fp8_kernel(which: int) -> int:
    """Process-wide kernel for FP8-cache decodes (pkv_set_fp8_kernel); returns the previous choice."""
    prev = load_library().pkv_set_fp8_kernel(int(which))
    if prev < 0:
        raise PkvError("pkv_set_fp8_kernel", -prev)
    return prev


def default_partitions(head_dim, block_size, num_heads, num_kv_heads, kv_dtype) -> int:
    code = kv_dtype if isinstance(kv_dtype, int) else _TORCH_DTYPE[kv_dtype]
    n = load_library().pkv_default_partitions(head_dim, block_size, num_heads, num_kv_heads, code)
    if n <= 0:
        raise PkvError("pkv_default_partitions", -n)
    return n


def paged_attention_decode(out, q, k_cache, v_cache, block_tables, seq_lens, scale,
                           k_scale=1.0, v_scale=1.0, num_partitions=0, workspace=None, stream=None) -> None:
    """out[s, g] = softmax(scale * q[s, g] . K) V over the seq_lens[s] cached tokens of sequence s.

    q, out: [num_seqs, num_heads, head_dim] (float32 or bfloat16);
    k_cache, v_cache: [num_blocks, num_kv_heads, block_size, head_dim]
    (float32, bfloat16, uint8/float8_e4m3fn E4M3 codes, float8_e5m2 codes or int8 codes, the
    8-bit ones with k_scale/v_scale);
    block_tables: int32 [num_seqs, max_blocks_per_seq]; seq_lens: int32 [num_seqs].
    """
    args = _decode_args(out, q, k_cache, v_cache, block_tables, seq_lens, scale, k_scale, v_scale,
                        num_partitions, workspace, stream)
    st = load_library().paged_attention_decode(*args, _stream_handle(stream))
    _check("paged_attention_decode", st)


def _decode_args(out, q, k_cache, v_cache, block_tables, seq_lens, scale, k_scale, v_scale, num_partitions,
                 workspace, stream=None):
    """Checked C arguments of a decode call, up to (not including) the stream."""
    dev = _launch_device("q", q)
    S, Hq, D = q.shape
    NB, Hkv, BS, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("shape mismatch between q/out and the caches")
    if out.dtype != q.dtype or v_cache.dtype != k_cache.dtype:
        raise TypeError("out must match q's dtype and v_cache k_cache's")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_tables and seq_lens must be int32")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_tables must be [num_seqs, max_blocks] and seq_lens [num_seqs]")
    if workspace is None:
        workspace = _cached_workspace(S, Hq, Hkv, D, num_partitions, dev, stream)
    return (_cuda("out", out, dev), _cuda("q", q, dev), _cuda("k_cache", k_cache, dev),
            _cuda("v_cache", v_cache, dev), _cuda("block_tables", block_tables, dev),
            _cuda("seq_lens", seq_lens, dev), S, Hq, Hkv, D, BS, float(scale),
            block_tables.shape[1], NB, _dtype_code(q), _dtype_code(k_cache), float(k_scale), float(v_scale),
            int(num_partitions), _cuda("workspace", workspace, dev), workspace.numel())


def paged_attention_decode_mq(out, q, k_cache, v_cache, block_tables, seq_lens, scale, k_scale=1.0, v_scale=1.0,
                              num_partitions=0, workspace=None, stream=None) -> None:
    """q_len new tokens per sequence, causal within the chunk: q, out [num_seqs, q_len, num_heads, head_dim]
    (bf16); query j of sequence s sits at position seq_lens[s] - q_len + j and attends every token
    up to itself. The new tokens' K/V must already be in the cache."""
    dev = _launch_device("q", q)
    S, QL, Hq, D = q.shape
    NB, Hkv, BS, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("shape mismatch between q/out and the caches")
    if out.dtype != q.dtype or v_cache.dtype != k_cache.dtype:
        raise TypeError("out must match q's dtype and v_cache k_cache's")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_tables and seq_lens must be int32")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_tables must be [num_seqs, max_blocks] and seq_lens [num_seqs]")
    if workspace is None:
        workspace = _cached_workspace(S, Hq * QL, Hkv, D, num_partitions, dev, stream)
    st = load_library().paged_attention_decode_mq(
        _cuda("out", out, dev), _cuda("q", q, dev), _cuda("k_cache", k_cache, dev), _cuda("v_cache", v_cache, dev),
        _cuda("block_tables", block_tables, dev), _cuda("seq_lens", seq_lens, dev), S, QL, Hq, Hkv, D, BS,
        float(scale), block_tables.shape[1], NB, _dtype_code(q), _dtype_code(k_cache), float(k_scale),
        float(v_scale), int(num_partitions), _cuda("workspace", workspace, dev), workspace.numel(),
        _stream_handle(stream))
    _check("paged_attention_decode_mq", st)


def withheld_unit_decode(out, q, k_cache, v_cache, block_tables, seq_lens, scale, withheld_unit, workspace,
                        k_scale=1.0, v_scale=1.0, num_partitions=0, stream=None) -> None:
    """Failure-path test hook: paged_attention_decode with unit `withheld_unit`'s stage never handed
    to its consumers, so their bounded wait runs out and the workspace error word gets
    DEVERR_TIMEOUT (read it with read_device_error, then workspace_init before reuse)."""
    args = _decode_args(out, q, k_cache, v_cache, block_tables, seq_lens, scale, k_scale, v_scale,
                        num_partitions, workspace, stream)
    st = load_library().pkv_test_decode_timeout(*args, int(withheld_unit), _stream_handle(stream))
    _check("pkv_test_decode_timeout", st)


def paged_decode_step(out, q, k_cache, v_cache, block_tables, seq_lens, new_k, new_v, slot_mapping, scale,
                      k_scale=1.0, v_scale=1.0, num_partitions=0, workspace=None, stream=None) -> None:
    """One decode step: append new_k/new_v row s at slot_mapping[s] (one new token per sequence,
    in its last block), then paged_attention_decode over the cache. One launch where the
    tensor-core decode kernel applies."""
    dev = _launch_device("q", q)
    S, Hq, D = q.shape
    NB, Hkv, BS, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("shape mismatch between q/out and the caches")
    if tuple(new_k.shape) != (S, Hkv, D) or tuple(new_v.shape) != (S, Hkv, D) or new_v.dtype != new_k.dtype:
        raise ValueError("new_k/new_v must be [num_seqs, num_kv_heads, head_dim] of one dtype")
    if slot_mapping.dtype != torch.int64 or slot_mapping.shape != (S,):
        raise TypeError("slot_mapping must be int64 [num_seqs]")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_tables and seq_lens must be int32")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_tables must be [num_seqs, max_blocks] and seq_lens [num_seqs]")
    if workspace is None:
        workspace = _cached_workspace(S, Hq, Hkv, D, num_partitions, dev, stream)
    st = load_library().paged_decode_step(
        _cuda("out", out, dev), _cuda("q", q, dev), _cuda("k_cache", k_cache, dev), _cuda("v_cache", v_cache, dev),
        _cuda("block_tables", block_tables, dev), _cuda("seq_lens", seq_lens, dev), S, Hq, Hkv, D, BS,
        float(scale), block_tables.shape[1], NB, _dtype_code(q), _dtype_code(k_cache), float(k_scale),
        float(v_scale), int(num_partitions), _cuda("workspace", workspace, dev), workspace.numel(),
        _cuda("new_k", new_k, dev), _cuda("new_v", new_v, dev), _cuda("slot_mapping", slot_mapping, dev),
        _dtype_code(new_k), _stream_handle(stream))
    _check("paged_decode_step", st)


def reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, k_scale=1.0, v_scale=1.0,
                      device_error=None, stream=None) -> None:
    """Write k[t], v[t] ([num_tokens, num_kv_heads, head_dim]) into slot slot_mapping[t] of the caches."""
    dev = _launch_device("k", k)
    T, Hkv, D = k.shape
    NB, Hkv2, BS, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or tuple(v.shape) != tuple(k.shape) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between rows and caches")
    if slot_mapping.dtype != torch.int64 or slot_mapping.shape != (T,):
        raise TypeError("slot_mapping must be int64 [num_tokens]")
    err = ctypes.c_void_p(None) if device_error is None else _cuda("device_error", device_error, dev)
    st = load_library().reshape_and_cache(
        _cuda("k", k, dev), _cuda("v", v, dev), _cuda("k_cache", k_cache, dev), _cuda("v_cache", v_cache, dev),
        _cuda("slot_mapping", slot_mapping, dev), T, Hkv, D, BS, NB, _dtype_code(k), _dtype_code(k_cache),
        float(k_scale), float(v_scale), err, _stream_handle(stream))
    _check("reshape_and_cache", st)


def _head_scales(name, t, Hkv, dev):
    if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or t.shape != (Hkv,):
        raise TypeError(f"{name} must be a float32 tensor of num_kv_heads scales")
    return _cuda(name, t, dev)


def reshape_and_cache_head_scales(k, v, k_cache, v_cache, slot_mapping, k_head_scales, v_head_scales,
                                  device_error=None, stream=None) -> None:
    """reshape_and_cache into an 8-bit cache with one scale per KV head (float32 [num_kv_heads] tensors)."""
    dev = _launch_device("k", k)
    T, Hkv, D = k.shape
    NB, Hkv2, BS, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or tuple(v.shape) != tuple(k.shape) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between rows and caches")
    if slot_mapping.dtype != torch.int64 or slot_mapping.shape != (T,):
        raise TypeError("slot_mapping must be int64 [num_tokens]")
    err = ctypes.c_void_p(None) if device_error is None else _cuda("device_error", device_error, dev)
    st = load_library().reshape_and_cache_head_scales(
        _cuda("k", k, dev), _cuda("v", v, dev), _cuda("k_cache", k_cache, dev), _cuda("v_cache", v_cache, dev),
        _cuda("slot_mapping", slot_mapping, dev), T, Hkv, D, BS, NB, _dtype_code(k), _dtype_code(k_cache),
        _head_scales("k_head_scales", k_head_scales, Hkv, dev), _head_scales("v_head_scales", v_head_scales, Hkv, dev),
        err, _stream_handle(stream))
    _check("reshape_and_cache_head_scales", st)


def paged_attention_decode_head_scales(out, q, k_cache, v_cache, block_tables, seq_lens, scale, k_head_scales,
                                       v_head_scales, num_partitions=0, workspace=None, stream=None) -> None:
    """paged_attention_decode over an 8-bit cache with one scale per KV head."""
    args = list(_decode_args(out, q, k_cache, v_cache, block_tables, seq_lens, scale, 1.0, 1.0, num_partitions,
                             workspace, stream))
    Hkv, dev = k_cache.shape[1], _launch_device("q", q)
    args[16:18] = [_head_scales("k_head_scales", k_head_scales, Hkv, dev),
                   _head_scales("v_head_scales", v_head_scales, Hkv, dev)]
    st = load_library().paged_attention_decode_head_scales(*args, _stream_handle(stream))
    _check("paged_attention_decode_head_scales", st)


def read_device_error(workspace: torch.Tensor, clear: bool = False, stream=None) -> int:
    """The workspace's device error word (PKV_DEVERR_* bits); synchronises the stream."""
    v = ctypes.c_int32(0)
    _check("pkv_read_device_error", load_library().pkv_read_device_error(
        _cuda("workspace", workspace), workspace.numel(), ctypes.byref(v), int(clear), _stream_handle(stream)))
    return int(v.value)


class DevicePrefixPlan:
    """A shared-prefix plan (``blocks.prefix_plan``'s result) copied to the device as the
    shared-prefix decode reads it: int32 members, offsets [groups + 1], tables [groups, max_blocks],
    lens [groups], shared [num_seqs]; ``max_group`` is the planner's group-size limit."""

    def __init__(self, plan, max_group: int, device=None):
        import numpy as np
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
        self.num_groups = int(plan.num_groups)
        self.max_group = int(max_group)
        self.members = t(plan.members)
        self.offsets = t(plan.offsets[: self.num_groups + 1])
        self.tables = t(plan.tables[: self.num_groups])
        self.lens = t(plan.lens[: self.num_groups])
        self.shared = t(plan.shared)

    def tensors(self):
        return (self.members, self.offsets, self.tables, self.lens, self.shared)


def shared_prefix_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, num_groups, num_partitions=0) -> int:
    n = load_library().paged_attention_shared_prefix_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim,
                                                                    num_groups, num_partitions)
    if n == 0:
        raise PkvError("paged_attention_shared_prefix_workspace_size", 2)
    return int(n)


def new_shared_prefix_workspace(num_seqs, num_heads, num_kv_heads, head_dim, num_groups, num_partitions=0,
                                device=None) -> torch.Tensor:
    """A zeroed workspace for the shared-prefix decode."""
    n = shared_prefix_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, num_groups, num_partitions)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def _plan_args(plan: DevicePrefixPlan, dev, S, MB):
    if not isinstance(plan, DevicePrefixPlan):
        raise TypeError("plan must be a DevicePrefixPlan")
    if plan.shared.shape != (S,) or (plan.num_groups and plan.tables.shape[1] != MB):
        raise ValueError("plan does not match the batch (shared [num_seqs], tables [groups, max_blocks])")
    ptr = lambda name, t: _cuda(name, t, dev) if t.numel() else ctypes.c_void_p(None)
    return (ptr("plan.members", plan.members), ptr("plan.offsets", plan.offsets), ptr("plan.tables", plan.tables),
            ptr("plan.lens", plan.lens), _cuda("plan.shared", plan.shared, dev), plan.num_groups, plan.max_group)


def _shared_prefix_workspace(workspace, S, Hq, Hkv, D, plan, num_partitions, dev):
    if workspace is not None:
        return workspace
    n = shared_prefix_workspace_size(S, Hq, Hkv, D, plan.num_groups, num_partitions)
    return torch.zeros(n, dtype=torch.uint8, device=torch.device("cuda", dev))


def paged_attention_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, seq_lens, plan, scale,
                                         k_scale=1.0, v_scale=1.0, num_partitions=0, workspace=None,
                                         stream=None) -> None:
    """paged_attention_decode with the blocks a plan shares read once per group (a prefix pass over
    the groups' shared rows, a suffix pass over each sequence's own blocks, a log-sum-exp merge)."""
    dev = _launch_device("q", q)
    S, Hq, D = q.shape
    NB, Hkv, BS, _ = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape) or k_cache.shape[3] != D:
        raise ValueError("shape mismatch between q/out and the caches")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32 or block_tables.dim() != 2 \
            or block_tables.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_tables must be int32 [num_seqs, max_blocks] and seq_lens int32 [num_seqs]")
    ws = _shared_prefix_workspace(workspace, S, Hq, Hkv, D, plan, num_partitions, dev)
    st = load_library().paged_attention_decode_shared_prefix(
        _cuda("out", out, dev), _cuda("q", q, dev), _cuda("k_cache", k_cache, dev), _cuda("v_cache", v_cache, dev),
        _cuda("block_tables", block_tables, dev), _cuda("seq_lens", seq_lens, dev), S, Hq, Hkv, D, BS,
        float(scale), block_tables.shape[1], NB, _dtype_code(q), _dtype_code(k_cache), float(k_scale),
        float(v_scale), *_plan_args(plan, dev, S, block_tables.shape[1]), int(num_partitions),
        _cuda("workspace", ws, dev), ws.numel(), _stream_handle(stream))
    _check("paged_attention_decode_shared_prefix", st)


def paged_decode_step_shared_prefix(out, q, k_cache, v_cache, block_tables, seq_lens, plan, new_k, new_v,
                                    slot_mapping, scale, k_scale=1.0, v_scale=1.0, num_partitions=0, workspace=None,
                                    stream=None) -> None:
    """paged_decode_step with the shared-prefix decode (the append rides in the suffix pass)."""
    dev = _launch_device("q", q)
    S, Hq, D = q.shape
    NB, Hkv, BS, _ = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape) or k_cache.shape[3] != D:
        raise ValueError("shape mismatch between q/out and the caches")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32 or block_tables.dim() != 2 \
            or block_tables.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_tables must be int32 [num_seqs, max_blocks] and seq_lens int32 [num_seqs]")
    if tuple(new_k.shape) != (S, Hkv, D) or tuple(new_v.shape) != (S, Hkv, D) or new_v.dtype != new_k.dtype:
        raise ValueError("new_k/new_v must be [num_seqs, num_kv_heads, head_dim] of one dtype")
    if slot_mapping.dtype != torch.int64 or slot_mapping.shape != (S,):
        raise TypeError("slot_mapping must be int64 [num_seqs]")
    ws = _shared_prefix_workspace(workspace, S, Hq, Hkv, D, plan, num_partitions, dev)
    st = load_library().paged_decode_step_shared_prefix(
        _cuda("out", out, dev), _cuda("q", q, dev), _cuda("k_cache", k_cache, dev), _cuda("v_cache", v_cache, dev),
        _cuda("block_tables", block_tables, dev), _cuda("seq_lens", seq_lens, dev), S, Hq, Hkv, D, BS,
        float(scale), block_tables.shape[1], NB, _dtype_code(q), _dtype_code(k_cache), float(k_scale),
        float(v_scale), *_plan_args(plan, dev, S, block_tables.shape[1]), int(num_partitions),
        _cuda("workspace", ws, dev), ws.numel(), _cuda("new_k", new_k, dev), _cuda("new_v", new_v, dev),
        _cuda("slot_mapping", slot_mapping, dev), _dtype_code(new_k), _stream_handle(stream))
    _check("paged_decode_step_shared_prefix", st)


def validate_tables(block_tables, seq_lens, block_size: int, num_blocks: int, slot_mapping=None):
    """Host check of a batch's tables (numpy or CPU tensors): (PKV_DEVERR_* bits found, first
    offending sequence or -1). See pkv_validate_tables."""
    import numpy as np
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    sm = None if slot_mapping is None else np.ascontiguousarray(slot_mapping, dtype=np.int64)
    if bt.ndim != 2 or bt.shape[0] != sl.shape[0] or (sm is not None and sm.shape != sl.shape):
        raise ValueError("block_tables [n, max_blocks], seq_lens [n], slot_mapping [n]")
    bits, first = ctypes.c_int32(0), ctypes.c_int32(-1)
    _check("pkv_validate_tables", load_library().pkv_validate_tables(
        bt.ctypes.data, sl.ctypes.data, sl.shape[0], max(1, bt.shape[1]), int(block_size), int(num_blocks),
        None if sm is None else sm.ctypes.data, ctypes.byref(bits), ctypes.byref(first)))
    return int(bits.value), int(first.value)


_ws_cache: dict = {}


def _cached_workspace(S, Hq, Hkv, D, parts, dev, stream):
    """A workspace kept per (device, partitions, stream), so calls on different streams never share
    one; a new one is zeroed by the library on the stream that will use it."""
    n = workspace_size(S, Hq, Hkv, D, parts)
    handle = _stream_handle(stream)
    key = (dev, parts, handle.value)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < n:
        if ws is not None:
            torch.cuda.synchronize(dev)   # the smaller one may still be in use on its stream
        ws = torch.empty(n, dtype=torch.uint8, device=torch.device("cuda", dev))
        _check("pkv_workspace_init", load_library().pkv_workspace_init(_cuda("workspace", ws), n, handle))
        _ws_cache[key] = ws
    return ws


__all__ = [
    "paged_attention_decode", "paged_decode_step", "paged_attention_decode_mq", "paged_attention_decode_head_scales",
    "reshape_and_cache", "reshape_and_cache_head_scales", "workspace_size", "new_workspace", "workspace_init",
    "read_device_error", "default_partitions", "status_string", "load_library", "PkvError",
    "paged_attention_decode_shared_prefix", "paged_decode_step_shared_prefix", "DevicePrefixPlan",
    "shared_prefix_workspace_size", "new_shared_prefix_workspace", "validate_tables",
    "F32", "BF16", "FP8_E4M3", "FP8_E5M2", "INT8",
]

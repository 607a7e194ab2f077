"""paged_attention_decode_static: the decode entry point that allocates nothing.

It serves callers that cannot allocate device memory (plug-ins whose host
framework owns every allocation, hosts that reserve all memory at start-up);
its scratch is a fixed array inside the library. Called through the C ABI, twice in a row, it must give the output of
paged_attention_decode with a caller workspace, within the parity tolerance.
This file is collected last so that a failure here comes after every other test.
"""
import ctypes

import pytest
import torch

import paged_kv_cache_462_b200 as pkv
import workloads as W
from gpu_harness import TOL, GpuStep

pytestmark = pytest.mark.gpu

P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
CODE = {torch.float32: 0, torch.bfloat16: 1, torch.uint8: 2}


def _fn():
    fn = pkv.load_library().paged_attention_decode_static
    fn.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, I, I, I, I, F, F, I, P]
    fn.restype = I
    return fn


def _call_static(g: GpuStep, out: torch.Tensor, parts: int = 0) -> int:
    b, sp = g.b, g.b.spec
    return _fn()(out.data_ptr(), g.q.data_ptr(), g.kc.data_ptr(), g.vc.data_ptr(), g.bt.data_ptr(), g.sl.data_ptr(),
                 b.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, sp.block_size, float(b.scale),
                 b.max_blocks_per_seq, b.num_blocks, CODE[g.q.dtype], CODE[g.kc.dtype], float(b.k_scale),
                 float(b.v_scale), parts, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("cfg", [0, 1, 4])
def test_static_matches_workspace_entry_point_twice(cfg):
    b = W.config_batch(cfg) if cfg == 0 else W.config_batch(cfg, num_seqs=24)
    g = GpuStep(b)
    g.append()
    ref = g.decode(0).clone()                       # existing entry point, caller-owned workspace
    torch.cuda.synchronize()
    for _ in range(2):                              # the array keeps the last call's contents
        out = torch.full_like(ref, float("nan"))
        assert _call_static(g, out) == 0
        torch.cuda.synchronize()
        err = (out.double() - ref.double()).abs().max().item()
        assert err <= TOL[b.spec.kv_dtype], err


@pytest.mark.parametrize("cfg", [1, 4])
def test_static_call_leaves_device_memory_unchanged(cfg):
    """After two warm-up calls (the first resolves the array's address), further calls change
    neither the device's free memory nor torch's allocation count: nothing is allocated."""
    b = W.config_batch(cfg, num_seqs=24)
    g = GpuStep(b)
    g.append()
    out = torch.empty_like(g.q)
    for _ in range(2):
        assert _call_static(g, out) == 0
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(3):
        assert _call_static(g, out) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0


def test_static_rejects_oversized_batch():
    # 16384 sequences x 8 KV heads need far more than the 32 MiB array: refused before any launch
    assert _fn()(None, None, None, None, None, None, 16384, 32, 8, 128, 16, 0.1, 64, 1024, 1, 1, 1.0, 1.0, 0,
                 None) == 4

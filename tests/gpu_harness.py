"""Run a synthetic decode step through the CUDA library, and the same step through the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_462_b200 as pkv

TOL = {"f32": 1e-5, "bf16": 1e-2, "e4m3": 3e-2, "e5m2": 3e-2, "int8": 3e-2}   # max |gpu - oracle| per cache dtype
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8, "e5m2": torch.float8_e5m2,
            "int8": torch.int8}


def to_dev(a: np.ndarray, name: str, device="cuda") -> torch.Tensor:
    if name == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    if name == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    if name == "int8":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int8)).to(device)
    if name == "e5m2":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(device).view(torch.float8_e5m2)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(device)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def cache_bytes(t: torch.Tensor) -> np.ndarray:
    """Raw bytes of a device cache tensor as a numpy array with the oracle's element type."""
    c = t.detach().cpu()
    if c.dtype == torch.bfloat16:
        return c.view(torch.int16).numpy().view(np.uint16)
    if c.dtype in (torch.float8_e5m2, torch.float8_e4m3fn):
        return c.view(torch.uint8).numpy()
    return c.numpy()


class GpuStep:
    """Device state of one batch: caches filled with the history, then the step."""

    def __init__(self, batch, device="cuda"):
        sp = batch.spec
        self.b = batch
        self.dev = device
        self.q = to_dev(batch.q, sp.q_dtype, device)
        self.bt = torch.from_numpy(batch.block_tables).to(device)
        self.sl = torch.from_numpy(batch.seq_lens).to(device)
        self.new_k = to_dev(batch.new_k, sp.in_dtype, device)
        self.new_v = to_dev(batch.new_v, sp.in_dtype, device)
        self.new_slots = torch.from_numpy(batch.new_slots).to(device)
        shape = (batch.num_blocks, sp.num_kv_heads, sp.block_size, sp.head_dim)
        self.kc = torch.zeros(shape, dtype=TORCH_DT[sp.kv_dtype], device=device)
        self.vc = torch.zeros(shape, dtype=TORCH_DT[sp.kv_dtype], device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.out = torch.empty_like(self.q)
        self.fill_history()

    def fill_history(self, chunk=1 << 16):
        b, sp = self.b, self.b.spec
        for i in range(0, b.hist_slots.size, chunk):
            k = to_dev(b.hist_k[i:i + chunk], sp.in_dtype, self.dev)
            v = to_dev(b.hist_v[i:i + chunk], sp.in_dtype, self.dev)
            s = torch.from_numpy(b.hist_slots[i:i + chunk]).to(self.dev)
            pkv.reshape_and_cache(k, v, self.kc, self.vc, s, float(b.k_scale), float(b.v_scale), self.err)

    def append(self):
        b = self.b
        pkv.reshape_and_cache(self.new_k, self.new_v, self.kc, self.vc, self.new_slots,
                              float(b.k_scale), float(b.v_scale), self.err)

    def decode(self, num_partitions=0, workspace=None):
        b = self.b
        sp = b.spec
        if workspace is None:
            workspace = pkv.new_workspace(b.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, num_partitions)
        self.ws = workspace
        pkv.paged_attention_decode(self.out, self.q, self.kc, self.vc, self.bt, self.sl, float(b.scale),
                                   float(b.k_scale), float(b.v_scale), num_partitions, workspace)
        return self.out

    def step(self, num_partitions=0):
        self.append()
        return self.decode(num_partitions)

    def fused_step(self, num_partitions=0, workspace=None):
        """The step through paged_decode_step (append fused into the decode launch where it applies)."""
        b = self.b
        sp = b.spec
        if workspace is None:
            workspace = pkv.new_workspace(b.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, num_partitions)
        self.ws = workspace
        pkv.paged_decode_step(self.out, self.q, self.kc, self.vc, self.bt, self.sl, self.new_k, self.new_v,
                              self.new_slots, float(b.scale), float(b.k_scale), float(b.v_scale), num_partitions,
                              workspace)
        return self.out

    def device_errors(self):
        torch.cuda.synchronize()
        e = int(self.err.item())
        if getattr(self, "ws", None) is not None:
            e |= pkv.read_device_error(self.ws)
        return e


def max_err(gpu_out: torch.Tensor, ref: np.ndarray, seqs=None) -> float:
    g = to_f64(gpu_out)
    if seqs is not None:
        g = g[np.asarray(seqs)]
    return float(np.max(np.abs(g - ref))) if ref.size else 0.0

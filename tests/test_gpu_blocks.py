"""Decode steps driven by the host block manager: prompts, forks that share prefix blocks,
copy on write of a shared last block, appends through paged_decode_step. The GPU caches
must equal the oracle's byte for byte and the outputs must match the oracle's attention."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_harness import TOL, cache_bytes, max_err, to_dev
import paged_kv_cache_462_b200 as pkv
from paged_kv_cache_462_b200.blocks import BlockManager

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
@pytest.mark.parametrize("bs", [16, 32])
def test_manager_driven_decode_steps(kv, bs):
    rng = np.random.default_rng(11 + bs)
    Hq, Hkv, D, NB, MB = 8, 2, 128, 48, 8
    scale = 1.0 / np.sqrt(D)
    ks, vs = (np.float32(0.02), np.float32(0.03)) if kv == "e4m3" else (np.float32(1.0), np.float32(1.0))
    bm = BlockManager(NB, bs, MB)
    kc_o = oracle.empty_cache(NB, Hkv, bs, D, kv)
    vc_o = oracle.empty_cache(NB, Hkv, bs, D, kv)
    kc = torch.from_numpy(kc_o.view(np.int16) if kv == "bf16" else kc_o.copy()).cuda()
    vc = torch.from_numpy(vc_o.view(np.int16) if kv == "bf16" else vc_o.copy()).cuda()
    if kv == "bf16":
        kc, vc = kc.view(torch.bfloat16), vc.view(torch.bfloat16)

    def write(slots, n):
        """n random bf16 K/V rows at `slots`, on both sides (each with its own implementation)."""
        k = W.f32_to_bf16_bits(rng.standard_normal((n, Hkv, D)).astype(np.float32))
        v = W.f32_to_bf16_bits(rng.standard_normal((n, Hkv, D)).astype(np.float32))
        sl = np.asarray(slots, dtype=np.int64)
        oracle.reshape_and_cache(k, v, "bf16", kc_o, vc_o, kv, sl, Hkv, D, bs, NB, ks, vs)
        return k, v, sl

    # prompts, then forks: 3 and 4 share 0's blocks (last one partly filled), 5 shares 2's (full)
    prompts = {0: bs + 5, 1: 2 * bs + 1, 2: 2 * bs}
    for sid, L in prompts.items():
        assert bm.add(sid, L) == 0
        st, tables, lens = bm.tables([sid])
        slots = [int(tables[0][p // bs]) * bs + p % bs for p in range(L)]
        k, v, sl = write(slots, L)
        pkv.reshape_and_cache(to_dev(k, "bf16"), to_dev(v, "bf16"), kc, vc, torch.from_numpy(sl).cuda(),
                              float(ks), float(vs))
    for parent, child in ((0, 3), (0, 4), (2, 5)):
        assert bm.fork(parent, child) == 0
    ids = [0, 1, 2, 3, 4, 5]
    n_cow = 0
    for step in range(2 * bs + 3):
        st, slots, tables, lens, cows, n_done = bm.step(ids)
        assert st == 0 and n_done == len(ids)
        n_cow += len(cows)
        for src, dst in cows.tolist():    # copy on write: the caller copies the shared block first
            kc[dst].copy_(kc[src])
            vc[dst].copy_(vc[src])
            kc_o[dst] = kc_o[src]
            vc_o[dst] = vc_o[src]
        k, v, sl = write(slots, len(ids))
        q = W.f32_to_bf16_bits(rng.standard_normal((len(ids), Hq, D)).astype(np.float32))
        out = torch.empty((len(ids), Hq, D), dtype=torch.bfloat16, device="cuda")
        ws = pkv.new_workspace(len(ids), Hq, Hkv, D, 0)
        pkv.paged_decode_step(out, to_dev(q, "bf16"), kc, vc, torch.from_numpy(tables).cuda(),
                              torch.from_numpy(lens).cuda(), to_dev(k, "bf16"), to_dev(v, "bf16"),
                              torch.from_numpy(sl).cuda(), float(scale), float(ks), float(vs), 0, ws)
        torch.cuda.synchronize()
        assert pkv.read_device_error(ws) == 0
        ref = oracle.paged_decode(q, "bf16", kc_o, vc_o, kv, tables, lens, Hq, Hkv, D, bs, NB, scale, ks, vs)
        assert max_err(out, ref) <= TOL[kv], step
        assert np.array_equal(cache_bytes(kc), kc_o) and np.array_equal(cache_bytes(vc), vc_o), step
    assert n_cow == 2   # 0 and 3 each copy the shared, partly filled last block; 4 then holds it alone
    for sid in ids:
        assert bm.free(sid) == 0
    assert bm.num_free() == NB

"""The C ABI without a GPU: the library loads, exports every declared symbol and
rejects bad host-visible arguments before touching a device."""
import ctypes
import os
import re

import pytest

import paged_kv_cache_462_b200 as pkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
           if h.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"PKV_API\s+[\w\s\*]+?\b(\w+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_462_b200 import build
    build.build()
    return pkv.load_library()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) >= {"paged_attention_decode", "reshape_and_cache", "paged_attention_workspace_size",
                          "paged_decode_step", "pkv_bm_create", "pkv_bm_step"}
    for n in names:
        assert hasattr(lib, n), n


def test_fp8_kernel_choice(lib):
    """The process-wide FP8 kernel choice: unknown values rejected, the previous value returned."""
    assert lib.pkv_set_fp8_kernel(7) == -2
    assert lib.pkv_set_fp8_kernel(-1) == -2
    prev = lib.pkv_set_fp8_kernel(pkv.FP8_KERNEL_TCGEN05)
    assert prev == pkv.FP8_KERNEL_MMA                      # the default
    assert lib.pkv_set_fp8_kernel(pkv.FP8_KERNEL_MMA) == pkv.FP8_KERNEL_TCGEN05
    assert pkv.set_fp8_kernel(pkv.FP8_KERNEL_MMA) == pkv.FP8_KERNEL_MMA
    with pytest.raises(pkv.PkvError):
        pkv.set_fp8_kernel(3)


def test_status_strings(lib):
    for code in range(7):
        assert pkv.status_string(code)
    assert pkv.status_string(0) == "ok"


def test_workspace_size_with_explicit_partitions(lib):
    # 64 seqs, 32/8 heads, d=128, 296 runs of up to 5 chunks: header + counters + a completion stamp per
    # chunk (296 * 5 * 8 bytes, rounded to 256) + (296 * 5 * 4 + 512) slots of 4*(128+2) floats
    n = lib.paged_attention_workspace_size(64, 32, 8, 128, 296)
    slot = 4 * (128 + 2)
    assert n == 256 + 2048 + (296 * 5 * 8 + 255) // 256 * 256 + (296 * 5 * 4 + 512) * slot * 4
    assert lib.paged_attention_workspace_size(64, 30, 8, 128, 296) == 0     # 30 % 8 != 0
    assert lib.paged_attention_workspace_size(64, 24, 8, 128, 296) == 0     # group 3 unsupported
    assert lib.paged_attention_workspace_size(64, 32, 8, 96, 296) == 0      # head_dim 96 unsupported


def _decode(lib, **kw):
    a = dict(out=None, q=None, k=None, v=None, bt=None, sl=None, S=4, Hq=8, Hkv=2, D=64, BS=16, scale=0.125,
             MB=4, NB=32, qdt=0, kvdt=0, ks=1.0, vs=1.0, parts=0, ws=None, wsb=0, stream=None)
    a.update(kw)
    return lib.paged_attention_decode(a["out"], a["q"], a["k"], a["v"], a["bt"], a["sl"], a["S"], a["Hq"], a["Hkv"],
                                      a["D"], a["BS"], a["scale"], a["MB"], a["NB"], a["qdt"], a["kvdt"], a["ks"],
                                      a["vs"], a["parts"], a["ws"], a["wsb"], a["stream"])


FAKE = 0x10000  # never dereferenced: every case below fails host validation first


def test_decode_host_validation(lib):
    ptrs = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, sl=FAKE, ws=FAKE, wsb=1 << 20)
    assert _decode(lib, **ptrs, Hq=6, Hkv=4) == 2          # heads not a multiple
    assert _decode(lib, **ptrs, D=96) == 2                  # head_dim
    assert _decode(lib, **ptrs, BS=12) == 2                 # block size
    assert _decode(lib, **ptrs, qdt=1, kvdt=0) == 3         # dtype pair
    assert _decode(lib, **ptrs, qdt=2, kvdt=2) == 3
    assert _decode(lib, **dict(ptrs, q=None)) == 1          # null
    assert _decode(lib, **dict(ptrs, ws=None)) == 4         # no workspace
    assert _decode(lib, **ptrs, MB=0) == 2
    assert _decode(lib, **dict(ptrs, k=FAKE + 8)) == 2      # misaligned cache for the bulk copies
    assert _decode(lib, S=0) == 0                           # empty batch: nothing to do


def test_append_host_validation(lib):
    f = lib.reshape_and_cache
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 96, 16, 8, 0, 0, 1.0, 1.0, None, None) == 2
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, 1, 0, 1.0, 1.0, None, None) == 3   # bf16 -> f32
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, 2, 2, 1.0, 1.0, None, None) == 3   # e4m3 input
    assert f(FAKE, FAKE, FAKE, FAKE, None, 4, 2, 64, 16, 8, 0, 0, 1.0, 1.0, None, None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, 1, 2, 0.0, 1.0, None, None) == 2   # zero fp8 scale
    assert f(None, None, None, None, None, 0, 2, 64, 16, 8, 0, 0, 1.0, 1.0, None, None) == 0   # nothing to append


def test_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 8, 64)
    kc = torch.zeros(4, 2, 16, 64)
    with pytest.raises(ValueError):
        pkv.paged_attention_decode(q.clone(), q, kc, kc.clone(), torch.zeros(1, 4, dtype=torch.int32),
                                   torch.ones(1, dtype=torch.int32), 0.125, workspace=torch.zeros(1 << 20, dtype=torch.uint8))


def test_multi_query_and_head_scale_host_validation(lib):
    mq = lib.paged_attention_decode_mq
    args = lambda **kw: [kw.get(n, d) for n, d in (
        ("out", FAKE), ("q", FAKE), ("k", FAKE), ("v", FAKE), ("bt", FAKE), ("sl", FAKE), ("S", 4), ("QL", 2),
        ("Hq", 8), ("Hkv", 2), ("D", 128), ("BS", 16), ("scale", 0.1), ("MB", 4), ("NB", 32), ("qdt", 1),
        ("kvdt", 1), ("ks", 1.0), ("vs", 1.0), ("parts", 0), ("ws", FAKE), ("wsb", 1 << 20), ("stream", None))]
    assert mq(*args(QL=0)) == 2 and mq(*args(QL=9)) == 2      # 1 <= q_len <= 8
    assert mq(*args(QL=3, Hq=4)) == 2                          # 3 tokens x 2 heads = 6 columns
    assert mq(*args(QL=2, BS=8)) == 2                          # tensor-core shapes only
    assert mq(*args(QL=2, qdt=0, kvdt=0)) == 2                 # f32: no multi-query form
    hs = lib.paged_attention_decode_head_scales
    base = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 2, 128, 16, 0.1, 4, 32, 1]
    assert hs(*base, 2, None, FAKE, 0, FAKE, 1 << 20, None) == 1             # a scale array missing
    assert hs(*base, 1, FAKE, FAKE, 0, FAKE, 1 << 20, None) == 2             # bf16 cache: no head scales
    rc = lib.reshape_and_cache_head_scales
    assert rc(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, 1, 1, FAKE, FAKE, None, None) == 3   # bf16 cache
    assert rc(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, 1, 4, None, FAKE, None, None) == 1   # null scales


def test_int8_and_e5m2_dtype_pairs(lib):
    ptrs = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, sl=FAKE, ws=FAKE, wsb=1 << 20)
    assert _decode(lib, **ptrs, qdt=0, kvdt=4) == 3            # f32 q with an INT8 cache
    assert _decode(lib, **ptrs, qdt=4, kvdt=4) == 3            # INT8 q
    assert _decode(lib, **ptrs, qdt=3, kvdt=3) == 3            # E5M2 q
    f = lib.reshape_and_cache
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, 1, 4, 0.0, 1.0, None, None) == 2   # zero INT8 scale
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 64, 16, 8, 4, 4, 1.0, 1.0, None, None) == 3   # INT8 input rows


def _shared(lib, **kw):
    a = dict(S=4, Hq=8, Hkv=2, D=128, BS=16, MB=4, NB=32, qdt=1, kvdt=1, groups=1, max_group=4, parts=7,
             ptr=ctypes.c_void_p(16), ws=ctypes.c_void_p(256), wsb=1 << 30)
    a.update(kw)
    p = a["ptr"]
    return lib.paged_attention_decode_shared_prefix(p, p, p, p, p, p, a["S"], a["Hq"], a["Hkv"], a["D"], a["BS"],
                                                    0.1, a["MB"], a["NB"], a["qdt"], a["kvdt"], 1.0, 1.0, p, p, p, p,
                                                    a.get("shared", p), a["groups"], a["max_group"], a["parts"],
                                                    a["ws"], a["wsb"], None)


def test_shared_prefix_host_validation(lib):
    """Shared-prefix decode: rejected before any device access."""
    assert _shared(lib, max_group=9) == 2                  # 9 members x 4 query heads > 32 columns
    assert _shared(lib, max_group=0) == 2
    assert _shared(lib, groups=5) == 2                     # more groups than sequences
    assert _shared(lib, groups=-1) == 2
    assert _shared(lib, Hq=16, max_group=5) == 2           # 5 x 8 > 32
    assert _shared(lib, qdt=0, kvdt=0) == 3                # f32 caches: no tensor-core kernel
    assert _shared(lib, BS=8) == 2                         # block 8: no tensor-core kernel
    assert _shared(lib, shared=ctypes.c_void_p(None)) == 1
    assert _shared(lib, S=0, groups=0) == 0                # nothing to do


def test_shared_prefix_workspace_size(lib):
    base = lib.paged_attention_workspace_size(64, 32, 8, 128, 296)
    n = lib.paged_attention_shared_prefix_workspace_size(64, 32, 8, 128, 8, 296)
    slot = 4 * 8 * (128 + 2)                               # 8 columns x (d + 2) floats
    assert n == (base + 255) // 256 * 256 + (296 * 5 + 8 * 8) * 4 * slot
    assert lib.paged_attention_shared_prefix_workspace_size(64, 32, 8, 128, 0, 296) == (base + 255) // 256 * 256
    assert lib.paged_attention_shared_prefix_workspace_size(64, 32, 8, 128, -1, 296) == 0
    assert lib.paged_attention_shared_prefix_workspace_size(64, 24, 8, 128, 4, 296) == 0

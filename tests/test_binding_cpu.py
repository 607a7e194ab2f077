"""The Python binding's marshalling, on the CPU: tensors that claim to live on a CUDA device
(their storage stays on the host and is never read) and a stand-in for the C library that
records each call. Checks the C argument order, the device and contiguity checks, and the
per-stream cached workspace. No GPU and no kernel launch."""
import ctypes

import pytest
import torch

import paged_kv_cache_462_b200 as pkv


class FakeCuda(torch.Tensor):
    """A host tensor that reports itself as living on cuda:<_dev>."""
    _dev = 0

    @property
    def is_cuda(self):
        return True

    @property
    def device(self):
        return torch.device("cuda", self._dev)


def cuda(t, dev=0):
    f = torch.Tensor._make_subclass(FakeCuda, t)
    f._dev = dev
    return f


class FakeLib:
    """Records every C call as (name, args); returns `status`."""

    def __init__(self):
        self.calls = []
        self.status = 0

    def __getattr__(self, name):
        if name.startswith("__"):
            raise AttributeError(name)

        def call(*args):
            self.calls.append((name, args))
            if name == "paged_attention_workspace_size":
                return 1 << 16
            if name == "pkv_status_string":
                return b"stand-in"
            return self.status
        return call


class Stream:
    def __init__(self, handle):
        self.cuda_stream = handle


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(pkv, "load_library", lambda: lib)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: Stream(0))
    monkeypatch.setattr(pkv, "_ws_cache", {})
    return lib


def decode_inputs(S=3, Hq=8, Hkv=2, D=64, NB=10, BS=16, MB=4, dev=0, kv=torch.bfloat16):
    return dict(out=cuda(torch.zeros(S, Hq, D, dtype=torch.bfloat16), dev),
                q=cuda(torch.zeros(S, Hq, D, dtype=torch.bfloat16), dev),
                k_cache=cuda(torch.zeros(NB, Hkv, BS, D, dtype=kv), dev),
                v_cache=cuda(torch.zeros(NB, Hkv, BS, D, dtype=kv), dev),
                block_tables=cuda(torch.zeros(S, MB, dtype=torch.int32), dev),
                seq_lens=cuda(torch.ones(S, dtype=torch.int32), dev))


def test_decode_argument_order(fake):
    x = decode_inputs()
    ws = cuda(torch.zeros(1 << 16, dtype=torch.uint8))
    pkv.paged_attention_decode(**x, scale=0.125, k_scale=2.0, v_scale=3.0, num_partitions=7, workspace=ws,
                               stream=Stream(1234))
    name, a = fake.calls[-1]
    assert name == "paged_attention_decode"
    assert [v.value for v in a[:6]] == [x[n].data_ptr() for n in ("out", "q", "k_cache", "v_cache", "block_tables",
                                                                  "seq_lens")]
    assert a[6:19] == (3, 8, 2, 64, 16, 0.125, 4, 10, pkv.BF16, pkv.BF16, 2.0, 3.0, 7)
    assert a[19].value == ws.data_ptr() and a[20] == ws.numel() and a[21].value == 1234


@pytest.mark.parametrize("kv, code", [(torch.uint8, pkv.FP8_E4M3), (torch.float8_e4m3fn, pkv.FP8_E4M3),
                                      (torch.float8_e5m2, pkv.FP8_E5M2), (torch.int8, pkv.INT8)])
def test_cache_dtype_codes(fake, kv, code):
    x = decode_inputs(kv=kv)
    pkv.paged_attention_decode(**x, scale=0.1, workspace=cuda(torch.zeros(1 << 16, dtype=torch.uint8)))
    assert fake.calls[-1][1][15] == code


def test_refuses_host_foreign_device_and_strided_tensors(fake):
    ws = cuda(torch.zeros(1 << 16, dtype=torch.uint8))
    x = decode_inputs()
    x["q"] = torch.zeros(3, 8, 64, dtype=torch.bfloat16)                 # host tensor
    with pytest.raises(ValueError, match="CUDA tensor"):
        pkv.paged_attention_decode(**x, scale=0.1, workspace=ws)
    x = decode_inputs()
    x["k_cache"] = cuda(torch.zeros(10, 2, 16, 64, dtype=torch.bfloat16), dev=1)
    with pytest.raises(ValueError, match="cuda:1"):
        pkv.paged_attention_decode(**x, scale=0.1, workspace=ws)
    x = decode_inputs()
    x["block_tables"] = cuda(torch.zeros(4, 3, dtype=torch.int32)).t()   # [3, 4], not contiguous
    with pytest.raises(ValueError, match="contiguous"):
        pkv.paged_attention_decode(**x, scale=0.1, workspace=ws)
    k = cuda(torch.zeros(5, 2, 64, dtype=torch.bfloat16))
    kc = cuda(torch.zeros(10, 2, 16, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="slot_mapping is on cuda:1"):
        pkv.reshape_and_cache(k, k.clone(), kc, kc.clone(), cuda(torch.zeros(5, dtype=torch.int64), dev=1))
    assert not [c for c in fake.calls if c[0] in ("paged_attention_decode", "reshape_and_cache")]


def test_cached_workspace_per_stream(fake, monkeypatch):
    made = []
    real_empty = torch.empty

    def empty(n, dtype=None, device=None):
        assert device == torch.device("cuda", 0)
        t = cuda(real_empty(n, dtype=dtype))
        made.append(t)
        return t
    monkeypatch.setattr(torch, "empty", empty)
    x = decode_inputs()
    for h in (11, 11, 22):
        pkv.paged_attention_decode(**x, scale=0.1, stream=Stream(h))
    assert len(made) == 2                                   # one workspace per stream, reused on stream 11
    inits = [a for n, a in fake.calls if n == "pkv_workspace_init"]
    assert [a[2].value for a in inits] == [11, 22]          # zeroed on the stream that uses it
    used = [a[19].value for n, a in fake.calls if n == "paged_attention_decode"]
    assert used == [made[0].data_ptr(), made[0].data_ptr(), made[1].data_ptr()]


def test_multi_query_workspace_and_order(fake):
    S, QL, Hq, Hkv, D = 2, 2, 8, 2, 128
    q = cuda(torch.zeros(S, QL, Hq, D, dtype=torch.bfloat16))
    kc = cuda(torch.zeros(6, Hkv, 16, D, dtype=torch.bfloat16))
    pkv.paged_attention_decode_mq(q.clone(), q, kc, kc.clone(), cuda(torch.zeros(S, 3, dtype=torch.int32)),
                                  cuda(torch.ones(S, dtype=torch.int32)), 0.1,
                                  workspace=cuda(torch.zeros(1 << 16, dtype=torch.uint8)))
    name, a = fake.calls[-1]
    assert name == "paged_attention_decode_mq" and a[6:12] == (S, QL, Hq, Hkv, D, 16)


def test_head_scales_replace_per_tensor_scales(fake):
    x = decode_inputs(kv=torch.uint8)
    ks, vs = cuda(torch.ones(2)), cuda(torch.ones(2))
    pkv.paged_attention_decode_head_scales(**x, scale=0.1, k_head_scales=ks, v_head_scales=vs,
                                           workspace=cuda(torch.zeros(1 << 16, dtype=torch.uint8)))
    name, a = fake.calls[-1]
    assert name == "paged_attention_decode_head_scales"
    assert (a[16].value, a[17].value) == (ks.data_ptr(), vs.data_ptr())
    with pytest.raises(TypeError):
        pkv.paged_attention_decode_head_scales(**x, scale=0.1, k_head_scales=cuda(torch.ones(3)), v_head_scales=vs,
                                               workspace=cuda(torch.zeros(1 << 16, dtype=torch.uint8)))


def test_status_becomes_exception(fake):
    fake.status = 2
    with pytest.raises(pkv.PkvError) as e:
        pkv.paged_attention_decode(**decode_inputs(), scale=0.1,
                                   workspace=cuda(torch.zeros(1 << 16, dtype=torch.uint8)))
    assert e.value.status == 2

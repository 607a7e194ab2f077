"""bench.py contract pieces that run without a GPU: the reference (CPU oracle) arm's JSON line
and the byte accounting the roofline uses, pinned to the pages' arithmetic."""
import json
import os
import subprocess
import sys

import numpy as np

from paged_kv_cache_462_b200 import accounting as acct

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_kv_bytes_per_token_matches_the_pages():
    # 32 layers x 8 KV heads x 128 x 2 (K,V) x 2 bytes = 131072 B = 128 KB; 4 KB per layer
    # ("vLLM inference cost optimisation", section 2.1; wzjinhao.cn write-up, section 2.1)
    assert acct.kv_bytes_per_token(32, 8, 128, 2) == 131072
    assert acct.kv_bytes_per_token(1, 8, 128, 2) == 4096
    # 8192 tokens x 128 KB = 1 GiB, "about 1 GB" per 8K-token request
    assert 8192 * acct.kv_bytes_per_token(32, 8, 128, 2) == 1 << 30


def test_decode_bytes_counts_shared_blocks_once():
    bt = np.array([[3, 5, -1], [3, 7, -1]], np.int32)     # block 3 shared
    sl = np.array([20, 17], np.int32)                       # 2 blocks each at block size 16
    d = acct.decode_bytes(sl, bt, 8, 2, 64, 16, "bf16", "bf16")
    per_tok = 2 * 2 * 64 * 2
    assert d["unique_blocks"] == 3
    assert d["kv_unique"] == 3 * 16 * per_tok
    assert d["kv_logical"] == 37 * per_tok
    assert d["q_out"] == 2 * 2 * 8 * 64 * 2
    assert d["tables"] == 4 * 4 + 2 * 4
    assert d["total"] == d["kv_unique"] + d["q_out"] + d["tables"]


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "5",
                        "--warmup", "1", "--config", "0"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["steps"] == 5 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_oracle_timing_on_all_cores():
    """The all-cores oracle sample: every thread does work, the attention-only bytes are the
    decode accounting of that sequence, and the same problems run on one or more threads."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    b = W.config_batch(0)
    items = bench.oracle_pair_sampler(b)
    run, nbytes, L, attend, attn_bytes = items[0]
    assert nbytes > attn_bytes > 0
    one = bench.time_oracle_threads(items, 0.3, 1)
    many = bench.time_oracle_threads(items, 0.3, 4)
    assert one[0] > 0 and one[1] > 0 and many[1] >= 4


def test_prefix_sharing_choice():
    """`--prefix-sharing auto` takes the shared-prefix step for bf16 caches of workloads that share
    prefix blocks and the plain step for 8-bit caches; `on` / `off` override it, and multi-query
    decode and f32 caches never take it."""
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    import workloads as W
    spec = W.config_spec(3)
    assert spec.share_group > 1 and spec.kv_dtype == "bf16"

    def args(mode="auto", q_len=1):
        return argparse.Namespace(prefix_sharing=mode, q_len=q_len)

    def typed(kv):
        s = W.config_spec(3)
        s.kv_dtype = kv
        return s

    assert bench.use_prefix_plan(args(), spec)
    for kv in ("e4m3", "e5m2", "int8"):
        assert not bench.use_prefix_plan(args(), typed(kv))
        assert bench.use_prefix_plan(args("on"), typed(kv))
    assert not bench.use_prefix_plan(args("off"), spec)
    assert not bench.use_prefix_plan(args(q_len=2), spec)
    assert not bench.use_prefix_plan(args("on"), typed("f32"))
    assert not bench.use_prefix_plan(args(), W.config_spec(2))   # no shared prefixes

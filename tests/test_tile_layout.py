"""Compile-time checks of the 8-bit consumer's token order within a 16-token tile (no GPU).

The warp-MMA kernel reads the K rows of a tile in the order tok_of_row and the V rows (through
the transposed byte ldmatrix) in the order v_tok. The p.V product is only right if, for every
lane (g, t), the P^T word it receives from the q.K accumulators holds exactly the two tokens its
MMA k pair multiplies:

* m16n8k16 B operand b0 = k (2t, 2t + 1), b1 = k (2t + 8, 2t + 9) of column g;
* the transposed byte load gives lane (g, t) bytes 0..3 = rows 4t .. 4t + 3 of the V tile, the
  low half feeding k (2t, 2t + 1) and the high half k (2t + 8, 2t + 9);
* the q.K accumulator of lane (g', t') holds rows g' and g' + 8, and lane 4(2t) + g/2 packs its
  two rows into one word (row g' low), as does lane 4(2t + 1) + g/2.

So v_tok(4t), v_tok(4t + 1) must be the tokens of q.K rows 2t, 2t + 8 and v_tok(4t + 2),
v_tok(4t + 3) those of rows 2t + 1, 2t + 9. Both orders must be permutations of the 16 tokens,
and each group of 8 rows a single ldmatrix phase reads must fall on 8 distinct 16-byte positions
of the 128-byte swizzle (token & 7), or the loads conflict on shared-memory banks. The checks are
static_asserts on the kernel header's own constexpr functions, compiled by nvcc for sm_100a."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "paged_kv_cache_462_b200", "csrc")

CHECK = r"""
#include "decode_mma.cuh"

namespace {
using pkv::tok_of_row;
using pkv::v_tok;

constexpr bool permutations()
{
    bool k[16] = {}, v[16] = {};
    for (int r = 0; r < 16; ++r) {
        const int a = tok_of_row(r), b = v_tok(r);
        if (a < 0 || a > 15 || b < 0 || b > 15 || k[a] || v[b])
            return false;
        k[a] = v[b] = true;
    }
    return true;
}

constexpr bool pv_pairs_match_scores()
{
    for (int t = 0; t < 4; ++t)
        if (v_tok(4 * t) != tok_of_row(2 * t) || v_tok(4 * t + 1) != tok_of_row(2 * t + 8) ||
            v_tok(4 * t + 2) != tok_of_row(2 * t + 1) || v_tok(4 * t + 3) != tok_of_row(2 * t + 9))
            return false;
    return true;
}

constexpr bool swizzle_positions_distinct()
{
    for (int half = 0; half < 2; ++half) {
        bool k[8] = {}, v[8] = {};
        for (int i = 0; i < 8; ++i) {
            const int a = tok_of_row(8 * half + i) & 7, b = v_tok(8 * half + i) & 7;
            if (k[a] || v[b])
                return false;
            k[a] = v[b] = true;
        }
    }
    return true;
}
}  // namespace

static_assert(permutations(), "tile token orders must be permutations of 0..15");
static_assert(pv_pairs_match_scores(), "P^T words must carry the tokens of the p.V k pairs");
static_assert(swizzle_positions_distinct(), "8-row ldmatrix phases must hit distinct swizzle positions");
"""

MUTANT = r"""
#define tok_of_row tok_of_row_unused
#include "decode_mma.cuh"
#undef tok_of_row
// the q.K row order without the permutation: the pairing check must reject it
constexpr int tok_of_row(int r) { return r; }
constexpr bool pv_pairs_match_scores()
{
    for (int t = 0; t < 4; ++t)
        if (pkv::v_tok(4 * t) != tok_of_row(2 * t) || pkv::v_tok(4 * t + 1) != tok_of_row(2 * t + 8))
            return false;
    return true;
}
static_assert(pv_pairs_match_scores(), "expected to fail");
"""


def _compile(tmp_path, name, src):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    cu = tmp_path / f"{name}.cu"
    cu.write_text(src)
    return subprocess.run([nvcc, "-std=c++17", "--expt-relaxed-constexpr", "-gencode",
                           "arch=compute_100a,code=sm_100a", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                           "-c", str(cu), "-o", str(tmp_path / f"{name}.o")],
                          capture_output=True, text=True, timeout=300)


def test_tile_token_orders(tmp_path):
    r = _compile(tmp_path, "layout_check", CHECK)
    assert r.returncode == 0, r.stderr[-3000:]


def test_identity_row_order_is_rejected(tmp_path):
    r = _compile(tmp_path, "layout_mutant", MUTANT)
    assert r.returncode != 0 and "expected to fail" in r.stderr, r.stderr[-3000:]

// Shape dispatch of the warp-MMA decode kernels: run-time (head_dim, block size, group, head
// group) -> template instantiation, for one cache type per translation unit (decode_mma_*.cu).
#pragma once

#include "decode_mma.cuh"

namespace pkv {

template <class KV, int D, int BS, int G, int HG>
int mma_run(const MmaOp& op)
{
    using L = MmaLauncher<KV, __nv_bfloat16, D, BS, G, HG>;
    switch (op.kind) {
    case MmaOp::kLaunch:
        return L::launch(*op.p, op.nruns, op.stream);
    case MmaOp::kOccupancy:
        *op.occ = L::occupancy(op.p->num_seqs);
        return PKV_OK;
    case MmaOp::kLaunchSharedPrefix:
        return L::launch_shared_prefix(*op.p, *op.pp, op.nruns, op.runs_p, op.stream);
    case MmaOp::kPrefixOccupancy:
        *op.occ = MmaLauncher<KV, __nv_bfloat16, D, BS, 8, 1, true>::occupancy(op.p->num_seqs);
        return PKV_OK;
    default:
        return PKV_ERR_SHAPE;
    }
}

template <class KV, int D, int BS, int G>
int mma_by_hg(int HG, const MmaOp& op)
{
    switch (HG) {
    case 1: return mma_run<KV, D, BS, G, 1>(op);
    case 2: return mma_run<KV, D, BS, G, 2>(op);
    case 4: return mma_run<KV, D, BS, G, 4>(op);
    default: return PKV_ERR_SHAPE;
    }
}

template <class KV, int D, int BS>
int mma_by_g(int G, int HG, const MmaOp& op)
{
    switch (G) {
    case 1: return mma_by_hg<KV, D, BS, 1>(HG, op);
    case 2: return mma_by_hg<KV, D, BS, 2>(HG, op);
    case 4: return mma_by_hg<KV, D, BS, 4>(HG, op);
    case 5: return mma_by_hg<KV, D, BS, 5>(HG, op);
    case 8: return mma_by_hg<KV, D, BS, 8>(HG, op);
    default: return PKV_ERR_SHAPE;
    }
}

template <class KV, int D>
int mma_by_bs(int BS, int G, int HG, const MmaOp& op)
{
    switch (BS) {
    case 16: return mma_by_g<KV, D, 16>(G, HG, op);
    case 32: return mma_by_g<KV, D, 32>(G, HG, op);
    default: return PKV_ERR_SHAPE;
    }
}

// head_dim 128 for every cache type; 64 as well for bf16 caches (WITH_D64)
template <class KV, bool WITH_D64>
int mma_by_d(int D, int BS, int G, int HG, const MmaOp& op)
{
    if (D == 128)
        return mma_by_bs<KV, 128>(BS, G, HG, op);
    if constexpr (WITH_D64) {
        if (D == 64)
            return mma_by_bs<KV, 64>(BS, G, HG, op);
    }
    return PKV_ERR_SHAPE;
}

}  // namespace pkv

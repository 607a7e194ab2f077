// Instantiations of the warp-MMA paged decode kernels for KvBF16 caches.
#include "decode_mma_dispatch.cuh"

namespace pkv {

int decode_mma_dispatch_bf16(int D, int BS, int G, int HG, const MmaOp& op)
{
    return mma_by_d<KvBF16, true>(D, BS, G, HG, op);
}

}  // namespace pkv

// Instantiations of the warp-MMA paged decode kernels for KvE5M2 caches.
#include "decode_mma_dispatch.cuh"

namespace pkv {

int decode_mma_dispatch_e5m2(int D, int BS, int G, int HG, const MmaOp& op)
{
    return mma_by_d<KvE5M2, false>(D, BS, G, HG, op);
}

}  // namespace pkv

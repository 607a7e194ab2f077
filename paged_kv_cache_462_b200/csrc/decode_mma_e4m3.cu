// Instantiations of the warp-MMA paged decode kernels for KvE4M3 caches.
#include "decode_mma_dispatch.cuh"

namespace pkv {

int decode_mma_dispatch_e4m3(int D, int BS, int G, int HG, const MmaOp& op)
{
    return mma_by_d<KvE4M3, false>(D, BS, G, HG, op);
}

}  // namespace pkv

// Instantiations of the warp-MMA paged decode kernels for KvI8 caches.
#include "decode_mma_dispatch.cuh"

namespace pkv {

int decode_mma_dispatch_i8(int D, int BS, int G, int HG, const MmaOp& op)
{
    return mma_by_d<KvI8, false>(D, BS, G, HG, op);
}

}  // namespace pkv

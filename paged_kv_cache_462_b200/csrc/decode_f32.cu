// Instantiations of the paged decode kernel for KvF32 caches (one translation
// unit per cache dtype so the library builds in parallel).
#include "decode_kernel.cuh"

namespace pkv {

int decode_dispatch_f32(int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    return dispatch_d<KvF32, float>(D, BS, G, p, nruns, st, occ);
}

}  // namespace pkv

// Instantiations of the paged decode kernel for KvE4M3 caches (one translation
// unit per cache dtype so the library builds in parallel).
#include "decode_kernel.cuh"

namespace pkv {

int decode_dispatch_e4m3(int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    return dispatch_d<KvE4M3, __nv_bfloat16>(D, BS, G, p, nruns, st, occ);
}

}  // namespace pkv

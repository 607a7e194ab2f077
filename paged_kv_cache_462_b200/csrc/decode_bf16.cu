// Instantiations of the paged decode kernel for KvBF16 caches (one translation
// unit per cache dtype so the library builds in parallel).
#include "decode_kernel.cuh"

namespace pkv {

int decode_dispatch_bf16(int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    return dispatch_d<KvBF16, __nv_bfloat16>(D, BS, G, p, nruns, st, occ);
}

}  // namespace pkv

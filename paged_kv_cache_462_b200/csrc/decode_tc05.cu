// Instantiations of the tcgen05 paged decode kernel for FP8 (E4M3 / E5M2) caches.
#include "decode_tc05.cuh"

namespace pkv {

namespace {

template <class KV, int BS>
int by_g(int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    switch (G) {
#define PKV_TC_G(GG)                                                                      \
    case GG:                                                                              \
        if (occ) {                                                                        \
            *occ = TcLauncher<KV, __nv_bfloat16, BS, GG>::occupancy(p.num_seqs);          \
            return PKV_OK;                                                                \
        }                                                                                 \
        return TcLauncher<KV, __nv_bfloat16, BS, GG>::launch(p, nruns, st);
        PKV_TC_G(1)
        PKV_TC_G(2)
        PKV_TC_G(4)
        PKV_TC_G(5)
        PKV_TC_G(8)
#undef PKV_TC_G
    default:
        return PKV_ERR_SHAPE;
    }
}

template <class KV>
int by_bs(int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    switch (BS) {
    case 16: return by_g<KV, 16>(G, p, nruns, st, occ);
    case 32: return by_g<KV, 32>(G, p, nruns, st, occ);
    default: return PKV_ERR_SHAPE;
    }
}

}  // namespace

// FP8 caches with head_dim 128 and block size 16 or 32 on the tcgen05 kernel
int decode_tc05_dispatch(int kv_dtype, int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st,
                         int* occ)
{
    if (D != 128)
        return PKV_ERR_SHAPE;
    if (kv_dtype == PKV_FP8_E4M3)
        return by_bs<KvE4M3>(BS, G, p, nruns, st, occ);
    if (kv_dtype == PKV_FP8_E5M2)
        return by_bs<KvE5M2>(BS, G, p, nruns, st, occ);
    return PKV_ERR_DTYPE;
}

}  // namespace pkv

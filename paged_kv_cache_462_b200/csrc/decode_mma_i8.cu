// Instantiations of the warp-MMA paged decode kernel for KvI8 caches.
#include "decode_mma.cuh"

namespace pkv {

namespace {

template <int D, int BS, int G>
int by_hg(int HG, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    switch (HG) {
#define PKV_HG(H)                                                                          \
    case H:                                                                                \
        if (occ) {                                                                         \
            *occ = MmaLauncher<KvI8, __nv_bfloat16, D, BS, G, H>::occupancy(p.num_seqs);    \
            return PKV_OK;                                                                 \
        }                                                                                  \
        return MmaLauncher<KvI8, __nv_bfloat16, D, BS, G, H>::launch(p, nruns, st);
        PKV_HG(1)
        PKV_HG(2)
        PKV_HG(4)
#undef PKV_HG
    default:
        return PKV_ERR_SHAPE;
    }
}

template <int D, int BS>
int by_g(int G, int HG, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    switch (G) {
    case 1: return by_hg<D, BS, 1>(HG, p, nruns, st, occ);
    case 2: return by_hg<D, BS, 2>(HG, p, nruns, st, occ);
    case 4: return by_hg<D, BS, 4>(HG, p, nruns, st, occ);
    case 5: return by_hg<D, BS, 5>(HG, p, nruns, st, occ);
    case 8: return by_hg<D, BS, 8>(HG, p, nruns, st, occ);
    default: return PKV_ERR_SHAPE;
    }
}

template <int D>
int by_bs(int BS, int G, int HG, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    switch (BS) {
    case 16: return by_g<D, 16>(G, HG, p, nruns, st, occ);
    case 32: return by_g<D, 32>(G, HG, p, nruns, st, occ);
    default: return PKV_ERR_SHAPE;
    }
}

}  // namespace

int decode_mma_dispatch_i8(int D, int BS, int G, int HG, const DecodeParams& p, int nruns, cudaStream_t st, int* occ)
{
    switch (D) {
    case 128: return by_bs<128>(BS, G, HG, p, nruns, st, occ);
    default: return PKV_ERR_SHAPE;
    }
}

}  // namespace pkv

// Dispatch of paged_attention_decode to the kernel instantiation for the
// (q dtype, cache dtype) pair; the kernel itself is in decode_kernel.cuh.
#include "decode_kernel.cuh"

namespace pkv {

int decode_dispatch_f32(int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ);
int decode_dispatch_bf16(int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ);
int decode_dispatch_e4m3(int D, int BS, int G, const DecodeParams& p, int nruns, cudaStream_t st, int* occ);

int decode_dispatch(int q_dtype, int kv_dtype, int D, int BS, int G, const DecodeParams& p, int nruns,
                    cudaStream_t st, int* occupancy_out)
{
    if (q_dtype == PKV_F32 && kv_dtype == PKV_F32)
        return decode_dispatch_f32(D, BS, G, p, nruns, st, occupancy_out);
    if (q_dtype == PKV_BF16 && kv_dtype == PKV_BF16)
        return decode_dispatch_bf16(D, BS, G, p, nruns, st, occupancy_out);
    if (q_dtype == PKV_BF16 && kv_dtype == PKV_FP8_E4M3)
        return decode_dispatch_e4m3(D, BS, G, p, nruns, st, occupancy_out);
    return PKV_ERR_DTYPE;
}

float kv_unbias(int kv_dtype) { return kv_dtype == PKV_FP8_E4M3 ? kE4M3Unbias : 1.0f; }

}  // namespace pkv

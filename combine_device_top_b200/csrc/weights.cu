// weights.cu -- one-time preparation of expert weights (not on the per-step
// path): the fp16 copy of W_down used by the down projection.
//
// Every bf16 value whose magnitude lies in fp16's normal range
// [2^-14, 65504] is exactly representable in fp16 (8 significant bits fit in
// 11), so the copy is exact there; smaller magnitudes round to fp16's
// subnormal grid (spacing 2^-24), larger ones saturate to +-65504.
#include "mok_device.cuh"
#include "mok_internal.h"

namespace mok {

__global__ void __launch_bounds__(256) k_bf16_to_fp16(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                      size_t n_vec, const __nv_bfloat16* __restrict__ tail_src,
                                                      __half* __restrict__ tail_dst, int n_tail) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec; i += stride) {
        const uint4 v = __ldcs(src + i);
        const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&v);
        uint4 o;
        uint32_t* op = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(b[q]);
            op[q] = pack_half2_sat(f.x, f.y);
        }
        __stcs(dst + i, o);
    }
    if (blockIdx.x == 0 && (int)threadIdx.x < n_tail) {
        const float f = fminf(fmaxf(__bfloat162float(tail_src[threadIdx.x]), -65504.f), 65504.f);
        tail_dst[threadIdx.x] = __float2half_rn(f);
    }
}

cudaError_t launch_bf16_to_fp16(const void* src, void* dst, size_t n, int num_sms, cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const size_t n_vec = n / 8;
    const int n_tail = (int)(n - n_vec * 8);
    size_t want = (n_vec + 255) / 256;
    const size_t cap = (size_t)num_sms * 8;
    const int grid = (int)(want < 1 ? 1 : (want > cap ? cap : want));
    k_bf16_to_fp16<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst),
                                             n_vec, reinterpret_cast<const __nv_bfloat16*>(src) + n_vec * 8,
                                             reinterpret_cast<__half*>(dst) + n_vec * 8, n_tail);
    return cudaGetLastError();
}

}  // namespace mok

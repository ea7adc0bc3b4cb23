// mxfp8.cu -- standalone MXFP8 quantisers: activation rows (blocks of 32
// along each row) and weights (blocks of 32 along the contraction index K
// of each output column).  The forward's fused quantisation (gather, SwiGLU
// epilogue) uses the same device functions (mxfp8.cuh).
#include "mok_internal.h"
#include "mxfp8.cuh"

namespace mok {

template <class T>
__device__ __forceinline__ float mx_load(const T* p);
template <>
__device__ __forceinline__ float mx_load<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float mx_load<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Blocks along rows: one warp per row, each lane 8 consecutive elements, 4
// lanes per 32-element block (warp-uniform trip count; lanes past the end
// take part in the shuffles with zeros and store nothing).
template <class T>
__global__ void __launch_bounds__(256) k_mx_quant_rows(const T* __restrict__ src, int rows, int K,
                                                       uint8_t* __restrict__ q, uint8_t* __restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x / 32);
    for (int r = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
        const T* row = src + (size_t)r * K;
        for (int c0 = 0; c0 < K; c0 += 256) {
            const int c = c0 + lane * 8;
            const bool live = c < K;
            float v[8];
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                v[i] = live ? mx_load<T>(row + c + i) : 0.f;
                amax = fmaxf(amax, fabsf(v[i]));
            }
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            const int s = mx_block_exponent(amax);
            const float inv = mx_pow2(-s);
            if (live) {
                uint32_t w0 = 0, w1 = 0;
#pragma unroll
                for (int i = 0; i < 4; i += 2) {
                    w0 |= (uint32_t)mx_e4m3x2(v[i] * inv, v[i + 1] * inv) << (8 * i);
                    w1 |= (uint32_t)mx_e4m3x2(v[4 + i] * inv, v[5 + i] * inv) << (8 * i);
                }
                *reinterpret_cast<uint2*>(q + (size_t)r * K + c) = make_uint2(w0, w1);
                if ((lane & 3) == 0) scales[(size_t)r * (K / 32) + c / 32] = (uint8_t)(s + 127);
            }
        }
    }
}

// Blocks along K of each column: src [rows_total, N] with rows_total = E*K;
// one thread per (32-row block, column), columns fastest (coalesced).
__global__ void __launch_bounds__(256) k_mx_quant_cols(const __nv_bfloat16* __restrict__ src, int nblocks, int N,
                                                       uint8_t* __restrict__ q, uint8_t* __restrict__ scales) {
    const size_t total = (size_t)nblocks * N;
    for (size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (size_t)gridDim.x * blockDim.x) {
        const size_t b = t / N, n = t - b * N;
        const __nv_bfloat16* p = src + b * 32 * N + n;
        float v[32];
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            v[i] = __bfloat162float(p[(size_t)i * N]);
            amax = fmaxf(amax, fabsf(v[i]));
        }
        const int s = mx_block_exponent(amax);
        const float inv = mx_pow2(-s);
        uint8_t* qo = q + b * 32 * N + n;
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            const uint16_t pr = mx_e4m3x2(v[i] * inv, v[i + 1] * inv);
            qo[(size_t)i * N] = (uint8_t)(pr & 0xff);
            qo[(size_t)(i + 1) * N] = (uint8_t)(pr >> 8);
        }
        scales[t] = (uint8_t)(s + 127);
    }
}

cudaError_t launch_mx_quant_rows(const void* src, bool f32, int rows, int K, void* q, void* scales, int num_sms,
                                 cudaStream_t stream) {
    if (rows <= 0) return cudaSuccess;
    const int want = (rows + 7) / 8;
    const int grid = want < num_sms * 8 ? want : num_sms * 8;
    if (f32)
        k_mx_quant_rows<float><<<grid, 256, 0, stream>>>(reinterpret_cast<const float*>(src), rows, K,
                                                         reinterpret_cast<uint8_t*>(q),
                                                         reinterpret_cast<uint8_t*>(scales));
    else
        k_mx_quant_rows<__nv_bfloat16><<<grid, 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16*>(src), rows,
                                                                 K, reinterpret_cast<uint8_t*>(q),
                                                                 reinterpret_cast<uint8_t*>(scales));
    return cudaGetLastError();
}

cudaError_t launch_mx_quant_cols(const void* src, int nblocks, int N, void* q, void* scales, int num_sms,
                                 cudaStream_t stream) {
    if (nblocks <= 0 || N <= 0) return cudaSuccess;
    const size_t total = (size_t)nblocks * N;
    const size_t want = (total + 255) / 256;
    const int grid = (int)(want < (size_t)num_sms * 8 ? want : (size_t)num_sms * 8);
    k_mx_quant_cols<<<grid, 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16*>(src), nblocks, N,
                                              reinterpret_cast<uint8_t*>(q), reinterpret_cast<uint8_t*>(scales));
    return cudaGetLastError();
}

}  // namespace mok

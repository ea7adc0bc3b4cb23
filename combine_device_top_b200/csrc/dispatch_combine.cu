// dispatch_combine.cu -- step 3 (pull dispatch / gather) and step 5
// (weighted combine) of the forward MoE layer as standalone kernels.  The
// warp bodies are in dispatch_combine.cuh.
//
// Both kernels are HBM-bound streams of 16-byte vectors: one warp per token,
// a grid of a few CTAs per SM looping over the tokens.  The gather reads each
// token once and writes it to its k rows (T*H*2 bytes in, N_s*H*2 out); the
// combine reads N_s*H*4 bytes of fp32 per-slot outputs and writes T*H*2
// bytes of bf16 y, rounding once.
#include "dispatch_combine.cuh"
#include "mok_internal.h"

namespace mok {

constexpr int DC_THREADS = 256;

// Token-major form of the same copy: one warp per token reads the token's
// row once and writes it to each of its k rows (pos[t*k + j]).  Every source
// row is read from HBM once instead of k times (with 940 MB of rows streaming
// out, x does not stay in L2 between its k reads).
__global__ void __launch_bounds__(DC_THREADS) k_gather_tokens(ShardsIn xs, int S_r, int H, int T, int k,
                                                              const int32_t* __restrict__ pos,
                                                              uint4* __restrict__ rows) {
    const int lane = threadIdx.x & 31;
    const int nvec = H >> 3;
    const int warps = gridDim.x * (DC_THREADS / 32);
    for (int t = blockIdx.x * (DC_THREADS / 32) + (threadIdx.x >> 5); t < T; t += warps) {
        const int r = t / S_r;
        const uint4* src = reinterpret_cast<const uint4*>(xs.p[r]) + (size_t)(t - r * S_r) * nvec;
        const int my_row = lane < k ? __ldg(pos + (size_t)t * k + lane) : 0;
        int v0 = 0;
        for (; v0 + 128 <= nvec; v0 += 128) {  // warp-uniform trip count
            const int v = v0 + lane;
            const uint4 a = __ldg(src + v), b = __ldg(src + v + 32), c = __ldg(src + v + 64), d = __ldg(src + v + 96);
            for (int j = 0; j < k; ++j) {
                uint4* dst = rows + (size_t)__shfl_sync(0xffffffffu, my_row, j) * nvec;
                dst[v] = a;
                dst[v + 32] = b;
                dst[v + 64] = c;
                dst[v + 96] = d;
            }
        }
        // tail: lanes may differ in trip count, so no warp collectives here
        for (int v = v0 + lane; v < nvec; v += 32) {
            const uint4 a = __ldg(src + v);
            for (int j = 0; j < k; ++j) rows[(size_t)__ldg(pos + (size_t)t * k + j) * nvec + v] = a;
        }
    }
}

template <int KMAX>
__global__ void __launch_bounds__(DC_THREADS) k_combine(const float4* __restrict__ out, const float* __restrict__ gates,
                                                        int T, int k, int H, int S_r, ShardsOut ys) {
    const int lane = threadIdx.x & 31;
    const int nvec = H >> 3;
    const int warps = gridDim.x * (DC_THREADS / 32);
    for (int t = blockIdx.x * (DC_THREADS / 32) + (threadIdx.x >> 5); t < T; t += warps) {
        const int r = t / S_r;
        uint4* dst = reinterpret_cast<uint4*>(ys.p[r]) + (size_t)(t - r * S_r) * nvec;
        warp_combine_token<KMAX>(out, gates, t, k, nvec, dst, lane);
    }
}

cudaError_t launch_gather(const ShardsIn& xs, int S_r, int H, int T, int k, const int32_t* pos, void* rows,
                          int num_sms, cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    const int want = (T + (DC_THREADS / 32) - 1) / (DC_THREADS / 32);
    const int grid = want < num_sms * 8 ? want : num_sms * 8;
    k_gather_tokens<<<grid, DC_THREADS, 0, stream>>>(xs, S_r, H, T, k, pos, reinterpret_cast<uint4*>(rows));
    return cudaGetLastError();
}

cudaError_t launch_combine(const void* out, const float* gates, int T, int k, int H, int S_r, const ShardsOut& ys,
                           int num_sms, cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    const int want = (T + (DC_THREADS / 32) - 1) / (DC_THREADS / 32);
    const int grid = want < num_sms * 8 ? want : num_sms * 8;
    const float4* o = reinterpret_cast<const float4*>(out);
    if (k <= 2)
        k_combine<2><<<grid, DC_THREADS, 0, stream>>>(o, gates, T, k, H, S_r, ys);
    else
        k_combine<8><<<grid, DC_THREADS, 0, stream>>>(o, gates, T, k, H, S_r, ys);
    return cudaGetLastError();
}

}  // namespace mok

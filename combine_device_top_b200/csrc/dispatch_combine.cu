// dispatch_combine.cu -- step 3 (pull dispatch / gather) and step 5
// (weighted combine) of the forward MoE layer as standalone kernels.  The
// warp bodies are in dispatch_combine.cuh.
//
// Both kernels are HBM-bound streams of 16-byte vectors: one warp per row
// (gather) or per token (combine), a grid of a few CTAs per SM looping over
// the rows.  The gather reads each token k times (L2 absorbs part of the
// reuse) and writes N_s*H*2 bytes; the combine reads N_s*H*4 bytes of fp32
// per-slot outputs and writes T*H*2 bytes of bf16 y, rounding once.
#include "dispatch_combine.cuh"
#include "mok_internal.h"

namespace mok {

constexpr int DC_THREADS = 256;

__global__ void __launch_bounds__(DC_THREADS) k_gather(ShardsIn xs, int S_r, int H,
                                                       const int32_t* __restrict__ src_rank,
                                                       const int32_t* __restrict__ src_index, int n_rows,
                                                       uint4* __restrict__ rows) {
    const int lane = threadIdx.x & 31;
    const int nvec = H >> 3;  // 16-byte vectors per row
    const int warps = gridDim.x * (DC_THREADS / 32);
    for (int row = blockIdx.x * (DC_THREADS / 32) + (threadIdx.x >> 5); row < n_rows; row += warps) {
        const int r = __ldg(src_rank + row);
        const int i = __ldg(src_index + row);
        warp_copy_row(reinterpret_cast<const uint4*>(xs.p[r]) + (size_t)i * nvec, rows + (size_t)row * nvec, nvec,
                      lane);
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

cudaError_t launch_gather(const ShardsIn& xs, int S_r, int H, const int32_t* src_rank, const int32_t* src_index,
                          int n_rows, void* rows, int num_sms, cudaStream_t stream) {
    if (n_rows <= 0) return cudaSuccess;
    const int want = (n_rows + (DC_THREADS / 32) - 1) / (DC_THREADS / 32);
    const int grid = want < num_sms * 8 ? want : num_sms * 8;
    k_gather<<<grid, DC_THREADS, 0, stream>>>(xs, S_r, H, src_rank, src_index, n_rows,
                                              reinterpret_cast<uint4*>(rows));
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

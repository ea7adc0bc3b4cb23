// dispatch_combine.cu -- step 3 (pull dispatch / gather) and step 5
// (weighted combine) of the forward MoE layer as standalone kernels.
// The combine reads the fp32 per-slot expert outputs pushed by the down
// GEMM and rounds y to bf16 once.
//
// MoK article (tahou.com), pull paragraph: the GPU holding the experts reads
// the tokens it needs, knowing only the source rank and the offset there,
// and lays its memory out itself.  Push-combine paragraph: each result goes
// straight back to its token.  Benchmark paragraph: the layer ends with the
// weighted merge.
//
// Both kernels are HBM-bound streams of 16-byte vectors: one warp per row
// (gather) or per token (combine), a grid of a few CTAs per SM looping over
// the rows.  The gather reads each token k times (L2 absorbs part of the
// reuse) and writes N_s*H*2 bytes; the combine reads N_s*H*4 bytes and
// writes T*H*2.
#include "mok_device.cuh"
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
        const uint4* src = reinterpret_cast<const uint4*>(xs.p[r]) + (size_t)i * nvec;
        uint4* dst = rows + (size_t)row * nvec;
        int v = lane;
        for (; v + 96 < nvec; v += 128) {
            const uint4 a = __ldg(src + v), b = __ldg(src + v + 32), c = __ldg(src + v + 64), d = __ldg(src + v + 96);
            dst[v] = a;
            dst[v + 32] = b;
            dst[v + 64] = c;
            dst[v + 96] = d;
        }
        for (; v < nvec; v += 32) dst[v] = __ldg(src + v);
    }
}

// y[t] = bf16(sum_{j<k} g[t,j] * out[t,j,:]), fp32 (out is fp32), j ascending.
// Each lane owns 8 consecutive features: two 16-byte loads per slot, one
// 16-byte store.
template <int KMAX>
__global__ void __launch_bounds__(DC_THREADS) k_combine(const float4* __restrict__ out, const float* __restrict__ gates,
                                                        int T, int k, int H, int S_r, ShardsOut ys) {
    const int lane = threadIdx.x & 31;
    const int nvec = H >> 3;  // 8-feature groups per row
    const int warps = gridDim.x * (DC_THREADS / 32);
    for (int t = blockIdx.x * (DC_THREADS / 32) + (threadIdx.x >> 5); t < T; t += warps) {
        const float gl = (lane < k) ? __ldg(gates + (size_t)t * k + lane) : 0.f;
        float g[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) g[j] = __shfl_sync(0xffffffffu, gl, j);
        const float4* src = out + (size_t)t * k * (2 * nvec);
        const int r = t / S_r;
        uint4* dst = reinterpret_cast<uint4*>(ys.p[r]) + (size_t)(t - r * S_r) * nvec;
        for (int v = lane; v < nvec; v += 32) {
            float4 a[KMAX], b[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                if (j < k) {
                    a[j] = __ldcs(src + (size_t)j * 2 * nvec + 2 * v);
                    b[j] = __ldcs(src + (size_t)j * 2 * nvec + 2 * v + 1);
                }
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                if (j < k) {
                    acc[0] = fmaf(g[j], a[j].x, acc[0]);
                    acc[1] = fmaf(g[j], a[j].y, acc[1]);
                    acc[2] = fmaf(g[j], a[j].z, acc[2]);
                    acc[3] = fmaf(g[j], a[j].w, acc[3]);
                    acc[4] = fmaf(g[j], b[j].x, acc[4]);
                    acc[5] = fmaf(g[j], b[j].y, acc[5]);
                    acc[6] = fmaf(g[j], b[j].z, acc[6]);
                    acc[7] = fmaf(g[j], b[j].w, acc[7]);
                }
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            dst[v] = o;
        }
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
    else if (k <= 8)
        k_combine<8><<<grid, DC_THREADS, 0, stream>>>(o, gates, T, k, H, S_r, ys);
    else if (k <= 16)
        k_combine<16><<<grid, DC_THREADS, 0, stream>>>(o, gates, T, k, H, S_r, ys);
    else
        k_combine<MOK_MAX_TOPK><<<grid, DC_THREADS, 0, stream>>>(o, gates, T, k, H, S_r, ys);
    return cudaGetLastError();
}

}  // namespace mok

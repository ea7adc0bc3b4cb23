// dispatch_combine.cuh -- warp-level bodies of step 3 (pull dispatch: copy
// one token row from its source shard) and step 5 (fixed-order weighted
// combine of one token), shared by the standalone kernels
// (dispatch_combine.cu) and the persistent kernel (persistent.cu).
//
// MoK article (tahou.com), pull paragraph: the GPU holding the experts reads
// the tokens it needs, knowing only the source rank and the offset there.
// Push-combine paragraph: each result goes straight back to its token.
// Benchmark paragraph: the layer ends with the weighted merge.
#pragma once

#include "mok_device.cuh"

namespace mok {

// One warp copies one row of nvec 16-byte vectors, four loads in flight per lane.
__device__ __forceinline__ void warp_copy_row(const uint4* __restrict__ src, uint4* __restrict__ dst, int nvec,
                                              int lane) {
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

// One warp: y[t] = bf16(sum_{j<k} g[t,j] * out[t,j,:]) in fp32, j ascending.
// out is fp32 [T, k, H]; each lane owns 8 consecutive features (two 16-byte
// loads per slot, one 16-byte store).  nvec = H / 8.  Slots are loaded KB at
// a time (KB loads in flight), then accumulated in order.
template <int KB>
__device__ __forceinline__ void warp_combine_token(const float4* __restrict__ out, const float* __restrict__ gates,
                                                   int t, int k, int nvec, uint4* __restrict__ dst, int lane) {
    const float4* src = out + (size_t)t * k * (2 * nvec);
    const float* gt = gates + (size_t)t * k;
    // lanes may run different numbers of iterations (nvec % 32 != 0): no
    // warp collectives inside; the gates are broadcast loads (L1 hits)
    for (int v = lane; v < nvec; v += 32) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j0 = 0; j0 < k; j0 += KB) {
            float4 a[KB], b[KB];
            float g[KB];
#pragma unroll
            for (int jj = 0; jj < KB; ++jj) {
                const int j = j0 + jj;
                if (j < k) {
                    g[jj] = __ldg(gt + j);
                    a[jj] = __ldcs(src + (size_t)j * 2 * nvec + 2 * v);
                    b[jj] = __ldcs(src + (size_t)j * 2 * nvec + 2 * v + 1);
                }
            }
#pragma unroll
            for (int jj = 0; jj < KB; ++jj)
                if (j0 + jj < k) {
                    acc[0] = fmaf(g[jj], a[jj].x, acc[0]);
                    acc[1] = fmaf(g[jj], a[jj].y, acc[1]);
                    acc[2] = fmaf(g[jj], a[jj].z, acc[2]);
                    acc[3] = fmaf(g[jj], a[jj].w, acc[3]);
                    acc[4] = fmaf(g[jj], b[jj].x, acc[4]);
                    acc[5] = fmaf(g[jj], b[jj].y, acc[5]);
                    acc[6] = fmaf(g[jj], b[jj].z, acc[6]);
                    acc[7] = fmaf(g[jj], b[jj].w, acc[7]);
                }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        dst[v] = o;
    }
}

}  // namespace mok

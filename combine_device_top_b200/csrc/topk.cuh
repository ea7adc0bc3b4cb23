// topk.cuh -- the per-token body of step 1 (router top-k and gates), shared
// by the top-k kernel over given logits (plan.cu) and the router GEMM's
// epilogue (router.cu), so both select and weigh identically.
//
// MoK article (tahou.com), routing paragraph: the router sends every token
// to its k experts.  Selection: the k largest logits, ties to the lower
// expert index, in rank order; gates: softmax over the k selected logits.
#pragma once

#include "mok_device.cuh"

namespace mok {

__device__ __forceinline__ bool better(float v, int e, float bv, int be) {
    return v > bv || (v == bv && e < be);
}

// One warp, one token: the E logits at `row` (global or shared memory) are
// held in registers (lane owns experts c * 32 + lane, c < NC; ceil(E / 32)
// <= NC), k rounds of a warp arg-max pick the experts, lanes 0..k-1 write
// idx[j] and the softmax gate g[j].  All 32 lanes must call it.
template <int NC>
__device__ __forceinline__ void warp_topk_token(const float* row, int E, int k, int lane, int32_t* idx, float* g) {
    float v[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int e = c * 32 + lane;
        float x = -INFINITY;
        if (e < E) {
            x = row[e];
            if (x != x) x = -INFINITY;  // NaN compares as -inf
        }
        v[c] = x;
    }
    uint32_t taken = 0;
    int my_idx = 0;
    float my_val = 0.f, m = 0.f;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int e = c * 32 + lane;
            if (e < E && !((taken >> c) & 1u) && better(v[c], e, bv, be)) {
                bv = v[c];
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (better(ov, oe, bv, be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (j == 0) m = bv;
        if (lane == j) {
            my_idx = be;
            my_val = bv;
        }
    }
    // softmax over the k selected logits (the first is the maximum)
    float ex = (lane < k) ? expf(my_val - m) : 0.f;
    float s = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane < k) {
        idx[lane] = my_idx;
        g[lane] = ex / s;
    }
}

}  // namespace mok

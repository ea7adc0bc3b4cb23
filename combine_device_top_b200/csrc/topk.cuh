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
// <= NC), and k rounds of a warp arg-max pick the experts: lane j < k gets
// the j-th selected logit and its expert index + e_base (lanes past the
// experts there are get -inf and INT_MAX).  Returns the first selected (the
// maximum).  All 32 lanes must call it.
template <int NC>
__device__ __forceinline__ float warp_topk_select(const float* row, int E, int k, int lane, int e_base, float& my_val,
                                                  int& my_idx) {
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
    float m = 0.f;
    my_idx = 0x7fffffff;
    my_val = -INFINITY;
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
        if (be != 0x7fffffff && (be & 31) == lane) taken |= 1u << (be >> 5);
        if (j == 0) m = bv;
        if (lane == j) {
            my_idx = be == 0x7fffffff ? be : be + e_base;
            my_val = bv;
        }
    }
    return m;
}

// The k best of two selections (lane j < k holds the j-th of each, as
// warp_topk_select leaves them; expert indices distinct): the same k
// rounds of a warp arg-max over the 2k candidates, so the result is the
// selection over the union of their experts.  Returns the first selected.
__device__ __forceinline__ float warp_topk_merge(float a_val, int a_idx, float b_val, int b_idx, int k, int lane,
                                                 float& my_val, int& my_idx) {
    const float v[2] = {lane < k ? a_val : -INFINITY, lane < k ? b_val : -INFINITY};
    const int e[2] = {lane < k ? a_idx : 0x7fffffff, lane < k ? b_idx : 0x7fffffff};
    uint32_t taken = 0;
    float m = 0.f;
    my_idx = 0x7fffffff;
    my_val = -INFINITY;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            if (!((taken >> c) & 1u) && better(v[c], e[c], bv, be)) {
                bv = v[c];
                be = e[c];
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
#pragma unroll
        for (int c = 0; c < 2; ++c)
            if (be != 0x7fffffff && e[c] == be) taken |= 1u << c;
        if (j == 0) m = bv;
        if (lane == j) {
            my_idx = be;
            my_val = bv;
        }
    }
    return m;
}

// Softmax over the k selected logits (lane j < k holds the j-th; m is the
// first, the maximum); lanes 0..k-1 write idx[j] and the gate g[j].
__device__ __forceinline__ void warp_topk_gates(float my_val, int my_idx, float m, int k, int lane, int32_t* idx,
                                                float* g) {
    float ex = (lane < k) ? expf(my_val - m) : 0.f;
    float s = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane < k) {
        idx[lane] = my_idx;
        g[lane] = ex / s;
    }
}

// One warp, one token: the k experts of the E logits at `row` and their
// softmax gates; lanes 0..k-1 write idx[j] and g[j].  All 32 lanes must
// call it.
template <int NC>
__device__ __forceinline__ void warp_topk_token(const float* row, int E, int k, int lane, int32_t* idx, float* g) {
    float my_val;
    int my_idx;
    const float m = warp_topk_select<NC>(row, E, k, lane, 0, my_val, my_idx);
    warp_topk_gates(my_val, my_idx, m, k, lane, idx, g);
}

}  // namespace mok

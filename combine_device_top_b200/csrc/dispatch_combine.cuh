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
#include "mxfp8.cuh"

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

// Bulk stores allowed to be still reading shared memory while the next rows load.
constexpr int BULK_STORES_IN_FLIGHT = 4;

// One thread streams n rows of row_bytes through S shared-memory slots with
// bulk async copies: row i is loaded from src_row(i) into a slot and stored
// from there to dst_row(i).  About S - BULK_STORES_IN_FLIGHT rows load while
// the previous stores drain, so one thread keeps ~200 KB in flight.
// `loads` counts the loads ever issued through these slots (it fixes the
// mbarrier phases across calls) and is advanced.  Returns false if a wait
// gave up; the thread's own copies are drained either way before it returns,
// and every store has completed when it returns true.  Needs
// S > BULK_STORES_IN_FLIGHT.
template <class SrcF, class DstF>
__device__ __forceinline__ bool bulk_stream_rows(int n, SrcF src_row, DstF dst_row, uint32_t row_bytes,
                                                 unsigned char* slots, uint64_t* full, int S, uint32_t& loads,
                                                 DevStatus* st, uint64_t timeout_ns, uint64_t drain_ns) {
    constexpr int D = BULK_STORES_IN_FLIGHT;
    const uint32_t base = loads;
    int loaded = 0;
    for (; loaded < n && loaded < S; ++loaded) {
        const int slot = (int)((base + loaded) % (uint32_t)S);
        mbar_arrive_expect_tx(&full[slot], row_bytes);
        bulk_load(slots + (size_t)slot * row_bytes, src_row(loaded), row_bytes, &full[slot]);
    }
    bool ok = true;
    int s = 0;
    for (; s < n; ++s) {
        const uint32_t g = base + s;
        const int slot = (int)(g % (uint32_t)S);
        if (!mbar_wait(&full[slot], (g / (uint32_t)S) & 1u, st, timeout_ns, 70)) {
            ok = false;
            break;
        }
        bulk_store(dst_row(s), slots + (size_t)slot * row_bytes, row_bytes);
        bulk_commit();
        if (s >= D) {
            bulk_wait_read<D>();  // the store of row s - D has read its slot
            const int i = s - D + S;
            if (i < n) {
                const int slot2 = (int)((base + i) % (uint32_t)S);
                mbar_arrive_expect_tx(&full[slot2], row_bytes);
                bulk_load(slots + (size_t)slot2 * row_bytes, src_row(i), row_bytes, &full[slot2]);
                loaded = i + 1;
            }
        }
    }
    // a wait gave up: let every load already issued land before leaving
    for (int i = s; i < loaded; ++i) {
        const uint32_t g = base + i;
        mbar_wait(&full[g % (uint32_t)S], (g / (uint32_t)S) & 1u, nullptr, drain_ns, 71);
    }
    bulk_wait_all();
    loads = base + loaded;
    return ok;
}

// MXFP8 quantisation of 256 consecutive elements of a bf16 row by one warp
// (OCP MX: 32-element blocks, E8M0 scale, E4M3 values; mxfp8.cuh).  Lane l
// holds elements 8l .. 8l + 7 in raw (zeros past the row's end), so 4 lanes
// form a block.  Returns the lane's 8 E4M3 bytes in q and, in word, the 4
// block scales of the lane's half-warp (block 4g + b of the half-warp in
// byte b), valid on every lane.  All 32 lanes must call it.
__device__ __forceinline__ void warp_mx_quant8(const uint4& raw, uint2& q, uint32_t& word, int lane) {
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
    float v[8];
    float amax = 0.f;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float2 f = __bfloat1622float2(b2[p]);
        v[2 * p] = f.x;
        v[2 * p + 1] = f.y;
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int s = mx_block_exponent(amax);
    const float inv = mx_pow2(-s);
    q = make_uint2((uint32_t)mx_e4m3x2(v[0] * inv, v[1] * inv) | ((uint32_t)mx_e4m3x2(v[2] * inv, v[3] * inv) << 16),
                   (uint32_t)mx_e4m3x2(v[4] * inv, v[5] * inv) | ((uint32_t)mx_e4m3x2(v[6] * inv, v[7] * inv) << 16));
    const uint32_t sb = (uint32_t)(s + 127);
    const int h0 = lane & 16;
    word = __shfl_sync(0xffffffffu, sb, h0) | (__shfl_sync(0xffffffffu, sb, h0 + 4) << 8) |
           (__shfl_sync(0xffffffffu, sb, h0 + 8) << 16) | (__shfl_sync(0xffffffffu, sb, h0 + 12) << 24);
}

// Slot outputs as the grouped GEMM stores them: fp16 with one exponent per
// 128-feature block of a row (bf16 path, SlotF16S), bf16 (MXFP8 path) or
// fp32 (the backward's dx rows).  A lane owns 8 consecutive features of a
// slot row (v = index of the 8-feature group, block v / 16): load() issues
// the raw loads, widen() turns them into 8 floats.  The combine issues every
// load of a round before it widens any, so all of them are in flight.
struct SlotSrc {
    const void* out;     // [N_s, H] slot rows
    const int8_t* exps;  // SlotF16S: [N_s, H/128] block exponents
};
struct SlotF32 {
    struct Raw {
        float4 a, b;
    };
    __device__ static __forceinline__ Raw load(const SlotSrc& s, size_t row, int nvec, int v) {
        const float4* p = reinterpret_cast<const float4*>(s.out) + (row * nvec + v) * 2;
        return Raw{__ldcs(p), __ldcs(p + 1)};
    }
    __device__ static __forceinline__ void widen(const Raw& r, float (&f)[8]) {
        f[0] = r.a.x; f[1] = r.a.y; f[2] = r.a.z; f[3] = r.a.w;
        f[4] = r.b.x; f[5] = r.b.y; f[6] = r.b.z; f[7] = r.b.w;
    }
};
struct SlotBf16 {
    using Raw = uint4;
    __device__ static __forceinline__ Raw load(const SlotSrc& s, size_t row, int nvec, int v) {
        return __ldcs(reinterpret_cast<const uint4*>(s.out) + row * nvec + v);
    }
    __device__ static __forceinline__ void widen(const Raw& r, float (&f)[8]) {
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 x = __bfloat1622float2(b2[p]);
            f[2 * p] = x.x;
            f[2 * p + 1] = x.y;
        }
    }
};
struct SlotF16S {
    struct Raw {
        uint4 v;
        int e;
    };
    __device__ static __forceinline__ Raw load(const SlotSrc& s, size_t row, int nvec, int v) {
        return Raw{__ldcs(reinterpret_cast<const uint4*>(s.out) + row * nvec + v),
                   (int)__ldg(s.exps + row * (size_t)(nvec >> 4) + (v >> 4))};
    }
    __device__ static __forceinline__ void widen(const Raw& r, float (&f)[8]) {
        const __half2* h2 = reinterpret_cast<const __half2*>(&r.v);
        const float sc = __int_as_float((r.e + 127) << 23);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 x = __half22float2(h2[p]);
            f[2 * p] = x.x * sc;
            f[2 * p + 1] = x.y * sc;
        }
    }
};

// One warp: y[t] = bf16(sum_{j<k} g[t,j] * out[t,j,:]) in fp32, j ascending
// (gates == nullptr: every g = 1, the backward's reverse-dispatch sum).
// out is [T, k, H] of slot type S; each lane owns 8 consecutive features
// (one 16-byte store of y).  nvec = H / 8.  Slots are loaded KB at a time
// (KB loads in flight), then accumulated in order; k > KB takes several
// rounds of KB.
template <int KB, class S>
__device__ __forceinline__ void warp_combine_token(const SlotSrc& src, const float* __restrict__ gates, int t, int k,
                                                   int nvec, uint4* __restrict__ dst, int lane) {
    const size_t row0 = (size_t)t * k;
    const float* gt = gates ? gates + row0 : nullptr;
    // lanes may run different numbers of iterations (nvec % 32 != 0): no
    // warp collectives inside; the gates are broadcast loads (L1 hits)
    for (int v = lane; v < nvec; v += 32) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j0 = 0; j0 < k; j0 += KB) {
            typename S::Raw raw[KB];
            float g[KB];
#pragma unroll
            for (int jj = 0; jj < KB; ++jj) {
                const int j = j0 + jj;
                if (j < k) {
                    g[jj] = gates ? __ldg(gt + j) : 1.f;
                    raw[jj] = S::load(src, row0 + j, nvec, v);
                }
            }
#pragma unroll
            for (int jj = 0; jj < KB; ++jj)
                if (j0 + jj < k) {
                    float f[8];
                    S::widen(raw[jj], f);
#pragma unroll
                    for (int p = 0; p < 8; ++p) acc[p] = fmaf(g[jj], f[p], acc[p]);
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

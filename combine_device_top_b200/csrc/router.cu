// router.cu -- the router projection on the tensor cores, fused with step 1
// (top-k and gates) of the forward MoE layer.
//
// MoK article (tahou.com), routing paragraph: a router assigns every token
// to its experts.  The plain reading (the same one the oracle's router
// follows): logits[t, e] = sum_h x[t, h] W_r[h, e] + prior[e], x bf16, W_r
// fp32, then the top-k and softmax gates of step 1.
//
// Precision.  W_r is split once into two bf16 arrays, hi = bf16(W_r) and
// lo = bf16(W_r - hi) (about 16 significant bits together, with fp32's
// exponent range); x is exact in bf16, so x W_r = x hi + x lo up to
// 2^-17 |x| |W_r| per term, and both products accumulate in one fp32 TMEM
// accumulator.  The top-k then sees logits within that bound plus fp32
// accumulation rounding of the exact ones; near-ties inside the bound may
// order either way.
//
// One CTA per tile of 128 tokens, all E (<= 384) experts of the tile in TMEM:
//   warp 0      TMA loads of the W_hi / W_lo tiles ([E_pad, H] bf16,
//               K-major, 128-byte swizzle: 128 experts x 64 K per box);
//   warp 1      allocates TMEM; one thread issues tcgen05.mma: per 64-wide
//               K step, for every 128-expert tile, 4 MMAs of K = 16 with
//               W_hi and 4 with W_lo into the tile's accumulator;
//   warps 2-5   load the tokens' x rows from their shards (16-byte loads,
//               the next step's loads in flight while this step's are
//               stored) into the 128-byte-swizzled K-major A tile, then,
//               after the last MMA, move the accumulators to shared memory
//               (token-major, + prior);
//   all warps   the top-k and gates of each token from shared memory (the
//               same warp body as the top-k over given logits), and the
//               logits to global memory when asked for.
// Every wait is bounded; a wait that gives up records MOK_ERR_TIMEOUT in
// the status word and the CTA leaves after draining its own loads and MMAs.
#include "mok_device.cuh"
#include "mok_internal.h"
#include "topk.cuh"

namespace mok {

constexpr int RT_THREADS = 192;
constexpr int RT_BK = 64;                    // K per stage
constexpr int RT_A_BYTES = 128 * RT_BK * 2;  // 16 KB: 128 tokens x 64 K bf16
constexpr int RT_NB = 128;                   // experts per N tile
constexpr int RT_B_BYTES = RT_NB * RT_BK * 2;  // 16 KB per tile and part (hi or lo)
constexpr int RT_SMEM_MAX = 227 * 1024;      // opt-in shared memory per CTA on sm_100
constexpr int RT_BAR_BYTES = 256;
constexpr int RT_STAGE_BUDGET = RT_SMEM_MAX - 1024 - RT_BAR_BYTES;  // minus alignment slack and barriers
constexpr uint64_t RT_DRAIN_NS = 1000000000ull;

struct RouterArgs {
    ShardsIn xs;
    int S_r, T, H, E, k;
    int nt;       // 128-expert tiles (E_pad = 128 nt)
    int nst;      // stages
    int stage;    // bytes per stage: A + 2 nt B tiles
    int ld;       // shared-memory pitch of the logits tile (floats)
    const float* prior;
    float* logits;  // [T, E] or nullptr
    int32_t* topk_idx;
    float* gates;
    DevStatus* st;
    uint64_t timeout_ns;
};

// TMEM columns for nt 128-column accumulators (a power of two)
__device__ __forceinline__ uint32_t rt_tmem_cols(int nt) { return nt == 1 ? 128u : nt == 2 ? 256u : 512u; }

__device__ __forceinline__ void rt_load_x(const RouterArgs& a, int t, int kb, uint4 (&r)[8]) {
    if (t < a.T) {
        const int s = t / a.S_r;
        const uint4* src =
            reinterpret_cast<const uint4*>(a.xs.p[s]) + ((size_t)(t - s * a.S_r) * a.H + (size_t)kb * RT_BK) / 8;
#pragma unroll
        for (int c = 0; c < 8; ++c) r[c] = __ldg(src + c);
    } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) r[c] = make_uint4(0, 0, 0, 0);
    }
}

template <int NC>
__global__ void __launch_bounds__(RT_THREADS, 1)
    k_router(const __grid_constant__ CUtensorMap map_hi, const __grid_constant__ CUtensorMap map_lo,
             const RouterArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                           ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.nst * a.stage);  // TMA bytes of W
    uint64_t* afull = full + a.nst;                                         // x tile stored (128 arrivals)
    uint64_t* empty = afull + a.nst;                                        // stage consumed (MMA commit)
    uint64_t* done = empty + a.nst;                                         // every MMA complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    int* ok_flag = reinterpret_cast<int*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = a.H / RT_BK;
    const int t0 = blockIdx.x * 128;

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.nst; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&afull[s], 128);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *ok_flag = 1;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_hi);
        tma_prefetch_desc(&map_lo);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, rt_tmem_cols(a.nt));
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---- W tiles
            const uint32_t bytes = (uint32_t)(2 * a.nt * RT_B_BYTES);
            int issued = 0;
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % a.nst;
                if (!mbar_wait(&empty[s], ((kb / a.nst) & 1u) ^ 1u, a.st, a.timeout_ns, 90)) break;
                unsigned char* b = smem + s * a.stage + RT_A_BYTES;
                mbar_arrive_expect_tx(&full[s], bytes);
                for (int j = 0; j < a.nt; ++j) {
                    tma_load_2d(b + (2 * j) * RT_B_BYTES, &map_hi, &full[s], kb * RT_BK, j * RT_NB);
                    tma_load_2d(b + (2 * j + 1) * RT_B_BYTES, &map_lo, &full[s], kb * RT_BK, j * RT_NB);
                }
                issued = kb + 1;
            }
            // never leave with a load in flight into this CTA's shared memory
            for (int kb = issued > a.nst ? issued - a.nst : 0; kb < issued; ++kb)
                mbar_wait(&full[kb % a.nst], (kb / a.nst) & 1u, nullptr, RT_DRAIN_NS, 91);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issue
            const uint32_t idesc = umma_idesc_f16(128, RT_NB, /*A K-major*/ 0, /*B K-major*/ 0, /*bf16*/ 1);
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % a.nst;
                const uint32_t par = (kb / a.nst) & 1u;
                if (!mbar_wait(&full[s], par, a.st, a.timeout_ns, 92)) break;
                if (!mbar_wait(&afull[s], par, a.st, a.timeout_ns, 93)) break;
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + s * a.stage);
                const uint32_t sb = sa + RT_A_BYTES;
#pragma unroll
                for (int ks = 0; ks < RT_BK / 16; ++ks) {
                    // K-major SW128: 16 K = 32 bytes inside the atom; 8-row groups 1 KB apart
                    const uint64_t ad = umma_desc_sw128(sa + ks * 32, 16, 1024);
                    for (int j = 0; j < a.nt; ++j) {
                        const uint32_t acc = (kb | ks) != 0 ? 1u : 0u;
                        const uint64_t bh = umma_desc_sw128(sb + (2 * j) * RT_B_BYTES + ks * 32, 16, 1024);
                        const uint64_t bl = umma_desc_sw128(sb + (2 * j + 1) * RT_B_BYTES + ks * 32, 16, 1024);
                        umma_bf16(tmem + j * RT_NB, ad, bh, idesc, acc);
                        umma_bf16(tmem + j * RT_NB, ad, bl, idesc, 1u);
                    }
                }
                umma_commit(&empty[s]);
            }
            // the accumulators are final once every MMA issued has completed
            umma_commit(done);
        }
    } else {
        // ---- x tile: thread et loads token t0 + et, row by row of 128 bytes per step
        const int et = threadIdx.x - 64;
        const int t = t0 + et;
        uint4 cur[8], nxt[8];
        rt_load_x(a, t, 0, cur);
        for (int kb = 0; kb < KB; ++kb) {
            const int s = kb % a.nst;
            if (kb + 1 < KB) rt_load_x(a, t, kb + 1, nxt);
            if (!mbar_wait(&empty[s], ((kb / a.nst) & 1u) ^ 1u, a.st, a.timeout_ns, 94)) break;
            // K-major, 128-byte swizzle: row et at et * 128 bytes, 16-byte chunk c at slot c ^ (et & 7)
            unsigned char* row = smem + s * a.stage + et * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(row + ((c ^ (et & 7)) << 4)) = cur[c];
            fence_proxy_async_shared();  // generic stores -> the MMA (async proxy) reads them
            mbar_arrive(&afull[s]);
            if (kb + 1 < KB) {
#pragma unroll
                for (int c = 0; c < 8; ++c) cur[c] = nxt[c];
            }
        }
    }

    // ---- every MMA done (or a failure recorded): accumulators to shared memory
    if (warp >= 2) {
        const int et = threadIdx.x - 64;
        if (et == 0) *ok_flag = mbar_wait(done, 0, a.st, a.timeout_ns, 95) ? 1 : 0;
    }
    __syncthreads();
    const bool ok = *ok_flag != 0 && !failed(a.st);
    float* tile = reinterpret_cast<float*>(smem);  // [128 tokens][ld], over the (now idle) stages
    if (ok && warp >= 2) {
        tc_fence_after();
        const int q = warp & 3;  // TMEM lane quadrant of this warp: tokens 32 q .. 32 q + 31
        const int tok = q * 32 + lane;
        for (int c = 0; c < a.nt * RT_NB / 32; ++c) {
            float v[32];
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(c * 32), v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int e = c * 32 + i;
                if (e < a.E) tile[tok * a.ld + e] = v[i] + (a.prior ? __ldg(a.prior + e) : 0.f);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, rt_tmem_cols(a.nt));
    }
    if (!ok) return;
    // ---- top-k and gates, a warp per token; the logits out when asked for
    for (int i = warp; i < 128; i += RT_THREADS / 32) {
        const int t = t0 + i;
        if (t >= a.T) break;
        const float* row = tile + i * a.ld;
        warp_topk_token<NC>(row, a.E, a.k, lane, a.topk_idx + (size_t)t * a.k, a.gates + (size_t)t * a.k);
        if (a.logits)
            for (int e = lane; e < a.E; e += 32) a.logits[(size_t)t * a.E + e] = row[e];
    }
}

// ------------------------------------------------------------------ weight preparation
// w [H, E] fp32 -> hi, lo [E_pad, H] bf16 (E_pad = E rounded up to 128; the
// padding rows are zero): hi = bf16(w), lo = bf16(w - hi).
__global__ void k_router_split(const float* __restrict__ w, int H, int E, int E_pad, uint16_t* __restrict__ hi,
                               uint16_t* __restrict__ lo) {
    const size_t n = (size_t)E_pad * H;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int e = (int)(i / H), h = (int)(i % H);
        const float v = e < E ? __ldg(w + (size_t)h * E + e) : 0.f;
        const __nv_bfloat16 bh = __float2bfloat16_rn(v);
        const __nv_bfloat16 bl = __float2bfloat16_rn(v - __bfloat162float(bh));
        hi[i] = *reinterpret_cast<const uint16_t*>(&bh);
        lo[i] = *reinterpret_cast<const uint16_t*>(&bl);
    }
}

// ------------------------------------------------------------------ host side
int router_e_pad(int E) { return (E + RT_NB - 1) / RT_NB * RT_NB; }

cudaError_t launch_router_split(const float* w, int H, int E, void* hi, void* lo, int num_sms, cudaStream_t stream) {
    const size_t n = (size_t)router_e_pad(E) * H;
    const int grid = (int)((n + 255) / 256 < (size_t)num_sms * 8 ? (n + 255) / 256 : (size_t)num_sms * 8);
    k_router_split<<<grid, 256, 0, stream>>>(w, H, E, router_e_pad(E), reinterpret_cast<uint16_t*>(hi),
                                             reinterpret_cast<uint16_t*>(lo));
    return cudaGetLastError();
}

template <int NC>
static cudaError_t launch_router_nc(const CUtensorMap& mh, const CUtensorMap& ml, const RouterArgs& a, int smem,
                                   cudaStream_t stream) {
    static bool attr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr[dev]) {
        e = cudaFuncSetAttribute(k_router<NC>, cudaFuncAttributeMaxDynamicSharedMemorySize, RT_SMEM_MAX);
        if (e != cudaSuccess) return e;
        attr[dev] = true;
    }
    const int grid = (a.T + 127) / 128;
    k_router<NC><<<grid, RT_THREADS, smem, stream>>>(mh, ml, a);
    return cudaGetLastError();
}

cudaError_t launch_router(const ShardsIn& xs, int S_r, int T, int H, int E, int k, const void* w_hi,
                          const void* w_lo, const float* prior, float* logits, int32_t* topk_idx, float* gates,
                          void* status, uint64_t timeout_ns, const char** err, cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    RouterArgs a{};
    a.xs = xs;
    a.S_r = S_r;
    a.T = T;
    a.H = H;
    a.E = E;
    a.k = k;
    a.nt = router_e_pad(E) / RT_NB;
    a.stage = RT_A_BYTES + 2 * a.nt * RT_B_BYTES;
    a.nst = RT_STAGE_BUDGET / a.stage;
    if (a.nst > 4) a.nst = 4;
    a.ld = a.nt * RT_NB + 1;  // odd pitch: a warp's 32 tokens hit 32 different banks
    if (a.nst < 2 || 128 * a.ld * 4 > a.nst * a.stage) {
        *err = "router tile does not fit in shared memory";
        return cudaErrorInvalidValue;
    }
    a.prior = prior;
    a.logits = logits;
    a.topk_idx = topk_idx;
    a.gates = gates;
    a.st = reinterpret_cast<DevStatus*>(status);
    a.timeout_ns = timeout_ns;
    CUtensorMap mh, ml;
    const int ep = router_e_pad(E);
    if (!encode_tmap_2d_bf16(&mh, w_hi, (uint64_t)H, (uint64_t)ep, RT_BK, RT_NB, err) ||
        !encode_tmap_2d_bf16(&ml, w_lo, (uint64_t)H, (uint64_t)ep, RT_BK, RT_NB, err))
        return cudaErrorInvalidValue;
    const int smem = a.nst * a.stage + RT_BAR_BYTES + 1024;
    const int nc = (E + 31) / 32;
    *err = "router launch";
    if (nc <= 4) return launch_router_nc<4>(mh, ml, a, smem, stream);
    if (nc <= 8) return launch_router_nc<8>(mh, ml, a, smem, stream);
    return launch_router_nc<12>(mh, ml, a, smem, stream);
}

}  // namespace mok

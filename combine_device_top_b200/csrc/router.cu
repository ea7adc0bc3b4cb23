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
// A pair of CTAs (a cluster of two) per tile of 128 tokens; CTA r computes
// the logits of experts [r EH, (r + 1) EH) (EH = E rounded up to 64, halved:
// at most 256) in one TMEM accumulator, so 2 (T / 128) SMs share the work
// and each streams only its half of W:
//   warp 0      TMA loads of the CTA's W_hi / W_lo tiles ([E_pad, H] bf16,
//               K-major, 128-byte swizzle: EH experts x 64 K per box);
//   warp 1      allocates TMEM; one thread issues tcgen05.mma: per 64-wide
//               K step, 4 MMAs of K = 16 with W_hi and 4 with W_lo into the
//               accumulator (M = 128 tokens, N = EH);
//   warps 2-5   load the tokens' x rows from their shards (16-byte loads,
//               the next step's loads in flight while this step's are
//               stored) into the 128-byte-swizzled K-major A tile, then,
//               after the last MMA, move the accumulator to shared memory
//               (token-major, + prior);
//   all warps   per token, the k best of the CTA's experts (the top-k warp
//               body of the top-k over given logits), into the FIRST CTA's
//               candidate buffer (the second CTA through distributed shared
//               memory), and the logits to global memory when asked for;
//   first CTA   after a cluster barrier, per token the k best of the two
//               candidate lists and their softmax gates: the same selection
//               and arithmetic as the top-k over the whole row.
// Every wait is bounded; a wait that gives up records MOK_ERR_TIMEOUT in
// the status word and the CTA skips to the end after draining its own loads
// and MMAs (both CTAs still meet at the cluster barrier).
#include <cstring>

#include "mok_device.cuh"
#include "mok_internal.h"
#include "topk.cuh"

namespace mok {

constexpr int RT_THREADS = 192;
constexpr int RT_BK = 64;                    // K per stage
constexpr int RT_A_BYTES = 128 * RT_BK * 2;  // 16 KB: 128 tokens x 64 K bf16
constexpr int RT_EH_MAX = 256;               // experts per CTA (one MMA of N <= 256)
constexpr int RT_SMEM_MAX = 227 * 1024;      // opt-in shared memory per CTA on sm_100
constexpr int RT_BAR_BYTES = 256;
constexpr int RT_STAGE_BUDGET = RT_SMEM_MAX - 1024 - RT_BAR_BYTES;  // minus alignment slack and barriers
constexpr uint64_t RT_DRAIN_NS = 1000000000ull;

// x tiles by TMA when no 128-token tile straddles two shards (S_r % 128 == 0):
// one {64 K, 128 tokens} box per shard map and stage
struct RouterXMaps {
    CUtensorMap m[MOK_MAX_SHARDS];
};

struct RouterArgs {
    ShardsIn xs;
    int S_r, T, H, E, k;
    int x_tma;    // 1: x tiles by TMA (maps in RouterXMaps), else by the copy warps
    int eh;       // experts per CTA (a multiple of 32, <= 256)
    int nst;      // stages
    int stage;    // bytes per stage: A + the hi and lo B tiles
    int ld;       // shared-memory pitch of the logits tile (floats)
    int cand_off; // byte offset of the candidate buffer [2][128][k] (value, index)
    const float* prior;
    float* logits;  // [T, E] or nullptr
    int32_t* topk_idx;
    float* gates;
    DevStatus* st;
    uint64_t timeout_ns;
};

// TMEM columns for an accumulator of n columns (a power of two >= 32)
__device__ __forceinline__ uint32_t rt_tmem_cols(int n) { return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : 256u; }

// 16-byte asynchronous copy global -> shared (bytes = 16, or 0: zeros)
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void st_cluster_b32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

template <int NC>
__global__ void __launch_bounds__(RT_THREADS, 1)
    k_router(const __grid_constant__ CUtensorMap map_hi, const __grid_constant__ CUtensorMap map_lo,
             const __grid_constant__ RouterXMaps xmaps, const RouterArgs a) {
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
    const uint32_t rank = cluster_ctarank();
    const int t0 = (blockIdx.x >> 1) * 128;
    const int e_base = (int)rank * a.eh;
    const int e_here = max(0, min(a.eh, a.E - e_base));  // this CTA's experts

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
        tmem_alloc(tmem_slot, rt_tmem_cols(a.eh));
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---- W tiles of this CTA's experts (and the x tile, by TMA)
            const uint32_t bytes = (uint32_t)(2 * a.eh * RT_BK * 2 + (a.x_tma ? RT_A_BYTES : 0));
            const int shard = t0 / a.S_r, srow = t0 - shard * a.S_r;
            int issued = 0;
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % a.nst;
                if (!mbar_wait(&empty[s], ((kb / a.nst) & 1u) ^ 1u, a.st, a.timeout_ns, 90)) break;
                unsigned char* b = smem + s * a.stage + RT_A_BYTES;
                mbar_arrive_expect_tx(&full[s], bytes);
                if (a.x_tma) tma_load_2d(smem + s * a.stage, &xmaps.m[shard], &full[s], kb * RT_BK, srow);
                tma_load_2d(b, &map_hi, &full[s], kb * RT_BK, e_base);
                tma_load_2d(b + a.eh * RT_BK * 2, &map_lo, &full[s], kb * RT_BK, e_base);
                issued = kb + 1;
            }
            // never leave with a load in flight into this CTA's shared memory
            for (int kb = issued > a.nst ? issued - a.nst : 0; kb < issued; ++kb)
                mbar_wait(&full[kb % a.nst], (kb / a.nst) & 1u, nullptr, RT_DRAIN_NS, 91);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issue
            const uint32_t idesc = umma_idesc_f16(128, a.eh, /*A K-major*/ 0, /*B K-major*/ 0, /*bf16*/ 1);
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % a.nst;
                const uint32_t par = (kb / a.nst) & 1u;
                if (!mbar_wait(&full[s], par, a.st, a.timeout_ns, 92)) break;
                if (!a.x_tma && !mbar_wait(&afull[s], par, a.st, a.timeout_ns, 93)) break;
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + s * a.stage);
                const uint32_t sb = sa + RT_A_BYTES;
#pragma unroll
                for (int ks = 0; ks < RT_BK / 16; ++ks) {
                    // K-major SW128: 16 K = 32 bytes inside the atom; 8-row groups 1 KB apart
                    const uint64_t ad = umma_desc_sw128(sa + ks * 32, 16, 1024);
                    const uint64_t bh = umma_desc_sw128(sb + ks * 32, 16, 1024);
                    const uint64_t bl = umma_desc_sw128(sb + a.eh * RT_BK * 2 + ks * 32, 16, 1024);
                    umma_bf16(tmem, ad, bh, idesc, (kb | ks) != 0 ? 1u : 0u);
                    umma_bf16(tmem, ad, bl, idesc, 1u);
                }
                umma_commit(&empty[s]);
            }
            // the accumulator is final once every MMA issued has completed
            umma_commit(done);
        }
    } else if (!a.x_tma) {
        // ---- x tile: thread et copies token t0 + et's 128 bytes of each K step
        // into its row of the stage's A tile (K-major, 128-byte swizzle: 16-byte
        // chunk c at slot c ^ (et & 7)) with asynchronous copies, the steps of
        // all nst stages in flight; a step is handed to the MMA (afull) once
        // its copies have landed.
        const int et = threadIdx.x - 64;
        const int t = t0 + et;
        const bool live = t < a.T;
        const int sh = live ? t / a.S_r : 0;
        const unsigned char* src =
            reinterpret_cast<const unsigned char*>(a.xs.p[sh]) + (live ? (size_t)(t - sh * a.S_r) * a.H * 2 : 0);
        const int D = a.nst;  // steps in flight
        int handed = 0;       // steps passed on to the MMA
        bool ok_x = true;
        for (int kb = 0; kb < KB; ++kb) {
            const int s = kb % a.nst;
            if (!mbar_wait(&empty[s], ((kb / a.nst) & 1u) ^ 1u, a.st, a.timeout_ns, 94)) {
                ok_x = false;
                break;
            }
            unsigned char* row = smem + s * a.stage + et * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                cp_async16(row + ((c ^ (et & 7)) << 4), src + (size_t)kb * RT_BK * 2 + c * 16, live ? 16 : 0);
            cp_async_commit();
            if (kb - handed == D - 1) {
                // the oldest step in flight has landed
                if (D == 4) cp_async_wait<3>();
                else if (D == 3) cp_async_wait<2>();
                else cp_async_wait<1>();
                fence_proxy_async_shared();  // the copies' writes -> the MMA (async proxy) reads them
                mbar_arrive(&afull[handed % a.nst]);
                ++handed;
            }
        }
        // the rest (also on failure: no copy stays in flight into shared memory)
        cp_async_wait<0>();
        fence_proxy_async_shared();
        if (ok_x)
            for (; handed < KB; ++handed) mbar_arrive(&afull[handed % a.nst]);
    }

    // ---- every MMA done (or a failure recorded): the accumulator to shared memory
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
        for (int c = 0; c < a.eh / 32; ++c) {
            float v[32];
            tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(c * 32), v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int e = c * 32 + i;
                if (e < e_here) tile[tok * a.ld + e] = v[i] + (a.prior ? __ldg(a.prior + e_base + e) : 0.f);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, rt_tmem_cols(a.eh));
    }
    // ---- per token, the k best of this CTA's experts into the first CTA's
    // candidate buffer: cand[rank][token][j] = (value, expert)
    unsigned char* cand = smem + a.cand_off;
    if (ok) {
        for (int i = warp; i < 128; i += RT_THREADS / 32) {
            const int t = t0 + i;
            if (t >= a.T) break;
            const float* row = tile + i * a.ld;
            float v;
            int e;
            warp_topk_select<NC>(row, e_here, a.k, lane, e_base, v, e);
            if (lane < a.k) {
                const size_t at = ((size_t)(rank * 128 + i) * a.k + lane) * 8;
                if (rank == 0) {
                    *reinterpret_cast<float*>(cand + at) = v;
                    *reinterpret_cast<int*>(cand + at + 4) = e;
                } else {
                    const uint32_t dst = smem_in_rank(cand + at, 0);
                    st_cluster_b32(dst, __float_as_uint(v));
                    st_cluster_b32(dst + 4, (uint32_t)e);
                }
            }
            if (a.logits)
                for (int x = lane; x < e_here; x += 32) a.logits[(size_t)t * a.E + e_base + x] = row[x];
        }
    }
    // both CTAs' candidates are in the first CTA's shared memory (and the
    // second CTA leaves only after its remote stores are done)
    cluster_sync_all();
    if (!ok || rank != 0 || failed(a.st)) return;
    // ---- the k best of the two lists and their gates, a warp per token
    for (int i = warp; i < 128; i += RT_THREADS / 32) {
        const int t = t0 + i;
        if (t >= a.T) break;
        const unsigned char* c0 = cand + ((size_t)i * a.k + lane) * 8;
        const unsigned char* c1 = cand + ((size_t)(128 + i) * a.k + lane) * 8;
        float av = -INFINITY, bv = -INFINITY;
        int ae = 0x7fffffff, be = 0x7fffffff;
        if (lane < a.k) {
            av = *reinterpret_cast<const float*>(c0);
            ae = *reinterpret_cast<const int*>(c0 + 4);
            bv = *reinterpret_cast<const float*>(c1);
            be = *reinterpret_cast<const int*>(c1 + 4);
        }
        float v;
        int e;
        const float m = warp_topk_merge(av, ae, bv, be, a.k, lane, v, e);
        warp_topk_gates(v, e, m, a.k, lane, a.topk_idx + (size_t)t * a.k, a.gates + (size_t)t * a.k);
    }
}

// ------------------------------------------------------------------ weight preparation
// w [H, E] fp32 -> hi, lo [E_pad, H] bf16 (E_pad = E rounded up to 64; the
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
// two halves of EH experts each, EH a multiple of 32
int router_e_pad(int E) { return (E + 63) / 64 * 64; }

cudaError_t launch_router_split(const float* w, int H, int E, void* hi, void* lo, int num_sms, cudaStream_t stream) {
    const size_t n = (size_t)router_e_pad(E) * H;
    const int grid = (int)((n + 255) / 256 < (size_t)num_sms * 8 ? (n + 255) / 256 : (size_t)num_sms * 8);
    k_router_split<<<grid, 256, 0, stream>>>(w, H, E, router_e_pad(E), reinterpret_cast<uint16_t*>(hi),
                                             reinterpret_cast<uint16_t*>(lo));
    return cudaGetLastError();
}

template <int NC>
static cudaError_t launch_router_nc(const CUtensorMap& mh, const CUtensorMap& ml, const RouterXMaps& xm,
                                   const RouterArgs& a, int smem, cudaStream_t stream) {
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
    // a cluster of two CTAs per 128-token tile
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(2 * ((a.T + 127) / 128)));
    cfg.blockDim = dim3(RT_THREADS);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_router<NC>, mh, ml, xm, a);
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
    a.eh = router_e_pad(E) / 2;
    if (a.eh > RT_EH_MAX || k > 32) {
        *err = "router shape";
        return cudaErrorInvalidValue;
    }
    a.stage = RT_A_BYTES + 2 * a.eh * RT_BK * 2;
    a.nst = RT_STAGE_BUDGET / a.stage;
    if (a.nst > 4) a.nst = 4;
    a.ld = a.eh + 1;  // odd pitch: a warp's 32 tokens hit 32 different banks
    a.cand_off = (128 * a.ld * 4 + 15) & ~15;
    if (a.nst < 2 || a.cand_off + 2 * 128 * k * 8 > a.nst * a.stage) {
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
    if (!encode_tmap_2d_bf16(&mh, w_hi, (uint64_t)H, (uint64_t)ep, RT_BK, (uint32_t)a.eh, err) ||
        !encode_tmap_2d_bf16(&ml, w_lo, (uint64_t)H, (uint64_t)ep, RT_BK, (uint32_t)a.eh, err))
        return cudaErrorInvalidValue;
    RouterXMaps xm;  // the kernel parameter (only the first R maps are read)
    memset(&xm, 0, sizeof xm);
    const int R = T / S_r;
    a.x_tma = S_r % 128 == 0 ? 1 : 0;
    if (a.x_tma)
        for (int r = 0; r < R && a.x_tma; ++r)
            if (!encode_tmap_2d_bf16(&xm.m[r], xs.p[r], (uint64_t)H, (uint64_t)S_r, RT_BK, 128, err)) a.x_tma = 0;
    const int smem = a.nst * a.stage + RT_BAR_BYTES + 1024;
    const int nc = a.eh / 32;
    *err = "router launch";
    if (nc <= 2) return launch_router_nc<2>(mh, ml, xm, a, smem, stream);
    if (nc <= 4) return launch_router_nc<4>(mh, ml, xm, a, smem, stream);
    return launch_router_nc<8>(mh, ml, xm, a, smem, stream);
}

}  // namespace mok

// persistent.cu -- step a6: the SM-partitioned persistent forward kernel.
//
// MoK article (tahou.com): megakernel paragraph (the SMs are split into a
// part doing dispatch, combine and state handling and a part doing the
// expert FFN; the communication side tells the compute side through a
// GPU-local counter that a batch of tokens is complete, and the compute side
// tells the communication side that results are ready), minibatch paragraphs
// (the minibatch handed to the expert computation should form at least two
// full waves), ring-buffer paragraph (a fixed-size token buffer whose space
// is reused by the next batch once the previous one's results have left;
// the GPU state machine advances without the CPU).  MoK wiki summary, key
// points (SM split, local counters).
//
// One launch (cooperative, so every CTA is resident), one CTA per SM:
//   CTAs [0, D)  dispatch/combine side: for each minibatch b, wait until ring
//                half b % 2 is free (all down units of minibatch b - 2 done),
//                gather b's rows into it, publish gathered[b].
//   CTAs [D, G)  GEMM side: the tcgen05 core of gemm_core.cuh over the units
//                of every minibatch in order -- gate/up units of b, then its
//                down units -- dealt round-robin.  A gate/up unit waits for
//                gathered[b] == D; a down unit waits for its chunk's gate/up
//                units (g_done[c] == their count); completions are published with
//                release atomics.
//   all CTAs     after every down unit is done: the fixed-order combine.
// Dependencies only point to lower unit indices (or to the dispatch side,
// which waits only on lower indices), so the lowest unfinished unit can
// always proceed: no deadlock without any host involvement.  Every wait is
// bounded; a wait that gives up records MOK_ERR_TIMEOUT and the kernel
// leaves its loops.
//
// Memory ordering: rows and h are written with generic stores and read by
// TMA (async proxy) in other CTAs.  Writers fence.proxy.async + threadfence,
// then one thread does a release add; readers do an acquire load, then
// fence.proxy.async, then issue TMA.
#include "dispatch_combine.cuh"
#include "gemm_core.cuh"

namespace mok {

struct PersistParams {
    // work list
    const Chunk* chunks;
    const Minibatch* mbs;
    const int* counts2;  // [0] chunks, [1] minibatches
    int cap;             // rows per ring half
    int MTG, MTD;        // units (groups of Bf16Cfg::SUB M tiles) per chunk of the gate/up and down phases
    int dispatch_ctas;
    // counters (zeroed before the launch)
    int* gathered;  // [max_mb]  dispatch CTAs done with minibatch b
    int* d_done;    // [max_mb]  down units done in minibatch b
    int* g_done;    // [max_chunks] gate/up units done for chunk c
    int* d_total;   // [1]       down units done overall
    // token data
    ShardsIn xs;
    ShardsOut ys;
    int S_r, T, k;
    const int32_t* src_rank;
    const int32_t* src_index;
    const float* gates;
    __nv_bfloat16* ring;  // [2 * cap, H]
};

struct PersistSched {
    static constexpr bool kSignals = true;
    const PersistParams* p;
    int nch, nmb, gidx, gctas, total;

    __device__ bool get(int i, Unit& u) const {
        const int idx = gidx + i * gctas;
        if (idx >= total) return false;
        const int upc = p->MTG + p->MTD;  // units per chunk
        // minibatch b: chunk0 * upc <= idx < chunk1 * upc
        int lo = 0, hi = nmb - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p->mbs[mid].chunk0 * upc <= idx) lo = mid; else hi = mid - 1;
        }
        const Minibatch mb = p->mbs[lo];
        const int n = mb.chunk1 - mb.chunk0;
        if (n <= 0) return false;  // only after a capacity error (status already set)
        int local = idx - mb.chunk0 * upc;
        if (local < n * p->MTG) {
            u.phase = 0;
        } else {
            u.phase = 1;
            local -= n * p->MTG;
        }
        // M tile runs fastest: a chunk's gate/up units finish together early
        // in the minibatch, so its down units (ordered the same way) rarely wait
        const int MT = u.phase == 0 ? p->MTG : p->MTD;
        const int c = mb.chunk0 + local / MT;
        const Chunk ck = p->chunks[c];
        u.m = local % MT;
        u.chunk = c;
        u.mb = lo;
        u.expert = ck.expert;
        u.rows = ck.rows;
        u.grow0 = ck.row0;
        u.brow0 = ck.row0 - mb.row0 + (lo & 1) * p->cap;
        return true;
    }

    __device__ bool wait_inputs(const Unit& u, DevStatus* st, uint64_t timeout_ns) const {
        const bool ok = u.phase == 0 ? flag_wait_geq(&p->gathered[u.mb], p->dispatch_ctas, st, timeout_ns, 40)
                                     : flag_wait_geq(&p->g_done[u.chunk], p->MTG, st, timeout_ns, 41);
        fence_proxy_async_global();
        return ok;
    }

    __device__ void unit_done(const Unit& u) const {
        if (u.phase == 0) {
            red_release_gpu_add(&p->g_done[u.chunk], 1);
        } else {
            red_release_gpu_add(&p->d_done[u.mb], 1);
            red_release_gpu_add(p->d_total, 1);
        }
    }
};

// C: the GEMM CTAs' configuration (one M tile per unit, or pairs); both
// share the thread count and shared-memory layout the dispatch side uses.
template <int KMAX, class C>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_moe_persistent(const __grid_constant__ GemmMaps maps, const CoreArgs a, const __grid_constant__ PersistParams p) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ int s_ok;
    unsigned char* smem = align_smem_1024(smem_raw);
    const int nch = reinterpret_cast<volatile const int*>(p.counts2)[0];
    const int nmb = reinterpret_cast<volatile const int*>(p.counts2)[1];
    const int D = p.dispatch_ctas;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nvec = a.H >> 3;  // 16-byte vectors per token row

    if ((int)blockIdx.x < D) {
        // ---------------------------------------- dispatch side: fill the ring
        // One thread streams rows through the CTA's otherwise idle shared
        // memory with bulk async copies (about 200 KB in flight per CTA);
        // rows too wide for enough slots fall back to warp copies.
        const uint32_t row_bytes = (uint32_t)a.H * 2u;
        const int S = min(16, SMEM_BAR_OFF / (int)row_bytes);
        const bool bulk = S > BULK_STORES_IN_FLIGHT;
        uint64_t* slot_full = reinterpret_cast<uint64_t*>(smem + SMEM_BAR_OFF);
        if (threadIdx.x == 0 && bulk) {
            for (int i = 0; i < S; ++i) mbar_init(&slot_full[i], 1);
            fence_mbar_init();
        }
        __syncthreads();
        uint32_t loads = 0;
        for (int b = 0; b < nmb; ++b) {
            if (threadIdx.x == 0) {
                bool ok = !failed(a.st);
                if (ok && b >= 2) {  // ring half b % 2 is free once minibatch b - 2 is fully consumed
                    const Minibatch old = p.mbs[b - 2];
                    ok = flag_wait_geq(&p.d_done[b - 2], (old.chunk1 - old.chunk0) * p.MTD, a.st, a.timeout_ns, 50);
                }
                s_ok = ok ? 1 : 0;
            }
            __syncthreads();
            const int ok = s_ok;
            __syncthreads();
            if (!ok) break;
            const Minibatch mb = p.mbs[b];
            const int n = mb.row1 - mb.row0;
            const int r0 = mb.row0 + (int)((long long)n * blockIdx.x / D);
            const int r1 = mb.row0 + (int)((long long)n * (blockIdx.x + 1) / D);
            uint4* half = reinterpret_cast<uint4*>(p.ring) + (size_t)((b & 1) * p.cap) * nvec;
            if (bulk) {
                if (threadIdx.x == 0) {
                    auto src = [&](int i) -> const void* {
                        const int r = r0 + i;
                        return reinterpret_cast<const uint4*>(p.xs.p[__ldg(p.src_rank + r)]) +
                               (size_t)__ldg(p.src_index + r) * nvec;
                    };
                    auto dst = [&](int i) -> void* { return half + (size_t)(r0 + i - mb.row0) * nvec; };
                    bulk_stream_rows(r1 - r0, src, dst, row_bytes, smem, slot_full, S, loads, a.st, a.timeout_ns,
                                     DRAIN_TIMEOUT_NS);
                }
            } else {
                for (int r = r0 + warp; r < r1; r += GEMM_THREADS / 32) {
                    const int sr = __ldg(p.src_rank + r), si = __ldg(p.src_index + r);
                    warp_copy_row(reinterpret_cast<const uint4*>(p.xs.p[sr]) + (size_t)si * nvec,
                                  half + (size_t)(r - mb.row0) * nvec, nvec, lane);
                }
            }
            // the rows are read next by TMA in the GEMM CTAs
            fence_proxy_async_global();
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0 && !failed(a.st)) red_release_gpu_add(&p.gathered[b], 1);
        }
    } else {
        // ---------------------------------------- GEMM side
        PersistSched s;
        s.p = &p;
        s.nch = nch;
        s.nmb = nmb;
        s.gidx = blockIdx.x - D;
        s.gctas = gridDim.x - D;
        s.total = nch * (p.MTG + p.MTD);
        gemm_cta<PersistSched, C>(maps, nullptr, a, s, smem);
    }

    // -------------------------------------------- combine, once every down unit is done
    if (threadIdx.x == 0)
        s_ok = (!failed(a.st) && flag_wait_geq(p.d_total, nch * p.MTD, a.st, a.timeout_ns, 60)) ? 1 : 0;
    __syncthreads();
    if (!s_ok) return;
    const int warps = gridDim.x * (GEMM_THREADS / 32);
    for (int t = blockIdx.x * (GEMM_THREADS / 32) + warp; t < p.T; t += warps) {
        const int r = t / p.S_r;
        uint4* dst = reinterpret_cast<uint4*>(p.ys.p[r]) + (size_t)(t - r * p.S_r) * nvec;
        warp_combine_token<KMAX>(reinterpret_cast<const uint4*>(a.out), p.gates, t, p.k, nvec, dst, lane);
    }
}

template <int KMAX, class C>
static cudaError_t launch_persistent_k(int grid, const GemmMaps& maps, const CoreArgs& a, const PersistParams& p,
                                       cudaStream_t stream) {
    static_assert(C::THREADS == GEMM_THREADS && C::SMEM == SMEM_ALLOC && C::BAR_OFF == SMEM_BAR_OFF,
                  "the dispatch side assumes the GEMM side's block shape");
    static bool attr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr[dev]) {
        e = cudaFuncSetAttribute(k_moe_persistent<KMAX, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
        if (e != cudaSuccess) return e;
        attr[dev] = true;
    }
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_moe_persistent<KMAX, C>, GEMM_THREADS, SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (per_sm < 1 || grid > per_sm * sms) return cudaErrorCooperativeLaunchTooLarge;
    void* args[] = {const_cast<GemmMaps*>(&maps), const_cast<CoreArgs*>(&a), const_cast<PersistParams*>(&p)};
    return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(k_moe_persistent<KMAX, C>), dim3(grid),
                                       dim3(GEMM_THREADS), args, SMEM_ALLOC, stream);
}

cudaError_t launch_forward_persistent(const PersistLaunch& L, const char** err, cudaStream_t stream) {
    GemmMaps maps;
    if (!encode_gemm_maps(&maps, L.wg, L.wu, L.wd, L.ring, L.h, L.H, L.I, L.E, 2 * L.cap, err))
        return cudaErrorInvalidValue;
    CoreArgs a{};
    a.H = L.H;
    a.I = L.I;
    a.h = L.h;
    a.out = L.out;
    a.row_slot = L.row_slot;
    a.st = reinterpret_cast<DevStatus*>(L.status);
    a.timeout_ns = L.timeout_ns;
    PersistParams p;
    p.chunks = L.chunks;
    p.mbs = L.mbs;
    p.counts2 = L.counts2;
    p.cap = L.cap;
    // the staged GEMM's rule for M-tile pairs: mean rows per expert <= 192
    const bool pair = gemm_tuning(L.T * L.k, L.E).pair != 0;
    const int sub = pair ? Bf16PairCfg::SUB : Bf16Cfg::SUB;
    // units per chunk (with pairs the last one may be single)
    p.MTG = (L.I / MT_G_FEATURES + sub - 1) / sub;
    p.MTD = (L.H / MT_D_FEATURES + sub - 1) / sub;
    p.dispatch_ctas = L.dispatch_ctas;
    p.gathered = L.gathered;
    p.d_done = L.d_done;
    p.g_done = L.g_done;
    p.d_total = L.d_total;
    p.xs = L.xs;
    p.ys = L.ys;
    p.S_r = L.S_r;
    p.T = L.T;
    p.k = L.k;
    p.src_rank = L.src_rank;
    p.src_index = L.src_index;
    p.gates = L.gates;
    p.ring = reinterpret_cast<__nv_bfloat16*>(L.ring);
    *err = "persistent launch";
    if (pair) {
        if (L.k <= 2) return launch_persistent_k<2, Bf16PairCfg>(L.grid, maps, a, p, stream);
        return launch_persistent_k<8, Bf16PairCfg>(L.grid, maps, a, p, stream);
    }
    if (L.k <= 2) return launch_persistent_k<2, Bf16Cfg>(L.grid, maps, a, p, stream);
    return launch_persistent_k<8, Bf16Cfg>(L.grid, maps, a, p, stream);
}

}  // namespace mok

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
//   CTAs [0, D)  dispatch side: for each minibatch b, wait until ring half
//                b % 2 is free (all down units of minibatch b - 2 done), then
//                copy b's chunks into it, chunks dealt round-robin to the D
//                CTAs (MXFP8 path: quantised to E4M3 rows plus the ring's
//                scale planes), publishing chunk_ready[c] after each chunk.
//   CTAs [D, G)  GEMM side: the tcgen05 core of gemm_core.cuh over the units
//                of every minibatch in order -- gate/up units of b, then its
//                down units -- dealt round-robin.  A gate/up unit waits for
//                its chunk's rows (chunk_ready[c]); a down unit waits for its
//                chunk's gate/up units (g_done[c] == their count).  When the
//                last down unit of a chunk is published, its epilogue group
//                counts each of the chunk's rows into its token (tok_cnt);
//                a token whose k slots are complete is appended to ready_q.
//   all CTAs     once their own role is done, combine tokens from ready_q in
//                queue order (a warp per token): the combine of early
//                tokens overlaps the GEMM of later experts (macrobatch
//                overlap), and the rest runs on every SM at the end.
// Warp layout (dispatch_warps > 0): no dispatch CTAs.  Every CTA runs the
// GEMM roles and, beside them, dispatch_warps warps that claim the
// expert-major rows in pieces of PIECE_ROWS from one device counter, in
// row order, copy (MXFP8: quantise) them into the ring and add the rows
// they wrote to chunk_ready[c]; a gate/up unit then waits for all of its
// chunk's rows.  The GEMM keeps every SM, and the dispatch warps join the
// combine as soon as the last piece is claimed.
// Dependencies only point to lower unit indices (or to the dispatch side,
// which waits only on lower indices), and the combine waits only on the GEMM
// side, so the lowest unfinished unit can always proceed: no deadlock
// without any host involvement.  Every wait is bounded; a wait that gives up
// records MOK_ERR_TIMEOUT and the kernel leaves its loops.
//
// Memory ordering: rows and h (and, MXFP8, their scale planes) are written
// with generic stores or bulk copies and read by TMA or bulk copies (async
// proxy) in other CTAs.  Writers fence.proxy.async + threadfence, then one
// thread does a release add; readers do an acquire load, then
// fence.proxy.async, then issue TMA.  Slot outputs reach the combine through
// a chain of release/acquire atomics: each down unit's publication (release),
// the chunk's completing acquire-release add, the token counter's
// acquire-release add, the queue entry's release store and the combining
// warp's acquire load.
#include <cstring>

#include "dispatch_combine.cuh"
#include "gemm_core.cuh"

namespace mok {

struct PersistParams {
    // work list
    const Chunk* chunks;
    const Minibatch* mbs;
    const int* counts2;  // [0] chunks, [1] minibatches
    int cap;             // rows per ring half
    int MTG, MTD;        // units (groups of C::SUB M tiles) per chunk of the gate/up and down phases
    int dispatch_ctas;
    int dispatch_warps;  // per CTA, warp layout (then dispatch_ctas == 0); 0: dispatch CTAs
    // counters (zeroed before the launch)
    int* chunk_ready;  // [max_chunks] 1 once the chunk's rows are in the ring
    int* g_done;       // [max_chunks] gate/up units done for chunk c
    int* d_chunk;      // [max_chunks] down units done for chunk c
    int* d_done;       // [max_mb]     down units done in minibatch b (ring half reuse)
    int* tok_cnt;      // [T] slots of token t whose outputs are complete
    int* ready_q;      // [T] 1 + token, in the order tokens became complete (0: not yet)
    int* q_tail;       // tokens appended to ready_q
    int* q_claim;      // queue positions claimed by combining warps
    int* d_claim;      // warp layout: pieces of rows claimed by dispatch warps
    // token data
    ShardsIn xs;
    ShardsOut ys;
    int S_r, T, k;
    const int32_t* src_rank;
    const int32_t* src_index;
    const int32_t* row_slot;
    const float* gates;
    void* ring;        // [2 * cap, H] bf16, or E4M3 bytes (MXFP8 path)
    uint8_t* ring_sc;  // MXFP8 path: the ring rows' scale planes [H/128][sc_rows][4]
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
        // chunk_ready counts rows in the warp layout, whole chunks otherwise
        const int need = p->dispatch_warps > 0 ? u.rows : 1;
        const bool ok = u.phase == 0 ? flag_wait_geq(&p->chunk_ready[u.chunk], need, st, timeout_ns, 40)
                                     : flag_wait_geq(&p->g_done[u.chunk], p->MTG, st, timeout_ns, 41);
        fence_proxy_async_global();
        return ok;
    }

    // Publishes a finished unit; true when it was the last down unit of its chunk.
    __device__ bool unit_done(const Unit& u) const {
        if (u.phase == 0) {
            red_release_gpu_add(&p->g_done[u.chunk], 1);
            return false;
        }
        red_release_gpu_add(&p->d_done[u.mb], 1);
        return atom_acq_rel_gpu_add(&p->d_chunk[u.chunk], 1) == p->MTD - 1;
    }

    // Every output of the chunk's rows is stored: count each row into its
    // token; a token whose k slots are all counted joins the combine queue.
    // Called by the n threads of one epilogue group (thread `tid`).
    __device__ void chunk_done(const Unit& u, int tid, int n) const {
        __threadfence();
        for (int r = tid; r < u.rows; r += n) {
            const int t = __ldg(p->row_slot + u.grow0 + r) / p->k;
            if (atom_acq_rel_gpu_add(&p->tok_cnt[t], 1) == p->k - 1) {
                const int at = atomicAdd(p->q_tail, 1);
                st_release_gpu(&p->ready_q[at], t + 1);
            }
        }
    }
};

// Rows a dispatch warp claims at a time (warp layout).
constexpr int PIECE_ROWS = 16;
constexpr int MAX_DISPATCH_WARPS = 2;  // 12 bf16 warps keep 168 registers a thread (3 warps per SM sub-partition)

// MXFP8: one warp quantises source row src into E4M3 ring row brow and its
// H/32 block scales into the scale planes; four 256-element steps' loads in
// flight per lane.
__device__ __forceinline__ void mx_dispatch_row(const PersistParams& p, const CoreArgs& a, const uint4* src,
                                                int brow, int lane) {
    uint32_t* planes = reinterpret_cast<uint32_t*>(p.ring_sc);
    uint8_t* dst = reinterpret_cast<uint8_t*>(p.ring) + (size_t)brow * a.H;
    for (int c0 = 0; c0 < a.H; c0 += 1024) {
        uint4 raw[4];
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
            const int cc = c0 + 256 * s4 + lane * 8;
            raw[s4] = cc < a.H ? __ldg(src + (cc >> 3)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
            const int cs = c0 + 256 * s4;
            if (cs < a.H) {  // warp-uniform
                uint2 q;
                uint32_t word;
                warp_mx_quant8(raw[s4], q, word, lane);
                const int cc = cs + lane * 8;
                if (cc < a.H) {
                    *reinterpret_cast<uint2*>(dst + cc) = q;
                    if ((lane & 15) == 0) planes[(size_t)((cs >> 7) + (lane >> 4)) * a.sc_rows + brow] = word;
                }
            }
        }
    }
}

// bf16: one warp copies a row of nvec 16-byte vectors, eight per lane in
// flight (4 KB per warp).
__device__ __forceinline__ void warp_copy_row_deep(const uint4* __restrict__ src, uint4* __restrict__ dst, int nvec,
                                                   int lane) {
    for (int v0 = 0; v0 < nvec; v0 += 256) {
        uint4 t[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int v = v0 + 32 * j + lane;
            if (v < nvec) t[j] = __ldg(src + v);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int v = v0 + 32 * j + lane;
            if (v < nvec) dst[v] = t[j];
        }
    }
}

// Warp layout: a dispatch warp claims pieces of PIECE_ROWS expert-major
// rows in order, and for each chunk a piece touches waits (once per
// minibatch, lane 0, bounded) for the ring half to be free, writes the rows
// and publishes them: every lane fences its own stores (generic -> async
// proxy, then GPU scope), the warp converges, and lane 0 adds the row count
// to chunk_ready[c] with release semantics.  Pieces are claimed in order, so
// every piece below a claimed one is already claimed by a running warp:
// the lowest unfinished piece waits only on the GEMM of minibatch b - 2,
// which waits only on lower pieces.
template <class C>
__device__ __forceinline__ void warp_dispatch(const PersistParams& p, const CoreArgs& a, int nch, int nmb, int lane) {
    if (nmb <= 0 || nch <= 0) return;
    const int total = p.mbs[nmb - 1].row1;
    const int nvec = a.H >> 3;
    int ready_b = 1;  // ring halves of minibatches 0 and 1 start free
    while (true) {
        int piece = 0;
        if (lane == 0) piece = atomicAdd(p.d_claim, 1);
        piece = __shfl_sync(0xffffffffu, piece, 0);
        const int r0 = piece * PIECE_ROWS;
        if (r0 >= total || failed(a.st)) return;
        const int r1 = min(r0 + PIECE_ROWS, total);
        // the chunk holding row r0: chunks are in row order
        int lo = 0, hi = nch - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.chunks[mid].row0 <= r0) lo = mid; else hi = mid - 1;
        }
        int c = lo;
        int r = r0;
        while (r < r1 && c < nch) {
            const Chunk ck = p.chunks[c];
            const int e1 = min(r1, ck.row0 + ck.rows);
            const int b = ck.mb;
            if (b > ready_b) {
                int ok = 1;
                if (lane == 0) {
                    const Minibatch old = p.mbs[b - 2];
                    ok = flag_wait_geq(&p.d_done[b - 2], (old.chunk1 - old.chunk0) * p.MTD, a.st, a.timeout_ns, 51)
                             ? 1 : 0;
                }
                if (__shfl_sync(0xffffffffu, ok, 0) == 0) return;
                ready_b = b;
            }
            const Minibatch mb = p.mbs[b];
            for (int rr = r; rr < e1; ++rr) {
                const int sr = __ldg(p.src_rank + rr), si = __ldg(p.src_index + rr);
                const uint4* src = reinterpret_cast<const uint4*>(p.xs.p[sr]) + (size_t)si * nvec;
                const int brow = (b & 1) * p.cap + (rr - mb.row0);
                if constexpr (C::MX)
                    mx_dispatch_row(p, a, src, brow, lane);
                else
                    warp_copy_row_deep(src, reinterpret_cast<uint4*>(p.ring) + (size_t)brow * nvec, nvec, lane);
            }
            // the rows are read next by TMA in the GEMM CTAs
            fence_proxy_async_global();
            __threadfence();
            __syncwarp();
            if (lane == 0) red_release_gpu_add(&p.chunk_ready[c], e1 - r);
            r = e1;
            ++c;
        }
    }
}

// C: the GEMM CTAs' configuration (bf16 with one M tile per unit or pairs,
// or MXFP8); the dispatch CTAs run with the same block shape.  In the warp
// layout the block has C::THREADS + 32 * dispatch_warps threads.
template <int KMAX, class C>
__global__ void __launch_bounds__(C::THREADS + 32 * MAX_DISPATCH_WARPS, 1)
    k_moe_persistent(const __grid_constant__ GemmMaps maps, const __grid_constant__ MxMaps mx, const CoreArgs a,
                     const __grid_constant__ PersistParams p) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ int s_ok;
    unsigned char* smem = align_smem_1024(smem_raw);
    const int nch = reinterpret_cast<volatile const int*>(p.counts2)[0];
    const int nmb = reinterpret_cast<volatile const int*>(p.counts2)[1];
    const int D = p.dispatch_ctas;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nvec = a.H >> 3;  // 16-byte vectors per token row

    if (p.dispatch_warps > 0) {
        // ---------------------------------------- warp layout
        if (warp >= C::THREADS / 32) {
            __syncthreads();  // the GEMM roles' set-up barrier (barrier 0 counts every thread)
            warp_dispatch<C>(p, a, nch, nmb, lane);
        } else {
            PersistSched s;
            s.p = &p;
            s.nch = nch;
            s.nmb = nmb;
            s.gidx = blockIdx.x;
            s.gctas = gridDim.x;
            s.total = nch * (p.MTG + p.MTD);
            gemm_cta<PersistSched, C>(maps, &mx, a, s, smem);
        }
    } else if ((int)blockIdx.x < D) {
        // ---------------------------------------- dispatch side: fill the ring
        // bf16: one thread streams rows through the CTA's otherwise idle
        // shared memory with bulk async copies (about 200 KB in flight per
        // CTA); rows too wide for enough slots fall back to warp copies.
        // MXFP8: a warp per row quantises it on the way (registers only).
        const uint32_t row_bytes = (uint32_t)a.H * 2u;
        const int S = min(16, C::BAR_OFF / (int)row_bytes);
        const bool bulk = !C::MX && S > BULK_STORES_IN_FLIGHT;
        uint64_t* slot_full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
        if (threadIdx.x == 0 && bulk) {
            for (int i = 0; i < S; ++i) mbar_init(&slot_full[i], 1);
            fence_mbar_init();
        }
        __syncthreads();
        uint32_t loads = 0;
        bool ok = true;
        for (int b = 0; b < nmb && ok; ++b) {
            if (threadIdx.x == 0) {
                bool w = !failed(a.st);
                if (w && b >= 2) {  // ring half b % 2 is free once minibatch b - 2 is fully consumed
                    const Minibatch old = p.mbs[b - 2];
                    w = flag_wait_geq(&p.d_done[b - 2], (old.chunk1 - old.chunk0) * p.MTD, a.st, a.timeout_ns, 50);
                }
                s_ok = w ? 1 : 0;
            }
            __syncthreads();
            ok = s_ok != 0;
            __syncthreads();
            if (!ok) break;
            const Minibatch mb = p.mbs[b];
            uint4* half = reinterpret_cast<uint4*>(p.ring) + (size_t)((b & 1) * p.cap) * nvec;
            for (int c = mb.chunk0 + (int)blockIdx.x; c < mb.chunk1; c += D) {
                const Chunk ck = p.chunks[c];
                const int r0 = ck.row0, r1 = ck.row0 + ck.rows;
                if constexpr (C::MX) {
                    for (int r = r0 + warp; r < r1; r += C::THREADS / 32) {
                        const int sr = __ldg(p.src_rank + r), si = __ldg(p.src_index + r);
                        mx_dispatch_row(p, a, reinterpret_cast<const uint4*>(p.xs.p[sr]) + (size_t)si * nvec,
                                        (b & 1) * p.cap + (r - mb.row0), lane);
                    }
                } else if (bulk) {
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
                    for (int r = r0 + warp; r < r1; r += C::THREADS / 32) {
                        const int sr = __ldg(p.src_rank + r), si = __ldg(p.src_index + r);
                        warp_copy_row(reinterpret_cast<const uint4*>(p.xs.p[sr]) + (size_t)si * nvec,
                                      half + (size_t)(r - mb.row0) * nvec, nvec, lane);
                    }
                }
                // the rows are read next by TMA in the GEMM CTAs
                fence_proxy_async_global();
                __threadfence();
                __syncthreads();
                if (threadIdx.x == 0 && !failed(a.st)) red_release_gpu_add(&p.chunk_ready[c], 1);
            }
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
        gemm_cta<PersistSched, C>(maps, &mx, a, s, smem);
    }

    // -------------------------------------------- combine tokens as they complete
    // A warp claims the next queue position and waits (bounded) for the
    // token that completes there; the fixed-order sum itself is the staged
    // combine's, so y does not depend on which warp combines a token or when.
    while (true) {
        int at = 0;
        if (lane == 0) at = atomicAdd(p.q_claim, 1);
        at = __shfl_sync(0xffffffffu, at, 0);
        if (at >= p.T) break;
        // lane 0 waits; the warp leaves or goes on as one
        int ready = 0;
        if (lane == 0) ready = flag_wait_geq(&p.ready_q[at], 1, a.st, a.timeout_ns, 60) ? 1 : 0;
        if (__shfl_sync(0xffffffffu, ready, 0) == 0) break;
        // every lane acquires the entry, so its loads of the slot rows come after it
        const int t = ld_acquire_gpu(&p.ready_q[at]) - 1;
        const int r = t / p.S_r;
        uint4* dst = reinterpret_cast<uint4*>(p.ys.p[r]) + (size_t)(t - r * p.S_r) * nvec;
        const SlotSrc src{a.out, a.out_exp};
        if constexpr (C::MX)
            warp_combine_token<KMAX, SlotBf16>(src, p.gates, t, p.k, nvec, dst, lane);
        else
            warp_combine_token<KMAX, SlotF16S>(src, p.gates, t, p.k, nvec, dst, lane);
    }
}

template <int KMAX, class C>
static cudaError_t launch_persistent_k(int grid, const GemmMaps& maps, const MxMaps& mx, const CoreArgs& a,
                                       const PersistParams& p, cudaStream_t stream) {
    const int threads = C::THREADS + 32 * p.dispatch_warps;
    static bool attr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr[dev]) {
        e = cudaFuncSetAttribute(k_moe_persistent<KMAX, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr[dev] = true;
    }
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_moe_persistent<KMAX, C>, threads, C::SMEM);
    if (e != cudaSuccess) return e;
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (per_sm < 1 || grid > per_sm * sms) return cudaErrorCooperativeLaunchTooLarge;
    void* args[] = {const_cast<GemmMaps*>(&maps), const_cast<MxMaps*>(&mx), const_cast<CoreArgs*>(&a),
                    const_cast<PersistParams*>(&p)};
    return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(k_moe_persistent<KMAX, C>), dim3(grid),
                                       dim3(threads), args, C::SMEM, stream);
}

cudaError_t launch_forward_persistent(const PersistLaunch& L, const char** err, cudaStream_t stream) {
    GemmMaps maps;
    MxMaps mx;
    memset(&maps, 0, sizeof maps);
    memset(&mx, 0, sizeof mx);
    if (L.mxw) {
        if (!encode_mx_maps(&mx, *L.mxw, L.H, L.I, L.E, err) ||
            !encode_bmaps_u8(&maps.rows, L.ring, (uint64_t)L.H, (uint64_t)2 * L.cap, err) ||
            !encode_bmaps_u8(&maps.h, L.h, (uint64_t)L.I, (uint64_t)2 * L.cap, err))
            return cudaErrorInvalidValue;
    } else if (!encode_gemm_maps(&maps, L.wg, L.wu, L.wd, L.ring, L.h, L.H, L.I, L.E, 2 * L.cap, err)) {
        return cudaErrorInvalidValue;
    }
    CoreArgs a{};
    a.H = L.H;
    a.I = L.I;
    a.h = L.h;
    a.out = L.out;
    if (!L.mxw) a.out_exp = reinterpret_cast<int8_t*>(L.out) + slot_exp_offset((size_t)L.T * L.k, L.H);
    a.row_slot = L.row_slot;
    a.st = reinterpret_cast<DevStatus*>(L.status);
    a.timeout_ns = L.timeout_ns;
    if (L.mxw) {
        a.xsc = L.ring_sc;
        a.hsc = L.h_sc;
        a.sc_rows = L.sc_rows;
    }
    PersistParams p;
    p.chunks = L.chunks;
    p.mbs = L.mbs;
    p.counts2 = L.counts2;
    p.cap = L.cap;
    // the staged GEMM's rule for M-tile pairs (mean rows per expert <= 192),
    // decided by the caller with the work list; bf16 only, the MXFP8 path
    // runs one M tile per unit
    const bool pair = !L.mxw && L.pair;
    const int sub = pair ? Bf16PairCfg::SUB : Bf16Cfg::SUB;
    // units per chunk (with pairs the last one may be single)
    p.MTG = (L.I / MT_G_FEATURES + sub - 1) / sub;
    p.MTD = (L.H / MT_D_FEATURES + sub - 1) / sub;
    p.dispatch_ctas = L.dispatch_ctas;
    p.dispatch_warps = L.dispatch_warps;
    if (p.dispatch_warps < 0 || p.dispatch_warps > MAX_DISPATCH_WARPS || (p.dispatch_warps > 0 && p.dispatch_ctas != 0))
        return cudaErrorInvalidValue;
    p.chunk_ready = L.chunk_ready;
    p.g_done = L.g_done;
    p.d_chunk = L.d_chunk;
    p.d_done = L.d_done;
    p.tok_cnt = L.tok_cnt;
    p.ready_q = L.ready_q;
    p.q_tail = L.q_tail;
    p.q_claim = L.q_claim;
    p.d_claim = L.d_claim;
    p.xs = L.xs;
    p.ys = L.ys;
    p.S_r = L.S_r;
    p.T = L.T;
    p.k = L.k;
    p.src_rank = L.src_rank;
    p.src_index = L.src_index;
    p.row_slot = L.row_slot;
    p.gates = L.gates;
    p.ring = L.ring;
    p.ring_sc = L.ring_sc;
    *err = "persistent launch";
    // KMAX slots' loads in flight per lane in the combine (k > KMAX: several rounds)
    if (L.mxw) {
        if (L.k <= 2) return launch_persistent_k<2, MxCfg>(L.grid, maps, mx, a, p, stream);
        return launch_persistent_k<8, MxCfg>(L.grid, maps, mx, a, p, stream);
    }
    if (pair) {
        if (L.k <= 2) return launch_persistent_k<2, Bf16PairCfg>(L.grid, maps, mx, a, p, stream);
        return launch_persistent_k<8, Bf16PairCfg>(L.grid, maps, mx, a, p, stream);
    }
    if (L.k <= 2) return launch_persistent_k<2, Bf16Cfg>(L.grid, maps, mx, a, p, stream);
    return launch_persistent_k<8, Bf16Cfg>(L.grid, maps, mx, a, p, stream);
}

}  // namespace mok

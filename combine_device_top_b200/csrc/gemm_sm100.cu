// gemm_sm100.cu -- step 4 of the forward MoE layer: the grouped expert GEMM
// with SwiGLU fused, on 5th-generation tensor cores (tcgen05 + TMEM, TMA).
//
// MoK article (tahou.com): routing paragraph (tokens of one expert laid out
// contiguously so the grouped GEMM runs efficiently), the paragraph on
// MXFP8 (SwiGLU inside the GEMM data path), push-combine paragraph (each
// result goes back to its token's slot).
//
// Orientation.  Expert segments are short (about 171 rows per expert at
// 384 experts, top-8, 8192 tokens), so the weights take the M = 128 side of
// every MMA and the tokens the N side (16..256 in steps of 16): an expert
// with 171 rows pads to N = 176 instead of two 128-row tiles, and each
// weight tile is streamed from HBM once per chunk of <= 256 rows.
//   gate/up unit (phase 0): A = 64 columns of Wg stacked on the same 64
//     columns of Wu (M = 128, K = H, read MN-major straight from the
//     [E, H, I] layout), B = the chunk's token rows (K-major).  Accumulator
//     lanes 0-63 hold gate, 64-127 up; the epilogue forms
//     h = silu(gate) * up and stores fp16 h rows.
//   down unit (phase 1): A = 128 columns of the fp16 copy of Wd (MN-major
//     from [E, I, H]), B = the chunk's fp16 h rows; fp16 keeps 3 more
//     mantissa bits of h than bf16 would, which is what keeps the largest
//     element error of y near the floor set by rounding y itself to bf16.
//     The epilogue stores fp32 rows to
//     out[row_slot[row]] (the push combine).  fp32 rather than bf16: with a
//     bf16 slot buffer the three bf16 roundings (h, o, y) put the largest
//     element error of y above 2e-2 * rms(y) on heavy-tailed outputs.
//
// Roles in a CTA of 6 warps: warp 0 issues TMA loads into a 4-stage ring
// of 48 KB stages, warp 1 allocates 512 TMEM columns and one thread of it
// issues tcgen05.mma into one of two 256-column accumulators, warps 2-5
// drain the other accumulator (tcgen05.ld) through shared memory to global.
// The grid is persistent (one CTA per SM) over the unit list built on the
// device; every wait is bounded.
#include "mok_device.cuh"
#include "mok_internal.h"

namespace mok {

constexpr int GEMM_THREADS = 192;
constexpr int NSTAGE = 4;
constexpr int BK = 64;                       // K per stage: one 128-byte swizzle atom of bf16
constexpr int A_BYTES = 128 * BK * 2;        // 16 KB: two {64 MN x 64 K} boxes
constexpr int B_ROWS_MAX = CHUNK_MAX_ROWS;   // 256
constexpr int B_ROW_BYTES = BK * 2;               // 128 bytes of one token row per stage
constexpr int B_BYTES = B_ROWS_MAX * BK * 2;       // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;     // 48 KB
constexpr int EPI_LD = 33;                          // fp32 staging row pitch (bank-conflict free)
constexpr int EPI_BYTES = 128 * EPI_LD * 4;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 256;

constexpr int SMEM_STAGES_OFF = 0;
constexpr int SMEM_EPI_OFF = NSTAGE * STAGE_BYTES;
constexpr int SMEM_BAR_OFF = SMEM_EPI_OFF + EPI_BYTES;
constexpr int SMEM_BYTES_USED = SMEM_BAR_OFF + 256;
constexpr int SMEM_ALLOC = SMEM_BYTES_USED + 1024;  // slack for 1024-byte alignment

struct GemmParams {
    const Chunk* chunks;
    const int* counts2;  // [0] = number of chunks
    int K;               // contraction length (H or I)
    int MT;              // M tiles per chunk
    int w_rows;          // rows per expert in the A tensor map (H or I)
    int I, H;
    __half* h_out;            // phase 0: [rows, I] fp16
    float* out;               // phase 1: [N_s, H] fp32, slot-indexed
    const int32_t* row_slot;  // phase 1
    DevStatus* st;
    uint64_t timeout_ns;
    int l2_prefetch;     // k-steps of weight tiles prefetched into L2 ahead of the loads
    int group_chunks;    // raster: chunks per group (see unit_map)
};

// Unit u -> (chunk c, M tile m).  Units are rastered in groups of GC chunks:
// inside a group the chunk index runs fastest, so the CTAs running at one
// time share a few chunks' token tiles (L2) while streaming distinct weight
// tiles.
__device__ __forceinline__ void unit_map(int u, int nch, int MT, int GC, int& c, int& m) {
    const int grp = u / (GC * MT);
    const int rem = u - grp * GC * MT;
    const int c0 = grp * GC;
    const int gsz = min(GC, nch - c0);
    m = rem / gsz;
    c = c0 + (rem - m * gsz);
}

template <int PHASE>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ BMaps tmB, const GemmParams p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + SMEM_BAR_OFF);
    uint64_t* empty = full + NSTAGE;
    uint64_t* tfull = empty + NSTAGE;
    uint64_t* tempty = tfull + 2;
    uint64_t* fin = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
    volatile int* ok_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(fin, 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA0);
        tma_prefetch_desc(&tmA1);
        for (int i = 0; i < B_MAPS; ++i) tma_prefetch_desc(&tmB.m[i]);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int nch = *reinterpret_cast<volatile const int*>(p.counts2);
    const int nunits = nch * p.MT;
    const int KB = p.K / BK;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_phase = 0;  // bit s: stage s holds a load of phase bit s
            bool ok = true;
            const uint64_t evict_first = l2_policy_evict_first();
            // Look-ahead cursor: the weight tiles of the k-step p.l2_prefetch
            // steps ahead are prefetched into L2, so that more weight bytes are
            // in flight per SM than the shared-memory stages alone hold.
            int pu = blockIdx.x, pkb = 0, pm = 0, pe = 0, pu_mapped = -1;
            auto prefetch_next = [&]() {
                if (pu >= nunits) return;
                if (pu != pu_mapped) {
                    int c;
                    unit_map(pu, nch, p.MT, p.group_chunks, c, pm);
                    pe = p.chunks[c].expert;
                    pu_mapped = pu;
                }
                const int ky = pe * p.w_rows + pkb * BK;
                if (PHASE == 0) {
                    tma_prefetch_l2_2d(&tmA0, pm * 64, ky);
                    tma_prefetch_l2_2d(&tmA1, pm * 64, ky);
                } else {
                    tma_prefetch_l2_2d(&tmA0, pm * 128, ky);
                    tma_prefetch_l2_2d(&tmA0, pm * 128 + 64, ky);
                }
                if (++pkb == KB) {
                    pkb = 0;
                    pu += gridDim.x;
                }
            };
            for (int i = 0; i < p.l2_prefetch; ++i) prefetch_next();
            for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
                int c, m;
                unit_map(u, nch, p.MT, p.group_chunks, c, m);
                const Chunk ck = p.chunks[c];
                // token rows rounded up to 16, loaded as one box per set bit
                // (256, 128, 64, 32, 16 rows): at most 5 TMA ops per stage
                const int r16 = (ck.rows + 15) & ~15;
                const uint32_t bytes = A_BYTES + r16 * B_ROW_BYTES;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.st, p.timeout_ns, 10)) {
                        ok = false;
                        break;
                    }
                    unsigned char* sa = smem + SMEM_STAGES_OFF + stage * STAGE_BYTES;
                    unsigned char* sb = sa + A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    const int ky = ck.expert * p.w_rows + kb * BK;
                    if (PHASE == 0) {
                        tma_load_2d_hint(sa, &tmA0, &full[stage], m * 64, ky, evict_first);
                        tma_load_2d_hint(sa + A_BYTES / 2, &tmA1, &full[stage], m * 64, ky, evict_first);
                    } else {
                        tma_load_2d_hint(sa, &tmA0, &full[stage], m * 128, ky, evict_first);
                        tma_load_2d_hint(sa + A_BYTES / 2, &tmA0, &full[stage], m * 128 + 64, ky, evict_first);
                    }
                    if (p.l2_prefetch > 0) prefetch_next();
                    int roff = 0;
#pragma unroll
                    for (int i = 0; i < B_MAPS; ++i) {
                        const int sz = B_MAX_BOX >> i;
                        if (r16 & sz) {
                            tma_load_2d(sb + roff * B_ROW_BYTES, &tmB.m[i], &full[stage], kb * BK, ck.row0 + roff);
                            roff += sz;
                        }
                    }
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == NSTAGE) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // never leave with a load in flight into this CTA's shared memory
            for (int s = 0; s < NSTAGE; ++s)
                if ((issued >> s) & 1u) mbar_wait(&full[s], (issued_phase >> s) & 1u, nullptr, p.timeout_ns, 11);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int tb = 0;
            uint32_t tph = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
                int c, m;
                unit_map(u, nch, p.MT, p.group_chunks, c, m);
                const Chunk ck = p.chunks[c];
                const int N = (ck.rows + 15) & ~15;
                // gate/up: bf16 x bf16; down: fp16 x fp16 (fp16 W_down copy, fp16 h)
                const uint32_t idesc = umma_idesc_f16(128, N, /*A MN-major*/ 1, /*B K-major*/ 0, PHASE == 0);
                if (!mbar_wait(&tempty[tb], tph ^ 1u, p.st, p.timeout_ns, 20)) break;
                tc_fence_after();
                const uint32_t dt = tmem_base + (uint32_t)(tb * ACC_COLS);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&full[stage], phase, p.st, p.timeout_ns, 21)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + SMEM_STAGES_OFF + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int ks = 0; ks < BK / 16; ++ks) {
                        // A: MN-major SW128, 16 K rows per MMA = 2 atoms of 1 KB;
                        //    the two 64-wide MN halves are 8 KB apart (LBO).
                        const uint64_t ad = umma_desc_sw128(sa + ks * 2048, A_BYTES / 2, 1024);
                        // B: K-major SW128, 16 K = 32 bytes inside the atom; 8-row groups 1 KB apart.
                        const uint64_t bd = umma_desc_sw128(sb + ks * 32, 16, 1024);
                        umma_bf16(dt, ad, bd, idesc, (kb | ks) != 0 ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == NSTAGE) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&tfull[tb]);
                if (++tb == 2) {
                    tb = 0;
                    tph ^= 1u;
                }
            }
            // wait for every MMA this thread issued before TMEM is released
            umma_commit(fin);
            mbar_wait(fin, 0, nullptr, p.timeout_ns, 22);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5)
        const int q = warp & 3;             // TMEM lane quadrant this warp may access
        const int et = threadIdx.x - 64;    // 0..127
        float* epi = reinterpret_cast<float*>(smem + SMEM_EPI_OFF);
        int tb = 0;
        uint32_t tph = 0;
        for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
            if (et == 0) *ok_flag = mbar_wait(&tfull[tb], tph, p.st, p.timeout_ns, 30) ? 1 : 0;
            named_bar_sync(1, 128);
            const int ok = *ok_flag;
            named_bar_sync(1, 128);
            if (!ok) break;
            tc_fence_after();
            int c, m;
            unit_map(u, nch, p.MT, p.group_chunks, c, m);
            const Chunk ck = p.chunks[c];
            const int ncc = (ck.rows + 31) >> 5;
            const int tok = et & 31, fq = et >> 5;
            for (int cc = 0; cc < ncc; ++cc) {
                float v[32];
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(tb * ACC_COLS + cc * 32), v);
                float* myrow = epi + (q * 32 + lane) * EPI_LD;
#pragma unroll
                for (int i = 0; i < 32; ++i) myrow[i] = v[i];
                named_bar_sync(1, 128);
                const int col = cc * 32 + tok;
                if (col < ck.rows) {
                    if (PHASE == 0) {
                        // features m*64 + fq*16 .. +15 : gate rows fq*16+i, up rows 64+fq*16+i
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 16; i += 2) {
                            const float g0 = epi[(fq * 16 + i) * EPI_LD + tok];
                            const float g1 = epi[(fq * 16 + i + 1) * EPI_LD + tok];
                            const float u0 = epi[(64 + fq * 16 + i) * EPI_LD + tok];
                            const float u1 = epi[(64 + fq * 16 + i + 1) * EPI_LD + tok];
                            const float h0 = g0 / (1.0f + __expf(-g0)) * u0;
                            const float h1 = g1 / (1.0f + __expf(-g1)) * u1;
                            pk[i >> 1] = pack_half2_sat(h0, h1);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(p.h_out + (size_t)(ck.row0 + col) * p.I + m * 64 + fq * 16);
                        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    } else {
                        // fp32 push: the combine reads these once more and rounds y once
                        const int slot = __ldg(p.row_slot + ck.row0 + col);
                        float4* dst = reinterpret_cast<float4*>(p.out + (size_t)slot * p.H + m * 128 + fq * 32);
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) {
                            const int f = fq * 32 + q4 * 4;
                            dst[q4] = make_float4(epi[f * EPI_LD + tok], epi[(f + 1) * EPI_LD + tok],
                                                  epi[(f + 2) * EPI_LD + tok], epi[(f + 3) * EPI_LD + tok]);
                        }
                    }
                }
                named_bar_sync(1, 128);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[tb]);
            if (++tb == 2) {
                tb = 0;
                tph ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ work list
// One block.  Minibatch boundaries: from row b0, the first expert boundary at
// or after b0 + minibatch, but never more than `cap` rows; then every
// (expert, minibatch) piece is cut into ceil(len / 256) chunks of nearly
// equal size (multiples of 16 rows except the last).
__device__ __forceinline__ int piece_chunks(int L) { return (L + CHUNK_MAX_ROWS - 1) / CHUNK_MAX_ROWS; }
__device__ __forceinline__ int piece_base(int L) {
    const int n = piece_chunks(L);
    int base = (((L + n - 1) / n) + 15) & ~15;
    if ((n - 1) * base >= L) base = CHUNK_MAX_ROWS;
    return base;
}

__global__ void __launch_bounds__(1024) k_build_chunks(const int32_t* __restrict__ offsets, int E, int n_slots,
                                                       int M, int cap, Chunk* __restrict__ chunks, int max_chunks,
                                                       Minibatch* __restrict__ mbs, int max_mb,
                                                       int* __restrict__ counts2, DevStatus* st) {
    __shared__ int s_nmb;
    __shared__ int warp_sums[32];
    if (threadIdx.x == 0) {
        int b0 = 0, n = 0;
        while (b0 < n_slots) {
            int b1;
            const int target = b0 + M;
            if (target >= n_slots) {
                b1 = n_slots;
            } else {
                int lo = 0, hi = E;
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (offsets[mid] >= target) hi = mid; else lo = mid + 1;
                }
                b1 = offsets[lo];
                if (b1 > b0 + cap) b1 = b0 + cap;
            }
            if (n >= max_mb) {
                set_status(st, MOK_ERR_CAPACITY, 1, n, max_mb);
                break;
            }
            mbs[n] = Minibatch{b0, b1, 0, 0};
            ++n;
            b0 = b1;
        }
        s_nmb = n;
    }
    __syncthreads();
    const int nmb = s_nmb;

    // per expert: count chunks (thread e; E <= 1024)
    const int e = threadIdx.x;
    int a = 0, b = 0, first_mb = 0, cnt = 0;
    if (e < E) {
        a = offsets[e];
        b = offsets[e + 1];
        if (b > a) {
            int lo = 0, hi = nmb - 1;  // last minibatch with row0 <= a
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (mbs[mid].row0 <= a) lo = mid; else hi = mid - 1;
            }
            first_mb = lo;
            for (int mb = first_mb; mb < nmb && mbs[mb].row0 < b; ++mb) {
                const int L = min(b, mbs[mb].row1) - max(a, mbs[mb].row0);
                if (L > 0) cnt += piece_chunks(L);
            }
        }
    }
    // exclusive scan of cnt over threads
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = warp_sums[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        warp_sums[lane] = w;
    }
    __syncthreads();
    int idx = incl - cnt + (warp > 0 ? warp_sums[warp - 1] : 0);
    const int total = warp_sums[31];
    if (e < E && b > a) {
        for (int mb = first_mb; mb < nmb && mbs[mb].row0 < b; ++mb) {
            const int r0 = max(a, mbs[mb].row0);
            const int L = min(b, mbs[mb].row1) - r0;
            if (L <= 0) continue;
            const int n = piece_chunks(L), base = piece_base(L);
            for (int i = 0; i < n; ++i, ++idx) {
                const int rr = (i < n - 1) ? base : L - (n - 1) * base;
                if (idx < max_chunks) chunks[idx] = Chunk{e, r0 + i * base, rr, mb};
            }
        }
    }
    if (threadIdx.x == 0) {
        if (total > max_chunks) set_status(st, MOK_ERR_CAPACITY, 2, total, max_chunks);
        counts2[0] = min(total, max_chunks);
        counts2[1] = nmb;
    }
    __syncthreads();
    const int nck = min(total, max_chunks);
    for (int i = threadIdx.x; i < nck; i += blockDim.x) {
        const int mb = chunks[i].mb;
        if (i == 0 || chunks[i - 1].mb != mb) mbs[mb].chunk0 = i;
        if (i == nck - 1 || chunks[i + 1].mb != mb) mbs[mb].chunk1 = i + 1;
    }
}

// ------------------------------------------------------------------ host side
int max_minibatches(int n_slots, int minibatch) {
    if (minibatch <= 0) minibatch = 1;
    return n_slots / minibatch + 2;
}
int max_chunks(int n_slots, int E, int n_mb) { return n_slots / CHUNK_MAX_ROWS + E + n_mb + 2; }

cudaError_t launch_build_chunks(const int32_t* offsets, int E, int n_slots, int minibatch, int cap, Chunk* chunks,
                                int max_ch, Minibatch* mbs, int max_mb, int* counts2, void* status,
                                cudaStream_t stream) {
    k_build_chunks<<<1, 1024, 0, stream>>>(offsets, E, n_slots, minibatch, cap, chunks, max_ch, mbs, max_mb, counts2,
                                           reinterpret_cast<DevStatus*>(status));
    return cudaGetLastError();
}

size_t gemm_smem_bytes() { return SMEM_ALLOC; }

// Defaults measured on B200 (page shape and a 512-rows-per-expert case):
// L2 prefetch of weight tiles did not pay (the token-side TMA op count was
// the limit), small raster groups did.  MOK_GEMM_L2_PREFETCH and
// MOK_GEMM_GROUP override them (tuning knobs only, results do not change).
GemmTuning gemm_tuning() {
    GemmTuning v{0, 2};
    if (const char* s = getenv("MOK_GEMM_L2_PREFETCH")) v.l2_prefetch = atoi(s) < 0 ? 0 : atoi(s);
    if (const char* s = getenv("MOK_GEMM_GROUP")) v.group_chunks = atoi(s) < 1 ? 1 : atoi(s);
    return v;
}

cudaError_t gemm_configure(int dev) {
    static bool done[64] = {};
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (done[dev]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_grouped_gemm<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
    if (e == cudaSuccess) done[dev] = true;
    return e;
}

cudaError_t launch_gemm_phase(int phase, const CUtensorMap& tmA0, const CUtensorMap& tmA1, const BMaps& tmB,
                              const GemmShape& sh, const Chunk* chunks, const int* counts2, void* h_out, void* out,
                              const int32_t* row_slot, void* status, uint64_t timeout_ns, int grid,
                              const GemmTuning& tune, cudaStream_t stream) {
    GemmParams p;
    p.chunks = chunks;
    p.counts2 = counts2;
    p.K = phase == 0 ? sh.H : sh.I;
    p.MT = phase == 0 ? sh.I / 64 : sh.H / 128;
    p.w_rows = phase == 0 ? sh.H : sh.I;
    p.I = sh.I;
    p.H = sh.H;
    p.h_out = reinterpret_cast<__half*>(h_out);
    p.out = reinterpret_cast<float*>(out);
    p.row_slot = row_slot;
    p.st = reinterpret_cast<DevStatus*>(status);
    p.timeout_ns = timeout_ns;
    p.l2_prefetch = tune.l2_prefetch;
    p.group_chunks = tune.group_chunks > 0 ? tune.group_chunks : 1;
    if (phase == 0)
        k_grouped_gemm<0><<<grid, GEMM_THREADS, SMEM_ALLOC, stream>>>(tmA0, tmA1, tmB, p);
    else
        k_grouped_gemm<1><<<grid, GEMM_THREADS, SMEM_ALLOC, stream>>>(tmA0, tmA1, tmB, p);
    return cudaGetLastError();
}

}  // namespace mok

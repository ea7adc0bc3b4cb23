// bwd.cu -- the backward of the forward MoE layer (bf16 path): the pull
// reverse-combine and the weight-gradient grouped GEMM.  The data-gradient
// GEMMs (dh with the SwiGLU backward, dx pushed to the token slots) are
// phases 2 and 3 of the grouped-GEMM core (gemm_core.cuh); the push
// reverse-dispatch sum is the combine with unit weights.
//
// MoK article (tahou.com), the Pull/Push paragraph: the backward pairs a
// pull reverse-combine (the expert side reads the output gradient of every
// token it served) with a push reverse-dispatch (each row's input gradient
// goes straight back to its token).  The arithmetic is the chain rule of
// the forward layer, in that order of steps:
//   do_tj = g_tj dy_t,  dg_tj = <dy_t, o_tj>          (reverse combine)
//   dh = do Wd^T;  da = dh b silu'(a),  db = dh silu(a)
//   dx_row = da Wg^T + db Wu^T,  dx_t = sum_j dx_row(t, j) (reverse dispatch)
//   dWd = h^T do,  dWg = x^T da,  dWu = x^T db          (per expert, over its rows)
//   dl_tj = g_tj (dg_tj - sum_i g_ti dg_ti)              (softmax backward)
#include "mok_device.cuh"
#include "mok_internal.h"

namespace mok {

// ------------------------------------------------------------------ reverse combine
// One warp per token: dy_t is read once (16-byte vectors, 8 features per
// lane); for each of its k slots the warp writes the bf16 row do = g dy_t to
// the slot's expert-major row and accumulates <dy_t, o_slot> from the
// forward's slot rows (fp16 with block exponents); then the softmax backward over the k gates
// gives the token's dlogits row (zeros outside its selection).
template <int KB>
__global__ void __launch_bounds__(256) k_reverse_combine(ShardsIn dys, int S_r, int H, int T, int k, int E,
                                                         const int32_t* __restrict__ pos,
                                                         const float* __restrict__ gates,
                                                         const int32_t* __restrict__ topk_idx,
                                                         const uint16_t* __restrict__ o_slots,
                                                         const int8_t* __restrict__ o_exps,
                                                         uint4* __restrict__ do_rows, float* __restrict__ dlogits) {
    const int lane = threadIdx.x & 31;
    const int nvec = H >> 3;
    const int warps = gridDim.x * 8;
    for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < T; t += warps) {
        const int r = t / S_r;
        const uint4* dy = reinterpret_cast<const uint4*>(dys.p[r]) + (size_t)(t - r * S_r) * nvec;
        const int my_row = lane < k ? __ldg(pos + (size_t)t * k + lane) : 0;
        const float my_g = lane < k ? __ldg(gates + (size_t)t * k + lane) : 0.f;
        int rows[KB];
        float gs[KB], dgp[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            rows[j] = __shfl_sync(0xffffffffu, my_row, j & 31);
            gs[j] = __shfl_sync(0xffffffffu, my_g, j & 31);
            dgp[j] = 0.f;
        }
        // lanes may run different numbers of iterations: no warp collectives inside
        for (int v = lane; v < nvec; v += 32) {
            const uint4 raw = __ldg(dy + v);
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
            float d[8];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                d[2 * p] = __uint_as_float(w[p] << 16);
                d[2 * p + 1] = __uint_as_float(w[p] & 0xffff0000u);
            }
            // the forward's slot rows: fp16 values, one power-of-two exponent per
            // 128 features; the loads of up to 8 slots are issued before any is used
            constexpr int C = KB < 8 ? KB : 8;
#pragma unroll
            for (int j0 = 0; j0 < KB; j0 += C) {
                if (j0 >= k) break;
                uint4 ovs[C];
                int exs[C];
#pragma unroll
                for (int c = 0; c < C; ++c) {
                    if (j0 + c < k) {
                        const size_t slot = (size_t)t * k + j0 + c;
                        ovs[c] = __ldcs(reinterpret_cast<const uint4*>(o_slots + slot * H) + v);
                        exs[c] = __ldg(o_exps + slot * (H >> 7) + (v >> 4));
                    }
                }
#pragma unroll
            for (int c = 0; c < C; ++c) {
                const int j = j0 + c;
                if (j < k) {
                    const uint4 ov = ovs[c];
                    const float sc = __int_as_float((exs[c] + 127) << 23);
                    const __half2* oh = reinterpret_cast<const __half2*>(&ov);
                    float acc = 0.f;
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float2 of = __half22float2(oh[p]);
                        acc += d[2 * p] * of.x + d[2 * p + 1] * of.y;
                    }
                    dgp[j] += acc * sc;
                    const float g = gs[j];
                    do_rows[(size_t)rows[j] * nvec + v] =
                        make_uint4(pack_bf16x2(g * d[0], g * d[1]), pack_bf16x2(g * d[2], g * d[3]),
                                   pack_bf16x2(g * d[4], g * d[5]), pack_bf16x2(g * d[6], g * d[7]));
                }
            }
            }
        }
        // dg_j over the warp; every lane ends with every sum
#pragma unroll
        for (int j = 0; j < KB; ++j) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dgp[j] += __shfl_xor_sync(0xffffffffu, dgp[j], off);
        }
        float dot = 0.f;
#pragma unroll
        for (int j = 0; j < KB; ++j)
            if (j < k) dot += gs[j] * dgp[j];
        float* dl = dlogits + (size_t)t * E;
        for (int e = lane; e < E; e += 32) dl[e] = 0.f;
        __syncwarp();
#pragma unroll
        for (int j = 0; j < KB; ++j)
            if (j < k && lane == (j & 31)) dl[__ldg(topk_idx + (size_t)t * k + j)] = gs[j] * (dgp[j] - dot);
    }
}

cudaError_t launch_reverse_combine(const ShardsIn& dys, int S_r, int H, int T, int k, int E, const int32_t* pos,
                                   const float* gates, const int32_t* topk_idx, const uint16_t* o_slots,
                                   const int8_t* o_exps, void* do_rows, float* dlogits, int num_sms,
                                   cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    const int want = (T + 7) / 8;
    const int grid = want < num_sms * 8 ? want : num_sms * 8;
    uint4* d = reinterpret_cast<uint4*>(do_rows);
    if (k <= 2)
        k_reverse_combine<2><<<grid, 256, 0, stream>>>(dys, S_r, H, T, k, E, pos, gates, topk_idx, o_slots, o_exps, d,
                                                       dlogits);
    else if (k <= 8)
        k_reverse_combine<8><<<grid, 256, 0, stream>>>(dys, S_r, H, T, k, E, pos, gates, topk_idx, o_slots, o_exps, d,
                                                       dlogits);
    else
        k_reverse_combine<32><<<grid, 256, 0, stream>>>(dys, S_r, H, T, k, E, pos, gates, topk_idx, o_slots, o_exps,
                                                        d, dlogits);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ weight gradients
// Units (expert e, gradient, M tile of 128 output rows, N tile of NB output
// columns), expert-major so that the CTAs working at one time share an
// expert's rows in L2:
//   dWd[e] [I, H] = h^T do:   M = i, N = h, A = h rows, B = do rows
//   dWg[e] [H, I] = x^T da:   M = h, N = i, A = x rows, B = da (dab cols 0..I)
//   dWu[e] [H, I] = x^T db:   M = h, N = i, A = x rows, B = db (dab cols I..2I)
// K = the expert's rows, 64 per stage; both operands are MN-major tiles
// (128-byte swizzle), each loaded as ONE 3D box of its 64-column blocks
// ({64 columns, 64 rows, blocks}).  Work is dealt in "rows of tiles": one
// (expert, gradient, M tile) and all its N tiles, so a CTA loads the A
// tile (x or h rows of its 128 features, up to 4 K stages: 256 rows) once
// and keeps it in shared memory while the B tiles of the N tiles stream
// through a ring (an expert taller than that reloads A for every tile
// through the same four slots).  Rows of the last stage past the expert
// belong to the next expert (or are TMA zero fill): the MMA warp zeroes
// them in the A tile (then every product with those rows is 0), once per
// load, before it issues that stage.  Accumulators: two of NB columns in
// TMEM, so one tile's epilogue overlaps the next's MMAs.  The epilogue
// writes the bf16 tile 64 columns at a time into a ring of two
// 128-byte-swizzled staging blocks and stores each block with one TMA op.
constexpr int WG_THREADS = 192;  // warp 0 TMA, 1 MMA (and tail zeroing), 2-5 epilogue
constexpr int WG_NST = 4;        // B stages
constexpr int WG_AS = 4;         // A slots (K stages of the resident A tile)
constexpr int WG_A_BYTES = 128 * 64 * 2;  // 16 KB
constexpr int WG_NB_MAX = 256;
constexpr int WG_B_MAX = WG_NB_MAX * 128;                    // 32 KB
constexpr int WG_OUT_BLOCK = 128 * 64 * 2;                   // one 64-column block of the tile, 16 KB
constexpr int WG_OUT_BYTES = 2 * WG_OUT_BLOCK;               // ring of two blocks
constexpr int WG_SMEM = WG_NST * WG_B_MAX + WG_AS * WG_A_BYTES + WG_OUT_BYTES + 256 + 1024;
static_assert(WG_SMEM <= 232448, "weight-gradient layout exceeds shared memory");
// bound of the waits that drain this CTA's own loads and MMAs before it leaves
constexpr uint64_t DRAIN_NS_WG = 1000000000ull;

// Two 32-column TMEM loads of this warp's 32 lanes (columns t0.. and
// t1..), one wait.
__device__ __forceinline__ void tmem_ld2_32x32b_x32(uint32_t t0, uint32_t t1, float (&v)[64]) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]),
          "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]),
          "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]),
          "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]),
          "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(t0), "r"(t1)
        : "memory");
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

struct WgradMaps {
    // operands: {64, rows, blocks} views of x [N_s, H], h [N_s, I], do [N_s, H], dab [N_s, 2I]
    CUtensorMap x, h, dor, dab;
    // outputs: {64, 128} boxes of dWd [E*I, H], dWg / dWu [E*H, I]
    CUtensorMap owd, owg, owu;
};

struct WgradArgs {
    int H, I, E, nb;             // nb: N tile (256 or 128)
    int dm_t, dn_t, gm_t, gn_t;  // M / N tiles of dWd and of dWg (= dWu)
    int spe;                     // rows of tiles per expert: dm_t + 2 gm_t
    const int32_t* offsets;      // [E+1]
    DevStatus* st;
    uint64_t timeout_ns;
};

// One row of tiles: expert e, gradient g (0 dWd, 1 dWg, 2 dWu), M tile m0,
// nt N tiles; the expert's rows r0 .. r0 + rows.
struct WgRow {
    int e, g, m0, nt, r0, rows;
};

__device__ __forceinline__ bool wg_row(const WgradArgs& a, int s, WgRow& w) {
    if (s >= a.E * a.spe) return false;
    w.e = s / a.spe;
    int r = s - w.e * a.spe;
    if (r < a.dm_t) {
        w.g = 0;
        w.m0 = r * 128;
        w.nt = a.dn_t;
    } else {
        r -= a.dm_t;
        w.g = r < a.gm_t ? 1 : 2;
        if (r >= a.gm_t) r -= a.gm_t;
        w.m0 = r * 128;
        w.nt = a.gn_t;
    }
    w.r0 = __ldg(a.offsets + w.e);
    w.rows = __ldg(a.offsets + w.e + 1) - w.r0;
    return true;
}

__global__ void __launch_bounds__(WG_THREADS, 1)
    k_wgrad(const __grid_constant__ WgradMaps maps, const WgradArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                           ~uintptr_t(1023));
    const uint32_t b_bytes = (uint32_t)a.nb * 64 * 2;
    unsigned char* ares = smem + WG_NST * WG_B_MAX;                        // A slots, 16 KB each
    unsigned char* otile = ares + WG_AS * WG_A_BYTES;                      // 2 x [128 rows][128 B], swizzled
    uint64_t* full = reinterpret_cast<uint64_t*>(otile + WG_OUT_BYTES);  // B bytes landed
    uint64_t* empty = full + WG_NST;                                     // B stage consumed (MMA commit)
    uint64_t* afull = empty + WG_NST;                                    // A slot landed
    uint64_t* aempty = afull + WG_AS;                                    // A slot's last use consumed
    uint64_t* tfull = aempty + WG_AS;
    uint64_t* tempty = tfull + 2;
    uint64_t* fin = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
    volatile int* ok_flags = reinterpret_cast<volatile int*>(tmem_slot + 1);  // one per epilogue warp
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < WG_NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < WG_AS; ++s) {
            mbar_init(&afull[s], 1);
            mbar_init(&aempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);  // one arrival per epilogue warp
        }
        mbar_init(fin, 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&maps.x);
        tma_prefetch_desc(&maps.h);
        tma_prefetch_desc(&maps.dor);
        tma_prefetch_desc(&maps.dab);
        tma_prefetch_desc(&maps.owd);
        tma_prefetch_desc(&maps.owg);
        tma_prefetch_desc(&maps.owu);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    WgRow w;

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA: the A tile of each row of tiles (once when it fits the
            // slots), the B tile of every N tile
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_phase = 0;
            uint32_t aph = 0, a_issued = 0, a_issued_phase = 0;  // bit s: loads into A slot s so far, mod 2
            bool ok = true;
            for (int i = 0; ok && wg_row(a, blockIdx.x + i * gridDim.x, w); ++i) {
                if (w.rows == 0) continue;  // the epilogue writes zeros
                const int KB = (w.rows + 63) / 64;
                const bool res = KB <= WG_AS;
                const CUtensorMap* am = w.g == 0 ? &maps.h : &maps.x;
                const CUtensorMap* bm = w.g == 0 ? &maps.dor : &maps.dab;
                for (int n = 0; ok && n < w.nt; ++n) {
                    const int bz0 = (n * a.nb + (w.g == 2 ? a.I : 0)) / 64;  // first 64-column block of B
                    for (int kb = 0; kb < KB; ++kb) {
                        const int y = w.r0 + kb * 64;
                        if (n == 0 || !res) {
                            const int sl = kb & (WG_AS - 1);
                            const uint32_t p = (aph >> sl) & 1u;
                            if (!mbar_wait(&aempty[sl], p ^ 1u, a.st, a.timeout_ns, 107)) {
                                ok = false;
                                break;
                            }
                            mbar_arrive_expect_tx(&afull[sl], (uint32_t)WG_A_BYTES);
                            tma_load_3d(ares + sl * WG_A_BYTES, am, &afull[sl], 0, y, w.m0 / 64);
                            a_issued |= 1u << sl;
                            a_issued_phase = (a_issued_phase & ~(1u << sl)) | (p << sl);
                            aph ^= 1u << sl;
                        }
                        if (!mbar_wait(&empty[stage], phase ^ 1u, a.st, a.timeout_ns, 100)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&full[stage], b_bytes);
                        tma_load_3d(smem + stage * WG_B_MAX, bm, &full[stage], 0, y, bz0);
                        issued |= 1u << stage;
                        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                        if (++stage == WG_NST) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
            // never leave with a load in flight into this CTA's shared memory
            for (int s = 0; s < WG_NST; ++s)
                if ((issued >> s) & 1u) mbar_wait(&full[s], (issued_phase >> s) & 1u, nullptr, DRAIN_NS_WG, 101);
            for (int s = 0; s < WG_AS; ++s)
                if ((a_issued >> s) & 1u) mbar_wait(&afull[s], (a_issued_phase >> s) & 1u, nullptr, DRAIN_NS_WG, 108);
        }
    } else if (warp == 1) {
        // ---- MMA, one thread: it also zeroes an A load's rows past the
        // expert before their first use (once per row of tiles when A stays
        // resident)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, tk = 0, aph = 0;
            const uint32_t idesc = umma_idesc_f16(128, a.nb, /*A MN-major*/ 1, /*B MN-major*/ 1, /*bf16*/ 1);
            bool ok = true;
            for (int i = 0; ok && wg_row(a, blockIdx.x + i * gridDim.x, w); ++i) {
                if (w.rows == 0) continue;  // the epilogue writes zeros; no accumulator is used
                const int KB = (w.rows + 63) / 64;
                const bool res = KB <= WG_AS;
                for (int n = 0; ok && n < w.nt; ++n) {
                    if (!mbar_wait(&tempty[tk & 1u], ((tk >> 1) & 1u) ^ 1u, a.st, a.timeout_ns, 102)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const bool last_use = !res || n == w.nt - 1;
                    for (int kb = 0; kb < KB; ++kb) {
                        const int sl = kb & (WG_AS - 1);
                        const int valid = min(64, w.rows - kb * 64);
                        const int nks = (valid + 15) >> 4;  // MMAs of 16 K rows that hold any of the expert's rows
                        if (n == 0 || !res) {
                            if (!mbar_wait(&afull[sl], (aph >> sl) & 1u, a.st, a.timeout_ns, 109)) {
                                ok = false;
                                break;
                            }
                            aph ^= 1u << sl;
                            if (valid < nks * 16) {
                                // a K row is one 128-byte line of each 64-column block (8 KB); only
                                // the rows of the last MMA's 16 need zeros, the MMAs past it are
                                // not issued
                                unsigned char* st = ares + sl * WG_A_BYTES;
                                for (int blk = 0; blk < 2; ++blk)
                                    for (int l = valid; l < nks * 16; ++l)
#pragma unroll
                                        for (int c = 0; c < 8; ++c)
                                            *reinterpret_cast<uint4*>(st + blk * 8192 + l * 128 + c * 16) =
                                                make_uint4(0, 0, 0, 0);
                                fence_proxy_async_shared();  // generic writes -> the MMA reads them
                            }
                        }
                        if (!mbar_wait(&full[stage], phase, a.st, a.timeout_ns, 103)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sa = smem_u32(ares + sl * WG_A_BYTES), sb = smem_u32(smem + stage * WG_B_MAX);
                        for (int ks = 0; ks < nks; ++ks) {
                            // both MN-major SW128: 16 K rows = 2 atoms of 1 KB; 64-wide blocks 8 KB apart
                            const uint64_t ad = umma_desc_sw128(sa + ks * 2048, 8192, 1024);
                            const uint64_t bd = umma_desc_sw128(sb + ks * 2048, 8192, 1024);
                            umma_bf16(tmem + (tk & 1u) * 256u, ad, bd, idesc, (kb | ks) != 0 ? 1u : 0u);
                        }
                        umma_commit(&empty[stage]);
                        if (last_use) umma_commit(&aempty[sl]);
                        if (++stage == WG_NST) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (!ok) break;
                    umma_commit(&tfull[tk & 1u]);
                    ++tk;
                }
            }
            umma_commit(fin);
            mbar_wait(fin, 0, nullptr, DRAIN_NS_WG, 104);
        }
    } else {
        // ---- epilogue (warps 2-5; a warp reads TMEM lanes 32 (warp % 4) + 0..31):
        // TMEM lane = output row m0 + 32 q + lane; bf16 into the swizzled
        // staging blocks, one TMA store (and one bulk group) per 64-column
        // block as soon as it is written.  A block buffer is written again
        // two blocks later, once its store has read it (the one younger
        // group may still be reading the other buffer).
        const int q = warp & 3;
        const int r = q * 32 + lane;  // row inside the tile
        const bool leader = warp == 3 && lane == 0;
        const int nblk = a.nb / 64;
        uint32_t tk = 0, gb = 0;
        bool all_ok = true;
        for (int i = 0; all_ok && wg_row(a, blockIdx.x + i * gridDim.x, w); ++i) {
            for (int n = 0; n < w.nt; ++n) {
                int ok = 1;
                if (w.rows > 0 && lane == 0) ok = mbar_wait(&tfull[tk & 1u], (tk >> 1) & 1u, a.st, a.timeout_ns, 105) ? 1 : 0;
                if (lane == 0) ok_flags[q] = ok;
                named_bar_sync(1, 128);
                // the four warps leave or go on together
                all_ok = (ok_flags[0] & ok_flags[1] & ok_flags[2] & ok_flags[3]) != 0;
                named_bar_sync(1, 128);  // the flags are written again at the next tile
                if (!all_ok) break;
                if (w.rows > 0) tc_fence_after();
                const CUtensorMap* om = w.g == 0 ? &maps.owd : (w.g == 1 ? &maps.owg : &maps.owu);
                const int y0 = w.e * (w.g == 0 ? a.I : a.H) + w.m0;
                const int n0 = n * a.nb;
                for (int b = 0; b < nblk; ++b, ++gb) {
                    float v[64];  // the block's 64 columns of this row: two TMEM loads, one wait
                    if (w.rows > 0) {
                        const uint32_t t = tmem + ((uint32_t)(q * 32) << 16) + (tk & 1u) * 256u + (uint32_t)(b * 64);
                        tmem_ld2_32x32b_x32(t, t + 32u, v);
                    } else {
#pragma unroll
                        for (int p = 0; p < 64; ++p) v[p] = 0.f;
                    }
                    unsigned char* buf = otile + (gb & 1u) * WG_OUT_BLOCK;
                    if (leader) bulk_wait_read<1>();
                    named_bar_sync(1, 128);  // the buffer is free
                    unsigned char* blk = buf + r * 128;
#pragma unroll
                    for (int p = 0; p < 8; ++p)  // 16-byte chunk p of the row's 128-byte line
                        *reinterpret_cast<uint4*>(blk + ((p ^ (r & 7)) << 4)) =
                            make_uint4(pack_bf16x2(v[8 * p], v[8 * p + 1]), pack_bf16x2(v[8 * p + 2], v[8 * p + 3]),
                                       pack_bf16x2(v[8 * p + 4], v[8 * p + 5]), pack_bf16x2(v[8 * p + 6], v[8 * p + 7]));
                    if (b == nblk - 1 && w.rows > 0) {
                        // every column of the accumulator has been read
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty[tk & 1u]);
                        ++tk;
                    }
                    fence_proxy_async_shared();  // generic writes of the block -> the TMA store reads them
                    named_bar_sync(1, 128);
                    if (leader) {
                        tma_store_2d(om, buf, n0 + b * 64, y0);
                        bulk_commit();
                    }
                }
            }
        }
        if (leader) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

cudaError_t launch_wgrad(const void* x_rows, const void* h_rows, const void* do_rows, const void* dab, int n_rows,
                         const int32_t* offsets, int H, int I, int E, void* dwg, void* dwu, void* dwd, void* status,
                         uint64_t timeout_ns, int num_sms, const char** err, cudaStream_t stream) {
    WgradArgs a{};
    a.H = H;
    a.I = I;
    a.E = E;
    a.nb = (H % 256 == 0 && I % 256 == 0) ? 256 : 128;
    WgradMaps maps;
    if (!encode_cols3d_bf16(&maps.x, x_rows, (uint64_t)H, (uint64_t)n_rows, 64, 2, err) ||
        !encode_cols3d_bf16(&maps.h, h_rows, (uint64_t)I, (uint64_t)n_rows, 64, 2, err) ||
        !encode_cols3d_bf16(&maps.dor, do_rows, (uint64_t)H, (uint64_t)n_rows, 64, a.nb / 64, err) ||
        !encode_cols3d_bf16(&maps.dab, dab, (uint64_t)2 * I, (uint64_t)n_rows, 64, a.nb / 64, err) ||
        !encode_tmap_2d_bf16(&maps.owd, dwd, (uint64_t)H, (uint64_t)E * I, 64, 128, err) ||
        !encode_tmap_2d_bf16(&maps.owg, dwg, (uint64_t)I, (uint64_t)E * H, 64, 128, err) ||
        !encode_tmap_2d_bf16(&maps.owu, dwu, (uint64_t)I, (uint64_t)E * H, 64, 128, err))
        return cudaErrorInvalidValue;
    a.dm_t = I / 128;
    a.dn_t = H / a.nb;
    a.gm_t = H / 128;
    a.gn_t = I / a.nb;
    a.spe = a.dm_t + 2 * a.gm_t;
    a.offsets = offsets;
    a.st = reinterpret_cast<DevStatus*>(status);
    a.timeout_ns = timeout_ns;
    static bool attr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr[dev]) {
        e = cudaFuncSetAttribute(k_wgrad, cudaFuncAttributeMaxDynamicSharedMemorySize, WG_SMEM);
        if (e != cudaSuccess) return e;
        attr[dev] = true;
    }
    const long long units = (long long)E * a.spe;  // rows of tiles
    const int grid = (int)(units < num_sms ? units : num_sms);
    *err = "weight-gradient launch";
    if (grid <= 0) return cudaSuccess;
    k_wgrad<<<grid, WG_THREADS, WG_SMEM, stream>>>(maps, a);
    return cudaGetLastError();
}

}  // namespace mok

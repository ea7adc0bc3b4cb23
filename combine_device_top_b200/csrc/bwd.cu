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
#pragma unroll
            for (int j = 0; j < KB; ++j) {
                if (j < k) {
                    // the forward's slot row: fp16 values, one power-of-two exponent per 128 features
                    const size_t slot = (size_t)t * k + j;
                    const uint4 ov = __ldcs(reinterpret_cast<const uint4*>(o_slots + slot * H) + v);
                    const float sc = __int_as_float(((int)__ldg(o_exps + slot * (H >> 7) + (v >> 4)) + 127) << 23);
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
// ({64 columns, 64 rows, blocks}).  Rows of the last stage past the expert
// belong to the next expert (or are TMA zero fill): the MMA warp zeroes
// them in the A tile (x or h rows; then every product with those rows is
// 0) before it issues that stage.  Accumulators: two of NB columns in TMEM,
// so one unit's epilogue overlaps the next's MMAs.  The epilogue writes the
// bf16 tile 64 columns at a time into a ring of two 128-byte-swizzled
// staging blocks and stores each block with one TMA op.
constexpr int WG_THREADS = 192;  // warp 0 TMA, 1 MMA (and tail zeroing), 2-5 epilogue
constexpr int WG_NST = 4;
constexpr int WG_A_BYTES = 128 * 64 * 2;  // 16 KB
constexpr int WG_NB_MAX = 256;
constexpr int WG_STAGE_MAX = WG_A_BYTES + WG_NB_MAX * 128;  // 48 KB
constexpr int WG_OUT_BLOCK = 128 * 64 * 2;                   // one 64-column block of the tile, 16 KB
constexpr int WG_OUT_BYTES = 2 * WG_OUT_BLOCK;               // ring of two blocks
constexpr int WG_SMEM = WG_NST * WG_STAGE_MAX + WG_OUT_BYTES + 256 + 1024;
static_assert(WG_SMEM <= 232448, "weight-gradient layout exceeds shared memory");
// bound of the waits that drain this CTA's own loads and MMAs before it leaves
constexpr uint64_t DRAIN_NS_WG = 1000000000ull;

struct WgradMaps {
    // operands: {64, rows, blocks} views of x [N_s, H], h [N_s, I], do [N_s, H], dab [N_s, 2I]
    CUtensorMap x, h, dor, dab;
    // outputs: {64, 128} boxes of dWd [E*I, H], dWg / dWu [E*H, I]
    CUtensorMap owd, owg, owu;
};

struct WgradArgs {
    int H, I, E, nb;             // nb: N tile (256 or 128)
    int dm_t, dn_t, gm_t, gn_t;  // M / N tiles of dWd and of dWg (= dWu)
    int upe;                     // units per expert
    const int32_t* offsets;      // [E+1]
    DevStatus* st;
    uint64_t timeout_ns;
};

struct WgUnit {
    int e, g, m0, n0, r0, rows;  // g: 0 dWd, 1 dWg, 2 dWu
};

__device__ __forceinline__ bool wg_unit(const WgradArgs& a, int u, WgUnit& w) {
    if (u >= a.E * a.upe) return false;
    w.e = u / a.upe;
    int r = u - w.e * a.upe;
    const int nd = a.dm_t * a.dn_t, ng = a.gm_t * a.gn_t;
    if (r < nd) {
        w.g = 0;
        w.m0 = (r / a.dn_t) * 128;
        w.n0 = (r % a.dn_t) * a.nb;
    } else {
        r -= nd;
        w.g = r < ng ? 1 : 2;
        if (r >= ng) r -= ng;
        w.m0 = (r / a.gn_t) * 128;
        w.n0 = (r % a.gn_t) * a.nb;
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
    const int b_bytes = a.nb * 64 * 2;
    const int stage_bytes = WG_A_BYTES + b_bytes;
    unsigned char* otile = smem + WG_NST * WG_STAGE_MAX;                  // 2 x [128 rows][128 B], swizzled
    uint64_t* full = reinterpret_cast<uint64_t*>(otile + WG_OUT_BYTES);  // TMA bytes landed
    uint64_t* empty = full + WG_NST;                                     // stage consumed (MMA commit)
    uint64_t* tfull = empty + WG_NST;
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
    WgUnit w;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_phase = 0;
            bool ok = true;
            for (int i = 0; ok && wg_unit(a, blockIdx.x + i * gridDim.x, w); ++i) {
                const int KB = (w.rows + 63) / 64;
                const CUtensorMap* am = w.g == 0 ? &maps.h : &maps.x;
                const CUtensorMap* bm = w.g == 0 ? &maps.dor : &maps.dab;
                const int bz0 = (w.n0 + (w.g == 2 ? a.I : 0)) / 64;  // first 64-column block of B
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, a.st, a.timeout_ns, 100)) {
                        ok = false;
                        break;
                    }
                    unsigned char* st = smem + stage * WG_STAGE_MAX;
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)stage_bytes);
                    const int y = w.r0 + kb * 64;
                    tma_load_3d(st, am, &full[stage], 0, y, w.m0 / 64);
                    tma_load_3d(st + WG_A_BYTES, bm, &full[stage], 0, y, bz0);
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == WG_NST) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < WG_NST; ++s)
                if ((issued >> s) & 1u) mbar_wait(&full[s], (issued_phase >> s) & 1u, nullptr, DRAIN_NS_WG, 101);
        }
    } else if (warp == 1) {
        // ---- MMA (lane 0 waits and issues); the whole warp zeroes the A
        // tile's rows past the expert in the unit's last stage first
        int stage = 0;
        uint32_t phase = 0, tk = 0;
        const uint32_t idesc = umma_idesc_f16(128, a.nb, /*A MN-major*/ 1, /*B MN-major*/ 1, /*bf16*/ 1);
        bool ok = true;
        for (int i = 0; ok && wg_unit(a, blockIdx.x + i * gridDim.x, w); ++i) {
            if (w.rows == 0) continue;  // the epilogue writes zeros; no accumulator is used
            const int KB = (w.rows + 63) / 64;
            int got = 0;
            if (lane == 0) got = mbar_wait(&tempty[tk & 1u], ((tk >> 1) & 1u) ^ 1u, a.st, a.timeout_ns, 102) ? 1 : 0;
            if (__shfl_sync(0xffffffffu, got, 0) == 0) break;
            tc_fence_after();
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) got = mbar_wait(&full[stage], phase, a.st, a.timeout_ns, 103) ? 1 : 0;
                if (__shfl_sync(0xffffffffu, got, 0) == 0) {
                    ok = false;
                    break;
                }
                const int valid = min(64, w.rows - kb * 64);
                const int nks = (valid + 15) >> 4;  // MMAs of 16 K rows that hold any of the expert's rows
                if (valid < nks * 16) {
                    // a K row is one 128-byte line of each 64-column block (8 KB); only the
                    // rows of the last MMA's 16 need zeros, the MMAs past it are not issued
                    unsigned char* st = smem + stage * WG_STAGE_MAX;
                    const int lines = nks * 16 - valid;
                    for (int i2 = lane; i2 < 2 * lines * 8; i2 += 32) {
                        const int blk = i2 / (lines * 8), rem = i2 - blk * lines * 8;
                        *reinterpret_cast<uint4*>(st + blk * 8192 + (valid + rem / 8) * 128 + (rem % 8) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_shared();  // generic writes -> the MMA reads them
                }
                __syncwarp();
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * WG_STAGE_MAX), sb = sa + WG_A_BYTES;
                    for (int ks = 0; ks < nks; ++ks) {
                        // both MN-major SW128: 16 K rows = 2 atoms of 1 KB; 64-wide blocks 8 KB apart
                        const uint64_t ad = umma_desc_sw128(sa + ks * 2048, 8192, 1024);
                        const uint64_t bd = umma_desc_sw128(sb + ks * 2048, 8192, 1024);
                        umma_bf16(tmem + (tk & 1u) * 256u, ad, bd, idesc, (kb | ks) != 0 ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);
                }
                __syncwarp();
                if (++stage == WG_NST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit(&tfull[tk & 1u]);
            ++tk;
        }
        if (lane == 0) {
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
        for (int i = 0; wg_unit(a, blockIdx.x + i * gridDim.x, w); ++i) {
            int ok = 1;
            if (w.rows > 0 && lane == 0) ok = mbar_wait(&tfull[tk & 1u], (tk >> 1) & 1u, a.st, a.timeout_ns, 105) ? 1 : 0;
            if (lane == 0) ok_flags[q] = ok;
            named_bar_sync(1, 128);
            // the four warps leave or go on together
            const int all_ok = ok_flags[0] & ok_flags[1] & ok_flags[2] & ok_flags[3];
            named_bar_sync(1, 128);  // the flags are written again at the next unit
            if (!all_ok) break;
            if (w.rows > 0) tc_fence_after();
            const CUtensorMap* om = w.g == 0 ? &maps.owd : (w.g == 1 ? &maps.owg : &maps.owu);
            const int y0 = w.e * (w.g == 0 ? a.I : a.H) + w.m0;
            for (int b = 0; b < nblk; ++b, ++gb) {
                unsigned char* buf = otile + (gb & 1u) * WG_OUT_BLOCK;
                if (leader) bulk_wait_read<1>();
                named_bar_sync(1, 128);  // the buffer is free
                unsigned char* blk = buf + r * 128;
#pragma unroll
                for (int c2 = 0; c2 < 64; c2 += 32) {
                    float v[32];
                    if (w.rows > 0) {
                        tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + (tk & 1u) * 256u + (uint32_t)(b * 64 + c2),
                                           v);
                    } else {
#pragma unroll
                        for (int p = 0; p < 32; ++p) v[p] = 0.f;
                    }
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const int chunk = c2 / 8 + p;  // 16-byte chunk of the row's 128-byte line
                        *reinterpret_cast<uint4*>(blk + ((chunk ^ (r & 7)) << 4)) =
                            make_uint4(pack_bf16x2(v[8 * p], v[8 * p + 1]), pack_bf16x2(v[8 * p + 2], v[8 * p + 3]),
                                       pack_bf16x2(v[8 * p + 4], v[8 * p + 5]), pack_bf16x2(v[8 * p + 6], v[8 * p + 7]));
                    }
                }
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
                    tma_store_2d(om, buf, w.n0 + b * 64, y0);
                    bulk_commit();
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
    a.upe = a.dm_t * a.dn_t + 2 * a.gm_t * a.gn_t;
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
    const long long units = (long long)E * a.upe;
    const int grid = (int)(units < num_sms ? units : num_sms);
    *err = "weight-gradient launch";
    if (grid <= 0) return cudaSuccess;
    k_wgrad<<<grid, WG_THREADS, WG_SMEM, stream>>>(maps, a);
    return cudaGetLastError();
}

}  // namespace mok

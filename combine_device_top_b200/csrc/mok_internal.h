// mok_internal.h -- host-side declarations shared by the translation units
// of libmok (workspace layouts and kernel launchers).  Not installed.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "mok.h"

namespace mok {

// ---- plan workspace (byte offsets from the workspace base)
struct PlanLayout {
    int nb;  // route blocks
    size_t status, counts, offsets, src_rank, src_index, row_slot, pos, topk, gates, blk_cnt, rank, total;
};
size_t plan_layout(int T, int E, int k, PlanLayout* L);
cudaError_t launch_plan(const float* logits, int T, int E, int k, int R, unsigned char* ws, const PlanLayout& L,
                        cudaStream_t stream);
int plan_route_blocks(int T);
cudaError_t launch_plan_parts(const float* logits, int T, int E, int k, int R, int32_t* counts, int32_t* offsets,
                              int32_t* src_rank, int32_t* src_index, int32_t* row_slot, int32_t* pos,
                              int32_t* topk_idx, float* gates, int32_t* blk_cnt, int32_t* rank,
                              cudaStream_t stream);
// Steps after the top-k (histogram, scan, schedule) from a given topk_idx.
cudaError_t launch_plan_schedule(int T, int E, int k, int R, int32_t* counts, int32_t* offsets, int32_t* src_rank,
                                 int32_t* src_index, int32_t* row_slot, int32_t* pos, const int32_t* topk_idx,
                                 int32_t* blk_cnt, int32_t* rank, cudaStream_t stream);
// Records a message for mok_last_error_string() and returns `code`.
int report_error(int code, const char* msg);

// ---- token shards as kernel parameters
struct ShardsIn {
    const void* p[MOK_MAX_SHARDS];
};
struct ShardsOut {
    void* p[MOK_MAX_SHARDS];
};

// rows[pos[t*k + j]] = x[t] for every slot (token-major walk of the pull schedule)
cudaError_t launch_gather(const ShardsIn& xs, int S_r, int H, int T, int k, const int32_t* pos, void* rows,
                          int num_sms, cudaStream_t stream);
// the same with MXFP8 quantisation of every 32-element block: rows [*, H]
// E4M3, block scales in planes [H/128][sc_rows][4] (see mx_sc_rows)
cudaError_t launch_gather_mx(const ShardsIn& xs, int S_r, int H, int T, int k, const int32_t* pos, void* rows,
                             void* xsc, int sc_rows, int num_sms, cudaStream_t stream);
// Slot rows in MOK_SLOTS_F16S form: [n_slots, H] fp16, then, at this byte
// offset, [n_slots, H/128] int8 block exponents.
inline size_t slot_exp_offset(size_t n_slots, int H) { return (n_slots * (size_t)H * 2 + 255) & ~(size_t)255; }
inline size_t slot_bytes(size_t n_slots, int H, int slot_type) {
    if (slot_type == MOK_SLOTS_F16S) return slot_exp_offset(n_slots, H) + n_slots * (size_t)(H / 128);
    return n_slots * (size_t)H * (slot_type == MOK_SLOTS_BF16 ? 2 : 4);
}
// y = fixed-order weighted sum of the slot outputs out [T*k, H] of type
// slot_type (MOK_SLOTS_*); gates == nullptr: unit weights
cudaError_t launch_combine(const void* out, int slot_type, const float* gates, int T, int k, int H, int S_r,
                           const ShardsOut& ys, int num_sms, cudaStream_t stream);

// ---- work decomposition of the grouped GEMM
// A chunk is <= 256 consecutive rows of one expert inside one minibatch.
struct Chunk {
    int expert, row0, rows, mb;
};
// A minibatch is a range of rows [row0, row1) with its chunk range.
struct Minibatch {
    int row0, row1, chunk0, chunk1;
};
constexpr int CHUNK_MAX_ROWS = 256;
// MXFP8 path: two accumulators of <= 224 columns leave TMEM room for the
// block scale factors.
constexpr int CHUNK_MAX_ROWS_MX = 224;

int max_chunks(int n_slots, int E, int n_mb);
int max_minibatches(int n_slots, int minibatch);
// Rows of the expert-major layout that give `waves` full waves of
// gemm_ctas CTAs when a unit is a tile of tile_rows rows x tile_features of
// the 2I gate+up output columns: ceil(waves * ctas * rows * features / 2I).
int two_wave_rows(int I, int gemm_ctas, int waves, int tile_rows, int tile_features);
// max_rows: chunk height cap, CHUNK_MAX_ROWS or CHUNK_MAX_ROWS_MX.  A
// minibatch ends at the first expert boundary where it holds at least
// `minibatch` rows and min_units gate/up units (units_per_chunk per chunk),
// or at `cap` rows.
cudaError_t launch_build_chunks(const int32_t* offsets, int E, int n_slots, int minibatch, int cap, int max_rows,
                                int min_units, int units_per_chunk, Chunk* chunks, int max_chunks, Minibatch* mbs,
                                int max_mb, int* counts2, void* status, cudaStream_t stream);

// ---- the grouped GEMM (tcgen05)
// Slot buffers of the ranks of an expert-parallel group, as this GPU
// addresses them (peer pointers): fp16 slot rows and their exponents.
struct PushDest {
    void* out[MOK_MAX_SHARDS];
    int8_t* exp[MOK_MAX_SHARDS];
};
struct GemmShape {
    int H, I, E;
};
struct GemmTuning {
    int group_chunks;  // raster group size in chunks
    int pair;          // 1: units of two M tiles sharing each token tile (bf16 path)
    int cta_pair;      // bf16 launches on CTA pairs (tcgen05 cta_group::2): 0 none, 1 all but gate/up,
                       // 2 all, 3 as 1 plus gate/up with two M tiles per CTA when pairing
    int mx_rings;      // MXFP8 staged launches: 2 = weight and token rings, 1 = one ring of stages
    int gate_up_pair2; // bf16 gate/up on CTA pairs of two M tiles at every shape (else where `pair` holds)
};
// defaults for `rows` expert-major rows over E experts, overridable by
// MOK_GEMM_GROUP / MOK_GEMM_PAIR / MOK_GEMM_CTA_PAIR / MOK_MX_RINGS
GemmTuning gemm_tuning(int rows, int E);
cudaError_t gemm_configure(int dev);
// Token-side (B operand) tensor maps of one buffer with box heights 16, 32,
// ..., 256 rows (map i has 16 * (i + 1) rows): a chunk of r rows is loaded
// as ONE box of r rounded up to 16.
constexpr int B_MAPS = 16;
constexpr int B_MAX_BOX = 256;
struct BMaps {
    CUtensorMap m[B_MAPS];
};
// box heights step, 2 step, ..., 16 step rows (step 16: a whole chunk's token
// tile; step 8: one CTA's half of it in a CTA pair)
bool encode_bmaps(BMaps* maps, const void* base, uint64_t inner, uint64_t rows, const char** err, int step = 16);

// Every tensor map the GEMM core reads.
struct GemmMaps {
    CUtensorMap wg, wu, wd;  // 64x64 boxes of Wg, Wu and Wd (bf16)
    CUtensorMap wd3;         // Wd as {64, E*I, H/64}: one op loads both 64-column halves of a down tile
    BMaps rows;              // token rows (bf16) of the row buffer
    BMaps h;                 // h rows (bf16) of the h buffer
    BMaps rows2, h2;         // the same with heights 8 .. 128 (half a token tile, CTA pairs)
    int has_wd3;             // wd3 could be encoded (else two 2D ops per down stage)
};
bool encode_gemm_maps(GemmMaps* m, const void* wg, const void* wu, const void* wd, const void* rows, const void* h,
                      int H, int I, int E, int buf_rows, const char** err);

// Extra maps of the MXFP8 GEMM: E4M3 weight bytes and E8M0 scale bytes.
struct MxMaps {
    CUtensorMap gq, uq;  // {64 columns, 128 K rows} boxes of Wg/Wu [E*H, I], 64-byte swizzle
    CUtensorMap dq;      // {128, 128} boxes of Wd [E*I, H], 128-byte swizzle
    CUtensorMap gs, us;  // scales: {64, 4} boxes of [E*H/32, I]
    CUtensorMap ds;      // scales: {128, 4} boxes of [E*I/32, H]
};
bool encode_mx_maps(MxMaps* m, const mok_mxfp8_weights& w, int H, int I, int E, const char** err);
// Token-side maps of the MXFP8 GEMM: E4M3 rows [rows, inner] in boxes of
// {128 bytes, 16 (i + 1) rows}, 128-byte swizzle.
bool encode_bmaps_u8(BMaps* maps, const void* base, uint64_t inner, uint64_t rows, const char** err);
// Token-side scale planes of the MXFP8 path: [ceil(K / 128)][sc_rows][4]
// bytes; sc_rows = rows rounded up to 4, plus 4 (a stage's copy may start up
// to 3 rows early and is rounded up to 16 bytes).
inline int mx_sc_rows(int rows) { return ((rows + 3) & ~3) + 4; }
inline size_t mx_sc_bytes(int rows, int K) { return (size_t)((K + 127) / 128) * mx_sc_rows(rows) * 4; }
struct MxTokenScales {
    const uint8_t* xsc;  // x rows, K = H (written by the gather)
    uint8_t* hsc;        // h rows, K = I (written by the gate/up epilogue)
    int sc_rows;
};

// Staged grouped GEMM over every chunk: phase 0 = gate/up + SwiGLU -> h,
// phase 1 = down -> out[row_slot] (fp16 slot rows with exponents; bf16 on
// the MXFP8 path), or, with `push` (a device array), to the slot's rank:
// push->out[d] / push->exp[d] at slot - d * push_slots, d = slot / push_slots.
struct MxMaps;
// mx: MXFP8 weight maps (MXFP8 path: rows and h are E4M3 with the scale
// planes of mxs), or nullptr (bf16 path).
// Buffers of the bf16 path kept for / used by the backward: a, b [rows, I]
// bf16 (phase 0 writes them when not null; phase 2 reads them) and
// dab = [da | db] rows [rows, 2I] bf16 (phase 2 writes, phase 3 reads).
struct BwdBuffers {
    uint16_t *save_a, *save_b, *dab;
};
// phase 2 (dh + SwiGLU backward -> dab) and 3 (dx rows -> out[row_slot])
// read maps.wd / maps.wg, maps.wu as K-major maps ({64 K, 128 rows} boxes
// of [E*I, H] / [E*H, I]) and B from maps.rows (do rows) / maps.h (dab).
cudaError_t launch_gemm_phase(int phase, const GemmMaps& maps, const MxMaps* mx, const MxTokenScales* mxs,
                              const GemmShape& sh, const Chunk* chunks, const int* counts2, void* h_out, void* out,
                              const int32_t* row_slot, void* status, uint64_t timeout_ns, int grid,
                              const GemmTuning& tune, cudaStream_t stream, const BwdBuffers* bwd = nullptr,
                              int8_t* out_exp = nullptr, const PushDest* push = nullptr, int push_slots = 0);

// ---- expert parallelism (ep.cu)
// offsets_loc[i] = offsets[e0 + i] - offsets[e0] (i <= e_loc); *push_dev = push
cudaError_t launch_ep_setup(const PushDest& push, PushDest* push_dev, const int32_t* offsets, int e0, int e_loc,
                            int32_t* offsets_loc, cudaStream_t stream);
// rows[i] = x[src_rank[row]][src_index[row]], row_slot_loc[i] = row_slot[row]
// for row = offsets[e0] + i < offsets[e0 + e_loc]; max_rows bounds the count
cudaError_t launch_ep_pull(const ShardsIn& xs, int H, const int32_t* offsets, int e0, int e_loc,
                           const int32_t* src_rank, const int32_t* src_index, const int32_t* row_slot, void* rows,
                           int32_t* row_slot_loc, int max_rows, int num_sms, cudaStream_t stream);
// the same pull quantised to MXFP8: rows_q [*, H] E4M3, scale planes
// [H/128][sc_rows][4] indexed by local row
cudaError_t launch_ep_pull_mx(const ShardsIn& xs, int H, const int32_t* offsets, int e0, int e_loc,
                              const int32_t* src_rank, const int32_t* src_index, const int32_t* row_slot,
                              void* rows_q, void* xsc, int sc_rows, int32_t* row_slot_loc, int max_rows, int num_sms,
                              cudaStream_t stream);
// one arrival on every rank's counter, then a bounded wait for this rank's
// counter (counters.p[g]) to reach target
cudaError_t launch_ep_barrier(const ShardsOut& counters, int G, int g, uint32_t target, void* status,
                              uint64_t timeout_ns, cudaStream_t stream);

// ---- the persistent SM-partitioned forward (persistent.cu)
struct PersistLaunch {
    int grid, dispatch_ctas, cap;  // CTAs, of which the first dispatch_ctas gather; ring half rows
    int dispatch_warps;            // > 0: no dispatch CTAs, this many dispatch warps in every CTA
    bool pair;                     // bf16 GEMM units of two M tiles (the work list counted units this way)
    int H, I, E, T, k, S_r;
    const void *wg, *wu, *wd;      // bf16 weights; unused on the MXFP8 path
    const mok_mxfp8_weights* mxw;  // MXFP8 weights, or nullptr (bf16 path)
    void* ring;                    // [2*cap, H] bf16, or E4M3 (MXFP8)
    void* h;                       // [2*cap, I] bf16, or E4M3 (MXFP8)
    uint8_t *ring_sc, *h_sc;       // MXFP8: scale planes of ring and h rows (sc_rows = mx_sc_rows(2*cap))
    int sc_rows;
    void* out;                     // [T*k, H] slot rows: MOK_SLOTS_F16S (bf16 path) or bf16 (MXFP8)
    const Chunk* chunks;
    const Minibatch* mbs;
    const int* counts2;
    // zeroed counters: chunk_ready, g_done, d_chunk [max_chunks]; d_done
    // [max_mb]; tok_cnt, ready_q [T]; q_tail, q_claim, d_claim [1]
    int *chunk_ready, *g_done, *d_chunk, *d_done, *tok_cnt, *ready_q, *q_tail, *q_claim, *d_claim;
    ShardsIn xs;
    ShardsOut ys;
    const int32_t *src_rank, *src_index, *row_slot;
    const float* gates;
    void* status;
    uint64_t timeout_ns;
};
cudaError_t launch_forward_persistent(const PersistLaunch& L, const char** err, cudaStream_t stream);

// ---- tensor maps (driver entry point fetched at run time)
// 2D tiled map of a row-major [outer, inner] array of bf16 elements,
// 128-byte swizzle, zero fill out of bounds.
bool encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                         uint32_t box_outer, const char** err);
// {64, rows, cols / 64} view of a row-major [rows, cols] bf16 array, boxes of
// box_blocks 64-column blocks x box_rows rows (128-byte swizzle)
bool encode_cols3d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
                        uint32_t box_blocks, const char** err);

// ---- the backward (bwd.cu)
// do rows (bf16, expert-major) = g dy_t; dlogits [T, E] by the softmax backward
cudaError_t launch_reverse_combine(const ShardsIn& dys, int S_r, int H, int T, int k, int E, const int32_t* pos,
                                   const float* gates, const int32_t* topk_idx, const uint16_t* o_slots,
                                   const int8_t* o_exps, void* do_rows, float* dlogits, int num_sms,
                                   cudaStream_t stream);
// dWd = h^T do, dWg = x^T da, dWu = x^T db per expert (bf16 outputs)
cudaError_t launch_wgrad(const void* x_rows, const void* h_rows, const void* do_rows, const void* dab, int n_rows,
                         const int32_t* offsets, int H, int I, int E, void* dwg, void* dwu, void* dwd, void* status,
                         uint64_t timeout_ns, int num_sms, const char** err, cudaStream_t stream);

// ---- the router projection fused with the top-k (router.cu)
// Experts rounded up to the 128-row tiles of the router weights.
int router_e_pad(int E);
// w [H, E] fp32 -> hi, lo [E_pad, H] bf16 (hi + lo = w to about 16 bits)
cudaError_t launch_router_split(const float* w, int H, int E, void* hi, void* lo, int num_sms, cudaStream_t stream);
// logits = x W_r (+ prior), then top-k and gates per token; logits may be nullptr
cudaError_t launch_router(const ShardsIn& xs, int S_r, int T, int H, int E, int k, const void* w_hi,
                          const void* w_lo, const float* prior, float* logits, int32_t* topk_idx, float* gates,
                          void* status, uint64_t timeout_ns, const char** err, cudaStream_t stream);

// ---- MXFP8 quantisers (mxfp8.cu)
cudaError_t launch_mx_quant_rows(const void* src, bool f32, int rows, int K, void* q, void* scales, int num_sms,
                                 cudaStream_t stream);
cudaError_t launch_mx_quant_cols(const void* src, int nblocks, int N, void* q, void* scales, int num_sms,
                                 cudaStream_t stream);

}  // namespace mok

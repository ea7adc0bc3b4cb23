// gemm_core.cuh -- the warp-specialised tcgen05 grouped-GEMM core shared by
// the staged kernels (gemm_sm100.cu) and the persistent SM-partitioned
// kernel (persistent.cu).  Step 4 of the forward MoE layer.
//
// MoK article (tahou.com): routing paragraph (tokens of one expert laid out
// contiguously so the grouped GEMM runs efficiently), MXFP8 paragraph
// (quantisation inside the GEMM / SwiGLU data path), push-combine paragraph
// (each result goes back to its token's slot).
//
// Orientation.  Expert segments are short (about 171 rows per expert at 384
// experts, top-8, 8192 tokens), so the weights take the M = 128 side of every
// MMA and the tokens the N side (16..256 in steps of 16): an expert with 171
// rows pads to N = 176 instead of two 128-row tiles, and each weight tile is
// streamed from HBM once per chunk of <= 256 rows.
//   gate/up unit (phase 0): A = 64 columns of Wg stacked on the same 64
//     columns of Wu (M = 128, K = H, read MN-major straight from the
//     [E, H, I] layout), B = the chunk's token rows (K-major).  Accumulator
//     lanes 0-63 hold gate, 64-127 up; the epilogue forms
//     h = silu(gate) * up and stores h rows.
//   down unit (phase 1): A = 128 columns of Wd (MN-major from [E, I, H]),
//     B = the chunk's h rows.  The epilogue pushes each row's 128 outputs
//     to out[row_slot[row]] (the push combine): fp16 with one power-of-two
//     exponent per 128 features on the bf16 path, bf16 on the MXFP8 path.
//     Under expert parallelism the slot's source rank owns the row: the
//     store goes to that rank's slot buffer (a peer pointer) at the slot's
//     index there.
// Precision: the bf16 path runs both GEMMs as bf16 x bf16 with fp32
// accumulation on the caller's bf16 weights; h = silu(gate) * up is rounded
// once to bf16 (the range of fp32, no saturation) and the slot outputs keep
// 11 significant bits with fp32's exponent range, so the roundings before
// y's own are h's and the slot rows'.  The MXFP8 path runs
// the block-scaled tensor-core MMA (kind::mxf8f6f4): E4M3 weights and E4M3
// token rows / h rows, each with one E8M0 scale per 32 K values, which the
// MMA reads from TMEM; the products are exact and accumulate in fp32.  The
// gather quantises x, the gate/up epilogue quantises h, and the slot
// outputs are bf16.
//
// Roles in a CTA: warp 0 issues TMA loads into a ring of stages, warp 1
// allocates 512 TMEM columns and one thread of it issues tcgen05.mma into
// one of two 256-column accumulators, warps 2-9 (two groups of four) drain
// the other accumulator (tcgen05.ld) through shared memory to global
// memory, and (MXFP8 only) warp 10 lays each stage's scales out for the
// copy into TMEM.  The token tile of a stage is ONE TMA box of exactly the
// 16-rounded row count, and a down unit's two 64-column weight halves come
// from one 3D map: measured on B200, the number of TMA ops per SM and then
// the bytes each SM takes in from L2 limited earlier versions.  With a unit
// of two M tiles (bf16 gate/up at <= 192 rows per expert) the tiles share
// every token tile.  Every wait is bounded.
//
// A schedule policy (template parameter) tells each role which units this
// CTA runs, what a unit's inputs wait for, and what its completion signals.
#pragma once

#include "mok_device.cuh"
#include "mok_internal.h"
#include "mxfp8.cuh"

namespace mok {

constexpr int BK = 64;                            // K per stage: one 128-byte swizzle atom
constexpr int A_BYTES = 128 * BK * 2;             // 16 KB: two {64 MN x 64 K} bf16 halves
constexpr int B_ROW_BYTES = BK * 2;               // 128 bytes of one token row per stage
constexpr int B_BYTES = CHUNK_MAX_ROWS * B_ROW_BYTES;  // 32 KB
constexpr int EPI_TLD = 132;                      // fp32 staging pitch: 32 tokens x 128 features (+4)
constexpr int EPI_BYTES = 32 * EPI_TLD * 4;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COLS = 256;
// Bound of the waits that drain this CTA's own TMA loads and MMAs before it
// leaves: those complete by themselves, so the bound is generous and does
// not follow the caller's (possibly tiny) timeout.
constexpr uint64_t DRAIN_TIMEOUT_NS = 1000000000ull;
constexpr int MT_G_FEATURES = 64;                 // gate/up unit: 64 gate + 64 up columns
constexpr int MT_D_FEATURES = 128;                // down unit: 128 output columns

// Stage layouts.  bf16 path, one M tile per unit: [A 16 KB][B 32 KB] x 4.
// bf16 path, pairs of M tiles sharing the token tile: [A0 16 KB][A1 16 KB]
// [B 32 KB] x 3.  MXFP8 path: [A bf16, converted 16 KB][B 32 KB][A E4M3
// bytes 8 KB][scales 1 KB] x 3.
// EXT_: the instantiation that also runs the backward phases (2, 3) and
// keeps the forward's gate/up pre-activations; the plain forward
// instantiations compile none of that code (measured: folding it into
// the forward kernels cost 12 % of the page-shape GEMM, in the
// single-thread TMA and MMA issue loops).
template <int SUB_, int NST_, bool EXT_ = false>
struct Bf16CfgT {
    static constexpr bool SPLIT = false;  // one ring of [weights | tokens] stages
    static constexpr bool MX = false;
    static constexpr bool EXT = EXT_;
    static constexpr bool CG2 = false;
    static constexpr int SUB = SUB_;  // M tiles per unit
    static constexpr int THREADS = 320;  // warps: 0 TMA, 1 MMA, 2-9 two epilogue groups
    static constexpr int NST = NST_;
    static constexpr int BKX = BK;  // K per stage
    static constexpr int STAGE = SUB * A_BYTES + B_BYTES;
    static constexpr int A_OFF = 0, B_OFF = SUB * A_BYTES;
    static constexpr int EPI_OFF = NST * STAGE;           // one staging tile per epilogue group
    static constexpr int BAR_OFF = EPI_OFF + 2 * EPI_BYTES;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM = BAR_OFF + BAR_BYTES + 1024;  // + slack for 1024-byte alignment
};
using Bf16Cfg = Bf16CfgT<1, 4>;
using Bf16PairCfg = Bf16CfgT<2, 3>;
using Bf16ExtCfg = Bf16CfgT<1, 4, true>;
using Bf16ExtPairCfg = Bf16CfgT<2, 3, true>;
static_assert(Bf16Cfg::BAR_OFF == Bf16PairCfg::BAR_OFF, "both bf16 layouts share the barrier offset");
// bf16 forward on CTA pairs (tcgen05 cta_group::2): a cluster of two CTAs
// runs each unit as one M = 256 MMA, CTA r holding M tile 2 m + r and half
// of the token tile: [A 16 KB][B half <= 128 rows x 128 B] x 6.  Per SM a
// stage carries 32 KB for the work a single-tile stage does with 48 KB,
// like a pair of M tiles in one CTA, while each CTA keeps two 256-column
// accumulators, so the epilogue still overlaps the next unit's MMAs.
// SUB_ = 2: each CTA holds two M tiles (a cluster covers four), sharing its
// half of the token tile: [A0 16 KB][A1 16 KB][B half] x 4.
template <int NST_, bool EXT_ = false, int SUB_ = 1>
struct Bf16Cta2CfgT {
    static constexpr bool SPLIT = false;  // one ring of [weights | tokens] stages
    static constexpr bool MX = false;
    static constexpr bool EXT = EXT_;  // also the backward's dh and dx phases (2, 3)
    static constexpr bool CG2 = true;
    static constexpr int SUB = SUB_;  // M tiles per CTA and unit
    static constexpr int THREADS = 320;  // warps: 0 TMA, 1 MMA (first CTA of the pair), 2-9 epilogue
    static constexpr int NST = NST_;
    static constexpr int BKX = BK;
    static constexpr int STAGE = SUB * A_BYTES + B_BYTES / 2;
    static constexpr int A_OFF = 0, B_OFF = SUB * A_BYTES;
    static constexpr int EPI_OFF = NST * STAGE;
    static constexpr int BAR_OFF = EPI_OFF + 2 * EPI_BYTES;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM = BAR_OFF + BAR_BYTES + 1024;
    static_assert(SMEM <= 232448, "CTA-pair layout exceeds shared memory");
};
using Bf16Cta2Cfg = Bf16Cta2CfgT<6>;
using Bf16Cta2ExtCfg = Bf16Cta2CfgT<6, true>;
using Bf16Cta2PairCfg = Bf16Cta2CfgT<4, false, 2>;
// MXFP8 path (block-scaled tcgen05 MMA, K = 128 per stage), SUB weight
// tiles per unit: [A E4M3 SUB x 16 KB][B E4M3 <= 224 rows x 128 B][A scales
// as loaded SUB x 512 B][B scales as loaded <= 1 KB][A scales, MMA layout
// SUB x 512 B][B scales, MMA layout 1 KB] x NST.
template <int SUB_, int NST_>
struct MxCfgT {
    static constexpr bool SPLIT = false;  // one ring of [weights | tokens] stages
    static constexpr bool MX = true;
    static constexpr bool EXT = false;
    static constexpr bool CG2 = false;
    static constexpr int SUB = SUB_;
    static constexpr int THREADS = 352;  // warps: 0 TMA, 1 MMA, 2-9 epilogue, 10 scale-factor layout
    static constexpr int NST = NST_;
    static constexpr int BKX = 128;      // K per stage
    static constexpr int A_OFF = 0, B_OFF = SUB * 16384;
    static constexpr int SFA_RAW_OFF = B_OFF + CHUNK_MAX_ROWS_MX * 128;  // per tile [4 K blocks][128 rows]
    static constexpr int SFB_RAW_OFF = SFA_RAW_OFF + SUB * 512;          // [rows][4 K blocks], 16-byte aligned copy
    static constexpr int SFA_OFF = SFB_RAW_OFF + 1024;                   // one 512-byte scale atom per tile
    static constexpr int SFB_OFF = SFA_OFF + SUB * 512;                  // two atoms (rows 0-127, 128-255)
    static constexpr int STAGE = SFB_OFF + 1024;
    static constexpr int EPI_OFF = NST * STAGE;           // one staging tile per epilogue group
    static constexpr int BAR_OFF = EPI_OFF + 2 * EPI_BYTES;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM = BAR_OFF + BAR_BYTES + 1024;
    // TMEM: accumulators in columns [0, 480) (N <= 224), then the scale
    // factors of the SUB weight tiles (4 columns each) and of the tokens (8)
    static constexpr uint32_t TM_SFA = 480, TM_SFB = 480 + 4 * SUB;
    static_assert(STAGE % 1024 == 0, "MXFP8 stages must keep 1024-byte alignment");
    static_assert(SMEM <= 232448, "MXFP8 layout exceeds shared memory");
    static_assert(TM_SFB + 8 <= 512, "scale factors must fit in TMEM");
};
using MxOneRingCfg = MxCfgT<1, 4>;
// MXFP8 path with two stage rings: a deep ring of weight tiles (E4M3 16 KB
// and their scales) streamed from HBM and a shallower ring of token tiles
// (<= 224 rows and their scales) mostly served by L2.  One ring of [weights
// | tokens] stages holds 4 stages, i.e. 64 KB of weights in flight per SM,
// which at HBM latency under load keeps the stream well below the HBM
// rate; NW = 6 weight slots keep 96 KB in flight with NT = 3 token slots.
// K step i of the CTA's unit sequence uses weight slot i % NW and token slot
// i % NT.  Warps: 0 loads the weight tiles, 11 the token tiles, 10 lays both
// scale sets out for the TMEM copy, 1 issues the MMAs, 2-9 drain.
template <int NW_, int NT_>
struct MxSplitCfgT {
    static constexpr bool SPLIT = true;
    static constexpr bool MX = true;
    static constexpr bool EXT = false;
    static constexpr bool CG2 = false;
    static constexpr int SUB = 1;
    static constexpr int THREADS = 384;  // warps: 0 weight TMA, 1 MMA, 2-9 epilogue, 10 scale layout, 11 token TMA
    static constexpr int NW = NW_, NT = NT_;
    static constexpr int NST = NT_;
    static constexpr int BKX = 128;  // K per stage
    // weight slot: [A E4M3 16 KB][A scales as loaded 512 B][A scales, MMA layout 512 B]
    static constexpr int A_OFF = 0, SFA_RAW_OFF = 16384, SFA_OFF = 16384 + 512, WSTAGE = 17408;
    // token slot: [B E4M3 <= 224 rows x 128 B][B scales as loaded 1 KB][B scales, MMA layout 1 KB]
    static constexpr int B_OFF = 0, SFB_RAW_OFF = CHUNK_MAX_ROWS_MX * 128, SFB_OFF = SFB_RAW_OFF + 1024;
    static constexpr int TSTAGE = SFB_OFF + 1024;
    static constexpr int T_BASE = NW * WSTAGE;
    static constexpr int EPI_OFF = T_BASE + NT * TSTAGE;  // one staging tile per epilogue group
    static constexpr int BAR_OFF = EPI_OFF + 2 * EPI_BYTES;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM = BAR_OFF + BAR_BYTES + 1024;
    // TMEM: accumulators in columns [0, 480) (N <= 224); two sets of scale
    // factors (the weight tile's 4 columns, the tokens' 8), used by
    // alternate K steps, so that the copy of step i + 1's scales does not
    // overwrite columns step i's MMAs still read
    static constexpr uint32_t TM_SFA = 480, TM_SFB = 484, TM_SF_SET = 12;
    static_assert(TM_SFB + TM_SF_SET + 8 <= 512, "scale factors must fit in TMEM");
    static_assert(WSTAGE % 1024 == 0 && TSTAGE % 1024 == 0, "MXFP8 slots must keep 1024-byte alignment");
    static_assert(SMEM <= 232448, "MXFP8 two-ring layout exceeds shared memory");
};
using MxSplitCfg = MxSplitCfgT<6, 3>;
using MxCfg = MxSplitCfg;

// One unit of work: C::SUB consecutive M tiles (fewer at the end of the M
// range) of one phase over one chunk; the tiles share every token tile.
struct Unit {
    int phase;   // 0 = gate/up, 1 = down
    int expert;
    int brow0;   // buffer row of the chunk's first row (token rows and h rows)
    int rows;    // valid rows, 1..256
    int m;       // unit index along M: first M tile = m * C::SUB
    int grow0;   // global expert-major row of the chunk's first row (row_slot index)
    int chunk;
    int mb;
};

struct CoreArgs {
    int H, I;
    void* h;                  // [buffer rows, I]: bf16 (bf16 path) or E4M3 (MXFP8 path)
    void* out;                // [N_s, H] slot-indexed: fp16 + block exponents (bf16 path and the
                              // backward's dx rows), bf16 (MXFP8 path)
    int8_t* out_exp;          // bf16 path: [N_s, H/128] exponents of the fp16 slot rows
    const int32_t* row_slot;  // [N_s]
    // Expert parallelism (nullptr: every slot goes to out / out_exp): slot s
    // belongs to rank d = s / push_slots and is stored at s - d * push_slots
    // of push->out[d] (fp16 rows) and push->exp[d] (their exponents).
    const PushDest* push;
    int push_slots;
    DevStatus* st;
    uint64_t timeout_ns;
    // MXFP8 path: E8M0 scales of the token side as planes [K/128][sc_rows][4]
    // (plane g, row r, byte b: the scale of K block 4g + b of row r)
    const uint8_t* xsc;       // token rows (gate/up B operand), K = H
    uint8_t* hsc;             // h rows (written by gate/up, read by down), K = I
    int sc_rows;              // rows per plane, a multiple of 4
    // bf16 path, kept for the backward: gate and up pre-activations a, b
    // [buffer rows, I] bf16 (written by gate/up when not null; read by the
    // dh phase), and the dh phase's output [da | db] rows [buffer rows, 2I]
    uint16_t* save_a;
    uint16_t* save_b;
    uint16_t* dab;
};

// Unit u -> (chunk c, M tile m) in raster groups of GC chunks: inside a group
// the chunk index runs fastest, so the CTAs running at one time share a few
// chunks' token tiles (L2) while streaming distinct weight tiles.
__device__ __forceinline__ void unit_map(int u, int nch, int MT, int GC, int& c, int& m) {
    const int grp = u / (GC * MT);
    const int rem = u - grp * GC * MT;
    const int c0 = grp * GC;
    const int gsz = min(GC, nch - c0);
    m = rem / gsz;
    c = c0 + (rem - m * gsz);
}

// Staged schedule: one phase over every chunk, units dealt round-robin to
// the CTAs of the grid; no waits, no signals (kernel boundaries order the
// phases).
struct StagedSched {
    static constexpr bool kSignals = false;
    int phase, nch, MT, GC;
    const Chunk* chunks;

    __device__ bool get(int i, Unit& u) const {
        const int idx = blockIdx.x + i * gridDim.x;
        if (idx >= nch * MT) return false;
        int c, m;
        unit_map(idx, nch, MT, GC, c, m);
        const Chunk ck = chunks[c];
        u.phase = phase;
        u.expert = ck.expert;
        u.brow0 = ck.row0;
        u.rows = ck.rows;
        u.m = m;
        u.grow0 = ck.row0;
        u.chunk = c;
        u.mb = ck.mb;
        return true;
    }
    __device__ bool wait_inputs(const Unit&, DevStatus*, uint64_t) const { return true; }
    __device__ bool unit_done(const Unit&) const { return false; }
    __device__ void chunk_done(const Unit&, int, int) const {}
};

// CTA-pair schedule: units are (chunk, 2 C::SUB M tiles), dealt round-robin
// to the clusters; both CTAs of a cluster walk the same units, CTA r taking
// M tiles (2 m + r) C::SUB + s (u.m = 2 m + r, in units of C::SUB tiles).
// MT counts cluster units.
struct StagedSched2 {
    static constexpr bool kSignals = false;
    int phase, nch, MT, GC;
    uint32_t rank;
    const Chunk* chunks;

    __device__ bool get(int i, Unit& u) const {
        const int idx = (int)(blockIdx.x >> 1) + i * (int)(gridDim.x >> 1);
        if (idx >= nch * MT) return false;
        int c, m;
        unit_map(idx, nch, MT, GC, c, m);
        const Chunk ck = chunks[c];
        u.phase = phase;
        u.expert = ck.expert;
        u.brow0 = ck.row0;
        u.rows = ck.rows;
        u.m = 2 * m + (int)rank;
        u.grow0 = ck.row0;
        u.chunk = c;
        u.mb = ck.mb;
        return true;
    }
    __device__ bool wait_inputs(const Unit&, DevStatus*, uint64_t) const { return true; }
    __device__ bool unit_done(const Unit&) const { return false; }
    __device__ void chunk_done(const Unit&, int, int) const {}
};

// M tiles of a phase (64 gate + 64 up features, or 128 down features, each),
// and how many of them unit u covers.
// Backward phases (bf16 path): 2 = dh = do Wd^T with the SwiGLU backward
// in the epilogue (M = I features), 3 = dx rows = da Wg^T + db Wu^T pushed
// to the token slots (M = H features); both read A K-major.
template <class C>
__device__ __forceinline__ int phase_tiles(const CoreArgs& a, int phase) {
    if constexpr (C::EXT)
        return phase == 0 ? a.I / MT_G_FEATURES : phase == 2 ? a.I / MT_D_FEATURES : a.H / MT_D_FEATURES;
    else
        return phase == 0 ? a.I / MT_G_FEATURES : a.H / MT_D_FEATURES;
}
// Contraction length of a phase.
template <class C>
__device__ __forceinline__ int phase_k(const CoreArgs& a, int phase) {
    if constexpr (C::EXT)
        return phase == 0 || phase == 2 ? a.H : phase == 1 ? a.I : 2 * a.I;
    else
        return phase == 0 ? a.H : a.I;
}
template <class C>
__device__ __forceinline__ int unit_subs(const CoreArgs& a, const Unit& u) {
    return min(C::SUB, phase_tiles<C>(a, u.phase) - u.m * C::SUB);
}

// Token tile of a unit: one box of the 16-rounded row count.  Returns the
// map index (box rows = 16 * (index + 1)); rows is 1..256.
__device__ __forceinline__ int token_box(int rows) { return ((rows + 15) >> 4) - 1; }

// ------------------------------------------------------------------ producer
// Loads the weight tile (bf16 halves, or MXFP8 bytes + scales) and the
// token tile of every k-step of every unit into the stage ring.
template <class S, class C>
__device__ __forceinline__ void gemm_producer(const GemmMaps& maps, const MxMaps* mx, const CoreArgs& a, const S& s,
                                              unsigned char* smem, uint64_t* full, uint64_t* empty) {
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, issued_phase = 0;  // bit s: stage s holds a load of phase bit s
    const uint64_t evict_first = l2_policy_evict_first();
    Unit u;
    for (int i = 0; s.get(i, u); ++i) {
        if (!s.wait_inputs(u, a.st, a.timeout_ns)) break;
        const int K = phase_k<C>(a, u.phase);
        const int KB = (K + C::BKX - 1) / C::BKX;
        const BMaps& bm = (u.phase == 0 || (C::EXT && u.phase == 2)) ? maps.rows : maps.h;
        const int bx = token_box(u.rows);
        const int nsub = unit_subs<C>(a, u);
        uint32_t bytes = (uint32_t)(16 * (bx + 1)) * B_ROW_BYTES;
        // MXFP8: the token side's scales for this stage are one 16-byte
        // aligned run of the plane, starting up to 3 rows before the chunk
        const int sc_lead = u.brow0 & 3;
        const uint32_t sc_bytes = (uint32_t)(4 * (sc_lead + u.rows) + 15) & ~15u;
        if (C::MX)
            bytes += (uint32_t)nsub * (16384 + 512) + sc_bytes;  // E4M3 weight tiles + their scales + token scales
        else
            bytes += (uint32_t)nsub * A_BYTES;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, a.st, a.timeout_ns, 10)) {
                ok = false;
                break;
            }
            unsigned char* st = smem + stage * C::STAGE;
            mbar_arrive_expect_tx(&full[stage], bytes);
            const int ky = u.expert * K + kb * C::BKX;
            if constexpr (C::MX) {
                const int kys = ky / 32;  // scale row of the stage's first K block
                for (int sub = 0; sub < nsub; ++sub) {
                    unsigned char* sa = st + C::A_OFF + sub * 16384;
                    unsigned char* sfa = st + C::SFA_RAW_OFF + sub * 512;
                    const int mt = u.m * C::SUB + sub;
                    if (u.phase == 0) {
                        // gate and up columns of the M tile: two 64-byte-swizzled 64-column boxes
                        tma_load_2d_hint(sa, &mx->gq, &full[stage], mt * MT_G_FEATURES, ky, evict_first);
                        tma_load_2d_hint(sa + 8192, &mx->uq, &full[stage], mt * MT_G_FEATURES, ky, evict_first);
                        tma_load_2d(sfa, &mx->gs, &full[stage], mt * MT_G_FEATURES, kys);
                        tma_load_2d(sfa + 256, &mx->us, &full[stage], mt * MT_G_FEATURES, kys);
                    } else {
                        tma_load_2d_hint(sa, &mx->dq, &full[stage], mt * MT_D_FEATURES, ky, evict_first);
                        tma_load_2d(sfa, &mx->ds, &full[stage], mt * MT_D_FEATURES, kys);
                    }
                }
                const uint8_t* plane = (u.phase == 0 ? a.xsc : a.hsc) + (size_t)kb * a.sc_rows * 4;
                bulk_load(st + C::SFB_RAW_OFF, plane + (size_t)(u.brow0 - sc_lead) * 4, sc_bytes, &full[stage]);
            } else {
                for (int sub = 0; sub < nsub; ++sub) {
                    unsigned char* sa = st + C::A_OFF + sub * A_BYTES;
                    const int mt = u.m * C::SUB + sub;
                    if (u.phase == 0) {
                        tma_load_2d_hint(sa, &maps.wg, &full[stage], mt * MT_G_FEATURES, ky, evict_first);
                        tma_load_2d_hint(sa + A_BYTES / 2, &maps.wu, &full[stage], mt * MT_G_FEATURES, ky,
                                         evict_first);
                    } else if (C::EXT && u.phase == 2) {
                        // Wd [E*I, H] K-major: 128 feature rows x 64 K in one box
                        tma_load_2d_hint(sa, &maps.wd, &full[stage], kb * BK, u.expert * a.I + mt * MT_D_FEATURES,
                                         evict_first);
                    } else if (C::EXT && u.phase == 3) {
                        // Wg then Wu [E*H, I] K-major: K runs over I twice
                        const int KI = a.I / BK;
                        const bool up = kb >= KI;
                        tma_load_2d_hint(sa, up ? &maps.wu : &maps.wg, &full[stage], (kb - (up ? KI : 0)) * BK,
                                         u.expert * a.H + mt * MT_D_FEATURES, evict_first);
                    } else if (maps.has_wd3) {
                        // both 64-column halves of the 128-column down tile in one op
                        tma_load_3d_hint(sa, &maps.wd3, &full[stage], 0, ky, mt * 2, evict_first);
                    } else {
                        tma_load_2d_hint(sa, &maps.wd, &full[stage], mt * MT_D_FEATURES, ky, evict_first);
                        tma_load_2d_hint(sa + A_BYTES / 2, &maps.wd, &full[stage], mt * MT_D_FEATURES + 64, ky,
                                         evict_first);
                    }
                }
            }
            tma_load_2d(st + C::B_OFF, &bm.m[bx], &full[stage], kb * C::BKX, u.brow0);
            issued |= 1u << stage;
            issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
            if (++stage == C::NST) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!ok) break;
    }
    // never leave with a load in flight into this CTA's shared memory
    for (int st = 0; st < C::NST; ++st)
        if ((issued >> st) & 1u) mbar_wait(&full[st], (issued_phase >> st) & 1u, nullptr, DRAIN_TIMEOUT_NS, 11);
}

// ------------------------------------------------------------------ producer, CTA pairs
// Each CTA of the pair loads its own M tile of weights and its half of the
// token tile (rows [r N/2, (r + 1) N/2) of the chunk, N the 16-rounded row
// count) into its own stage; both loads count their bytes on the FIRST
// CTA's full[stage], whose producer expects the pair's total.  A stage is
// reused once the MMA's commit has arrived on this CTA's empty[stage].
template <class S, class C>
__device__ __forceinline__ void gemm_producer_pair(const GemmMaps& maps, const CoreArgs& a, const S& s,
                                                   unsigned char* smem, uint64_t* full, uint64_t* empty,
                                                   uint32_t rank) {
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, issued_phase = 0;
    const uint64_t evict_first = l2_policy_evict_first();
    const uint64_t evict_normal = l2_policy_evict_normal();
    Unit u;
    for (int i = 0; s.get(i, u); ++i) {
        const int K = phase_k<C>(a, u.phase);
        const int KB = (K + C::BKX - 1) / C::BKX;
        const BMaps& bm = (u.phase == 0 || (C::EXT && u.phase == 2)) ? maps.rows2 : maps.h2;
        const int hb = ((u.rows + 15) >> 4) - 1;  // half tile of 8 (hb + 1) rows: map hb of the 8-row set
        const int brow = u.brow0 + (int)rank * 8 * (hb + 1);
        const int nsub = unit_subs<C>(a, u);  // the same in both CTAs (whole cluster units)
        const uint32_t bytes = 2u * ((uint32_t)(nsub * A_BYTES) + (uint32_t)(8 * (hb + 1)) * B_ROW_BYTES);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, a.st, a.timeout_ns, 12)) {
                ok = false;
                break;
            }
            unsigned char* st = smem + stage * C::STAGE;
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], bytes);
            const uint32_t full0 = smem_in_rank(&full[stage], 0);  // the first CTA's full[stage]
            const int ky = u.expert * K + kb * C::BKX;
            for (int sub = 0; sub < nsub; ++sub) {
                unsigned char* sa = st + C::A_OFF + sub * A_BYTES;
                const int mt = u.m * C::SUB + sub;
                if (u.phase == 0) {
                    tma_load_2d_pair(sa, &maps.wg, full0, mt * MT_G_FEATURES, ky, evict_first);
                    tma_load_2d_pair(sa + A_BYTES / 2, &maps.wu, full0, mt * MT_G_FEATURES, ky, evict_first);
                } else if (C::EXT && u.phase == 2) {
                    // Wd [E*I, H] K-major: 128 feature rows x 64 K in one box
                    tma_load_2d_pair(sa, &maps.wd, full0, kb * BK, u.expert * a.I + mt * MT_D_FEATURES, evict_first);
                } else if (C::EXT && u.phase == 3) {
                    // Wg then Wu [E*H, I] K-major: K runs over I twice
                    const int KI = a.I / BK;
                    const bool up = kb >= KI;
                    tma_load_2d_pair(sa, up ? &maps.wu : &maps.wg, full0, (kb - (up ? KI : 0)) * BK,
                                     u.expert * a.H + mt * MT_D_FEATURES, evict_first);
                } else if (maps.has_wd3) {
                    tma_load_3d_pair(sa, &maps.wd3, full0, 0, ky, mt * 2, evict_first);
                } else {
                    tma_load_2d_pair(sa, &maps.wd, full0, mt * MT_D_FEATURES, ky, evict_first);
                    tma_load_2d_pair(sa + A_BYTES / 2, &maps.wd, full0, mt * MT_D_FEATURES + 64, ky, evict_first);
                }
            }
            tma_load_2d_pair(st + C::B_OFF, &bm.m[hb], full0, kb * C::BKX, brow, evict_normal);
            issued |= 1u << stage;
            issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
            if (++stage == C::NST) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!ok) break;
    }
    // never leave with a load in flight into this CTA's shared memory: the
    // MMA's commit on empty[stage] follows the stage's loads (both CTAs')
    for (int st = 0; st < C::NST; ++st)
        if ((issued >> st) & 1u) mbar_wait(&empty[st], (issued_phase >> st) & 1u, nullptr, DRAIN_TIMEOUT_NS, 13);
}

// ------------------------------------------------------------------ MXFP8 scale-factor layout (warp 10)
// The block-scaled MMA reads the scales of a 128-row operand tile from TMEM
// as 32 lanes x 4 columns of 32-bit words: row r = r0 + 32 r1 at lane r0,
// column r1, byte b = K block b of the stage (the copy to TMEM takes them
// from shared memory as 32 rows of 16 bytes: row r0 = the 4 words r1 =
// 0..3).  Per stage this warp rearranges the scales as loaded into that
// atom layout:
//   weights (A): loaded [4 K blocks][128 features] (gate/up: [4][64] gate
//     then [4][64] up, features 0-63 gate and 64-127 up of the M tile);
//   tokens (B): loaded [rows][4 K blocks] starting sc_lead rows early; rows
//     past the chunk get scale 0 (their MMA columns are never stored);
//     rows 128-255 form a second atom.
template <class S, class C>
__device__ __forceinline__ void gemm_sf_layout(const CoreArgs& a, const S& s, unsigned char* smem, uint64_t* full,
                                               uint64_t* sfready) {
    const int lane = threadIdx.x & 31;
    int stage = 0;
    uint32_t phase = 0;
    Unit u;
    for (int i = 0; s.get(i, u); ++i) {
        const int K = phase_k<C>(a, u.phase);
        const int KB = (K + C::BKX - 1) / C::BKX;
        const int nsub = unit_subs<C>(a, u);
        const int lead = u.brow0 & 3;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            // the warp leaves or goes on as one (it synchronises below)
            if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, a.st, a.timeout_ns, 80))) {
                ok = false;
                break;
            }
            unsigned char* st = smem + stage * C::STAGE;
            const uint32_t* rb = reinterpret_cast<const uint32_t*>(st + C::SFB_RAW_OFF) + lead;
            for (int sub = 0; sub < nsub; ++sub) {
                const uint8_t* ra = st + C::SFA_RAW_OFF + sub * 512;
                uint32_t wa[4];
#pragma unroll
                for (int r1 = 0; r1 < 4; ++r1) {
                    const int r = lane + 32 * r1;
                    // feature r of the tile: gate/up keeps 64 gate then 64 up rows of 64 bytes
                    const uint8_t* col = u.phase == 0 ? ra + (r >> 6) * 256 + (r & 63) : ra + r;
                    const int pitch = u.phase == 0 ? 64 : 128;
                    wa[r1] = (uint32_t)col[0] | ((uint32_t)col[pitch] << 8) | ((uint32_t)col[2 * pitch] << 16) |
                             ((uint32_t)col[3 * pitch] << 24);
                }
                *reinterpret_cast<uint4*>(st + C::SFA_OFF + sub * 512 + 16 * lane) =
                    make_uint4(wa[0], wa[1], wa[2], wa[3]);
            }
#pragma unroll
            for (int r2 = 0; r2 < 2; ++r2) {
                uint32_t wb[4];
#pragma unroll
                for (int r1 = 0; r1 < 4; ++r1) {
                    const int r = lane + 32 * r1 + 128 * r2;
                    wb[r1] = r < u.rows ? rb[r] : 0u;
                }
                *reinterpret_cast<uint4*>(st + C::SFB_OFF + 512 * r2 + 16 * lane) =
                    make_uint4(wb[0], wb[1], wb[2], wb[3]);
            }
            fence_proxy_async_shared();  // generic writes -> the TMEM copy (async proxy) reads
            __syncwarp();                // every lane's writes and fence precede the one arrival
            if (lane == 0) mbar_arrive(&sfready[stage]);
            if (++stage == C::NST) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!ok) break;
    }
}

// ------------------------------------------------------------------ MXFP8, two rings
// Weight tiles of every K step of every unit into the weight ring (warp 0).
// Weights are read-only, so this producer does not wait for a unit's inputs
// (in the persistent kernel it runs ahead of the dispatch, bounded by the
// ring).
template <class S, class C>
__device__ __forceinline__ void mx_producer_w(const MxMaps* mx, const CoreArgs& a, const S& s, unsigned char* smem,
                                              uint64_t* wfull, uint64_t* wempty) {
    int slot = 0;
    uint32_t ph = 0;
    uint32_t issued = 0, issued_ph = 0;
    const uint64_t evict_first = l2_policy_evict_first();
    Unit u;
    for (int i = 0; s.get(i, u); ++i) {
        if (failed(a.st)) break;
        const int K = phase_k<C>(a, u.phase);
        const int KB = (K + C::BKX - 1) / C::BKX;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&wempty[slot], ph ^ 1u, a.st, a.timeout_ns, 14)) {
                ok = false;
                break;
            }
            unsigned char* w = smem + slot * C::WSTAGE;
            mbar_arrive_expect_tx(&wfull[slot], 16384u + 512u);
            const int ky = u.expert * K + kb * C::BKX;
            const int kys = ky / 32;  // scale row of the stage's first K block
            if (u.phase == 0) {
                // gate and up columns of the M tile: two 64-byte-swizzled 64-column boxes
                tma_load_2d_hint(w + C::A_OFF, &mx->gq, &wfull[slot], u.m * MT_G_FEATURES, ky, evict_first);
                tma_load_2d_hint(w + C::A_OFF + 8192, &mx->uq, &wfull[slot], u.m * MT_G_FEATURES, ky, evict_first);
                tma_load_2d(w + C::SFA_RAW_OFF, &mx->gs, &wfull[slot], u.m * MT_G_FEATURES, kys);
                tma_load_2d(w + C::SFA_RAW_OFF + 256, &mx->us, &wfull[slot], u.m * MT_G_FEATURES, kys);
            } else {
                tma_load_2d_hint(w + C::A_OFF, &mx->dq, &wfull[slot], u.m * MT_D_FEATURES, ky, evict_first);
                tma_load_2d(w + C::SFA_RAW_OFF, &mx->ds, &wfull[slot], u.m * MT_D_FEATURES, kys);
            }
            issued |= 1u << slot;
            issued_ph = (issued_ph & ~(1u << slot)) | (ph << slot);
            if (++slot == C::NW) {
                slot = 0;
                ph ^= 1u;
            }
        }
        if (!ok) break;
    }
    // never leave with a load in flight into this CTA's shared memory
    for (int st = 0; st < C::NW; ++st)
        if ((issued >> st) & 1u) mbar_wait(&wfull[st], (issued_ph >> st) & 1u, nullptr, DRAIN_TIMEOUT_NS, 15);
}

// Token tiles (E4M3 rows, one box of the 16-rounded row count) and their
// scales of every K step into the token ring (warp 11), after the unit's
// inputs are ready.
template <class S, class C>
__device__ __forceinline__ void mx_producer_t(const GemmMaps& maps, const CoreArgs& a, const S& s,
                                              unsigned char* smem, uint64_t* tkfull, uint64_t* tkempty) {
    int slot = 0;
    uint32_t ph = 0;
    uint32_t issued = 0, issued_ph = 0;
    Unit u;
    for (int i = 0; s.get(i, u); ++i) {
        if (!s.wait_inputs(u, a.st, a.timeout_ns)) break;
        const int K = phase_k<C>(a, u.phase);
        const int KB = (K + C::BKX - 1) / C::BKX;
        const BMaps& bm = u.phase == 0 ? maps.rows : maps.h;
        const int bx = token_box(u.rows);
        // the stage's token scales: one 16-byte aligned run of the plane,
        // starting up to 3 rows before the chunk
        const int sc_lead = u.brow0 & 3;
        const uint32_t sc_bytes = (uint32_t)(4 * (sc_lead + u.rows) + 15) & ~15u;
        const uint32_t bytes = (uint32_t)(16 * (bx + 1)) * B_ROW_BYTES + sc_bytes;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&tkempty[slot], ph ^ 1u, a.st, a.timeout_ns, 16)) {
                ok = false;
                break;
            }
            unsigned char* t = smem + C::T_BASE + slot * C::TSTAGE;
            mbar_arrive_expect_tx(&tkfull[slot], bytes);
            const uint8_t* plane = (u.phase == 0 ? a.xsc : a.hsc) + (size_t)kb * a.sc_rows * 4;
            bulk_load(t + C::SFB_RAW_OFF, plane + (size_t)(u.brow0 - sc_lead) * 4, sc_bytes, &tkfull[slot]);
            tma_load_2d(t + C::B_OFF, &bm.m[bx], &tkfull[slot], kb * C::BKX, u.brow0);
            issued |= 1u << slot;
            issued_ph = (issued_ph & ~(1u << slot)) | (ph << slot);
            if (++slot == C::NT) {
                slot = 0;
                ph ^= 1u;
            }
        }
        if (!ok) break;
    }
    for (int st = 0; st < C::NT; ++st)
        if ((issued >> st) & 1u) mbar_wait(&tkfull[st], (issued_ph >> st) & 1u, nullptr, DRAIN_TIMEOUT_NS, 17);
}

// Scale layout of the two-ring path (warp 10): as gemm_sf_layout, with the
// weight scales in the weight slot and the token scales in the token slot;
// arrives on sfready[token slot] once both slots' loads have landed.
template <class S, class C>
__device__ __forceinline__ void mx_sf_layout_split(const CoreArgs& a, const S& s, unsigned char* smem,
                                                   uint64_t* wfull, uint64_t* tkfull, uint64_t* sfready) {
    const int lane = threadIdx.x & 31;
    int ws = 0, ts = 0;
    uint32_t wph = 0, tph = 0;
    Unit u;
    for (int i = 0; s.get(i, u); ++i) {
        const int K = phase_k<C>(a, u.phase);
        const int KB = (K + C::BKX - 1) / C::BKX;
        const int lead = u.brow0 & 3;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            // the warp leaves or goes on as one (it synchronises below)
            const bool landed = mbar_wait(&wfull[ws], wph, a.st, a.timeout_ns, 81) &&
                                mbar_wait(&tkfull[ts], tph, a.st, a.timeout_ns, 82);
            if (!__all_sync(0xffffffffu, landed)) {
                ok = false;
                break;
            }
            unsigned char* w = smem + ws * C::WSTAGE;
            unsigned char* t = smem + C::T_BASE + ts * C::TSTAGE;
            const uint8_t* ra = w + C::SFA_RAW_OFF;
            uint32_t wa[4];
#pragma unroll
            for (int r1 = 0; r1 < 4; ++r1) {
                const int r = lane + 32 * r1;
                // feature r of the tile: gate/up keeps 64 gate then 64 up rows of 64 bytes
                const uint8_t* col = u.phase == 0 ? ra + (r >> 6) * 256 + (r & 63) : ra + r;
                const int pitch = u.phase == 0 ? 64 : 128;
                wa[r1] = (uint32_t)col[0] | ((uint32_t)col[pitch] << 8) | ((uint32_t)col[2 * pitch] << 16) |
                         ((uint32_t)col[3 * pitch] << 24);
            }
            *reinterpret_cast<uint4*>(w + C::SFA_OFF + 16 * lane) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
            const uint32_t* rb = reinterpret_cast<const uint32_t*>(t + C::SFB_RAW_OFF) + lead;
#pragma unroll
            for (int r2 = 0; r2 < 2; ++r2) {
                uint32_t wb[4];
#pragma unroll
                for (int r1 = 0; r1 < 4; ++r1) {
                    const int r = lane + 32 * r1 + 128 * r2;
                    wb[r1] = r < u.rows ? rb[r] : 0u;
                }
                *reinterpret_cast<uint4*>(t + C::SFB_OFF + 512 * r2 + 16 * lane) =
                    make_uint4(wb[0], wb[1], wb[2], wb[3]);
            }
            fence_proxy_async_shared();  // generic writes -> the TMEM copy (async proxy) reads
            __syncwarp();                // every lane's writes and fence precede the one arrival
            if (lane == 0) mbar_arrive(&sfready[ts]);
            if (++ws == C::NW) {
                ws = 0;
                wph ^= 1u;
            }
            if (++ts == C::NT) {
                ts = 0;
                tph ^= 1u;
            }
        }
        if (!ok) break;
    }
}

// ------------------------------------------------------------------ TMEM placement
// TMEM holds two 256-column accumulator buffers used in ring order; each use
// is a "ticket" (buffer = ticket & 1, barrier parity = (ticket >> 1) & 1).
// A unit whose M tiles fit in one buffer (one tile, or two tiles of N <= 128
// columns: tile s at column 128 s) takes one ticket; two tiles of N > 128
// take two consecutive tickets, one buffer each.
// A pair of tiles fits one buffer up to N = 128 columns each; the MXFP8
// path stops at 96 so that buffer 1's second tile ends below its scale
// factors (column 480).
template <class C>
__device__ __forceinline__ int unit_tickets(int nsub, int N) {
    return (nsub == 2 && N > (C::MX ? 96 : 128)) ? 2 : 1;
}
__device__ __forceinline__ uint32_t acc_col(uint32_t tk, int sub, bool wide) {
    return wide ? ((tk + (uint32_t)sub) & 1u) * ACC_COLS : (tk & 1u) * ACC_COLS + (uint32_t)sub * 128u;
}

// ------------------------------------------------------------------ MMA issuer
// ready[stage]: the TMA barrier (bf16) or the scale-layout barrier (MXFP8).
template <class S, class C>
__device__ __forceinline__ void gemm_mma(const CoreArgs& a, const S& s, unsigned char* smem, uint64_t* ready,
                                         uint64_t* empty, uint64_t* tfull, uint64_t* tempty, uint64_t* fin,
                                         uint32_t tmem_base) {
    int stage = 0;
    uint32_t phase = 0;
    uint32_t tk = 0;  // next accumulator ticket
    Unit u;
    for (int i = 0; s.get(i, u); ++i) {
        const int K = phase_k<C>(a, u.phase);
        const int KB = (K + C::BKX - 1) / C::BKX;
        const int N = (u.rows + 15) & ~15;
        const int nsub = unit_subs<C>(a, u);
        const int nt = unit_tickets<C>(nsub, N);
        const bool wide = nt == 2;
        // bf16 path: every phase bf16 x bf16; A MN-major (forward) or K-major (backward)
        const bool a_kmaj = C::EXT && u.phase >= 2;
        const uint32_t idesc = umma_idesc_f16(128, N, a_kmaj ? 0 : 1, /*B K-major*/ 0, /*bf16*/ 1);
        bool ok = true;
        for (int t = 0; t < nt && ok; ++t) {
            const uint32_t tkt = tk + (uint32_t)t;
            ok = mbar_wait(&tempty[tkt & 1u], ((tkt >> 1) & 1u) ^ 1u, a.st, a.timeout_ns, 20);
        }
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&ready[stage], phase, a.st, a.timeout_ns, 21)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + stage * C::STAGE + C::A_OFF);
            const uint32_t sb = smem_u32(smem + stage * C::STAGE + C::B_OFF);
            if constexpr (C::MX) {
                // scale factors of this stage into TMEM (executed in order with the MMAs)
                unsigned char* st = smem + stage * C::STAGE;
                for (int sub = 0; sub < nsub; ++sub)
                    tmem_cp_32x128b_warpx4(tmem_base + C::TM_SFA + 4 * sub, st + C::SFA_OFF + sub * 512);
                tmem_cp_32x128b_warpx4(tmem_base + C::TM_SFB, st + C::SFB_OFF);
                if (N > 128) tmem_cp_32x128b_warpx4(tmem_base + C::TM_SFB + 4, st + C::SFB_OFF + 512);
                const int nks = min(4, (K - kb * C::BKX) / 32);  // 32 K values per MMA
                for (int ks = 0; ks < nks; ++ks) {
                    // B: K-major E4M3 SW128, 32 K = 32 bytes inside the atom
                    const uint64_t bd = umma_desc_sw128(sb + ks * 32, 16, 1024);
                    const uint32_t sel = (uint32_t)ks << 30;  // scale byte of these 32 K values
                    const uint32_t idx = umma_idesc_mxf8(128, N, 1, 0, (uint32_t)ks);
                    for (int sub = 0; sub < nsub; ++sub) {
                        // A: MN-major E4M3; gate/up = two 64-byte-swizzled 64-column halves 8 KB
                        //    apart (8-row K groups 512 bytes apart), down = one 128-byte-swizzled
                        //    128-column tile (K groups 1 KB apart); 32 K rows per MMA.
                        const uint32_t a0 = sa + sub * 16384;
                        const uint64_t ad = u.phase == 0 ? umma_desc(a0 + ks * 2048, 8192, 512, UMMA_LAYOUT_SW64)
                                                         : umma_desc(a0 + ks * 4096, 0, 1024, UMMA_LAYOUT_SW128);
                        umma_mxf8(tmem_base + acc_col(tk, sub, wide), ad, bd, idx,
                                  tmem_base + C::TM_SFA + 4 * sub + sel, tmem_base + C::TM_SFB + sel,
                                  (kb | ks) != 0 ? 1u : 0u);
                    }
                }
            } else {
#pragma unroll
                for (int ks = 0; ks < BK / 16; ++ks) {
                    // B: K-major SW128, 16 K = 32 bytes inside the atom; 8-row groups 1 KB apart.
                    const uint64_t bd = umma_desc_sw128(sb + ks * 32, 16, 1024);
#pragma unroll
                    for (int sub = 0; sub < C::SUB; ++sub) {
                        if (sub < nsub) {
                            // A MN-major SW128: 16 K rows per MMA = 2 atoms of 1 KB, the two
                            //   64-wide MN halves 8 KB apart (LBO);
                            // A K-major SW128: 16 K = 32 bytes inside the atom, 8-row groups 1 KB apart.
                            const uint64_t ad =
                                a_kmaj ? umma_desc_sw128(sa + sub * A_BYTES + ks * 32, 16, 1024)
                                       : umma_desc_sw128(sa + sub * A_BYTES + ks * 2048, A_BYTES / 2, 1024);
                            umma_bf16(tmem_base + acc_col(tk, sub, wide), ad, bd, idesc, (kb | ks) != 0 ? 1u : 0u);
                        }
                    }
                }
            }
            umma_commit(&empty[stage]);
            if (++stage == C::NST) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!ok) break;
        for (int t = 0; t < nt; ++t) umma_commit(&tfull[(tk + (uint32_t)t) & 1u]);
        tk += (uint32_t)nt;
    }
    // wait for every MMA this thread issued before TMEM is released
    umma_commit(fin);
    mbar_wait(fin, 0, nullptr, DRAIN_TIMEOUT_NS, 22);
}

// ------------------------------------------------------------------ MMA issuer, MXFP8 two rings
// As gemm_mma's MXFP8 branch: per K step the scales of the weight slot and
// the token slot into TMEM, then 4 block-scaled MMAs (K = 32 each); the
// step's commits free both slots.
template <class S, class C>
__device__ __forceinline__ void gemm_mma_mx_split(const CoreArgs& a, const S& s, unsigned char* smem,
                                                  uint64_t* sfready, uint64_t* wempty, uint64_t* tkempty,
                                                  uint64_t* tfull, uint64_t* tempty, uint64_t* fin,
                                                  uint32_t tmem_base) {
    int ws = 0, ts = 0;
    uint32_t tph = 0;
    uint32_t tk = 0;  // next accumulator ticket
    uint32_t set = 0;  // scale-factor set of the next K step
    Unit u;
    for (int i = 0; s.get(i, u); ++i) {
        const int K = phase_k<C>(a, u.phase);
        const int KB = (K + C::BKX - 1) / C::BKX;
        const int N = (u.rows + 15) & ~15;
        bool ok = mbar_wait(&tempty[tk & 1u], ((tk >> 1) & 1u) ^ 1u, a.st, a.timeout_ns, 26);
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&sfready[ts], tph, a.st, a.timeout_ns, 27)) {
                ok = false;
                break;
            }
            tc_fence_after();
            unsigned char* w = smem + ws * C::WSTAGE;
            unsigned char* t = smem + C::T_BASE + ts * C::TSTAGE;
            const uint32_t sa = smem_u32(w + C::A_OFF);
            const uint32_t sb = smem_u32(t + C::B_OFF);
            // scale factors of this stage into TMEM (executed in order with the MMAs)
            const uint32_t sfa = tmem_base + C::TM_SFA + set * C::TM_SF_SET;
            const uint32_t sfb = tmem_base + C::TM_SFB + set * C::TM_SF_SET;
            set ^= 1u;
            tmem_cp_32x128b_warpx4(sfa, w + C::SFA_OFF);
            tmem_cp_32x128b_warpx4(sfb, t + C::SFB_OFF);
            if (N > 128) tmem_cp_32x128b_warpx4(sfb + 4, t + C::SFB_OFF + 512);
            const int nks = min(4, (K - kb * C::BKX) / 32);  // 32 K values per MMA
            for (int ks = 0; ks < nks; ++ks) {
                // B: K-major E4M3 SW128, 32 K = 32 bytes inside the atom
                const uint64_t bd = umma_desc_sw128(sb + ks * 32, 16, 1024);
                const uint32_t sel = (uint32_t)ks << 30;  // scale byte of these 32 K values
                const uint32_t idx = umma_idesc_mxf8(128, N, 1, 0, (uint32_t)ks);
                // A: MN-major E4M3; gate/up = two 64-byte-swizzled 64-column halves 8 KB apart
                // (8-row K groups 512 bytes apart), down = one 128-byte-swizzled 128-column tile
                // (K groups 1 KB apart); 32 K rows per MMA.
                const uint64_t ad = u.phase == 0 ? umma_desc(sa + ks * 2048, 8192, 512, UMMA_LAYOUT_SW64)
                                                 : umma_desc(sa + ks * 4096, 0, 1024, UMMA_LAYOUT_SW128);
                umma_mxf8(tmem_base + acc_col(tk, 0, false), ad, bd, idx, sfa + sel, sfb + sel,
                          (kb | ks) != 0 ? 1u : 0u);
            }
            umma_commit(&wempty[ws]);
            umma_commit(&tkempty[ts]);
            if (++ws == C::NW) ws = 0;
            if (++ts == C::NT) {
                ts = 0;
                tph ^= 1u;
            }
        }
        if (!ok) break;
        umma_commit(&tfull[tk & 1u]);
        ++tk;
    }
    // wait for every MMA this thread issued before TMEM is released
    umma_commit(fin);
    mbar_wait(fin, 0, nullptr, DRAIN_TIMEOUT_NS, 28);
}

// ------------------------------------------------------------------ MMA issuer, CTA pairs
// One thread of the pair's first CTA: per stage (both CTAs' loads counted
// on full[stage]) 4 MMAs of M = 256, N = the 16-rounded rows, K = 16 into
// both CTAs' accumulators; the stage's commit arrives on empty[stage] of
// both CTAs, the unit's on tfull[] of both.  tempty[] (this CTA's) counts
// the epilogue warps of both CTAs.
template <class S, class C>
__device__ __forceinline__ void gemm_mma_pair(const CoreArgs& a, const S& s, unsigned char* smem, uint64_t* full,
                                              uint64_t* empty, uint64_t* tfull, uint64_t* tempty, uint64_t* fin,
                                              uint32_t tmem_base) {
    int stage = 0;
    uint32_t phase = 0;
    uint32_t tk = 0;
    Unit u;
    for (int i = 0; s.get(i, u); ++i) {
        const int K = phase_k<C>(a, u.phase);
        const int KB = (K + C::BKX - 1) / C::BKX;
        const int N = (u.rows + 15) & ~15;
        const bool a_kmaj = C::EXT && u.phase >= 2;  // the backward reads the weights K-major
        const uint32_t idesc = umma_idesc_f16(256, N, a_kmaj ? 0 : 1, /*B K-major*/ 0, /*bf16*/ 1);
        const int nsub = unit_subs<C>(a, u);
        const int nt = unit_tickets<C>(nsub, N);
        const bool wide = nt == 2;
        bool ok = true;
        for (int t = 0; t < nt && ok; ++t) {
            const uint32_t tkt = tk + (uint32_t)t;
            ok = mbar_wait(&tempty[tkt & 1u], ((tkt >> 1) & 1u) ^ 1u, a.st, a.timeout_ns, 23);
        }
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb) {
            if (!mbar_wait(&full[stage], phase, a.st, a.timeout_ns, 24)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + stage * C::STAGE + C::A_OFF);
            const uint32_t sb = smem_u32(smem + stage * C::STAGE + C::B_OFF);
#pragma unroll
            for (int ks = 0; ks < BK / 16; ++ks) {
                // same descriptors as one CTA's: A MN-major SW128 (halves 8 KB apart), B K-major SW128;
                // the second CTA's rows sit at the same offsets in its shared memory
                const uint64_t bd = umma_desc_sw128(sb + ks * 32, 16, 1024);
#pragma unroll
                for (int sub = 0; sub < C::SUB; ++sub) {
                    if (sub < nsub) {
                        const uint32_t s0 = sa + sub * A_BYTES;
                        const uint64_t ad = a_kmaj ? umma_desc_sw128(s0 + ks * 32, 16, 1024)
                                                   : umma_desc_sw128(s0 + ks * 2048, A_BYTES / 2, 1024);
                        umma_bf16_pair(tmem_base + acc_col(tk, sub, wide), ad, bd, idesc, (kb | ks) != 0 ? 1u : 0u);
                    }
                }
            }
            umma_commit_pair_both(&empty[stage], 0x3);
            if (++stage == C::NST) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!ok) break;
        for (int t = 0; t < nt; ++t) umma_commit_pair_both(&tfull[(tk + (uint32_t)t) & 1u], 0x3);
        tk += (uint32_t)nt;
    }
    // wait for every MMA this thread issued before TMEM is released
    umma_commit_pair_local(fin);
    mbar_wait(fin, 0, nullptr, DRAIN_TIMEOUT_NS, 25);
}

// ------------------------------------------------------------------ epilogue (warps 2..9)
// Drains one M tile's accumulator (TMEM columns col0 .. col0 + rows), 32
// tokens at a time, through a token-major staging tile in shared memory
// (epi[token][feature], pitch EPI_TLD), so that every global store is a
// row-contiguous run: gate/up writes h rows (8 lanes per 64-feature row),
// down pushes a row's 128 outputs (a warp per row: 256 bytes of fp16 and one
// exponent byte, or 256 bytes of bf16 on the MXFP8 path) to the tokens'
// slots.
// Chunks cc0, cc0 + ccstep, ... of the tile are drained by this warpgroup
// (named barrier `bar`, staging tile `epi`).
template <class C>
__device__ __forceinline__ void epi_drain_tile(const CoreArgs& a, const Unit& u, int mt, uint32_t col0, float* epi,
                                               uint32_t tmem_base, int cc0, int ccstep, int bar) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3;  // TMEM lane quadrant this warp may access: features q*32 .. q*32+31
    const int ncc = (u.rows + 31) >> 5;
    for (int cc = cc0; cc < ncc; cc += ccstep) {
        float v[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + col0 + (uint32_t)(cc * 32), v);
        // token-major: lanes hold consecutive features, so each store row is contiguous
#pragma unroll
        for (int t = 0; t < 32; ++t) epi[t * EPI_TLD + q * 32 + lane] = v[t];
        named_bar_sync(bar, 128);
        if (u.phase == 0) {
            // h features mt*64 + j: gate in staging columns j, up in 64 + j.  Lane
            // group g = lane / 8 takes token rows; lane % 8 owns 8 features.
            const int j0 = (lane & 7) * 8;
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int t = it * 16 + q * 4 + (lane >> 3);  // token of this chunk
                const float* er = epi + t * EPI_TLD;
                const float4 g0 = *reinterpret_cast<const float4*>(er + j0);
                const float4 g1 = *reinterpret_cast<const float4*>(er + j0 + 4);
                const float4 u0 = *reinterpret_cast<const float4*>(er + 64 + j0);
                const float4 u1 = *reinterpret_cast<const float4*>(er + 64 + j0 + 4);
                const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                float hv[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) hv[k] = gv[k] / (1.0f + __expf(-gv[k])) * uv[k];
                const int col = cc * 32 + t;
                const bool live = col < u.rows;
                const size_t row = (size_t)(u.brow0 + col);
                if constexpr (C::MX) {
                    // MXFP8 h: a 32-feature block = 4 lanes of one row (lane % 8 in 0-3 or 4-7)
                    float amax = 0.f;
#pragma unroll
                    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(hv[k]));
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
                    const int sx = mx_block_exponent(amax);
                    const float inv = mx_pow2(-sx);
                    const uint2 pq = make_uint2((uint32_t)mx_e4m3x2(hv[0] * inv, hv[1] * inv) |
                                                    ((uint32_t)mx_e4m3x2(hv[2] * inv, hv[3] * inv) << 16),
                                                (uint32_t)mx_e4m3x2(hv[4] * inv, hv[5] * inv) |
                                                    ((uint32_t)mx_e4m3x2(hv[6] * inv, hv[7] * inv) << 16));
                    if (live) {
                        *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(a.h) + row * a.I + mt * MT_G_FEATURES +
                                                  j0) = pq;
                        if ((lane & 3) == 0) {
                            const int b = 2 * mt + ((lane & 7) >> 2);  // 32-feature block along I
                            a.hsc[((size_t)(b >> 2) * a.sc_rows + row) * 4 + (b & 3)] = (uint8_t)(sx + 127);
                        }
                    }
                } else {
                    const uint4 pk = make_uint4(pack_bf16x2(hv[0], hv[1]), pack_bf16x2(hv[2], hv[3]),
                                                pack_bf16x2(hv[4], hv[5]), pack_bf16x2(hv[6], hv[7]));
                    const size_t at = row * a.I + mt * MT_G_FEATURES + j0;
                    if (live) {
                        *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.h) + at) = pk;
                        if (C::EXT && a.save_a) {
                            *reinterpret_cast<uint4*>(a.save_a + at) =
                                make_uint4(pack_bf16x2(gv[0], gv[1]), pack_bf16x2(gv[2], gv[3]),
                                           pack_bf16x2(gv[4], gv[5]), pack_bf16x2(gv[6], gv[7]));
                            *reinterpret_cast<uint4*>(a.save_b + at) =
                                make_uint4(pack_bf16x2(uv[0], uv[1]), pack_bf16x2(uv[2], uv[3]),
                                           pack_bf16x2(uv[4], uv[5]), pack_bf16x2(uv[6], uv[7]));
                        }
                    }
                }
            }
        } else if (C::EXT && u.phase == 2) {
            // dh of features mt*128 + 4*lane .. +3, a warp per token: the SwiGLU backward with the
            // row's saved a, b (bf16); da and db rows pushed as bf16 into dab [rows, 2I]
#pragma unroll 2
            for (int it = 0; it < 8; ++it) {
                const int t = it * 4 + q;
                const int col = cc * 32 + t;
                if (col < u.rows) {
                    const size_t row = (size_t)(u.brow0 + col);
                    const int i0 = mt * MT_D_FEATURES + 4 * lane;
                    const float4 d4 = *reinterpret_cast<const float4*>(epi + t * EPI_TLD + 4 * lane);
                    const uint2 av = *reinterpret_cast<const uint2*>(a.save_a + row * a.I + i0);
                    const uint2 bv = *reinterpret_cast<const uint2*>(a.save_b + row * a.I + i0);
                    const float dh[4] = {d4.x, d4.y, d4.z, d4.w};
                    const float af[4] = {__uint_as_float(av.x << 16), __uint_as_float(av.x & 0xffff0000u),
                                         __uint_as_float(av.y << 16), __uint_as_float(av.y & 0xffff0000u)};
                    const float bf[4] = {__uint_as_float(bv.x << 16), __uint_as_float(bv.x & 0xffff0000u),
                                         __uint_as_float(bv.y << 16), __uint_as_float(bv.y & 0xffff0000u)};
                    float da[4], db[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        // silu(a) = a s, silu'(a) = s + a s (1 - s), s = 1 / (1 + e^-a)
                        const float sg = 1.0f / (1.0f + __expf(-af[p]));
                        db[p] = dh[p] * af[p] * sg;
                        da[p] = dh[p] * bf[p] * (sg + af[p] * sg * (1.0f - sg));
                    }
                    uint16_t* out = a.dab + row * (size_t)(2 * a.I) + i0;
                    *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16x2(da[0], da[1]), pack_bf16x2(da[2], da[3]));
                    *reinterpret_cast<uint2*>(out + a.I) =
                        make_uint2(pack_bf16x2(db[0], db[1]), pack_bf16x2(db[2], db[3]));
                }
            }
        } else {
            // push to the token's slot, one row per warp store (fp16 with the row's exponent for
            // these 128 features, or bf16 on the MXFP8 path: 256 bytes); the combine rounds y
            // once.  Phase 3 (the backward's dx rows) pushes the same way.
#pragma unroll 4
            for (int it = 0; it < 8; ++it) {
                const int t = it * 4 + q;
                const int col = cc * 32 + t;
                if (col < u.rows) {  // warp-uniform: t depends on the warp only
                    int slot = __ldg(a.row_slot + u.grow0 + col);
                    void* out = a.out;
                    int8_t* out_exp = a.out_exp;
                    if (a.push) {  // the slot's source rank
                        const int d = slot / a.push_slots;
                        slot -= d * a.push_slots;
                        out = a.push->out[d];
                        out_exp = a.push->exp[d];
                    }
                    const float4 o4 = *reinterpret_cast<const float4*>(epi + t * EPI_TLD + 4 * lane);
                    const size_t at = (size_t)slot * a.H + mt * MT_D_FEATURES;
                    if constexpr (C::MX) {
                        reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(out) + at)[lane] =
                            make_uint2(pack_bf16x2(o4.x, o4.y), pack_bf16x2(o4.z, o4.w));
                    } else {
                        // fp16 with one exponent for the row's 128 features of this tile
                        float m = fmaxf(fmaxf(fabsf(o4.x), fabsf(o4.y)), fmaxf(fabsf(o4.z), fabsf(o4.w)));
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
                        const int sx = slot_block_exponent(m);
                        const float inv = pow2f(-sx);
                        reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(out) + at)[lane] =
                            make_uint2(pack_half2(o4.x * inv, o4.y * inv), pack_half2(o4.z * inv, o4.w * inv));
                        if (lane == 0) out_exp[(size_t)slot * (a.H / MT_D_FEATURES) + mt] = (int8_t)sx;
                    }
                }
            }
        }
        named_bar_sync(bar, 128);
    }
}

// Two warpgroups drain each unit side by side (warps 2-5 and 6-9, each
// covering the four TMEM lane quadrants): a pair's tiles one each, a single
// tile's 32-token chunks alternately.  Each group arrives once on every
// ticket of the unit when it has finished its share (tempty counts 8).
template <class S, class C>
__device__ __forceinline__ void gemm_epilogue(const CoreArgs& a, const S& s, unsigned char* smem, uint64_t* tfull,
                                              uint64_t* tempty, volatile int* ok_flags, int* done_cnt,
                                              uint32_t tmem_base) {
    const int lane = threadIdx.x & 31;
    const int g = (threadIdx.x - 64) >> 7;     // warpgroup 0 or 1
    const int et = (threadIdx.x - 64) & 127;   // 0..127 inside the group
    const int bar = 1 + g;                     // the group's named barrier
    volatile int* ok_flag = ok_flags + g;
    float* epi = reinterpret_cast<float*>(smem + C::EPI_OFF + g * EPI_BYTES);
    uint32_t tk = 0;  // next accumulator ticket (the MMA issuer's sequence)
    bool ok = true;
    Unit u;
    for (int i = 0; ok && s.get(i, u); ++i) {
        const int nsub = unit_subs<C>(a, u);
        const int nt = unit_tickets<C>(nsub, (u.rows + 15) & ~15);
        const bool wide = nt == 2;
        // this group's share: tile `g` of a pair, or every other chunk of a single tile
        const int sub = nsub == 2 ? g : 0;
        {
            const uint32_t tkt = wide ? tk + (uint32_t)sub : tk;
            // one thread waits, all 128 of the group leave together on failure
            if (et == 0) *ok_flag = mbar_wait(&tfull[tkt & 1u], (tkt >> 1) & 1u, a.st, a.timeout_ns, 30) ? 1 : 0;
            named_bar_sync(bar, 128);
            ok = *ok_flag != 0;
            named_bar_sync(bar, 128);
            if (!ok) break;
            tc_fence_after();
            epi_drain_tile<C>(a, u, u.m * C::SUB + sub, acc_col(tk, sub, wide), epi, tmem_base,
                              nsub == 2 ? 0 : g, nsub == 2 ? 1 : 2, bar);
        }
        // this group is done with every buffer of the unit (CTA pairs: on
        // the first CTA's tempty, where the MMA issuer waits)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            for (int t = 0; t < nt; ++t) {
                if constexpr (C::CG2)
                    mbar_arrive_cluster(smem_in_rank(&tempty[(tk + (uint32_t)t) & 1u], 0));
                else
                    mbar_arrive(&tempty[(tk + (uint32_t)t) & 1u]);
            }
        }
        tk += (uint32_t)nt;
        if (S::kSignals) {
            // h rows are read next by TMA (async proxy) in some CTA: make this
            // group's stores visible to that proxy; the group that finishes
            // the unit second publishes it once.  The groups are at most one
            // unit apart (a buffer is reused only after both released it), so
            // two counters, by unit parity, pair their arrivals.  When that
            // publication completes a chunk's down units, the whole group
            // passes the chunk's rows on (s.chunk_done).
            fence_proxy_async_global();
            __threadfence();
            named_bar_sync(bar, 128);
            if (et == 0) {
                __threadfence();
                int fin = 0;
                if (atomicAdd(done_cnt + (i & 1), 1) & 1) {
                    __threadfence();
                    fin = s.unit_done(u) ? 1 : 0;
                }
                *ok_flag = fin;
            }
            named_bar_sync(bar, 128);
            const bool fin = *ok_flag != 0;
            named_bar_sync(bar, 128);  // ok_flag is written again at the next unit
            if (fin) s.chunk_done(u, et, 128);
        }
    }
}

// ------------------------------------------------------------------ one GEMM CTA
// Runs every unit the schedule gives this CTA.  Threads [0, C::THREADS) must
// call it; any further warps of the block take part in its first barrier
// (a __syncthreads of their own) and in nothing else.  It returns after TMEM
// is released.  mx: MXFP8 maps (C::MX only).
// Depth of the ring that `full` / `empty` index: the weight ring of the
// two-ring MXFP8 layout, else the one ring.
template <class C>
constexpr int ring_w() {
    if constexpr (C::SPLIT)
        return C::NW;
    else
        return C::NST;
}

template <class S, class C>
__device__ __forceinline__ void gemm_cta(const GemmMaps& maps, const MxMaps* mx, const CoreArgs& a, const S& s,
                                         unsigned char* smem) {
    // one ring: full, empty, sfready [NST] each; two rings (MXFP8): the
    // weight ring's full and empty [NW], the token ring's tkfull and tkempty
    // [NT = NST], and sfready [NT]
    constexpr int NWR = ring_w<C>();
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* empty = full + NWR;
    uint64_t* tkfull = empty + NWR;
    uint64_t* tkempty = tkfull + (C::SPLIT ? C::NST : 0);
    uint64_t* sfready = C::SPLIT ? tkempty + C::NST : empty + C::NST;  // MXFP8: stage scales in the MMA layout
    uint64_t* tfull = sfready + C::NST;
    uint64_t* tempty = tfull + 2;
    uint64_t* fin = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
    volatile int* ok_flags = reinterpret_cast<volatile int*>(tmem_slot + 1);  // one per epilogue group
    int* done_cnt = const_cast<int*>(ok_flags) + 2;                            // two, by unit parity
    static_assert(((C::SPLIT ? 2 * NWR + 3 * C::NST : 3 * C::NST) + 5) * 8 + 4 * 5 <= C::BAR_BYTES, "barrier region");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        done_cnt[0] = 0;
        done_cnt[1] = 0;
        if constexpr (C::SPLIT) {
            for (int st = 0; st < NWR; ++st) {
                mbar_init(&full[st], 1);
                mbar_init(&empty[st], 1);
            }
            for (int st = 0; st < C::NST; ++st) {
                mbar_init(&tkfull[st], 1);
                mbar_init(&tkempty[st], 1);
                mbar_init(&sfready[st], 1);
            }
        } else {
            for (int st = 0; st < C::NST; ++st) {
                mbar_init(&full[st], 1);
                mbar_init(&empty[st], 1);
                mbar_init(&sfready[st], 1);
            }
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], C::CG2 ? 16 : 8);  // 4 warps of each epilogue group (of both CTAs of a pair)
        }
        mbar_init(fin, 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        if constexpr (C::MX) {
            tma_prefetch_desc(&mx->gq);
            tma_prefetch_desc(&mx->uq);
            tma_prefetch_desc(&mx->dq);
            tma_prefetch_desc(&mx->gs);
            tma_prefetch_desc(&mx->us);
            tma_prefetch_desc(&mx->ds);
        } else {
            tma_prefetch_desc(&maps.wg);
            tma_prefetch_desc(&maps.wu);
            tma_prefetch_desc(&maps.wd);
            if (maps.has_wd3) tma_prefetch_desc(&maps.wd3);
        }
        for (int b = 0; b < B_MAPS; ++b) {
            tma_prefetch_desc(&maps.rows.m[b]);
            tma_prefetch_desc(&maps.h.m[b]);
        }
    }
    if (warp == 1) {
        if constexpr (C::CG2) {
            tmem_alloc_pair(tmem_slot, TMEM_COLS);  // both CTAs of the pair, same columns
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (C::CG2) cluster_sync_all();  // both CTAs' barriers and TMEM are set up
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    uint32_t rank = 0;
    if constexpr (C::CG2) rank = cluster_ctarank();

    if (warp == 0) {
        if (lane == 0) {
            if constexpr (C::CG2)
                gemm_producer_pair<S, C>(maps, a, s, smem, full, empty, rank);
            else if constexpr (C::SPLIT)
                mx_producer_w<S, C>(mx, a, s, smem, full, empty);
            else
                gemm_producer<S, C>(maps, mx, a, s, smem, full, empty);
        }
    } else if (warp == 1) {
        if constexpr (C::CG2) {
            if (lane == 0 && rank == 0) gemm_mma_pair<S, C>(a, s, smem, full, empty, tfull, tempty, fin, tmem_base);
        } else if constexpr (C::SPLIT) {
            if (lane == 0)
                gemm_mma_mx_split<S, C>(a, s, smem, sfready, empty, tkempty, tfull, tempty, fin, tmem_base);
        } else {
            if (lane == 0) gemm_mma<S, C>(a, s, smem, C::MX ? sfready : full, empty, tfull, tempty, fin, tmem_base);
        }
    } else if (warp < 10) {
        gemm_epilogue<S, C>(a, s, smem, tfull, tempty, ok_flags, done_cnt, tmem_base);
    } else if constexpr (C::SPLIT) {
        if (warp == 10)
            mx_sf_layout_split<S, C>(a, s, smem, full, tkfull, sfready);
        else if (lane == 0)
            mx_producer_t<S, C>(maps, a, s, smem, tkfull, tkempty);
    } else if constexpr (C::MX) {
        gemm_sf_layout<S, C>(a, s, smem, full, sfready);
    }

    // the GEMM roles' threads only: a persistent kernel may run other warps
    // beside them (barrier 3; the epilogue groups use 1 and 2)
    tc_fence_before();
    named_bar_sync(3, C::THREADS);
    if constexpr (C::CG2) {
        // the first CTA's MMAs (which read this CTA's shared memory and write
        // its TMEM) have completed, and no epilogue still reads TMEM
        cluster_sync_all();
        if (warp == 1) {
            tc_fence_after();
            tmem_dealloc_pair(tmem_base, TMEM_COLS);
        }
    } else if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

__device__ __forceinline__ unsigned char* align_smem_1024(unsigned char* p) {
    return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

}  // namespace mok

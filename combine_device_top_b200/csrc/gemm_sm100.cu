// gemm_sm100.cu -- the staged grouped-GEMM kernels (step 4 of the forward
// MoE layer as its own launches): one persistent launch per phase, gate/up
// + SwiGLU then down + push, over every chunk of the device-built work list.
// The tcgen05/TMEM/TMA core and its design notes are in gemm_core.cuh.
#include <cstring>

#include "gemm_core.cuh"

namespace mok {

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    k_grouped_gemm(const __grid_constant__ GemmMaps maps, const __grid_constant__ MxMaps mx, const CoreArgs a,
                   const Chunk* __restrict__ chunks, const int* __restrict__ counts2, int phase, int MT, int GC) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    StagedSched s;
    s.phase = phase;
    s.nch = *reinterpret_cast<volatile const int*>(counts2);
    s.MT = MT;
    s.GC = GC;
    s.chunks = chunks;
    gemm_cta<StagedSched, C>(maps, &mx, a, s, smem);
}

// The bf16 phases on CTA pairs (clusters of two): MT counts cluster units
// (2 C::SUB M tiles each).
template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    k_grouped_gemm_pair(const __grid_constant__ GemmMaps maps, const CoreArgs a, const Chunk* __restrict__ chunks,
                        const int* __restrict__ counts2, int phase, int MT, int GC) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    StagedSched2 s;
    s.phase = phase;
    s.nch = *reinterpret_cast<volatile const int*>(counts2);
    s.MT = MT;
    s.GC = GC;
    s.rank = cluster_ctarank();
    s.chunks = chunks;
    gemm_cta<StagedSched2, C>(maps, nullptr, a, s, smem);
}

template <class C>
static cudaError_t launch_pair_phase(int grid, const GemmMaps& maps, const CoreArgs& a, const Chunk* chunks,
                                     const int* counts2, int phase, int MT, int GC, cudaStream_t stream) {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)(grid & ~1));
    // as many pairs as can be resident at once (the grid walks its units)
    int clusters = 0;
    cudaError_t e = cudaOccupancyMaxActiveClusters(&clusters, k_grouped_gemm_pair<C>, &cfg);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    if (2 * clusters < grid) grid = 2 * clusters;
    cfg.gridDim = dim3((unsigned)(grid & ~1));
    return cudaLaunchKernelEx(&cfg, k_grouped_gemm_pair<C>, maps, a, chunks, counts2, phase, MT, GC);
}

// Defaults measured on B200 (page shape and a 512-rows-per-expert case):
// small raster groups paid.  Pairs of M tiles halve the token-tile bytes
// each SM takes in per weight byte, but a pair of chunks taller than 128 rows
// fills TMEM, so its epilogue no longer overlaps the next unit's MMAs: pairs
// paid at about 171 rows per expert and cost at 512 (measured), so they are
// used when the mean rows per expert is at most 192.  MOK_GEMM_GROUP and
// MOK_GEMM_PAIR (0/1) override (tuning knobs only: results do not change).
GemmTuning gemm_tuning(int rows, int E) {
    GemmTuning v{2, rows <= 192 * E ? 1 : 0, 3, 2, 1};
    if (const char* s = getenv("MOK_GEMM_GROUP")) v.group_chunks = atoi(s) < 1 ? 1 : atoi(s);
    if (const char* s = getenv("MOK_GEMM_PAIR")) {
        v.pair = atoi(s) != 0;
        v.gate_up_pair2 = 0;  // the explicit setting decides the gate/up unit shape too
    }
    if (const char* s = getenv("MOK_GEMM_CTA_PAIR")) v.cta_pair = atoi(s) < 0 ? 0 : atoi(s);
    if (const char* s = getenv("MOK_MX_RINGS")) v.mx_rings = atoi(s) == 1 ? 1 : 2;
    return v;
}

cudaError_t gemm_configure(int dev) {
    static bool done[64] = {};
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (done[dev]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm<Bf16Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Bf16Cfg::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_grouped_gemm<Bf16PairCfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Bf16PairCfg::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_grouped_gemm<MxCfg>, cudaFuncAttributeMaxDynamicSharedMemorySize, MxCfg::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_grouped_gemm<MxOneRingCfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 MxOneRingCfg::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_grouped_gemm<Bf16ExtCfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Bf16ExtCfg::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_grouped_gemm<Bf16ExtPairCfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Bf16ExtPairCfg::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_grouped_gemm_pair<Bf16Cta2Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Bf16Cta2Cfg::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_grouped_gemm_pair<Bf16Cta2ExtCfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Bf16Cta2ExtCfg::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k_grouped_gemm_pair<Bf16Cta2PairCfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Bf16Cta2PairCfg::SMEM);

    if (e == cudaSuccess) done[dev] = true;
    return e;
}

cudaError_t launch_gemm_phase(int phase, const GemmMaps& maps, const MxMaps* mx, const MxTokenScales* mxs,
                              const GemmShape& sh, const Chunk* chunks, const int* counts2, void* h_out, void* out,
                              const int32_t* row_slot, void* status, uint64_t timeout_ns, int grid,
                              const GemmTuning& tune, cudaStream_t stream, const BwdBuffers* bwd, int8_t* out_exp,
                              const PushDest* push, int push_slots) {
    if (mx && !mxs) return cudaErrorInvalidValue;
    if (push && push_slots <= 0) return cudaErrorInvalidValue;
    if (phase >= 2 && (mx || !bwd || !bwd->save_a || !bwd->save_b || !bwd->dab)) return cudaErrorInvalidValue;
    CoreArgs a{};
    if (bwd) {
        a.save_a = bwd->save_a;
        a.save_b = bwd->save_b;
        a.dab = bwd->dab;
    }
    if (mxs) {
        a.xsc = mxs->xsc;
        a.hsc = mxs->hsc;
        a.sc_rows = mxs->sc_rows;
    }
    a.H = sh.H;
    a.I = sh.I;
    a.h = h_out;
    a.out = out;
    a.out_exp = out_exp;
    if ((phase == 1 || phase == 3) && !mx && !out_exp && !push)
        return cudaErrorInvalidValue;  // fp16 slot rows need their exponents
    a.push = push;
    a.push_slots = push_slots;
    a.row_slot = row_slot;
    a.st = reinterpret_cast<DevStatus*>(status);
    a.timeout_ns = timeout_ns;
    const int tiles = phase == 0 ? sh.I / MT_G_FEATURES : phase == 2 ? sh.I / MT_D_FEATURES : sh.H / MT_D_FEATURES;
    // Pairs only for the bf16 gate/up launch.  MXFP8 keeps one tile per unit:
    // measured, pairs were 6-10 % slower there (a tall pair fills TMEM, and
    // its quantising epilogue then stalls the next unit's MMAs).  The down
    // launch's units are short (K = I), so that stall weighs more there:
    // pairs for gate/up only measured 3 % faster than pairs for both.  In
    // the backward's dh and dx launches pairs measured 2 % slower (two runs
    // each, one session).
    const bool pair = tune.pair && !mx && phase == 0;
    const int sub = pair ? 2 : 1;
    const int MT = (tiles + sub - 1) / sub;  // units along M
    const int GC = tune.group_chunks > 0 ? tune.group_chunks : 1;
    // CTA pairs (MOK_GEMM_CTA_PAIR): 0 none; 1 every bf16 launch but gate/up;
    // 2 all, one M tile per CTA; 3 (default) as 1, and gate/up on CTA pairs
    // of two M tiles per CTA (MOK_GEMM_PAIR=0 keeps gate/up on single CTAs
    // where the M-tile pairing rule does not hold).  Needs an even number of
    // M tiles (a multiple of 4 for two per CTA) and an even grid.  Measured
    // on B200 (ncu launch times or bench A/Bs, one session each): down on CTA
    // pairs 5 % faster than single tiles at the page shape and 1 % at the
    // zipf shape; gate/up on CTA pairs of one tile 4 % slower than M-tile
    // pairs (page) and 5 % slower than single tiles (zipf); gate/up on CTA
    // pairs of two tiles 3 % faster than M-tile pairs (page), 1-3 % faster
    // than single tiles at the zipf shape (512 rows per expert) and 1.5 % at
    // the Mixtral-shaped config (1024); down on CTA pairs of two tiles slower
    // than on CTA pairs of one (page).
    if (tune.cta_pair == 3 && phase == 0 && (pair || tune.gate_up_pair2) && !mx && !bwd && tiles % 4 == 0 &&
        grid >= 2)
        return launch_pair_phase<Bf16Cta2PairCfg>(grid, maps, a, chunks, counts2, phase, tiles / 4, GC, stream);
    const bool cta2 = tune.cta_pair == 2 || ((tune.cta_pair == 1 || tune.cta_pair == 3) && phase != 0);
    if (cta2 && !mx && tiles % 2 == 0 && grid >= 2) {
        if (phase >= 2)  // the backward's dh and dx phases
            return launch_pair_phase<Bf16Cta2ExtCfg>(grid, maps, a, chunks, counts2, phase, tiles / 2, GC, stream);
        if (!bwd)
            return launch_pair_phase<Bf16Cta2Cfg>(grid, maps, a, chunks, counts2, phase, tiles / 2, GC, stream);
    }
    if (mx) {
        if (tune.mx_rings == 1)
            k_grouped_gemm<MxOneRingCfg><<<grid, MxOneRingCfg::THREADS, MxOneRingCfg::SMEM, stream>>>(
                maps, *mx, a, chunks, counts2, phase, MT, GC);
        else
            k_grouped_gemm<MxCfg><<<grid, MxCfg::THREADS, MxCfg::SMEM, stream>>>(maps, *mx, a, chunks, counts2, phase,
                                                                                MT, GC);
    } else {
        MxMaps none;
        memset(&none, 0, sizeof none);
        // the backward phases and the forward that keeps a, b run the
        // instantiations with that code; the plain forward runs without it
        const bool ext = bwd != nullptr;
        if (pair && ext)
            k_grouped_gemm<Bf16ExtPairCfg><<<grid, Bf16ExtPairCfg::THREADS, Bf16ExtPairCfg::SMEM, stream>>>(
                maps, none, a, chunks, counts2, phase, MT, GC);
        else if (ext)
            k_grouped_gemm<Bf16ExtCfg><<<grid, Bf16ExtCfg::THREADS, Bf16ExtCfg::SMEM, stream>>>(
                maps, none, a, chunks, counts2, phase, MT, GC);
        else if (pair)
            k_grouped_gemm<Bf16PairCfg><<<grid, Bf16PairCfg::THREADS, Bf16PairCfg::SMEM, stream>>>(
                maps, none, a, chunks, counts2, phase, MT, GC);
        else
            k_grouped_gemm<Bf16Cfg><<<grid, Bf16Cfg::THREADS, Bf16Cfg::SMEM, stream>>>(maps, none, a, chunks,
                                                                                      counts2, phase, MT, GC);
    }
    return cudaGetLastError();
}

}  // namespace mok

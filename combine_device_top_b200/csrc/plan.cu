// plan.cu -- step 1 (router top-k, gates, histogram) and step 2 (pull
// schedule) of the forward MoE layer.
//
// MoK article (tahou.com), routing paragraph: the router sends every token
// to some experts; the system counts each expert's tokens, plans where they
// land and keeps one expert's tokens contiguous for the grouped GEMM.  MoK
// wiki summary, key points, schedule bullet: the pull schedule is a
// {src_rank, src_index} table built on the device with no sort and no
// CPU-GPU traffic.
//
// Four launches, all on the caller's stream, nothing read back:
//   k_topk    (one warp per token, every token in flight at once) top-k
//             over the E logits held in registers (k rounds of a warp
//             arg-max, ties to the lower index) and the softmax gates.
//   k_rank    (T/256 blocks) stable ranks of each token inside its block
//             per expert through shared-memory bit masks (one bit per token
//             of a 32-token warp tile) and per-block expert histograms.
//   k_scan    (1 block) per expert: exclusive prefix of the block
//             histograms, totals, the exclusive scan over experts ->
//             counts, offsets.
//   k_scatter (one thread per slot) row = offsets[e] + block prefix +
//             rank; writes the schedule, row_slot and pos.
// The row order inside an expert segment is ascending token index, which
// makes the schedule deterministic and independent of the launch shape.
#include "mok_device.cuh"
#include "mok_internal.h"
#include "topk.cuh"

namespace mok {

constexpr int PLAN_THREADS = 256;
constexpr int PLAN_WARPS = PLAN_THREADS / 32;
constexpr int PLAN_TOK = PLAN_WARPS * 32;  // tokens per block
constexpr int MAX_CHUNKS_PER_LANE = MOK_MAX_EXPERTS / 32;

// One warp per token (grid-stride over tokens).  NC: 32-expert chunks held
// per lane (ceil(E / 32) <= NC).
template <int NC>
__global__ void __launch_bounds__(PLAN_THREADS) k_topk(const float* __restrict__ logits, int T, int E, int k,
                                                       int32_t* __restrict__ topk_idx, float* __restrict__ gates) {
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * PLAN_WARPS;
    for (int t = blockIdx.x * PLAN_WARPS + (threadIdx.x >> 5); t < T; t += warps)
        warp_topk_token<NC>(logits + (size_t)t * E, E, k, lane, topk_idx + (size_t)t * k, gates + (size_t)t * k);
}

// dynamic smem: sel[PLAN_TOK][k] int32 | mask[PLAN_WARPS][E] uint32
__global__ void __launch_bounds__(PLAN_THREADS) k_rank(const int32_t* __restrict__ topk_idx, int T, int E, int k,
                                                       int32_t* __restrict__ blk_cnt, int32_t* __restrict__ rank_blk) {
    extern __shared__ __align__(16) unsigned char plan_smem[];
    int32_t* sel = reinterpret_cast<int32_t*>(plan_smem);
    uint32_t* mask = reinterpret_cast<uint32_t*>(sel + PLAN_TOK * k);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t_blk = blockIdx.x * PLAN_TOK;
    const int n_sel = min(PLAN_TOK, T - t_blk) * k;
    for (int i = threadIdx.x; i < n_sel; i += PLAN_THREADS) sel[i] = topk_idx[(size_t)t_blk * k + i];

    // ---- stable ranks inside the block, per expert
    uint32_t* my_mask = mask + warp * E;
    for (int e = lane; e < E; e += 32) my_mask[e] = 0u;
    __syncthreads();
    const int lt = warp * 32 + lane;
    const bool live = (t_blk + lt) < T;
    if (live)
        for (int j = 0; j < k; ++j) atomicOr(&my_mask[sel[lt * k + j]], 1u << lane);
    __syncthreads();
    if (live) {
        const uint32_t lower = (1u << lane) - 1u;
        for (int j = 0; j < k; ++j) {
            const int e = sel[lt * k + j];
            int r = __popc(my_mask[e] & lower);
            for (int w = 0; w < warp; ++w) r += __popc(mask[w * E + e]);
            rank_blk[(size_t)(t_blk + lt) * k + j] = r;
        }
    }
    for (int e = threadIdx.x; e < E; e += PLAN_THREADS) {
        int c = 0;
        for (int w = 0; w < PLAN_WARPS; ++w) c += __popc(mask[w * E + e]);
        blk_cnt[(size_t)blockIdx.x * E + e] = c;
    }
}

// One block: per-expert prefix over blocks (in place), counts, offsets.
__global__ void __launch_bounds__(1024) k_scan(int32_t* __restrict__ blk_cnt, int nb, int E, int n_slots,
                                               int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
    __shared__ int32_t warp_sums[32];
    const int e = threadIdx.x;  // E <= 1024
    int total = 0;
    if (e < E) {
        for (int b = 0; b < nb; ++b) {
            const int c = blk_cnt[(size_t)b * E + e];
            blk_cnt[(size_t)b * E + e] = total;
            total += c;
        }
        counts[e] = total;
    }
    // exclusive block scan of total over e
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = total;
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
        warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int excl = incl - total + (warp > 0 ? warp_sums[warp - 1] : 0);
    if (e < E) offsets[e] = excl;
    if (e == 0) offsets[E] = n_slots;
}

__global__ void __launch_bounds__(PLAN_THREADS) k_scatter(const int32_t* __restrict__ topk_idx,
                                                          const int32_t* __restrict__ rank_blk,
                                                          const int32_t* __restrict__ blk_pre,
                                                          const int32_t* __restrict__ offsets, int T, int E, int k,
                                                          int S_r, int32_t* __restrict__ src_rank,
                                                          int32_t* __restrict__ src_index,
                                                          int32_t* __restrict__ row_slot, int32_t* __restrict__ pos) {
    const int ns = T * k;
    for (int s = blockIdx.x * PLAN_THREADS + threadIdx.x; s < ns; s += gridDim.x * PLAN_THREADS) {
        const int t = s / k;
        const int e = topk_idx[s];
        const int row = offsets[e] + blk_pre[(size_t)(t / PLAN_TOK) * E + e] + rank_blk[s];
        src_rank[row] = t / S_r;
        src_index[row] = t - (t / S_r) * S_r;
        row_slot[row] = s;
        pos[s] = row;
    }
}

// ------------------------------------------------------------------ host side
size_t plan_layout(int T, int E, int k, PlanLayout* L) {
    const size_t ns = (size_t)T * k;
    const int nb = (T + PLAN_TOK - 1) / PLAN_TOK;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 255) & ~(size_t)255;
        return o;
    };
    PlanLayout l;
    l.nb = nb;
    l.status = take(64);  // device status word of the router kernel (mok_plan_router)
    l.counts = take(sizeof(int32_t) * E);
    l.offsets = take(sizeof(int32_t) * (E + 1));
    l.src_rank = take(sizeof(int32_t) * ns);
    l.src_index = take(sizeof(int32_t) * ns);
    l.row_slot = take(sizeof(int32_t) * ns);
    l.pos = take(sizeof(int32_t) * ns);
    l.topk = take(sizeof(int32_t) * ns);
    l.gates = take(sizeof(float) * ns);
    l.blk_cnt = take(sizeof(int32_t) * (size_t)nb * E);
    l.rank = take(sizeof(int32_t) * ns);
    l.total = off;
    if (L) *L = l;
    return off;
}

// Top-k launch: every token's warp resident at once where the GPU holds them.
static cudaError_t launch_topk(const float* logits, int T, int E, int k, int32_t* topk_idx, float* gates,
                               cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int want = (T + PLAN_WARPS - 1) / PLAN_WARPS;
    const int grid = want < sms * 8 ? want : sms * 8;
    const int nc = (E + 31) >> 5;
    if (nc <= 1) k_topk<1><<<grid, PLAN_THREADS, 0, stream>>>(logits, T, E, k, topk_idx, gates);
    else if (nc <= 2) k_topk<2><<<grid, PLAN_THREADS, 0, stream>>>(logits, T, E, k, topk_idx, gates);
    else if (nc <= 4) k_topk<4><<<grid, PLAN_THREADS, 0, stream>>>(logits, T, E, k, topk_idx, gates);
    else if (nc <= 8) k_topk<8><<<grid, PLAN_THREADS, 0, stream>>>(logits, T, E, k, topk_idx, gates);
    else if (nc <= 12) k_topk<12><<<grid, PLAN_THREADS, 0, stream>>>(logits, T, E, k, topk_idx, gates);
    else if (nc <= 16) k_topk<16><<<grid, PLAN_THREADS, 0, stream>>>(logits, T, E, k, topk_idx, gates);
    else k_topk<MAX_CHUNKS_PER_LANE><<<grid, PLAN_THREADS, 0, stream>>>(logits, T, E, k, topk_idx, gates);
    return cudaGetLastError();
}

static cudaError_t rank_configure() {
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_rank, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(sizeof(int32_t) * PLAN_TOK * MOK_MAX_TOPK +
                                                   sizeof(uint32_t) * PLAN_WARPS * MOK_MAX_EXPERTS));
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    return cudaSuccess;
}

cudaError_t launch_plan(const float* logits, int T, int E, int k, int R, unsigned char* ws, const PlanLayout& L,
                        cudaStream_t stream) {
    auto I32 = [&](size_t o) { return reinterpret_cast<int32_t*>(ws + o); };
    return launch_plan_parts(logits, T, E, k, R, I32(L.counts), I32(L.offsets), I32(L.src_rank), I32(L.src_index),
                             I32(L.row_slot), I32(L.pos), I32(L.topk), reinterpret_cast<float*>(ws + L.gates),
                             I32(L.blk_cnt), I32(L.rank), stream);
}

// The same launches with every array given explicitly (outputs and the two
// scratch arrays: blk_cnt [ceil(T/256), E] and rank [T*k]).
int plan_route_blocks(int T) { return (T + PLAN_TOK - 1) / PLAN_TOK; }

cudaError_t launch_plan_schedule(int T, int E, int k, int R, int32_t* counts, int32_t* offsets, int32_t* src_rank,
                                 int32_t* src_index, int32_t* row_slot, int32_t* pos, const int32_t* topk_idx,
                                 int32_t* blk_cnt, int32_t* rank, cudaStream_t stream) {
    cudaError_t e = rank_configure();
    if (e != cudaSuccess) return e;
    const size_t smem = sizeof(int32_t) * PLAN_TOK * k + sizeof(uint32_t) * PLAN_WARPS * E;
    const int nb = plan_route_blocks(T);
    if (T > 0) k_rank<<<nb, PLAN_THREADS, smem, stream>>>(topk_idx, T, E, k, blk_cnt, rank);
    k_scan<<<1, 1024, 0, stream>>>(blk_cnt, nb, E, T * k, counts, offsets);
    if (T > 0) {
        // one thread per slot
        const int blocks = (T * k + PLAN_THREADS - 1) / PLAN_THREADS;
        k_scatter<<<blocks < 4096 ? blocks : 4096, PLAN_THREADS, 0, stream>>>(
            topk_idx, rank, blk_cnt, offsets, T, E, k, T / R, src_rank, src_index, row_slot, pos);
    }
    return cudaGetLastError();
}

cudaError_t launch_plan_parts(const float* logits, int T, int E, int k, int R, int32_t* counts, int32_t* offsets,
                              int32_t* src_rank, int32_t* src_index, int32_t* row_slot, int32_t* pos,
                              int32_t* topk_idx, float* gates, int32_t* blk_cnt, int32_t* rank,
                              cudaStream_t stream) {
    cudaError_t e = rank_configure();
    if (e != cudaSuccess) return e;
    if ((e = launch_topk(logits, T, E, k, topk_idx, gates, stream)) != cudaSuccess) return e;
    return launch_plan_schedule(T, E, k, R, counts, offsets, src_rank, src_index, row_slot, pos, topk_idx, blk_cnt,
                                rank, stream);
}

}  // namespace mok

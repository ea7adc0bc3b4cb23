// worklist.cu -- the device-built work list of the grouped GEMM: minibatch
// boundaries over the expert-major rows and chunks of at most max_rows (256,
// or 224 on the MXFP8 path) rows of one expert inside one minibatch.  Built
// from `offsets` on the device, so the forward needs no host round trip (MoK
// wiki summary, key points: schedule built on the device without CPU-GPU
// traffic; MoK article, minibatch paragraph: a minibatch is the unit handed
// to the expert computation).
#include "mok_device.cuh"
#include "mok_internal.h"

namespace mok {

// ------------------------------------------------------------------ work list
// One block.  Minibatch boundaries: from row b0, walk the expert boundaries
// until the minibatch holds at least M rows AND at least min_units gate/up
// units (chunks x units per chunk: two full waves of the GEMM CTAs is the
// pages' rule), but never more than `cap` rows (one ring half); then every
// (expert, minibatch) piece is cut into ceil(len / maxr) chunks of nearly
// equal size (multiples of 16 rows except the last; maxr is a multiple of 16).
__device__ __forceinline__ int piece_chunks(int L, int maxr) { return (L + maxr - 1) / maxr; }
__device__ __forceinline__ int piece_base(int L, int maxr) {
    const int n = piece_chunks(L, maxr);
    int base = (((L + n - 1) / n) + 15) & ~15;
    if ((n - 1) * base >= L) base = maxr;
    return base;
}

__global__ void __launch_bounds__(1024) k_build_chunks(const int32_t* __restrict__ offsets, int E, int n_slots,
                                                       int M, int cap, int maxr, int min_units, int upc,
                                                       Chunk* __restrict__ chunks, int max_chunks,
                                                       Minibatch* __restrict__ mbs, int max_mb,
                                                       int* __restrict__ counts2, DevStatus* st) {
    __shared__ int s_nmb;
    __shared__ int warp_sums[32];
    __shared__ int s_off[1025];  // offsets[0..E] (E <= 1024): the serial walk below reads shared memory
    for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = offsets[i];
    __syncthreads();
    if (threadIdx.x == 0) {
        // the rows end at offsets[E]; n_slots bounds it (under expert
        // parallelism a rank's share of the rows is known on the device only)
        const int n_end = min(n_slots, s_off[E]);
        int b0 = 0, n = 0, e = 0;
        while (b0 < n_end) {
            while (e < E - 1 && s_off[e + 1] <= b0) ++e;  // expert holding row b0
            const int limit = min(n_end, b0 + cap);
            int b = b0, units = 0, ee = e;
            while (true) {
                const int end = min(s_off[ee + 1], limit);
                units += piece_chunks(end - b, maxr) * upc;
                b = end;
                if (b >= limit || (b >= b0 + M && units >= min_units) || ee == E - 1) break;
                ++ee;
            }
            if (n >= max_mb) {
                set_status(st, MOK_ERR_CAPACITY, 1, n, max_mb);
                break;
            }
            mbs[n] = Minibatch{b0, b, 0, 0};
            ++n;
            b0 = b;
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
                if (L > 0) cnt += piece_chunks(L, maxr);
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
            const int n = piece_chunks(L, maxr), base = piece_base(L, maxr);
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

int two_wave_rows(int I, int gemm_ctas, int waves, int tile_rows, int tile_features) {
    if (I <= 0 || gemm_ctas <= 0 || waves <= 0 || tile_rows <= 0 || tile_features <= 0) return 0;
    const long long num = (long long)waves * gemm_ctas * tile_rows * tile_features;
    const long long den = 2LL * I;
    return (int)((num + den - 1) / den);
}
// bound for every chunk height cap >= CHUNK_MAX_ROWS_MX
int max_chunks(int n_slots, int E, int n_mb) { return n_slots / CHUNK_MAX_ROWS_MX + E + n_mb + 2; }

cudaError_t launch_build_chunks(const int32_t* offsets, int E, int n_slots, int minibatch, int cap, int max_rows,
                                int min_units, int units_per_chunk, Chunk* chunks, int max_ch, Minibatch* mbs,
                                int max_mb, int* counts2, void* status, cudaStream_t stream) {
    if (max_rows < CHUNK_MAX_ROWS_MX || max_rows > CHUNK_MAX_ROWS || max_rows % 16) return cudaErrorInvalidValue;
    if (units_per_chunk < 1) return cudaErrorInvalidValue;
    k_build_chunks<<<1, 1024, 0, stream>>>(offsets, E, n_slots, minibatch, cap, max_rows, min_units, units_per_chunk,
                                           chunks, max_ch, mbs, max_mb, counts2, reinterpret_cast<DevStatus*>(status));
    return cudaGetLastError();
}

}  // namespace mok

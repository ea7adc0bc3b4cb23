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
// One block.  Minibatch boundaries: from row b0, the first expert boundary at
// or after b0 + minibatch, but never more than `cap` rows; then every
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
                                                       int M, int cap, int maxr, Chunk* __restrict__ chunks,
                                                       int max_chunks,
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
// bound for every chunk height cap >= CHUNK_MAX_ROWS_MX
int max_chunks(int n_slots, int E, int n_mb) { return n_slots / CHUNK_MAX_ROWS_MX + E + n_mb + 2; }

cudaError_t launch_build_chunks(const int32_t* offsets, int E, int n_slots, int minibatch, int cap, int max_rows,
                                Chunk* chunks, int max_ch, Minibatch* mbs, int max_mb, int* counts2, void* status,
                                cudaStream_t stream) {
    if (max_rows < CHUNK_MAX_ROWS_MX || max_rows > CHUNK_MAX_ROWS || max_rows % 16) return cudaErrorInvalidValue;
    k_build_chunks<<<1, 1024, 0, stream>>>(offsets, E, n_slots, minibatch, cap, max_rows, chunks, max_ch, mbs, max_mb,
                                           counts2, reinterpret_cast<DevStatus*>(status));
    return cudaGetLastError();
}

}  // namespace mok

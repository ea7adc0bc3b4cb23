// dispatch_combine.cu -- step 3 (pull dispatch / gather) and step 5
// (weighted combine) of the forward MoE layer as standalone kernels.  The
// warp bodies are in dispatch_combine.cuh.
//
// Both kernels are HBM-bound streams of 16-byte vectors: one warp per token,
// a grid of a few CTAs per SM looping over the tokens.  The gather reads each
// token once and writes it to its k rows (T*H*2 bytes in, N_s*H*2 out); the
// combine reads the per-slot outputs (N_s*H*2 bytes of fp16 plus N_s*H/128
// exponents on the bf16 path, N_s*H*2 of bf16 on the MXFP8 path) and writes
// T*H*2 bytes of bf16 y, rounding once.
#include "dispatch_combine.cuh"
#include "mok_internal.h"
#include "mxfp8.cuh"

namespace mok {

constexpr int DC_THREADS = 256;

// Token-major form of the same copy: one warp per token reads the token's
// row once and writes it to each of its k rows (pos[t*k + j]).  Every source
// row is read from HBM once instead of k times (with 940 MB of rows streaming
// out, x does not stay in L2 between its k reads).
__global__ void __launch_bounds__(DC_THREADS) k_gather_tokens(ShardsIn xs, int S_r, int H, int T, int k,
                                                              const int32_t* __restrict__ pos,
                                                              uint4* __restrict__ rows) {
    const int lane = threadIdx.x & 31;
    const int nvec = H >> 3;
    const int warps = gridDim.x * (DC_THREADS / 32);
    for (int t = blockIdx.x * (DC_THREADS / 32) + (threadIdx.x >> 5); t < T; t += warps) {
        const int r = t / S_r;
        const uint4* src = reinterpret_cast<const uint4*>(xs.p[r]) + (size_t)(t - r * S_r) * nvec;
        const int my_row = lane < k ? __ldg(pos + (size_t)t * k + lane) : 0;
        int v0 = 0;
        for (; v0 + 128 <= nvec; v0 += 128) {  // warp-uniform trip count
            const int v = v0 + lane;
            const uint4 a = __ldg(src + v), b = __ldg(src + v + 32), c = __ldg(src + v + 64), d = __ldg(src + v + 96);
            for (int j = 0; j < k; ++j) {
                uint4* dst = rows + (size_t)__shfl_sync(0xffffffffu, my_row, j) * nvec;
                dst[v] = a;
                dst[v + 32] = b;
                dst[v + 64] = c;
                dst[v + 96] = d;
            }
        }
        // tail: lanes may differ in trip count, so no warp collectives here
        for (int v = v0 + lane; v < nvec; v += 32) {
            const uint4 a = __ldg(src + v);
            for (int j = 0; j < k; ++j) rows[(size_t)__ldg(pos + (size_t)t * k + j) * nvec + v] = a;
        }
    }
}

// The same copy with MXFP8 quantisation fused in (MoK article: activation
// quantisation inside the dispatch): each 32-element block of the token row
// is quantised to E4M3 with its E8M0 scale; the k rows receive the E4M3
// bytes and the scale planes [H/128][sc_rows][4] the block scales (plane g,
// byte b: block 4g + b), the operand form of the block-scaled MMA.
// Each lane owns 8 consecutive elements, 4 lanes a block, a half-warp one
// 4-block scale word (warp_mx_quant8); the step loop is warp-uniform (lanes
// past the end join the shuffles with zeros).  Four 256-element steps'
// loads are in flight per lane before the first is quantised.
__global__ void __launch_bounds__(DC_THREADS) k_gather_tokens_mx(ShardsIn xs, int S_r, int H, int T, int k,
                                                                 const int32_t* __restrict__ pos,
                                                                 uint8_t* __restrict__ rows, uint8_t* __restrict__ xsc,
                                                                 int sc_rows) {
    const int lane = threadIdx.x & 31;
    const int nvec = H >> 3;
    const int warps = gridDim.x * (DC_THREADS / 32);
    for (int t = blockIdx.x * (DC_THREADS / 32) + (threadIdx.x >> 5); t < T; t += warps) {
        const int r = t / S_r;
        const uint4* src = reinterpret_cast<const uint4*>(xs.p[r]) + (size_t)(t - r * S_r) * nvec;
        const int my_row = lane < k ? __ldg(pos + (size_t)t * k + lane) : 0;
        for (int c00 = 0; c00 < H; c00 += 1024) {
            uint4 raw[4];
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) {
                const int c = c00 + 256 * s4 + lane * 8;
                raw[s4] = c < H ? __ldg(src + (c >> 3)) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) {
                const int c0 = c00 + 256 * s4;
                if (c0 >= H) break;  // warp-uniform
                const int c = c0 + lane * 8;
                const bool live = c < H;
                uint2 q;
                uint32_t word;
                warp_mx_quant8(raw[s4], q, word, lane);
                uint32_t* plane = reinterpret_cast<uint32_t*>(xsc) + (size_t)((c0 >> 7) + (lane >> 4)) * sc_rows;
                for (int j = 0; j < k; ++j) {
                    const int row = __shfl_sync(0xffffffffu, my_row, j);
                    if (live) {
                        *reinterpret_cast<uint2*>(rows + (size_t)row * H + c) = q;
                        if ((lane & 15) == 0) plane[row] = word;
                    }
                }
            }
        }
    }
}

cudaError_t launch_gather_mx(const ShardsIn& xs, int S_r, int H, int T, int k, const int32_t* pos, void* rows,
                             void* xsc, int sc_rows, int num_sms, cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    const int want = (T + (DC_THREADS / 32) - 1) / (DC_THREADS / 32);
    const int grid = want < num_sms * 8 ? want : num_sms * 8;
    k_gather_tokens_mx<<<grid, DC_THREADS, 0, stream>>>(xs, S_r, H, T, k, pos, reinterpret_cast<uint8_t*>(rows),
                                                         reinterpret_cast<uint8_t*>(xsc), sc_rows);
    return cudaGetLastError();
}

template <int KMAX, class S>
__global__ void __launch_bounds__(DC_THREADS) k_combine(SlotSrc src, const float* __restrict__ gates, int T, int k,
                                                        int H, int S_r, ShardsOut ys) {
    const int lane = threadIdx.x & 31;
    const int nvec = H >> 3;
    const int warps = gridDim.x * (DC_THREADS / 32);
    for (int t = blockIdx.x * (DC_THREADS / 32) + (threadIdx.x >> 5); t < T; t += warps) {
        const int r = t / S_r;
        uint4* dst = reinterpret_cast<uint4*>(ys.p[r]) + (size_t)(t - r * S_r) * nvec;
        warp_combine_token<KMAX, S>(src, gates, t, k, nvec, dst, lane);
    }
}

cudaError_t launch_gather(const ShardsIn& xs, int S_r, int H, int T, int k, const int32_t* pos, void* rows,
                          int num_sms, cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    const int want = (T + (DC_THREADS / 32) - 1) / (DC_THREADS / 32);
    const int grid = want < num_sms * 8 ? want : num_sms * 8;
    k_gather_tokens<<<grid, DC_THREADS, 0, stream>>>(xs, S_r, H, T, k, pos, reinterpret_cast<uint4*>(rows));
    return cudaGetLastError();
}

template <class S>
static void launch_combine_t(const SlotSrc& src, const float* gates, int T, int k, int H, int S_r,
                             const ShardsOut& ys, int grid, cudaStream_t stream) {
    // KB slots' loads in flight per lane: all of them up to 8; k > 8 takes
    // several rounds
    if (k <= 2)
        k_combine<2, S><<<grid, DC_THREADS, 0, stream>>>(src, gates, T, k, H, S_r, ys);
    else if (k <= 4)
        k_combine<4, S><<<grid, DC_THREADS, 0, stream>>>(src, gates, T, k, H, S_r, ys);
    else
        k_combine<8, S><<<grid, DC_THREADS, 0, stream>>>(src, gates, T, k, H, S_r, ys);
}

cudaError_t launch_combine(const void* out, int slot_type, const float* gates, int T, int k, int H, int S_r,
                           const ShardsOut& ys, int num_sms, cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    const int want = (T + (DC_THREADS / 32) - 1) / (DC_THREADS / 32);
    const int grid = want < num_sms * 8 ? want : num_sms * 8;
    SlotSrc src{out, nullptr};
    if (slot_type == MOK_SLOTS_F16S) {
        src.exps = reinterpret_cast<const int8_t*>(out) + slot_exp_offset(T * k, H);
        launch_combine_t<SlotF16S>(src, gates, T, k, H, S_r, ys, grid, stream);
    } else if (slot_type == MOK_SLOTS_BF16) {
        launch_combine_t<SlotBf16>(src, gates, T, k, H, S_r, ys, grid, stream);
    } else {
        launch_combine_t<SlotF32>(src, gates, T, k, H, S_r, ys, grid, stream);
    }
    return cudaGetLastError();
}

}  // namespace mok

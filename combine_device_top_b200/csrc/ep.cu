// ep.cu -- expert parallelism over G GPUs, one process per GPU: the forward
// layer with the source ranks on other GPUs instead of shards of one HBM.
//
// MoK article (tahou.com), pull-dispatch paragraph: the rank that owns an
// expert pulls that expert's tokens from the source ranks' memory, knowing
// only {src_rank, src_index}; push-combine paragraph: each expert output
// goes back to its token's rank, which merges the k results locally.  MoK
// wiki summary, key points: NVLink loads and stores issued from inside the
// kernels, no collective library on the data path.
//
// Every rank holds the same plan (built from the all-gathered logits), owns
// the experts [e0, e0 + e_loc) and reaches the other ranks' token shards and
// slot buffers through peer pointers (CUDA IPC over NVLink / NVSwitch).  A
// step on rank g:
//   k_ep_setup    this rank's expert offsets (rows relative to its first
//                 row) and the device copy of the slot-buffer pointers;
//   k_ep_pull     pull dispatch: its experts' rows, each read from the
//                 source rank's x (16-byte loads over NVLink) into a local
//                 expert-major buffer (k_ep_pull_mx on the MXFP8 path:
//                 quantised to E4M3 rows and block scales on the way);
//   the grouped GEMM of the single-GPU path over those rows, whose down
//                 epilogue stores every slot row into the source rank's slot
//                 buffer (the push);
//   k_ep_barrier  every rank's pushes have landed;
//   the combine   over its own tokens' slot rows, from local memory.
#include "dispatch_combine.cuh"
#include "mok_device.cuh"
#include "mok_internal.h"

namespace mok {

constexpr int EP_THREADS = 256;

// offsets_loc[i] = offsets[e0 + i] - offsets[e0] for i <= e_loc, and the
// device copy of the push destinations.  One block.
__global__ void k_ep_setup(const __grid_constant__ PushDest push, PushDest* __restrict__ push_dev,
                           const int32_t* __restrict__ offsets, int e0, int e_loc, int32_t* __restrict__ offsets_loc) {
    const int r0 = offsets[e0];
    for (int i = threadIdx.x; i <= e_loc; i += blockDim.x) offsets_loc[i] = offsets[e0 + i] - r0;
    for (int i = threadIdx.x; i < MOK_MAX_SHARDS; i += blockDim.x) {
        push_dev->out[i] = push.out[i];
        push_dev->exp[i] = push.exp[i];
    }
}

// Pull dispatch of this rank's rows: for i < n = offsets[e0 + e_loc] -
// offsets[e0] (row = offsets[e0] + i),
//   rows[i]         = x[src_rank[row]][src_index[row]]   (H bf16)
//   row_slot_loc[i] = row_slot[row].
// One warp per row; four 16-byte loads per lane in flight (4 CTAs of 8 warps
// per SM: 64 KB in flight per SM).  The source is a peer GPU's shard
// (NVLink) or this GPU's own; it is not written while the kernel runs, so
// the read-only path is used.
__global__ void __launch_bounds__(EP_THREADS, 4)
    k_ep_pull(const __grid_constant__ ShardsIn xs, int H, const int32_t* __restrict__ offsets, int e0, int e_loc,
              const int32_t* __restrict__ src_rank, const int32_t* __restrict__ src_index,
              const int32_t* __restrict__ row_slot, uint4* __restrict__ rows, int32_t* __restrict__ row_slot_loc) {
    const int r0 = __ldg(offsets + e0);
    const int n = __ldg(offsets + e0 + e_loc) - r0;
    const int lane = threadIdx.x & 31;
    const int nvec = H >> 3;
    const int warps = gridDim.x * (EP_THREADS / 32);
    for (int i = blockIdx.x * (EP_THREADS / 32) + (threadIdx.x >> 5); i < n; i += warps) {
        const int row = r0 + i;
        const uint4* src = reinterpret_cast<const uint4*>(xs.p[__ldg(src_rank + row)]) +
                           (size_t)__ldg(src_index + row) * nvec;
        uint4* dst = rows + (size_t)i * nvec;
        if (lane == 0) row_slot_loc[i] = __ldg(row_slot + row);
        int v0 = 0;
        for (; v0 + 128 <= nvec; v0 += 128) {
            const int v = v0 + lane;
            const uint4 a = __ldg(src + v), b = __ldg(src + v + 32), c = __ldg(src + v + 64), d = __ldg(src + v + 96);
            dst[v] = a;
            dst[v + 32] = b;
            dst[v + 64] = c;
            dst[v + 96] = d;
        }
        for (int v = v0 + lane; v < nvec; v += 32) dst[v] = __ldg(src + v);
    }
}

// The MXFP8 pull: as k_ep_pull, each row quantised on the way (32-element
// blocks, OCP MX): rows_q[i] the E4M3 bytes, the scale planes [H/128]
// [sc_rows][4] at row i.  A warp per row, four 256-element steps' loads in
// flight per lane.  H % 128 == 0.
__global__ void __launch_bounds__(EP_THREADS, 4)
    k_ep_pull_mx(const __grid_constant__ ShardsIn xs, int H, const int32_t* __restrict__ offsets, int e0, int e_loc,
                 const int32_t* __restrict__ src_rank, const int32_t* __restrict__ src_index,
                 const int32_t* __restrict__ row_slot, uint8_t* __restrict__ rows_q, uint8_t* __restrict__ xsc,
                 int sc_rows, int32_t* __restrict__ row_slot_loc) {
    const int r0 = __ldg(offsets + e0);
    const int n = __ldg(offsets + e0 + e_loc) - r0;
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (EP_THREADS / 32);
    uint32_t* planes = reinterpret_cast<uint32_t*>(xsc);
    for (int i = blockIdx.x * (EP_THREADS / 32) + (threadIdx.x >> 5); i < n; i += warps) {
        const int row = r0 + i;
        const uint4* src = reinterpret_cast<const uint4*>(xs.p[__ldg(src_rank + row)]) +
                           (size_t)__ldg(src_index + row) * (H >> 3);
        uint8_t* dst = rows_q + (size_t)i * H;
        if (lane == 0) row_slot_loc[i] = __ldg(row_slot + row);
        for (int c0 = 0; c0 < H; c0 += 1024) {
            uint4 raw[4];
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) {
                const int c = c0 + 256 * s4 + lane * 8;
                raw[s4] = c < H ? __ldg(src + (c >> 3)) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) {
                const int cs = c0 + 256 * s4;
                if (cs >= H) break;  // warp-uniform
                uint2 q;
                uint32_t word;
                warp_mx_quant8(raw[s4], q, word, lane);
                const int c = cs + lane * 8;
                if (c < H) {
                    *reinterpret_cast<uint2*>(dst + c) = q;
                    if ((lane & 15) == 0) planes[(size_t)((cs >> 7) + (lane >> 4)) * sc_rows + i] = word;
                }
            }
        }
    }
}

__device__ __forceinline__ void red_add_release_sys(uint32_t* p, uint32_t v) {
    asm volatile("red.release.sys.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// The group barrier: counters.p[h] is rank h's arrival counter as this GPU
// addresses it.  One thread makes this GPU's earlier writes (the previous
// kernels' pushes into peer slot buffers) visible at system scope, adds one
// to every rank's counter (release), then waits until its own counter
// reaches `target` = epoch * G (acquire): every rank has arrived `epoch`
// times.  The wait is bounded by timeout_ns (then MOK_ERR_TIMEOUT, where
// 201, aux = target and the count seen) and never spins forever.
__global__ void k_ep_barrier(ShardsOut counters, int G, int g, uint32_t target, DevStatus* st, uint64_t timeout_ns) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    __threadfence_system();
    for (int h = 0; h < G; ++h) red_add_release_sys(reinterpret_cast<uint32_t*>(counters.p[h]), 1u);
    const uint32_t* mine = reinterpret_cast<const uint32_t*>(counters.p[g]);
    const uint64_t t0 = globaltimer();
    uint32_t v;
    while ((int32_t)((v = ld_acquire_sys(mine)) - target) < 0) {
        if (globaltimer() - t0 > timeout_ns) {
            set_status(st, MOK_ERR_TIMEOUT, 201, (int)target, (int)v);
            break;
        }
        __nanosleep(64);
    }
    __threadfence_system();
}

cudaError_t launch_ep_setup(const PushDest& push, PushDest* push_dev, const int32_t* offsets, int e0, int e_loc,
                            int32_t* offsets_loc, cudaStream_t stream) {
    k_ep_setup<<<1, 256, 0, stream>>>(push, push_dev, offsets, e0, e_loc, offsets_loc);
    return cudaGetLastError();
}

cudaError_t launch_ep_pull(const ShardsIn& xs, int H, const int32_t* offsets, int e0, int e_loc,
                           const int32_t* src_rank, const int32_t* src_index, const int32_t* row_slot, void* rows,
                           int32_t* row_slot_loc, int max_rows, int num_sms, cudaStream_t stream) {
    if (max_rows <= 0) return cudaSuccess;
    const int want = (max_rows + (EP_THREADS / 32) - 1) / (EP_THREADS / 32);
    const int grid = want < num_sms * 4 ? want : num_sms * 4;
    k_ep_pull<<<grid, EP_THREADS, 0, stream>>>(xs, H, offsets, e0, e_loc, src_rank, src_index, row_slot,
                                               reinterpret_cast<uint4*>(rows), row_slot_loc);
    return cudaGetLastError();
}

cudaError_t launch_ep_pull_mx(const ShardsIn& xs, int H, const int32_t* offsets, int e0, int e_loc,
                              const int32_t* src_rank, const int32_t* src_index, const int32_t* row_slot,
                              void* rows_q, void* xsc, int sc_rows, int32_t* row_slot_loc, int max_rows, int num_sms,
                              cudaStream_t stream) {
    if (max_rows <= 0) return cudaSuccess;
    const int want = (max_rows + (EP_THREADS / 32) - 1) / (EP_THREADS / 32);
    const int grid = want < num_sms * 4 ? want : num_sms * 4;
    k_ep_pull_mx<<<grid, EP_THREADS, 0, stream>>>(xs, H, offsets, e0, e_loc, src_rank, src_index, row_slot,
                                                  reinterpret_cast<uint8_t*>(rows_q), reinterpret_cast<uint8_t*>(xsc),
                                                  sc_rows, row_slot_loc);
    return cudaGetLastError();
}

cudaError_t launch_ep_barrier(const ShardsOut& counters, int G, int g, uint32_t target, void* status,
                              uint64_t timeout_ns, cudaStream_t stream) {
    k_ep_barrier<<<1, 32, 0, stream>>>(counters, G, g, target, reinterpret_cast<DevStatus*>(status), timeout_ns);
    return cudaGetLastError();
}

}  // namespace mok

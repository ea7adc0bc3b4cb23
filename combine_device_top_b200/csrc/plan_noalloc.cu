// plan_noalloc.cu -- mok_plan_noalloc: the plan (router top-k, gates,
// histogram, pull schedule) for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they need a plan:
// code running inside a stream capture (allocation there is not allowed),
// an allocator-less runtime that hands out only pre-registered buffers, or
// a framework hook that must not touch the device allocator.  They can still
// provide the plan's outputs, but not the workspace mok_plan needs for its
// internal scratch (per-block expert histograms and in-block ranks).  This
// entry point keeps that scratch in a file-scope device array instead.
//
// The array is part of the library image: every GPU that loads the library
// holds MOK_PLAN_NOALLOC_SCRATCH_BYTES of it until the process exits.  Its
// device address is looked up once per device (cudaGetSymbolAddress, with
// that device current) on the first call made on that device; make that
// first call before any stream capture.  All calls on a device share the
// array, so calls whose kernels overlap on the GPU (different streams
// without ordering between them) race on it.  Each call writes every
// scratch entry it later reads, so nothing has to start at zero and the
// contents left by the previous call are never used.
#include <mutex>

#include "mok_device.cuh"
#include "mok_internal.h"

namespace mok {

static __device__ __align__(256) unsigned char g_plan_scratch[MOK_PLAN_NOALLOC_SCRATCH_BYTES];

static size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }

// Device address of g_plan_scratch for the current device (nullptr on failure).
static unsigned char* scratch_address(cudaError_t* err) {
    static std::mutex mu;
    static void* addr[64] = {};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_plan_scratch);
        if (*err != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return static_cast<unsigned char*>(addr[dev]);
}

}  // namespace mok

using namespace mok;

extern "C" int mok_plan_noalloc(const float* logits, int T, int E, int top_k, int R, int32_t* counts,
                                int32_t* offsets, int32_t* sched_src_rank, int32_t* sched_src_index,
                                int32_t* row_slot, int32_t* pos, int32_t* topk_idx, float* gates,
                                mok_stream_t stream) {
    if (T < 0 || E <= 0 || top_k <= 0 || R <= 0)
        return report_error(MOK_ERR_INVALID_ARG, "T, E, top_k, R out of range");
    if (E > MOK_MAX_EXPERTS) return report_error(MOK_ERR_UNSUPPORTED, "E above MOK_MAX_EXPERTS");
    if (top_k > E) return report_error(MOK_ERR_INVALID_ARG, "top_k > E");
    if (top_k > MOK_MAX_TOPK) return report_error(MOK_ERR_UNSUPPORTED, "top_k above MOK_MAX_TOPK");
    if (R > MOK_MAX_SHARDS) return report_error(MOK_ERR_UNSUPPORTED, "R above MOK_MAX_SHARDS");
    if (T % R) return report_error(MOK_ERR_UNSUPPORTED, "T % R != 0");
    if (!counts || !offsets)
        return report_error(MOK_ERR_INVALID_ARG, "NULL output pointer");
    if (T > 0 && (!logits || !sched_src_rank || !sched_src_index || !row_slot || !pos || !topk_idx || !gates))
        return report_error(MOK_ERR_INVALID_ARG, "NULL input or output pointer");
    const size_t ns = (size_t)T * (size_t)top_k;
    const size_t rank_bytes = round256(sizeof(int32_t) * ns);
    const size_t cnt_bytes = round256(sizeof(int32_t) * (size_t)plan_route_blocks(T) * (size_t)E);
    if (rank_bytes + cnt_bytes > (size_t)MOK_PLAN_NOALLOC_SCRATCH_BYTES)
        return report_error(MOK_ERR_UNSUPPORTED,
                            "mok_plan_noalloc: shape needs more than MOK_PLAN_NOALLOC_SCRATCH_BYTES of scratch "
                            "(4*T*k + 4*ceil(T/256)*E bytes); use mok_plan with a workspace");
    cudaError_t err = cudaSuccess;
    unsigned char* base = scratch_address(&err);
    if (base == nullptr) return report_error(MOK_ERR_CUDA, cudaGetErrorString(err));
    int32_t* rank = reinterpret_cast<int32_t*>(base);
    int32_t* blk_cnt = reinterpret_cast<int32_t*>(base + rank_bytes);
    err = launch_plan_parts(logits, T, E, top_k, R, counts, offsets, sched_src_rank, sched_src_index, row_slot, pos,
                            topk_idx, gates, blk_cnt, rank, reinterpret_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return report_error(MOK_ERR_CUDA, cudaGetErrorString(err));
    return MOK_OK;
}

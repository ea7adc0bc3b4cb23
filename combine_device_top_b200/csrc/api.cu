// api.cu -- the C ABI declared in include/mok.h: argument validation,
// workspace layout, tensor-map encoding and kernel launches.  No device
// memory is allocated here; every buffer lives in a caller-provided
// workspace.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "mok_device.cuh"
#include "mok_internal.h"

namespace mok {

// ------------------------------------------------------------------ errors
static thread_local std::string g_err = "no error";

static int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int report_error(int code, const char* msg) { return fail(code, "%s", msg); }

static int cuda_fail(cudaError_t e, const char* what) {
    return fail(MOK_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

#define MOK_CUDA(call, what)                       \
    do {                                           \
        cudaError_t e_ = (call);                   \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

static int device_sms(int* dev_out) {
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    if (sms[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
        sms[dev] = v;
    }
    if (dev_out) *dev_out = dev;
    return sms[dev];
}

// ------------------------------------------------------------------ tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                         uint32_t box_outer, const char** err) {
    auto enc = get_encode();
    if (!enc) {
        *err = "cuTensorMapEncodeTiled unavailable";
        return false;
    }
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *err = "cuTensorMapEncodeTiled failed";
        return false;
    }
    return true;
}

bool encode_bmaps(BMaps* maps, const void* base, uint64_t inner, uint64_t rows, const char** err, int step) {
    for (int i = 0; i < B_MAPS; ++i)
        if (!encode_tmap_2d_bf16(&maps->m[i], base, inner, rows, 64, (uint32_t)(step * (i + 1)), err))
            return false;
    return true;
}

// {64, rows, cols / 64} view of a row-major [rows, cols] bf16 array (strides
// {cols * 2, 128} bytes): a {64, box_rows, box_blocks} box is box_blocks
// consecutive 64-column blocks of box_rows rows, 128-byte swizzle, each block
// the MN-major operand layout of the MMA.
bool encode_cols3d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
                        uint32_t box_blocks, const char** err) {
    auto enc = get_encode();
    if (!enc) {
        *err = "cuTensorMapEncodeTiled unavailable";
        return false;
    }
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, box_rows, box_blocks};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        *err = "cuTensorMapEncodeTiled failed (3D column blocks)";
        return false;
    }
    return true;
}

// Wd viewed as {64 (columns inside a 64-wide block), E*I (rows), H/64 (column
// blocks)} with strides {H*2, 128} bytes: a {64, 64, 2} box is the MMA's
// two-atom MN-major tile of a 128-column down unit, in one TMA op.
static bool encode_wd3(CUtensorMap* map, const void* wd, int H, int I, int E) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {64, (cuuint64_t)E * I, (cuuint64_t)H / 64};
    cuuint64_t strides[2] = {(cuuint64_t)H * 2, 128};
    cuuint32_t box[3] = {64, 64, 2};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(wd), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_gemm_maps(GemmMaps* m, const void* wg, const void* wu, const void* wd, const void* rows, const void* h,
                      int H, int I, int E, int buf_rows, const char** err) {
    m->has_wd3 = encode_wd3(&m->wd3, wd, H, I, E) ? 1 : 0;
    return encode_tmap_2d_bf16(&m->wg, wg, (uint64_t)I, (uint64_t)E * H, 64, 64, err) &&
           encode_tmap_2d_bf16(&m->wu, wu, (uint64_t)I, (uint64_t)E * H, 64, 64, err) &&
           encode_tmap_2d_bf16(&m->wd, wd, (uint64_t)H, (uint64_t)E * I, 64, 64, err) &&
           encode_bmaps(&m->rows, rows, (uint64_t)H, (uint64_t)buf_rows, err) &&
           encode_bmaps(&m->h, h, (uint64_t)I, (uint64_t)buf_rows, err) &&
           encode_bmaps(&m->rows2, rows, (uint64_t)H, (uint64_t)buf_rows, err, 8) &&
           encode_bmaps(&m->h2, h, (uint64_t)I, (uint64_t)buf_rows, err, 8);
}

// 2D map of a row-major [outer, inner] byte array.
static bool encode_2d_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                         uint32_t box_outer, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_mx_maps(MxMaps* m, const mok_mxfp8_weights& w, int H, int I, int E, const char** err) {
    const bool ok =
        encode_2d_u8(&m->gq, w.gate, (uint64_t)I, (uint64_t)E * H, 64, 128, CU_TENSOR_MAP_SWIZZLE_64B) &&
        encode_2d_u8(&m->uq, w.up, (uint64_t)I, (uint64_t)E * H, 64, 128, CU_TENSOR_MAP_SWIZZLE_64B) &&
        encode_2d_u8(&m->dq, w.down, (uint64_t)H, (uint64_t)E * I, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_2d_u8(&m->gs, w.gate_scales, (uint64_t)I, (uint64_t)E * H / 32, 64, 4) &&
        encode_2d_u8(&m->us, w.up_scales, (uint64_t)I, (uint64_t)E * H / 32, 64, 4) &&
        encode_2d_u8(&m->ds, w.down_scales, (uint64_t)H, (uint64_t)E * I / 32, 128, 4);
    if (!ok) *err = "cuTensorMapEncodeTiled failed (MXFP8 weights)";
    return ok;
}

bool encode_bmaps_u8(BMaps* maps, const void* base, uint64_t inner, uint64_t rows, const char** err) {
    for (int i = 0; i < B_MAPS; ++i)
        if (!encode_2d_u8(&maps->m[i], base, inner, rows, 128, (uint32_t)(16 * (i + 1)),
                          CU_TENSOR_MAP_SWIZZLE_128B)) {
            *err = "cuTensorMapEncodeTiled failed (MXFP8 token rows)";
            return false;
        }
    return true;
}

// ------------------------------------------------------------------ layouts
static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

struct FwdLayout {
    size_t status, counts2, chunks, mbs, counters, counter_ints, rows, h, out, save_a, save_b, total;
    int save;
    size_t xsc, hsc;  // MXFP8 path: token-side scale planes
    int max_chunks, max_mb, buf_rows, cap, minibatch, mode, mx;
};

static const uint64_t kDefaultTimeoutNs = 2000000000ull;
// Dispatch CTAs of the persistent kernel by default.  On the bf16 path one
// thread per CTA streams rows with bulk copies (about 200 KB in flight, some
// 30 GB/s per CTA measured); at the page shape on B200, 2, 4, 8 and 16 CTAs
// gave 15.7, 9.7, 8.0 and 8.4 ms per forward in one session, and 5, 6, 7
// and 8 gave 8.61, 7.87, 7.90 and 7.93 ms in another.  The MXFP8 path
// quantises with every warp of its CTAs (16 measured best).
static const int kDefaultDispatchBf16 = 6;

static bool fwd_layout(int T, int H, int I, int E, int k, int minibatch, const mok_fwd_opts* o, FwdLayout* L) {
    if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0) return false;
    const int64_t ns = (int64_t)T * k;
    if (ns > 0x7fffffff / 2) return false;
    FwdLayout l{};
    l.mode = o ? o->mode : MOK_MODE_PERSISTENT;
    if (l.mode == MOK_MODE_STAGED) {
        l.minibatch = (int)(ns > 0 ? ns : 1);
        l.cap = l.minibatch;
        l.buf_rows = (int)ns;
    } else {
        // 0: the two-wave rule alone; at least 16 rows either way
        l.minibatch = minibatch > 16 ? minibatch : 16;
        const int ring = (o && o->ring_slots > 0) ? o->ring_slots : 2 * (minibatch > 4096 ? minibatch : 4096);
        l.cap = ring / 2;
        l.buf_rows = ring;
    }
    if (l.minibatch < 1) return false;
    l.max_mb = max_minibatches((int)ns, l.minibatch);
    l.max_chunks = max_chunks((int)ns, E, l.max_mb);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += align256(bytes);
        return at;
    };
    l.status = take(sizeof(DevStatus));
    l.counts2 = take(sizeof(int) * 4);
    l.chunks = take(sizeof(Chunk) * (size_t)l.max_chunks);
    l.mbs = take(sizeof(Minibatch) * (size_t)l.max_mb);
    // persistent-mode counters: chunk_ready, g_done, d_chunk [max_chunks],
    // d_done [max_mb], tok_cnt, ready_q [T], q_tail, q_claim
    l.counter_ints = 3 * (size_t)l.max_chunks + (size_t)l.max_mb + 2 * (size_t)T + 8;
    l.counters = take(sizeof(int) * l.counter_ints);
    l.mx = (o && o->mxfp8) ? 1 : 0;
    if (l.mx) {
        // E4M3 rows and h, with their scale planes
        l.rows = take((size_t)l.buf_rows * H);
        l.h = take((size_t)l.buf_rows * I);
        l.xsc = take(mx_sc_bytes(l.buf_rows, H));
        l.hsc = take(mx_sc_bytes(l.buf_rows, I));
    } else {
        l.rows = take((size_t)l.buf_rows * H * 2);
        l.h = take((size_t)l.buf_rows * I * 2);
    }
    l.out = take(slot_bytes((size_t)ns, H, l.mx ? MOK_SLOTS_BF16 : MOK_SLOTS_F16S));  // slot outputs
    // kept for the backward (staged bf16 path): gate and up pre-activations
    l.save = (o && o->save_for_backward) ? 1 : 0;
    if (l.save) {
        if (l.mx || l.mode != MOK_MODE_STAGED) return false;
        l.save_a = take((size_t)ns * I * 2);
        l.save_b = take((size_t)ns * I * 2);
    }
    l.total = off;
    *L = l;
    return true;
}

static int check_ws(const void* ws, size_t have, size_t need) {
    if (ws == nullptr) return fail(MOK_ERR_WORKSPACE, "workspace is NULL");
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(MOK_ERR_WORKSPACE, "workspace not 256-byte aligned");
    if (have < need) return fail(MOK_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", have, need);
    return MOK_OK;
}

static int check_plan(const mok_plan_t* p) {
    if (!p) return fail(MOK_ERR_INVALID_ARG, "plan is NULL");
    if (p->T < 0 || p->E <= 0 || p->k <= 0 || p->k > p->E || p->R <= 0 || p->R > MOK_MAX_SHARDS ||
        (p->T > 0 && p->T % p->R))
        return fail(MOK_ERR_INVALID_ARG, "plan holds an invalid shape");
    // a hand-filled plan (e.g. from mok_plan_noalloc's outputs) gets the same
    // limits as mok_plan: the work list and the combine are built for them
    if (p->E > MOK_MAX_EXPERTS) return fail(MOK_ERR_UNSUPPORTED, "plan E > %d", MOK_MAX_EXPERTS);
    if (p->k > MOK_MAX_TOPK) return fail(MOK_ERR_UNSUPPORTED, "plan k > %d", MOK_MAX_TOPK);
    if ((int64_t)p->T * p->k > 0x3fffffff) return fail(MOK_ERR_UNSUPPORTED, "plan T * k too large");
    if (!p->counts || !p->offsets || !p->sched_src_rank || !p->sched_src_index || !p->row_slot || !p->pos ||
        !p->topk_idx || !p->gates)
        return fail(MOK_ERR_INVALID_ARG, "plan has NULL views (was mok_plan called?)");
    return MOK_OK;
}

static int check_hi(int H, int I) {
    if (H <= 0 || I <= 0) return fail(MOK_ERR_INVALID_ARG, "H and I must be positive");
    if (H % 128) return fail(MOK_ERR_UNSUPPORTED, "H %% 128 != 0 (H = %d)", H);
    if (I % 64) return fail(MOK_ERR_UNSUPPORTED, "I %% 64 != 0 (I = %d)", I);
    return MOK_OK;
}

// ------------------------------------------------------------------ pieces
// mxw != nullptr: MXFP8 weights (wg/wu/wd are then ignored); rows and h are
// E4M3 with the token-side scale planes of mxs.
static int run_expert_ffn(const void* rows, int n_rows_buf, int H, int I, const void* wg, const void* wu,
                          const void* wd, int E, const int32_t* row_slot, const Chunk* chunks, const int* counts2,
                          void* h, void* out, DevStatus* status, uint64_t timeout_ns, cudaStream_t stream,
                          const mok_mxfp8_weights* mxw = nullptr, const MxTokenScales* mxs = nullptr,
                          const BwdBuffers* save = nullptr, const PushDest* push = nullptr, int push_slots = 0,
                          int tune_rows = -1) {
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    MOK_CUDA(gemm_configure(dev), "gemm configure");
    GemmMaps maps;
    memset(&maps, 0, sizeof maps);
    MxMaps mx;
    const char* err = nullptr;
    if (mxw) {
        if (!encode_mx_maps(&mx, *mxw, H, I, E, &err) ||
            !encode_bmaps_u8(&maps.rows, rows, (uint64_t)H, (uint64_t)n_rows_buf, &err) ||
            !encode_bmaps_u8(&maps.h, h, (uint64_t)I, (uint64_t)n_rows_buf, &err))
            return fail(MOK_ERR_CUDA, "tensor map: %s", err);
    } else if (!encode_gemm_maps(&maps, wg, wu, wd, rows, h, H, I, E, n_rows_buf, &err)) {
        return fail(MOK_ERR_CUDA, "tensor map: %s", err);
    }
    GemmShape sh{H, I, E};
    const GemmTuning tune = gemm_tuning(tune_rows >= 0 ? tune_rows : n_rows_buf, E);
    const MxMaps* mxp = mxw ? &mx : nullptr;
    MOK_CUDA(launch_gemm_phase(0, maps, mxp, mxs, sh, chunks, counts2, h, out, row_slot, status, timeout_ns, sms,
                               tune, stream, save),
             "gate/up GEMM launch");
    int8_t* out_exp =
        mxw || push ? nullptr : reinterpret_cast<int8_t*>(out) + slot_exp_offset((size_t)n_rows_buf, H);
    MOK_CUDA(launch_gemm_phase(1, maps, mxp, mxs, sh, chunks, counts2, h, out, row_slot, status, timeout_ns, sms,
                               tune, stream, nullptr, out_exp, push, push_slots),
             "down GEMM launch");
    return MOK_OK;
}

static bool all_aligned16(const void* const* p, int n) {
    for (int i = 0; i < n; ++i)
        if (reinterpret_cast<uintptr_t>(p[i]) & 15u) return false;
    return true;
}

static bool all_nonnull(const void* const* p, int n) {
    if (!p) return false;
    for (int i = 0; i < n; ++i)
        if (!p[i]) return false;
    return true;
}

}  // namespace mok

using namespace mok;

extern "C" {

const char* mok_last_error_string(void) { return g_err.c_str(); }

size_t mok_plan_workspace_bytes(int T, int E, int k) {
    if (T < 0 || E <= 0 || E > MOK_MAX_EXPERTS || k <= 0 || k > E || k > MOK_MAX_TOPK) return 0;
    return plan_layout(T, E, k, nullptr);
}

int mok_plan(const float* logits, int T, int E, int top_k, int R, void* ws, size_t ws_bytes, mok_plan_t* plan,
             mok_stream_t stream) {
    if (!plan) return fail(MOK_ERR_INVALID_ARG, "plan is NULL");
    if (T < 0 || E <= 0 || top_k <= 0 || R <= 0) return fail(MOK_ERR_INVALID_ARG, "T, E, top_k, R out of range");
    if (E > MOK_MAX_EXPERTS) return fail(MOK_ERR_UNSUPPORTED, "E > %d", MOK_MAX_EXPERTS);
    if (top_k > E) return fail(MOK_ERR_INVALID_ARG, "top_k > E");
    if (top_k > MOK_MAX_TOPK) return fail(MOK_ERR_UNSUPPORTED, "top_k > %d", MOK_MAX_TOPK);
    if (R > MOK_MAX_SHARDS) return fail(MOK_ERR_UNSUPPORTED, "R > %d", MOK_MAX_SHARDS);
    if (T % R) return fail(MOK_ERR_UNSUPPORTED, "T %% R != 0 (T = %d, R = %d)", T, R);
    if ((int64_t)T * top_k > 0x3fffffff) return fail(MOK_ERR_UNSUPPORTED, "T * top_k too large");
    if (T > 0 && !logits) return fail(MOK_ERR_INVALID_ARG, "logits is NULL");
    PlanLayout L;
    const size_t need = plan_layout(T, E, top_k, &L);
    int rc = check_ws(ws, ws_bytes, need);
    if (rc) return rc;
    unsigned char* base = static_cast<unsigned char*>(ws);
    plan->T = T;
    plan->E = E;
    plan->k = top_k;
    plan->R = R;
    plan->counts = reinterpret_cast<int32_t*>(base + L.counts);
    plan->offsets = reinterpret_cast<int32_t*>(base + L.offsets);
    plan->sched_src_rank = reinterpret_cast<int32_t*>(base + L.src_rank);
    plan->sched_src_index = reinterpret_cast<int32_t*>(base + L.src_index);
    plan->row_slot = reinterpret_cast<int32_t*>(base + L.row_slot);
    plan->pos = reinterpret_cast<int32_t*>(base + L.pos);
    plan->topk_idx = reinterpret_cast<int32_t*>(base + L.topk);
    plan->gates = reinterpret_cast<float*>(base + L.gates);
    if (device_sms(nullptr) <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    MOK_CUDA(launch_plan(logits, T, E, top_k, R, base, L, reinterpret_cast<cudaStream_t>(stream)), "plan launch");
    return MOK_OK;
}

size_t mok_slot_bytes(int n_slots, int H, int slot_type) {
    if (n_slots < 0 || H <= 0 || (slot_type != MOK_SLOTS_F32 && slot_type != MOK_SLOTS_BF16 &&
                                  slot_type != MOK_SLOTS_F16S))
        return 0;
    if (slot_type == MOK_SLOTS_F16S && H % 128) return 0;
    return slot_bytes((size_t)n_slots, H, slot_type);
}

size_t mok_slot_exp_offset(int n_slots, int H) {
    return (n_slots < 0 || H <= 0) ? 0 : slot_exp_offset((size_t)n_slots, H);
}

size_t mok_router_weights_bytes(int H, int E) {
    if (H <= 0 || E <= 0 || E > MOK_ROUTER_MAX_EXPERTS) return 0;
    return (size_t)router_e_pad(E) * H * 2;
}

int mok_router_prepare(const float* w_r, int H, int E, void* w_hi, void* w_lo, mok_stream_t stream) {
    if (H <= 0 || E <= 0) return fail(MOK_ERR_INVALID_ARG, "H, E out of range");
    if (E > MOK_ROUTER_MAX_EXPERTS) return fail(MOK_ERR_UNSUPPORTED, "E > %d", MOK_ROUTER_MAX_EXPERTS);
    if (H % 64) return fail(MOK_ERR_UNSUPPORTED, "H %% 64 != 0 (H = %d)", H);
    if (!w_r || !w_hi || !w_lo) return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    if ((reinterpret_cast<uintptr_t>(w_hi) | reinterpret_cast<uintptr_t>(w_lo)) & 15u)
        return fail(MOK_ERR_UNSUPPORTED, "w_hi and w_lo must be 16-byte aligned");
    const int sms = device_sms(nullptr);
    if (sms <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    MOK_CUDA(launch_router_split(w_r, H, E, w_hi, w_lo, sms, reinterpret_cast<cudaStream_t>(stream)),
             "router weight split launch");
    return MOK_OK;
}

int mok_plan_router(const void* const* x_shards, int H, const void* w_hi, const void* w_lo, const float* prior,
                    int T, int E, int top_k, int R, float* logits_out, void* ws, size_t ws_bytes, mok_plan_t* plan,
                    mok_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (!plan) return fail(MOK_ERR_INVALID_ARG, "plan is NULL");
    if (T < 0 || E <= 0 || top_k <= 0 || R <= 0 || H <= 0) return fail(MOK_ERR_INVALID_ARG, "T, E, top_k, R, H");
    if (E > MOK_ROUTER_MAX_EXPERTS) return fail(MOK_ERR_UNSUPPORTED, "E > %d", MOK_ROUTER_MAX_EXPERTS);
    if (top_k > E) return fail(MOK_ERR_INVALID_ARG, "top_k > E");
    if (top_k > MOK_MAX_TOPK) return fail(MOK_ERR_UNSUPPORTED, "top_k > %d", MOK_MAX_TOPK);
    if (R > MOK_MAX_SHARDS) return fail(MOK_ERR_UNSUPPORTED, "R > %d", MOK_MAX_SHARDS);
    if (T % R) return fail(MOK_ERR_UNSUPPORTED, "T %% R != 0 (T = %d, R = %d)", T, R);
    if (H % 64) return fail(MOK_ERR_UNSUPPORTED, "H %% 64 != 0 (H = %d)", H);
    if ((int64_t)T * top_k > 0x3fffffff) return fail(MOK_ERR_UNSUPPORTED, "T * top_k too large");
    if (!w_hi || !w_lo) return fail(MOK_ERR_INVALID_ARG, "NULL router weights");
    if ((reinterpret_cast<uintptr_t>(w_hi) | reinterpret_cast<uintptr_t>(w_lo)) & 15u)
        return fail(MOK_ERR_UNSUPPORTED, "w_hi and w_lo must be 16-byte aligned");
    if (T > 0) {
        if (!all_nonnull(x_shards, R)) return fail(MOK_ERR_INVALID_ARG, "NULL shard pointer");
        if (!all_aligned16(x_shards, R)) return fail(MOK_ERR_UNSUPPORTED, "shard pointers must be 16-byte aligned");
    }
    PlanLayout L;
    const size_t need = plan_layout(T, E, top_k, &L);
    int rc = check_ws(ws, ws_bytes, need);
    if (rc) return rc;
    unsigned char* base = static_cast<unsigned char*>(ws);
    auto I32 = [&](size_t o) { return reinterpret_cast<int32_t*>(base + o); };
    plan->T = T;
    plan->E = E;
    plan->k = top_k;
    plan->R = R;
    plan->counts = I32(L.counts);
    plan->offsets = I32(L.offsets);
    plan->sched_src_rank = I32(L.src_rank);
    plan->sched_src_index = I32(L.src_index);
    plan->row_slot = I32(L.row_slot);
    plan->pos = I32(L.pos);
    plan->topk_idx = I32(L.topk);
    plan->gates = reinterpret_cast<float*>(base + L.gates);
    if (device_sms(nullptr) <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    MOK_CUDA(cudaMemsetAsync(base + L.status, 0, sizeof(DevStatus), stream), "status reset");
    if (T > 0) {
        ShardsIn xs{};
        for (int r = 0; r < R; ++r) xs.p[r] = x_shards[r];
        const char* err = "";
        cudaError_t e = launch_router(xs, T / R, T, H, E, top_k, w_hi, w_lo, prior, logits_out, plan->topk_idx,
                                      plan->gates, base + L.status, kDefaultTimeoutNs, &err, stream);
        if (e != cudaSuccess) return fail(MOK_ERR_CUDA, "%s: %s", err, cudaGetErrorString(e));
    }
    MOK_CUDA(launch_plan_schedule(T, E, top_k, R, plan->counts, plan->offsets, plan->sched_src_rank,
                                  plan->sched_src_index, plan->row_slot, plan->pos, plan->topk_idx, I32(L.blk_cnt),
                                  I32(L.rank), stream),
             "plan launch");
    return MOK_OK;
}

size_t mok_forward_workspace_bytes(int T, int H, int I, int E, int k, int minibatch, const mok_fwd_opts* opts) {
    FwdLayout L;
    if (!fwd_layout(T, H, I, E, k, minibatch, opts, &L)) return 0;
    return L.total;
}

}  // extern "C"

namespace mok {

// Everything mok_moe_forward decides before its kernels: validated shape,
// workspace layout, SM split and the device-built work list (minibatches
// and chunks) in the workspace.
struct FwdSetup {
    FwdLayout L;
    int sms, dispatch, dwarps, gemm, upc, min_units;
    bool pair;
    uint64_t timeout;
    const mok_mxfp8_weights* mxw;
    DevStatus* status;
    int* counts2;
    Chunk* chunks;
    Minibatch* mbs;
};

static int setup_forward(int H, int I, const void* w_gate, const mok_plan_t* plan, int minibatch,
                         const mok_fwd_opts* opts, void* ws, size_t ws_bytes, cudaStream_t stream, FwdSetup* F) {
    int rc = check_plan(plan);
    if (rc) return rc;
    if ((rc = check_hi(H, I))) return rc;
    const int mode = opts ? opts->mode : MOK_MODE_PERSISTENT;
    if (mode != MOK_MODE_STAGED && mode != MOK_MODE_PERSISTENT)
        return fail(MOK_ERR_INVALID_ARG, "unknown mode %d", mode);
    F->mxw = nullptr;
    if (opts && opts->mxfp8) {
        F->mxw = static_cast<const mok_mxfp8_weights*>(w_gate);
        const mok_mxfp8_weights* m = F->mxw;
        if (!m || !m->gate || !m->gate_scales || !m->up || !m->up_scales || !m->down || !m->down_scales)
            return fail(MOK_ERR_INVALID_ARG, "MXFP8 weight pack with NULL members");
    }
    const int dwarps = opts ? opts->dispatch_warps : 0;
    if (dwarps < 0 || dwarps > 2) return fail(MOK_ERR_INVALID_ARG, "dispatch_warps must be in [0, 2]");
    if (dwarps > 0 && opts->dispatch_ctas > 0)
        return fail(MOK_ERR_INVALID_ARG, "dispatch_warps and dispatch_ctas exclude each other");
    if (opts && opts->save_for_backward && (mode != MOK_MODE_STAGED || (opts->mxfp8 != 0)))
        return fail(MOK_ERR_UNSUPPORTED, "save_for_backward needs the staged bf16 path");
    if (mode == MOK_MODE_PERSISTENT && minibatch != 0 && minibatch < 16)
        return fail(MOK_ERR_INVALID_ARG, "minibatch must be 0 (two-wave rule) or >= 16");
    if (minibatch < 0) return fail(MOK_ERR_INVALID_ARG, "minibatch < 0");
    const int T = plan->T, E = plan->E, k = plan->k;
    if (!fwd_layout(T, H, I, E, k, minibatch, opts, &F->L)) return fail(MOK_ERR_INVALID_ARG, "invalid shape");
    if (mode == MOK_MODE_PERSISTENT && F->L.cap < F->L.minibatch)
        return fail(MOK_ERR_INVALID_ARG, "ring_slots / 2 < minibatch");
    if ((rc = check_ws(ws, ws_bytes, F->L.total))) return rc;
    F->sms = device_sms(nullptr);
    if (F->sms <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    F->dispatch = 0;
    F->dwarps = 0;
    F->gemm = F->sms;
    if (mode == MOK_MODE_PERSISTENT && dwarps > 0) {
        // warp layout: every CTA runs the GEMM and dispatch warps
        F->dwarps = dwarps;
        F->gemm = (opts->gemm_ctas > 0) ? opts->gemm_ctas : F->sms;
        if (F->gemm > F->sms) return fail(MOK_ERR_INVALID_ARG, "gemm_ctas must be at most the %d SMs", F->sms);
    } else if (mode == MOK_MODE_PERSISTENT) {
        F->dispatch = (opts && opts->dispatch_ctas > 0) ? opts->dispatch_ctas : (F->mxw ? 16 : kDefaultDispatchBf16);
        F->gemm = (opts && opts->gemm_ctas > 0) ? opts->gemm_ctas : F->sms - F->dispatch;
        if (F->dispatch >= F->sms || F->gemm < 1 || F->dispatch + F->gemm > F->sms)
            return fail(MOK_ERR_INVALID_ARG, "dispatch_ctas + gemm_ctas must be at most the %d SMs", F->sms);
    }
    // gate/up units per chunk: M tiles of 64 gate + 64 up features, in
    // pairs where the pairing rule holds (bf16 path)
    const int ns = T * k;
    F->pair = !F->mxw && gemm_tuning(ns, E).pair != 0;
    const int sub = F->pair ? 2 : 1;
    F->upc = (I / 64 + sub - 1) / sub;
    // minibatches of at least `waves` full waves of gate/up units (the
    // pages' rule: two), persistent mode only
    const int waves = (opts && opts->min_waves != 0) ? opts->min_waves : 2;
    F->min_units = (mode == MOK_MODE_PERSISTENT && waves > 0) ? waves * F->gemm : 0;
    F->timeout = (opts && opts->timeout_ns) ? opts->timeout_ns : kDefaultTimeoutNs;
    unsigned char* base = static_cast<unsigned char*>(ws);
    F->status = reinterpret_cast<DevStatus*>(base + F->L.status);
    F->counts2 = reinterpret_cast<int*>(base + F->L.counts2);
    F->chunks = reinterpret_cast<Chunk*>(base + F->L.chunks);
    F->mbs = reinterpret_cast<Minibatch*>(base + F->L.mbs);
    if (T == 0) return MOK_OK;
    MOK_CUDA(cudaMemsetAsync(F->status, 0, sizeof(DevStatus), stream), "status reset");
    MOK_CUDA(launch_build_chunks(plan->offsets, E, ns, F->L.minibatch, F->L.cap,
                                 F->mxw ? CHUNK_MAX_ROWS_MX : CHUNK_MAX_ROWS, F->min_units, F->upc, F->chunks,
                                 F->L.max_chunks, F->mbs, F->L.max_mb, F->counts2, F->status, stream),
             "work list launch");
    return MOK_OK;
}

}  // namespace mok

extern "C" {

int mok_two_wave_rows(int I, int gemm_ctas, int tile_rows, int tile_features) {
    return two_wave_rows(I, gemm_ctas, 2, tile_rows, tile_features);
}

int mok_minibatch_bounds(const mok_plan_t* plan, int H, int I, const void* w_gate, int minibatch,
                         const mok_fwd_opts* opts, void* ws, size_t ws_bytes, int32_t* row0, int32_t* units,
                         int max_mb, int* n_mb, mok_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (!row0 || !n_mb || max_mb < 1) return fail(MOK_ERR_INVALID_ARG, "row0, n_mb, max_mb");
    FwdSetup F;
    int rc = setup_forward(H, I, w_gate, plan, minibatch, opts, ws, ws_bytes, stream, &F);
    if (rc) return rc;
    *n_mb = 0;
    if (plan->T == 0) return MOK_OK;
    MOK_CUDA(cudaStreamSynchronize(stream), "stream synchronize");
    int c2[2];
    MOK_CUDA(cudaMemcpy(c2, F.counts2, sizeof c2, cudaMemcpyDeviceToHost), "work list read");
    DevStatus st;
    MOK_CUDA(cudaMemcpy(&st, F.status, sizeof st, cudaMemcpyDeviceToHost), "status read");
    if (st.code != MOK_OK) return fail(st.code, "work list: device status %d", st.code);
    const int n = c2[1] < max_mb ? c2[1] : max_mb;
    for (int b = 0; b < n; ++b) {
        Minibatch m;
        MOK_CUDA(cudaMemcpy(&m, F.mbs + b, sizeof m, cudaMemcpyDeviceToHost), "work list read");
        row0[b] = m.row0;
        if (units) units[b] = (m.chunk1 - m.chunk0) * F.upc;
    }
    *n_mb = c2[1];
    return MOK_OK;
}

int mok_moe_forward(const void* const* x_shards, int H, int I, const void* w_gate, const void* w_up,
                    const void* w_down, const mok_plan_t* plan, int minibatch, const mok_fwd_opts* opts, void* ws,
                    size_t ws_bytes, void* const* y_shards, mok_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int rc = check_plan(plan);
    if (rc) return rc;
    if ((rc = check_hi(H, I))) return rc;
    if (opts && opts->mode != MOK_MODE_STAGED && opts->mode != MOK_MODE_PERSISTENT)
        return fail(MOK_ERR_INVALID_ARG, "unknown mode %d", opts->mode);
    if (plan->T > 0) {
        if (!all_nonnull(x_shards, plan->R) || !all_nonnull(y_shards, plan->R))
            return fail(MOK_ERR_INVALID_ARG, "NULL shard pointer");
        if (!all_aligned16(x_shards, plan->R) || !all_aligned16(y_shards, plan->R))
            return fail(MOK_ERR_UNSUPPORTED, "shard pointers must be 16-byte aligned");
    }
    const bool mx = opts && opts->mxfp8;
    if (!mx && (!w_gate || !w_up || !w_down)) return fail(MOK_ERR_INVALID_ARG, "NULL weight pointer");
    FwdSetup F;
    rc = setup_forward(H, I, w_gate, plan, minibatch, opts, ws, ws_bytes, stream, &F);
    if (rc) return rc;
    const int T = plan->T, E = plan->E, k = plan->k, R = plan->R;
    if (T == 0) return MOK_OK;
    const mok_mxfp8_weights* mxw = F.mxw;
    const FwdLayout& L = F.L;
    const int sms = F.sms;
    unsigned char* base = static_cast<unsigned char*>(ws);
    ShardsIn xs{};
    ShardsOut ys{};
    for (int r = 0; r < R; ++r) {
        xs.p[r] = x_shards[r];
        ys.p[r] = y_shards[r];
    }
    const int ns = T * k;
    if (L.mode == MOK_MODE_PERSISTENT) {
        int dev = 0;
        device_sms(&dev);
        int* counters = reinterpret_cast<int*>(base + L.counters);
        MOK_CUDA(cudaMemsetAsync(counters, 0, sizeof(int) * L.counter_ints, stream), "counter reset");
        PersistLaunch P{};
        P.grid = F.dispatch + F.gemm;
        P.dispatch_ctas = F.dispatch;
        P.dispatch_warps = F.dwarps;
        P.pair = F.pair;
        P.cap = L.cap;
        P.H = H;
        P.I = I;
        P.E = E;
        P.T = T;
        P.k = k;
        P.S_r = T / R;
        P.wg = w_gate;
        P.wu = w_up;
        P.wd = w_down;
        P.mxw = mxw;
        if (mxw) {
            P.ring_sc = base + L.xsc;
            P.h_sc = base + L.hsc;
            P.sc_rows = mx_sc_rows(L.buf_rows);
        }
        P.ring = base + L.rows;
        P.h = base + L.h;
        P.out = base + L.out;
        P.chunks = F.chunks;
        P.mbs = F.mbs;
        P.counts2 = F.counts2;
        P.chunk_ready = counters;
        P.g_done = counters + L.max_chunks;
        P.d_chunk = counters + 2 * (size_t)L.max_chunks;
        P.d_done = counters + 3 * (size_t)L.max_chunks;
        P.tok_cnt = P.d_done + L.max_mb;
        P.ready_q = P.tok_cnt + T;
        P.q_tail = P.ready_q + T;
        P.q_claim = P.q_tail + 1;
        P.d_claim = P.q_claim + 1;
        P.xs = xs;
        P.ys = ys;
        P.src_rank = plan->sched_src_rank;
        P.src_index = plan->sched_src_index;
        P.row_slot = plan->row_slot;
        P.gates = plan->gates;
        P.status = F.status;
        P.timeout_ns = F.timeout;
        MOK_CUDA(gemm_configure(dev), "gemm configure");
        const char* err = "";
        cudaError_t e = launch_forward_persistent(P, &err, stream);
        if (e != cudaSuccess) return fail(MOK_ERR_CUDA, "%s: %s", err, cudaGetErrorString(e));
        return MOK_OK;
    }
    MxTokenScales mxs{};
    if (mxw) {
        mxs.xsc = base + L.xsc;
        mxs.hsc = base + L.hsc;
        mxs.sc_rows = mx_sc_rows(L.buf_rows);
        MOK_CUDA(launch_gather_mx(xs, T / R, H, T, k, plan->pos, base + L.rows, base + L.xsc, mxs.sc_rows, sms,
                                  stream),
                 "gather launch");
    } else {
        MOK_CUDA(launch_gather(xs, T / R, H, T, k, plan->pos, base + L.rows, sms, stream), "gather launch");
    }
    BwdBuffers save{};
    if (L.save) {
        save.save_a = reinterpret_cast<uint16_t*>(base + L.save_a);
        save.save_b = reinterpret_cast<uint16_t*>(base + L.save_b);
    }
    rc = run_expert_ffn(base + L.rows, ns, H, I, w_gate, w_up, w_down, E, plan->row_slot, F.chunks, F.counts2,
                        base + L.h, base + L.out, F.status, F.timeout, stream, mxw, mxw ? &mxs : nullptr,
                        L.save ? &save : nullptr);
    if (rc) return rc;
    MOK_CUDA(launch_combine(base + L.out, mxw ? MOK_SLOTS_BF16 : MOK_SLOTS_F16S, plan->gates, T, k, H, T / R, ys,
                            sms, stream),
             "combine launch");
    return MOK_OK;
}

size_t mok_backward_workspace_bytes(int T, int H, int I, int E, int k) {
    if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0) return 0;
    const size_t ns = (size_t)T * k;
    return align256(sizeof(DevStatus)) + align256(ns * H * 2) + align256(ns * (size_t)I * 4) +
           align256(slot_bytes(ns, H, MOK_SLOTS_F16S));
}

int mok_moe_backward(const void* const* dy_shards, int H, int I, const void* w_gate, const void* w_up,
                     const void* w_down, const mok_plan_t* plan, const void* fwd_ws, size_t fwd_ws_bytes,
                     void* const* dx_shards, void* dw_gate, void* dw_up, void* dw_down, float* dlogits, void* ws,
                     size_t ws_bytes, mok_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int rc = check_plan(plan);
    if (rc) return rc;
    if ((rc = check_hi(H, I))) return rc;
    if (I % 128) return fail(MOK_ERR_UNSUPPORTED, "the backward needs I %% 128 == 0 (I = %d)", I);
    const int T = plan->T, E = plan->E, k = plan->k, R = plan->R;
    if (T == 0) return MOK_OK;
    if (!all_nonnull(dy_shards, R) || !all_nonnull(dx_shards, R)) return fail(MOK_ERR_INVALID_ARG, "NULL shard pointer");
    if (!all_aligned16(dy_shards, R) || !all_aligned16(dx_shards, R))
        return fail(MOK_ERR_UNSUPPORTED, "shard pointers must be 16-byte aligned");
    if (!w_gate || !w_up || !w_down || !dw_gate || !dw_up || !dw_down || !dlogits || !fwd_ws)
        return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    if ((reinterpret_cast<uintptr_t>(dw_gate) | reinterpret_cast<uintptr_t>(dw_up) |
         reinterpret_cast<uintptr_t>(dw_down)) & 15u)
        return fail(MOK_ERR_UNSUPPORTED, "weight gradients must be 16-byte aligned");
    // the forward workspace as a staged forward with save_for_backward laid it out
    mok_fwd_opts fo{};
    fo.mode = MOK_MODE_STAGED;
    fo.save_for_backward = 1;
    FwdLayout FL;
    if (!fwd_layout(T, H, I, E, k, 0, &fo, &FL)) return fail(MOK_ERR_INVALID_ARG, "invalid shape");
    if ((rc = check_ws(fwd_ws, fwd_ws_bytes, FL.total))) return rc;
    if ((rc = check_ws(ws, ws_bytes, mok_backward_workspace_bytes(T, H, I, E, k)))) return rc;
    const int sms = device_sms(nullptr);
    if (sms <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    int dev = 0;
    device_sms(&dev);
    const unsigned char* fb = static_cast<const unsigned char*>(fwd_ws);
    unsigned char* base = static_cast<unsigned char*>(ws);
    const size_t ns = (size_t)T * k;
    size_t off = 0;
    DevStatus* status = reinterpret_cast<DevStatus*>(base);
    off += align256(sizeof(DevStatus));
    void* do_rows = base + off;
    off += align256(ns * H * 2);
    uint16_t* dab = reinterpret_cast<uint16_t*>(base + off);
    off += align256(ns * (size_t)I * 4);
    unsigned char* dx_slots = base + off;  // fp16 rows with one exponent per 128 features (MOK_SLOTS_F16S)
    int8_t* dx_exps = reinterpret_cast<int8_t*>(dx_slots + slot_exp_offset(ns, H));
    ShardsIn dys{};
    ShardsOut dxs{};
    for (int r = 0; r < R; ++r) {
        dys.p[r] = dy_shards[r];
        dxs.p[r] = dx_shards[r];
    }
    MOK_CUDA(cudaMemsetAsync(status, 0, sizeof(DevStatus), stream), "status reset");
    // 1. pull reverse-combine: do rows, gate gradients, dlogits
    MOK_CUDA(launch_reverse_combine(dys, T / R, H, T, k, E, plan->pos, plan->gates, plan->topk_idx,
                                    reinterpret_cast<const uint16_t*>(fb + FL.out),
                                    reinterpret_cast<const int8_t*>(fb + FL.out + slot_exp_offset(ns, H)), do_rows,
                                    dlogits, sms, stream),
             "reverse combine launch");
    // 2. dh = do Wd^T with the SwiGLU backward -> [da | db]; 3. dx rows = da Wg^T + db Wu^T -> slots
    MOK_CUDA(gemm_configure(dev), "gemm configure");
    GemmMaps maps;
    memset(&maps, 0, sizeof maps);
    const char* err = nullptr;
    if (!encode_tmap_2d_bf16(&maps.wd, w_down, (uint64_t)H, (uint64_t)E * I, 64, 128, &err) ||
        !encode_tmap_2d_bf16(&maps.wg, w_gate, (uint64_t)I, (uint64_t)E * H, 64, 128, &err) ||
        !encode_tmap_2d_bf16(&maps.wu, w_up, (uint64_t)I, (uint64_t)E * H, 64, 128, &err) ||
        !encode_bmaps(&maps.rows, do_rows, (uint64_t)H, (uint64_t)ns, &err) ||
        !encode_bmaps(&maps.h, dab, (uint64_t)2 * I, (uint64_t)ns, &err) ||
        !encode_bmaps(&maps.rows2, do_rows, (uint64_t)H, (uint64_t)ns, &err, 8) ||
        !encode_bmaps(&maps.h2, dab, (uint64_t)2 * I, (uint64_t)ns, &err, 8))
        return fail(MOK_ERR_CUDA, "tensor map: %s", err);
    BwdBuffers bb{};
    bb.save_a = reinterpret_cast<uint16_t*>(const_cast<unsigned char*>(fb) + FL.save_a);
    bb.save_b = reinterpret_cast<uint16_t*>(const_cast<unsigned char*>(fb) + FL.save_b);
    bb.dab = dab;
    const Chunk* chunks = reinterpret_cast<const Chunk*>(fb + FL.chunks);
    const int* counts2 = reinterpret_cast<const int*>(fb + FL.counts2);
    GemmShape sh{H, I, E};
    GemmTuning tune = gemm_tuning((int)ns, E);
    MOK_CUDA(launch_gemm_phase(2, maps, nullptr, nullptr, sh, chunks, counts2, nullptr, nullptr, plan->row_slot, status,
                               kDefaultTimeoutNs, sms, tune, stream, &bb),
             "dh GEMM launch");
    MOK_CUDA(launch_gemm_phase(3, maps, nullptr, nullptr, sh, chunks, counts2, nullptr, dx_slots, plan->row_slot,
                               status, kDefaultTimeoutNs, sms, tune, stream, &bb, dx_exps),
             "dx GEMM launch");
    // 4. push reverse-dispatch: dx_t = sum of its k rows (the combine with unit weights)
    MOK_CUDA(launch_combine(dx_slots, MOK_SLOTS_F16S, nullptr, T, k, H, T / R, dxs, sms, stream),
             "reverse dispatch launch");
    // 5. weight gradients per expert over its rows
    cudaError_t e = launch_wgrad(fb + FL.rows, fb + FL.h, do_rows, dab, (int)ns, plan->offsets, H, I, E, dw_gate,
                                 dw_up, dw_down, status, kDefaultTimeoutNs, sms, &err, stream);
    if (e != cudaSuccess) return fail(MOK_ERR_CUDA, "%s: %s", err ? err : "", cudaGetErrorString(e));
    return MOK_OK;
}

int mok_mxfp8_quantize_rows(const void* src, int src_f32, int rows, int K, void* q, void* scales,
                            mok_stream_t stream) {
    if (rows < 0 || K <= 0) return fail(MOK_ERR_INVALID_ARG, "rows, K out of range");
    if (K % 32) return fail(MOK_ERR_UNSUPPORTED, "K %% 32 != 0");
    if (rows == 0) return MOK_OK;
    if (!src || !q || !scales) return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    if (reinterpret_cast<uintptr_t>(q) & 7u) return fail(MOK_ERR_UNSUPPORTED, "q must be 8-byte aligned");
    const int sms = device_sms(nullptr);
    if (sms <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    MOK_CUDA(launch_mx_quant_rows(src, src_f32 != 0, rows, K, q, scales, sms, reinterpret_cast<cudaStream_t>(stream)),
             "quantiser launch");
    return MOK_OK;
}

int mok_quantize_weights_mxfp8(const void* w_bf16, int E, int K, int N, void* q, void* scales,
                               mok_stream_t stream) {
    if (E <= 0 || K <= 0 || N <= 0) return fail(MOK_ERR_INVALID_ARG, "E, K, N out of range");
    if (K % 32) return fail(MOK_ERR_UNSUPPORTED, "K %% 32 != 0");
    if (!w_bf16 || !q || !scales) return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    const int sms = device_sms(nullptr);
    if (sms <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    MOK_CUDA(launch_mx_quant_cols(w_bf16, E * (K / 32), N, q, scales, sms, reinterpret_cast<cudaStream_t>(stream)),
             "quantiser launch");
    return MOK_OK;
}

int mok_get_status(const void* ws, size_t ws_bytes, mok_stream_t stream, int* device_code) {
    if (!device_code) return fail(MOK_ERR_INVALID_ARG, "device_code is NULL");
    int rc = check_ws(ws, ws_bytes, sizeof(DevStatus));
    if (rc) return rc;
    MOK_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)), "stream synchronize");
    DevStatus st;
    MOK_CUDA(cudaMemcpy(&st, ws, sizeof st, cudaMemcpyDeviceToHost), "status read");
    *device_code = st.code;
    if (st.code != MOK_OK)
        fail(st.code, "device status %d (where %d, aux %d %d)", st.code, st.where, st.aux0, st.aux1);
    return MOK_OK;
}

int mok_gather(const void* const* x_shards, int H, const mok_plan_t* plan, void* rows, mok_stream_t stream) {
    int rc = check_plan(plan);
    if (rc) return rc;
    if (H <= 0 || H % 8) return fail(MOK_ERR_UNSUPPORTED, "H %% 8 != 0");
    if (plan->T == 0) return MOK_OK;
    if (!rows || !all_nonnull(x_shards, plan->R)) return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    if (!all_aligned16(x_shards, plan->R) || (reinterpret_cast<uintptr_t>(rows) & 15u))
        return fail(MOK_ERR_UNSUPPORTED, "shard and row pointers must be 16-byte aligned");
    ShardsIn xs{};
    for (int r = 0; r < plan->R; ++r) xs.p[r] = x_shards[r];
    const int sms = device_sms(nullptr);
    if (sms <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    MOK_CUDA(launch_gather(xs, plan->T / plan->R, H, plan->T, plan->k, plan->pos, rows, sms,
                           reinterpret_cast<cudaStream_t>(stream)),
             "gather launch");
    return MOK_OK;
}

int mok_mxfp8_scale_rows(int n_rows) { return n_rows < 0 ? 0 : mx_sc_rows(n_rows); }

int mok_gather_mxfp8(const void* const* x_shards, int H, const mok_plan_t* plan, void* rows_q, void* scales,
                     mok_stream_t stream) {
    int rc = check_plan(plan);
    if (rc) return rc;
    if (H <= 0 || H % 128) return fail(MOK_ERR_UNSUPPORTED, "H %% 128 != 0");
    if (plan->T == 0) return MOK_OK;
    if (!rows_q || !scales || !all_nonnull(x_shards, plan->R)) return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    if (!all_aligned16(x_shards, plan->R) || ((reinterpret_cast<uintptr_t>(rows_q) |
                                               reinterpret_cast<uintptr_t>(scales)) & 15u))
        return fail(MOK_ERR_UNSUPPORTED, "shard, row and scale pointers must be 16-byte aligned");
    ShardsIn xs{};
    for (int r = 0; r < plan->R; ++r) xs.p[r] = x_shards[r];
    const int sms = device_sms(nullptr);
    if (sms <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    MOK_CUDA(launch_gather_mx(xs, plan->T / plan->R, H, plan->T, plan->k, plan->pos, rows_q, scales,
                              mx_sc_rows(plan->T * plan->k), sms, reinterpret_cast<cudaStream_t>(stream)),
             "gather launch");
    return MOK_OK;
}

size_t mok_expert_ffn_workspace_bytes(int n_rows, int I, int E) {
    if (n_rows < 0 || I <= 0 || E <= 0) return 0;
    const int mb = max_minibatches(n_rows, n_rows > 0 ? n_rows : 1);
    const int mc = max_chunks(n_rows, E, mb);
    return align256(sizeof(DevStatus)) + align256(sizeof(int) * 4) + align256(sizeof(Chunk) * (size_t)mc) +
           align256(sizeof(Minibatch) * (size_t)mb) + align256((size_t)n_rows * I * 2);
}

int mok_expert_ffn(const void* rows, int H, int I, const void* w_gate, const void* w_up, const void* w_down,
                   const mok_plan_t* plan, void* ws, size_t ws_bytes, void* out, mok_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int rc = check_plan(plan);
    if (rc) return rc;
    if ((rc = check_hi(H, I))) return rc;
    const int ns = plan->T * plan->k;
    if ((rc = check_ws(ws, ws_bytes, mok_expert_ffn_workspace_bytes(ns, I, plan->E)))) return rc;
    if (ns == 0) return MOK_OK;
    if (!rows || !out || !w_gate || !w_up || !w_down) return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    unsigned char* base = static_cast<unsigned char*>(ws);
    const int mb = max_minibatches(ns, ns);
    const int mc = max_chunks(ns, plan->E, mb);
    size_t off = 0;
    DevStatus* status = reinterpret_cast<DevStatus*>(base + off);
    off += align256(sizeof(DevStatus));
    int* counts2 = reinterpret_cast<int*>(base + off);
    off += align256(sizeof(int) * 4);
    Chunk* chunks = reinterpret_cast<Chunk*>(base + off);
    off += align256(sizeof(Chunk) * (size_t)mc);
    Minibatch* mbs = reinterpret_cast<Minibatch*>(base + off);
    off += align256(sizeof(Minibatch) * (size_t)mb);
    void* h = base + off;
    MOK_CUDA(cudaMemsetAsync(status, 0, sizeof(DevStatus), stream), "status reset");
    MOK_CUDA(launch_build_chunks(plan->offsets, plan->E, ns, ns, ns, CHUNK_MAX_ROWS, 0, 1, chunks, mc, mbs, mb,
                                 counts2, status, stream),
             "work list launch");
    return run_expert_ffn(rows, ns, H, I, w_gate, w_up, w_down, plan->E, plan->row_slot, chunks, counts2, h, out,
                          status, kDefaultTimeoutNs, stream);
}

size_t mok_expert_ffn_mxfp8_workspace_bytes(int n_rows, int I, int E) {
    if (n_rows < 0 || I <= 0 || E <= 0) return 0;
    const int mb = max_minibatches(n_rows, n_rows > 0 ? n_rows : 1);
    const int mc = max_chunks(n_rows, E, mb);
    return align256(sizeof(DevStatus)) + align256(sizeof(int) * 4) + align256(sizeof(Chunk) * (size_t)mc) +
           align256(sizeof(Minibatch) * (size_t)mb) + align256((size_t)n_rows * I) + align256(mx_sc_bytes(n_rows, I));
}

int mok_expert_ffn_mxfp8(const void* rows_q, const void* scales, int H, int I, const mok_mxfp8_weights* w,
                         const mok_plan_t* plan, void* ws, size_t ws_bytes, void* out, mok_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int rc = check_plan(plan);
    if (rc) return rc;
    if ((rc = check_hi(H, I))) return rc;
    const int ns = plan->T * plan->k;
    if ((rc = check_ws(ws, ws_bytes, mok_expert_ffn_mxfp8_workspace_bytes(ns, I, plan->E)))) return rc;
    if (ns == 0) return MOK_OK;
    if (!rows_q || !scales || !out || !w || !w->gate || !w->gate_scales || !w->up || !w->up_scales || !w->down ||
        !w->down_scales)
        return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    if ((reinterpret_cast<uintptr_t>(rows_q) | reinterpret_cast<uintptr_t>(scales)) & 15u)
        return fail(MOK_ERR_UNSUPPORTED, "row and scale pointers must be 16-byte aligned");
    unsigned char* base = static_cast<unsigned char*>(ws);
    const int mb = max_minibatches(ns, ns);
    const int mc = max_chunks(ns, plan->E, mb);
    size_t off = 0;
    DevStatus* status = reinterpret_cast<DevStatus*>(base + off);
    off += align256(sizeof(DevStatus));
    int* counts2 = reinterpret_cast<int*>(base + off);
    off += align256(sizeof(int) * 4);
    Chunk* chunks = reinterpret_cast<Chunk*>(base + off);
    off += align256(sizeof(Chunk) * (size_t)mc);
    Minibatch* mbs = reinterpret_cast<Minibatch*>(base + off);
    off += align256(sizeof(Minibatch) * (size_t)mb);
    void* h = base + off;
    off += align256((size_t)ns * I);
    MxTokenScales mxs{};
    mxs.xsc = static_cast<const uint8_t*>(scales);
    mxs.hsc = base + off;
    mxs.sc_rows = mx_sc_rows(ns);
    MOK_CUDA(cudaMemsetAsync(status, 0, sizeof(DevStatus), stream), "status reset");
    MOK_CUDA(launch_build_chunks(plan->offsets, plan->E, ns, ns, ns, CHUNK_MAX_ROWS_MX, 0, 1, chunks, mc, mbs, mb,
                                 counts2, status, stream),
             "work list launch");
    return run_expert_ffn(rows_q, ns, H, I, nullptr, nullptr, nullptr, plan->E, plan->row_slot, chunks, counts2, h,
                          out, status, kDefaultTimeoutNs, stream, w, &mxs);
}

int mok_combine(const void* out, int out_dtype, int H, const mok_plan_t* plan, void* const* y_shards,
                mok_stream_t stream) {
    int rc = check_plan(plan);
    if (rc) return rc;
    if (out_dtype != MOK_SLOTS_F32 && out_dtype != MOK_SLOTS_BF16 && out_dtype != MOK_SLOTS_F16S)
        return fail(MOK_ERR_INVALID_ARG, "unknown slot dtype %d", out_dtype);
    if (H <= 0 || H % 8) return fail(MOK_ERR_UNSUPPORTED, "H %% 8 != 0");
    if (out_dtype == MOK_SLOTS_F16S && H % 128) return fail(MOK_ERR_UNSUPPORTED, "H %% 128 != 0 (fp16 slot rows)");
    if (plan->T == 0) return MOK_OK;
    if (!out || !all_nonnull(y_shards, plan->R)) return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    if (!all_aligned16(y_shards, plan->R) || (reinterpret_cast<uintptr_t>(out) & 15u))
        return fail(MOK_ERR_UNSUPPORTED, "shard and output pointers must be 16-byte aligned");
    ShardsOut ys{};
    for (int r = 0; r < plan->R; ++r) ys.p[r] = y_shards[r];
    const int sms = device_sms(nullptr);
    if (sms <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    MOK_CUDA(launch_combine(out, out_dtype, plan->gates, plan->T, plan->k, H, plan->T / plan->R, ys, sms,
                            reinterpret_cast<cudaStream_t>(stream)),
             "combine launch");
    return MOK_OK;
}

}  // extern "C"

namespace mok {

// Host-buffer forward: nbuf sets of device staging buffers {x, y, logits}
// (256-byte aligned), one plan workspace and one forward workspace.
struct HostLayout {
    size_t xb, lb, set_bytes, plan_bytes, plan_off, fwd_off, total;
};

static bool host_layout(int T, int H, int I, int E, int k, int minibatch, const mok_fwd_opts* opts, int nbuf,
                        HostLayout* L) {
    const size_t p = mok_plan_workspace_bytes(T, E, k);
    const size_t f = mok_forward_workspace_bytes(T, H, I, E, k, minibatch, opts);
    if (!p || !f || T <= 0 || H <= 0) return false;
    L->xb = (size_t)T * H * 2;
    L->lb = (size_t)T * E * 4;
    L->set_bytes = align256(L->xb) * 2 + align256(L->lb);
    L->plan_bytes = align256(p);
    L->plan_off = L->set_bytes * nbuf;
    L->fwd_off = L->plan_off + L->plan_bytes;
    L->total = L->fwd_off + f;
    return true;
}

// Streams and events of the pipelined host forward, one set per device,
// made on first use and kept for the process; `mu` serialises the calls
// that use them.
struct HostPipe {
    std::mutex mu;
    bool ready = false;
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t uploaded[2], computed[2], downloaded[2];
};

static int host_pipe(int dev, HostPipe** out) {
    static HostPipe pipes[64];
    static std::mutex init_mu;
    if (dev < 0 || dev >= 64) return fail(MOK_ERR_CUDA, "device ordinal %d out of range", dev);
    HostPipe& hp = pipes[dev];
    std::lock_guard<std::mutex> g(init_mu);
    if (!hp.ready) {
        MOK_CUDA(cudaStreamCreateWithFlags(&hp.up, cudaStreamNonBlocking), "stream create");
        MOK_CUDA(cudaStreamCreateWithFlags(&hp.down, cudaStreamNonBlocking), "stream create");
        for (int b = 0; b < 2; ++b) {
            MOK_CUDA(cudaEventCreateWithFlags(&hp.uploaded[b], cudaEventDisableTiming), "event create");
            MOK_CUDA(cudaEventCreateWithFlags(&hp.computed[b], cudaEventDisableTiming), "event create");
            MOK_CUDA(cudaEventCreateWithFlags(&hp.downloaded[b], cudaEventDisableTiming), "event create");
        }
        hp.ready = true;
    }
    *out = &hp;
    return MOK_OK;
}

static int enqueue_host_batches(int n, const void* const* x_host, const float* const* logits_host,
                                void* const* y_host, int T, int H, int I, int E, int top_k, int R,
                                const void* w_gate, const void* w_up, const void* w_down, int minibatch,
                                const mok_fwd_opts* opts, unsigned char* base, const HostLayout& L, int nbuf,
                                HostPipe* hp, cudaStream_t stream, cudaStream_t up, cudaStream_t down) {
    unsigned char* plan_ws = base + L.plan_off;
    unsigned char* fwd_ws = base + L.fwd_off;
    const size_t fwd_bytes = L.total - L.fwd_off;
    const int S_r = T / R;
    int rc = MOK_OK;
    for (int i = 0; i < n; ++i) {
        const int b = i % nbuf;
        unsigned char* x_dev = base + (size_t)b * L.set_bytes;
        unsigned char* y_dev = x_dev + align256(L.xb);
        unsigned char* l_dev = y_dev + align256(L.xb);
        if (hp) MOK_CUDA(cudaStreamWaitEvent(up, hp->computed[b], 0), "stream wait");
        MOK_CUDA(cudaMemcpyAsync(l_dev, logits_host[i], L.lb, cudaMemcpyHostToDevice, up), "logits upload");
        MOK_CUDA(cudaMemcpyAsync(x_dev, x_host[i], L.xb, cudaMemcpyHostToDevice, up), "x upload");
        if (hp) {
            MOK_CUDA(cudaEventRecord(hp->uploaded[b], up), "event record");
            MOK_CUDA(cudaStreamWaitEvent(stream, hp->uploaded[b], 0), "stream wait");
            MOK_CUDA(cudaStreamWaitEvent(stream, hp->downloaded[b], 0), "stream wait");
        }
        mok_plan_t plan;
        if ((rc = mok_plan(reinterpret_cast<const float*>(l_dev), T, E, top_k, R, plan_ws, L.plan_bytes, &plan,
                           reinterpret_cast<mok_stream_t>(stream))))
            return rc;
        const void* xs[MOK_MAX_SHARDS];
        void* ys[MOK_MAX_SHARDS];
        for (int r = 0; r < R; ++r) {
            xs[r] = x_dev + (size_t)r * S_r * H * 2;
            ys[r] = y_dev + (size_t)r * S_r * H * 2;
        }
        if ((rc = mok_moe_forward(xs, H, I, w_gate, w_up, w_down, &plan, minibatch, opts, fwd_ws, fwd_bytes, ys,
                                  reinterpret_cast<mok_stream_t>(stream))))
            return rc;
        if (hp) {
            MOK_CUDA(cudaEventRecord(hp->computed[b], stream), "event record");
            MOK_CUDA(cudaStreamWaitEvent(down, hp->computed[b], 0), "stream wait");
        }
        MOK_CUDA(cudaMemcpyAsync(y_host[i], y_dev, L.xb, cudaMemcpyDeviceToHost, down), "y download");
        if (hp) MOK_CUDA(cudaEventRecord(hp->downloaded[b], down), "event record");
    }
    if (hp) {
        // `stream` ends after the last download
        MOK_CUDA(cudaStreamWaitEvent(stream, hp->downloaded[(n - 1) % 2], 0), "stream wait");
        MOK_CUDA(cudaStreamWaitEvent(stream, hp->downloaded[n % 2], 0), "stream wait");
    }
    return MOK_OK;
}

// n batches through plan + forward from host buffers.  Batch i uses staging
// set i % nbuf.  With nbuf = 2, batch i+1's upload (stream `up`) and batch
// i-1's download (stream `down`) run while batch i computes on `stream`:
//   up:     wait computed[b] (batch i-2 is done with x[b], logits[b]);
//           copy logits, x; record uploaded[b]
//   stream: wait uploaded[b], downloaded[b] (batch i-2's y[b] has left);
//           plan; forward; record computed[b]
//   down:   wait computed[b]; copy y; record downloaded[b]
// With nbuf = 1 everything runs on `stream` in order.
static int forward_host_batches(int n, const void* const* x_host, const float* const* logits_host,
                                void* const* y_host, int T, int H, int I, int E, int top_k, int R,
                                const void* w_gate, const void* w_up, const void* w_down, int minibatch,
                                const mok_fwd_opts* opts, void* ws, size_t ws_bytes, int nbuf,
                                cudaStream_t stream) {
    if (n < 0) return fail(MOK_ERR_INVALID_ARG, "n < 0");
    if (n == 0) return MOK_OK;
    if (!x_host || !logits_host || !y_host) return fail(MOK_ERR_INVALID_ARG, "NULL host pointer array");
    for (int i = 0; i < n; ++i)
        if (!x_host[i] || !logits_host[i] || !y_host[i]) return fail(MOK_ERR_INVALID_ARG, "NULL host pointer");
    if (T <= 0 || R <= 0 || R > MOK_MAX_SHARDS || T % R) return fail(MOK_ERR_INVALID_ARG, "T, R invalid");
    HostLayout L;
    if (!host_layout(T, H, I, E, top_k, minibatch, opts, nbuf, &L)) return fail(MOK_ERR_INVALID_ARG, "invalid shape");
    int rc = check_ws(ws, ws_bytes, L.total);
    if (rc) return rc;
    unsigned char* base = static_cast<unsigned char*>(ws);
    HostPipe* hp = nullptr;
    std::unique_lock<std::mutex> lock;
    if (nbuf == 2) {
        int dev = 0;
        MOK_CUDA(cudaGetDevice(&dev), "get device");
        if ((rc = host_pipe(dev, &hp))) return rc;
        lock = std::unique_lock<std::mutex>(hp->mu);
        // the copy streams start after the work already queued on `stream`
        MOK_CUDA(cudaEventRecord(hp->computed[0], stream), "event record");
        MOK_CUDA(cudaStreamWaitEvent(hp->up, hp->computed[0], 0), "stream wait");
        MOK_CUDA(cudaStreamWaitEvent(hp->down, hp->computed[0], 0), "stream wait");
        MOK_CUDA(cudaEventRecord(hp->computed[1], stream), "event record");
        MOK_CUDA(cudaEventRecord(hp->downloaded[0], stream), "event record");
        MOK_CUDA(cudaEventRecord(hp->downloaded[1], stream), "event record");
    }
    cudaStream_t up = hp ? hp->up : stream, down = hp ? hp->down : stream;
    rc = enqueue_host_batches(n, x_host, logits_host, y_host, T, H, I, E, top_k, R, w_gate, w_up, w_down, minibatch,
                              opts, base, L, nbuf, hp, stream, up, down);
    if (rc != MOK_OK) {
        // leave no copy in flight on the caller's host buffers
        if (hp) {
            cudaStreamSynchronize(up);
            cudaStreamSynchronize(down);
        }
        cudaStreamSynchronize(stream);
        return rc;
    }
    MOK_CUDA(cudaStreamSynchronize(stream), "stream synchronize");
    return MOK_OK;
}

}  // namespace mok

extern "C" {

size_t mok_forward_host_workspace_bytes(int T, int H, int I, int E, int k, int minibatch, const mok_fwd_opts* opts) {
    HostLayout L;
    return host_layout(T, H, I, E, k, minibatch, opts, 1, &L) ? L.total : 0;
}

int mok_moe_forward_host(const void* x_host, const float* logits_host, int T, int H, int I, int E, int top_k, int R,
                         const void* w_gate, const void* w_up, const void* w_down, int minibatch,
                         const mok_fwd_opts* opts, void* ws, size_t ws_bytes, void* y_host, mok_stream_t stream) {
    if (!x_host || !logits_host || !y_host) return fail(MOK_ERR_INVALID_ARG, "NULL host pointer");
    const void* xh[1] = {x_host};
    const float* lh[1] = {logits_host};
    void* yh[1] = {y_host};
    return forward_host_batches(1, xh, lh, yh, T, H, I, E, top_k, R, w_gate, w_up, w_down, minibatch, opts, ws,
                                ws_bytes, 1, reinterpret_cast<cudaStream_t>(stream));
}

size_t mok_forward_host_batches_workspace_bytes(int T, int H, int I, int E, int k, int minibatch,
                                                const mok_fwd_opts* opts) {
    HostLayout L;
    return host_layout(T, H, I, E, k, minibatch, opts, 2, &L) ? L.total : 0;
}

int mok_moe_forward_host_batches(int n, const void* const* x_host, const float* const* logits_host,
                                 void* const* y_host, int T, int H, int I, int E, int top_k, int R,
                                 const void* w_gate, const void* w_up, const void* w_down, int minibatch,
                                 const mok_fwd_opts* opts, void* ws, size_t ws_bytes, mok_stream_t stream) {
    return forward_host_batches(n, x_host, logits_host, y_host, T, H, I, E, top_k, R, w_gate, w_up, w_down, minibatch,
                                opts, ws, ws_bytes, 2, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ------------------------------------------------------------------ expert parallelism
namespace mok {

// Byte offset of the barrier counter in a rank's slot buffer.
static size_t ep_counter_offset(int S_r, int H, int k) {
    return align256(slot_bytes((size_t)S_r * k, H, MOK_SLOTS_F16S));
}

struct EpLayout {
    size_t status, push, offsets, row_slot, counts2, chunks, mbs, rows, h, total;
    int max_chunks, max_mb;
};

static size_t ep_layout(int T, int H, int I, int e_loc, int k, EpLayout* L) {
    const int ns = T * k;
    L->max_mb = max_minibatches(ns, ns > 0 ? ns : 1);
    L->max_chunks = max_chunks(ns, e_loc > 0 ? e_loc : 1, L->max_mb);
    size_t off = 0;
    L->status = off;
    off += align256(sizeof(DevStatus));
    L->push = off;
    off += align256(sizeof(PushDest));
    L->offsets = off;
    off += align256(sizeof(int32_t) * ((size_t)e_loc + 1));
    L->row_slot = off;
    off += align256(sizeof(int32_t) * (size_t)ns);
    L->counts2 = off;
    off += align256(sizeof(int) * 4);
    L->chunks = off;
    off += align256(sizeof(Chunk) * (size_t)L->max_chunks);
    L->mbs = off;
    off += align256(sizeof(Minibatch) * (size_t)L->max_mb);
    // rows and h: bf16, or (MXFP8 path) E4M3 bytes followed by their scale planes
    L->rows = off;
    off += std::max(align256((size_t)ns * H * 2), align256((size_t)ns * H) + align256(mx_sc_bytes(ns, H)));
    L->h = off;
    off += std::max(align256((size_t)ns * I * 2), align256((size_t)ns * I) + align256(mx_sc_bytes(ns, I)));
    L->total = off;
    return off;
}

static int check_ep(const mok_plan_t* plan, const mok_ep_t* ep, int H) {
    if (!ep) return fail(MOK_ERR_INVALID_ARG, "ep is NULL");
    if (ep->G < 1 || ep->G > MOK_MAX_SHARDS || ep->g < 0 || ep->g >= ep->G)
        return fail(MOK_ERR_INVALID_ARG, "EP rank %d of %d out of range", ep->g, ep->G);
    if (plan->R != ep->G) return fail(MOK_ERR_INVALID_ARG, "plan R (%d) must equal the group size (%d)", plan->R, ep->G);
    if (ep->e0 < 0 || ep->e_loc < 0 || ep->e0 + ep->e_loc > plan->E)
        return fail(MOK_ERR_INVALID_ARG, "experts [%d, %d) outside 0 .. %d", ep->e0, ep->e0 + ep->e_loc, plan->E);
    if (ep->sync != MOK_EP_SYNC_CALLER && ep->sync != MOK_EP_SYNC_DEVICE)
        return fail(MOK_ERR_INVALID_ARG, "unknown EP sync mode %d", ep->sync);
    if (ep->mxfp8 != 0 && ep->mxfp8 != 1) return fail(MOK_ERR_INVALID_ARG, "ep mxfp8 must be 0 or 1");
    if (H <= 0 || H % 128) return fail(MOK_ERR_UNSUPPORTED, "H %% 128 != 0 (H = %d)", H);
    for (int r = 0; r < ep->G; ++r) {
        if (!ep->x[r] || !ep->slots[r]) return fail(MOK_ERR_INVALID_ARG, "NULL pointer of rank %d", r);
        if (reinterpret_cast<uintptr_t>(ep->x[r]) & 15u)
            return fail(MOK_ERR_UNSUPPORTED, "x of rank %d is not 16-byte aligned", r);
        if (reinterpret_cast<uintptr_t>(ep->slots[r]) & 255u)
            return fail(MOK_ERR_UNSUPPORTED, "slot buffer of rank %d is not 256-byte aligned", r);
    }
    return MOK_OK;
}

// The group barrier of step `step`, half `half` (1: before the dispatch, 2:
// before the combine): waits for arrival number 2 * (step - 1) + half of
// every rank.
static int ep_barrier(const mok_plan_t* plan, const mok_ep_t* ep, int H, uint32_t step, int half,
                      uint64_t timeout_ns, void* status, cudaStream_t stream) {
    if (ep->sync != MOK_EP_SYNC_DEVICE) return MOK_OK;
    const int S_r = plan->T / plan->R;
    ShardsOut counters{};
    for (int r = 0; r < ep->G; ++r)
        counters.p[r] = static_cast<unsigned char*>(ep->slots[r]) + ep_counter_offset(S_r, H, plan->k);
    const uint32_t target = (2u * (step - 1u) + (uint32_t)half) * (uint32_t)ep->G;
    MOK_CUDA(launch_ep_barrier(counters, ep->G, ep->g, target, status, timeout_ns ? timeout_ns : kDefaultTimeoutNs,
                               stream),
             "EP barrier launch");
    return MOK_OK;
}

using AddrRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

static AddrRangeFn get_addr_range() {
    static AddrRangeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<AddrRangeFn>(p);
    });
    return fn;
}

}  // namespace mok

extern "C" {

size_t mok_ep_slot_bytes(int S_r, int H, int k) {
    if (S_r < 0 || H <= 0 || H % 128 || k <= 0) return 0;
    return ep_counter_offset(S_r, H, k) + 256;
}

size_t mok_ep_workspace_bytes(int T, int H, int I, int e_loc, int k) {
    if (T < 0 || H <= 0 || I <= 0 || e_loc < 0 || k <= 0) return 0;
    EpLayout L;
    return ep_layout(T, H, I, e_loc, k, &L);
}

}  // extern "C"

namespace mok {

// The body of both dispatch calls: barrier, set-up, work list, pull (bf16 or
// quantising) and the grouped FFN with push destinations.
static int ep_dispatch(const mok_plan_t* plan, const mok_ep_t* ep, int H, int I, const void* w_gate,
                       const void* w_up, const void* w_down, const mok_mxfp8_weights* mxw, uint32_t step,
                       uint64_t timeout_ns, void* ws, size_t ws_bytes, cudaStream_t stream) {
    int rc = check_plan(plan);
    if (rc) return rc;
    if ((rc = check_hi(H, I))) return rc;
    if ((rc = check_ep(plan, ep, H))) return rc;
    if (step < 1) return fail(MOK_ERR_INVALID_ARG, "step counts from 1");
    if ((ep->mxfp8 != 0) != (mxw != nullptr))
        return fail(MOK_ERR_INVALID_ARG, "ep->mxfp8 does not match the call (bf16 or MXFP8 weights)");
    EpLayout L;
    if ((rc = check_ws(ws, ws_bytes, ep_layout(plan->T, H, I, ep->e_loc, plan->k, &L)))) return rc;
    if (ep->e_loc > 0) {
        if (mxw ? (!mxw->gate || !mxw->gate_scales || !mxw->up || !mxw->up_scales || !mxw->down ||
                   !mxw->down_scales)
                : (!w_gate || !w_up || !w_down))
            return fail(MOK_ERR_INVALID_ARG, "NULL weight pointer");
    }
    unsigned char* base = static_cast<unsigned char*>(ws);
    DevStatus* status = reinterpret_cast<DevStatus*>(base + L.status);
    MOK_CUDA(cudaMemsetAsync(status, 0, sizeof(DevStatus), stream), "status reset");
    if ((rc = ep_barrier(plan, ep, H, step, 1, timeout_ns, status, stream))) return rc;
    const int ns = plan->T * plan->k;
    if (ns == 0 || ep->e_loc == 0) return MOK_OK;  // nothing to pull or compute on this rank
    const int S_r = plan->T / plan->R;
    const int sms = device_sms(nullptr);
    if (sms <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    PushDest pd{};
    ShardsIn xs{};
    for (int r = 0; r < ep->G; ++r) {
        pd.out[r] = ep->slots[r];
        pd.exp[r] = static_cast<int8_t*>(ep->slots[r]) + slot_exp_offset((size_t)S_r * plan->k, H);
        xs.p[r] = ep->x[r];
    }
    PushDest* push_dev = reinterpret_cast<PushDest*>(base + L.push);
    int32_t* offsets_loc = reinterpret_cast<int32_t*>(base + L.offsets);
    int32_t* row_slot_loc = reinterpret_cast<int32_t*>(base + L.row_slot);
    int* counts2 = reinterpret_cast<int*>(base + L.counts2);
    Chunk* chunks = reinterpret_cast<Chunk*>(base + L.chunks);
    Minibatch* mbs = reinterpret_cast<Minibatch*>(base + L.mbs);
    MOK_CUDA(launch_ep_setup(pd, push_dev, plan->offsets, ep->e0, ep->e_loc, offsets_loc, stream), "EP setup launch");
    MOK_CUDA(launch_build_chunks(offsets_loc, ep->e_loc, ns, ns, ns, mxw ? CHUNK_MAX_ROWS_MX : CHUNK_MAX_ROWS, 0, 1,
                                 chunks, L.max_chunks, mbs, L.max_mb, counts2, status, stream),
             "work list launch");
    // the GEMM's tuning sees the rows this rank's experts hold on average
    const int tune_rows = (int)((int64_t)ns * ep->e_loc / plan->E);
    if (mxw) {
        MxTokenScales mxs;
        mxs.sc_rows = mx_sc_rows(ns);
        mxs.xsc = base + L.rows + align256((size_t)ns * H);
        mxs.hsc = base + L.h + align256((size_t)ns * I);
        MOK_CUDA(launch_ep_pull_mx(xs, H, plan->offsets, ep->e0, ep->e_loc, plan->sched_src_rank,
                                   plan->sched_src_index, plan->row_slot, base + L.rows,
                                   const_cast<uint8_t*>(mxs.xsc), mxs.sc_rows, row_slot_loc, ns, sms, stream),
                 "pull dispatch launch");
        return run_expert_ffn(base + L.rows, ns, H, I, nullptr, nullptr, nullptr, ep->e_loc, row_slot_loc, chunks,
                              counts2, base + L.h, nullptr, status, kDefaultTimeoutNs, stream, mxw, &mxs, nullptr,
                              push_dev, S_r * plan->k, tune_rows);
    }
    MOK_CUDA(launch_ep_pull(xs, H, plan->offsets, ep->e0, ep->e_loc, plan->sched_src_rank, plan->sched_src_index,
                            plan->row_slot, base + L.rows, row_slot_loc, ns, sms, stream),
             "pull dispatch launch");
    return run_expert_ffn(base + L.rows, ns, H, I, w_gate, w_up, w_down, ep->e_loc, row_slot_loc, chunks, counts2,
                          base + L.h, nullptr, status, kDefaultTimeoutNs, stream, nullptr, nullptr, nullptr, push_dev,
                          S_r * plan->k, tune_rows);
}

}  // namespace mok

extern "C" {

int mok_ep_dispatch_ffn(const mok_plan_t* plan, const mok_ep_t* ep, int H, int I, const void* w_gate,
                        const void* w_up, const void* w_down, uint32_t step, uint64_t timeout_ns, void* ws,
                        size_t ws_bytes, mok_stream_t stream) {
    return ep_dispatch(plan, ep, H, I, w_gate, w_up, w_down, nullptr, step, timeout_ns, ws, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

int mok_ep_dispatch_ffn_mxfp8(const mok_plan_t* plan, const mok_ep_t* ep, int H, int I, const mok_mxfp8_weights* w,
                              uint32_t step, uint64_t timeout_ns, void* ws, size_t ws_bytes, mok_stream_t stream) {
    if (!w) return fail(MOK_ERR_INVALID_ARG, "NULL MXFP8 weights");
    return ep_dispatch(plan, ep, H, I, nullptr, nullptr, nullptr, w, step, timeout_ns, ws, ws_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

int mok_ep_combine(const mok_plan_t* plan, const mok_ep_t* ep, int H, uint32_t step, uint64_t timeout_ns, void* y,
                   void* ws, size_t ws_bytes, mok_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int rc = check_plan(plan);
    if (rc) return rc;
    if ((rc = check_ep(plan, ep, H))) return rc;
    if (step < 1) return fail(MOK_ERR_INVALID_ARG, "step counts from 1");
    if ((rc = check_ws(ws, ws_bytes, sizeof(DevStatus)))) return rc;
    if (!y) return fail(MOK_ERR_INVALID_ARG, "y is NULL");
    if (reinterpret_cast<uintptr_t>(y) & 15u) return fail(MOK_ERR_UNSUPPORTED, "y must be 16-byte aligned");
    DevStatus* status = static_cast<DevStatus*>(ws);
    if ((rc = ep_barrier(plan, ep, H, step, 2, timeout_ns, status, stream))) return rc;
    const int S_r = plan->T / plan->R;
    if (S_r == 0) return MOK_OK;
    const int sms = device_sms(nullptr);
    if (sms <= 0) return fail(MOK_ERR_CUDA, "no CUDA device");
    ShardsOut ys{};
    ys.p[0] = y;
    MOK_CUDA(launch_combine(ep->slots[ep->g], ep->mxfp8 ? MOK_SLOTS_BF16 : MOK_SLOTS_F16S,
                            plan->gates + (size_t)ep->g * S_r * plan->k, S_r, plan->k, H, S_r, ys, sms, stream),
             "combine launch");
    return MOK_OK;
}

int mok_ipc_export(const void* dptr, void* handle, size_t* offset) {
    if (!dptr || !handle || !offset) return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    static_assert(sizeof(cudaIpcMemHandle_t) == MOK_IPC_HANDLE_BYTES, "IPC handle size");
    AddrRangeFn range = get_addr_range();
    if (!range) return fail(MOK_ERR_CUDA, "cuMemGetAddressRange unavailable");
    CUdeviceptr b = 0;
    size_t size = 0;
    if (range(&b, &size, reinterpret_cast<CUdeviceptr>(dptr)) != CUDA_SUCCESS)
        return fail(MOK_ERR_CUDA, "cuMemGetAddressRange failed (not device memory?)");
    cudaIpcMemHandle_t h;
    MOK_CUDA(cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(b)), "cudaIpcGetMemHandle");
    memcpy(handle, &h, sizeof h);
    *offset = (size_t)(reinterpret_cast<CUdeviceptr>(dptr) - b);
    return MOK_OK;
}

int mok_ipc_import(const void* handle, void** base) {
    if (!handle || !base) return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, sizeof h);
    MOK_CUDA(cudaIpcOpenMemHandle(base, h, cudaIpcMemLazyEnablePeerAccess), "cudaIpcOpenMemHandle");
    return MOK_OK;
}

int mok_ipc_close(void* base) {
    if (!base) return fail(MOK_ERR_INVALID_ARG, "NULL pointer");
    MOK_CUDA(cudaIpcCloseMemHandle(base), "cudaIpcCloseMemHandle");
    return MOK_OK;
}

}  // extern "C"

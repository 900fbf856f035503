// capi.cu -- the extern "C" boundary of libmsa: argument validation on the host, workspace
// sizing, TMA descriptor encoding, and kernel launches on the caller's stream. Nothing here
// allocates device memory or synchronises (except msa_get_device_status, which must).
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "msa_common.cuh"

namespace msa {
// kernels (other translation units)
void launch_pool(const void*, int, int, int64_t, float*, int64_t, float*, cudaStream_t);
void launch_append(const void*, const void*, const void*, const int32_t*, int, int, void*, void*, int64_t,
                   float*, float*, int64_t, void*, cudaStream_t);
msa_status_t launch_select_prefill_tc(const void*, int, int, int64_t, int64_t, const float*, int64_t, int32_t*, void*,
                                      cudaStream_t);
size_t select_prefill_ws_bytes(int, int, int64_t);
void launch_pool_chunk(const void*, int, int, int64_t, int64_t, float*, int64_t, float*, cudaStream_t);
void launch_select_decode(const void*, const int32_t*, int64_t, int, int, const float*, int64_t, int32_t*,
                          void*, cudaStream_t);
size_t decode_select_ws_bytes(int, int, int64_t);
msa_status_t launch_attn_decode(const void*, const void*, const void*, int64_t, const int32_t*, int64_t, const int32_t*,
                                int, int, int, void*, float*, void*, cudaStream_t, const void*, const void*,
                                const float*, const float*, int64_t);
void launch_fp8_quantize(const void*, const void*, int64_t, int64_t, int, int, void*, void*, float*, float*, int64_t,
                         cudaStream_t);
void launch_fp8_close(const void*, const void*, int64_t, const int32_t*, int, int, void*, void*, float*, float*, int64_t,
                      void*, cudaStream_t);
size_t decode_attn_ws_bytes(int, int, int);
size_t prefill_attn_ws_bytes(int, int64_t, int, int, int64_t);
size_t backward_ws_bytes(int, int64_t, int, int);
msa_status_t launch_attn_backward(const void*, const void*, const void*, int64_t, int, int, int, const int32_t*,
                                  const void*, const float*, const void*, float*, float*, float*, void*, cudaStream_t);
msa_status_t launch_attn_prefill_tc(const void*, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, int64_t,
                                    int64_t, int, int, int, const int32_t*, void*, float*, void*, cudaStream_t);

static std::atomic<uint64_t> g_launches{0};
void count_launch(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// kernel timing records: (kernel id, start event, end event) in launch order
struct TimingRec {
    int kid;
    cudaEvent_t a, b;
};
static std::atomic<bool> g_timing{false};
static std::mutex g_timing_mu;
static std::vector<TimingRec> g_timing_recs;

KernelTimer::KernelTimer(int kid, cudaStream_t st) : kid_(kid), st_(st) {
    count_launch();
    if (!g_timing.load(std::memory_order_relaxed)) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return;
    if (cudaEventCreate(&a_) != cudaSuccess) {
        a_ = nullptr;
        return;
    }
    if (cudaEventCreate(&b_) != cudaSuccess) {
        cudaEventDestroy(a_);
        a_ = nullptr;
        return;
    }
    cudaEventRecord(a_, st);
}

KernelTimer::~KernelTimer() {
    if (a_ == nullptr) return;
    cudaEventRecord(b_, st_);
    std::lock_guard<std::mutex> lk(g_timing_mu);
    g_timing_recs.push_back(TimingRec{kid_, a_, b_});
}

thread_local int g_last_cuda_error = 0;

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> cached{nullptr};
    PFN_cuTensorMapEncodeTiled_v12000 fn = cached.load(std::memory_order_acquire);
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
            cached.store(fn, std::memory_order_release);
        }
    }
    return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

msa_status_t check_shape(const msa_shape_t* s) {
    if (s == nullptr) return MSA_ERR_INVALID_ARGUMENT;
    if (s->batch < 1 || s->n_q_heads < 1 || s->n_kv_groups < 1 || s->batch > 65535 || s->n_kv_groups > 65535)
        return MSA_ERR_INVALID_ARGUMENT;
    if (s->n_q_heads % s->n_kv_groups != 0) return MSA_ERR_INVALID_ARGUMENT;
    if (s->head_dim != kHeadDim || s->index_dim != kIndexDim || s->block_size != kBlock || s->top_k != kTopK)
        return MSA_ERR_UNSUPPORTED;
    const int hg = s->n_q_heads / s->n_kv_groups;
    if (!(hg == 1 || hg == 2 || hg == 4 || hg == 8 || hg == 16)) return MSA_ERR_UNSUPPORTED;
    return MSA_OK;
}

msa_status_t cuda_status() {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        g_last_cuda_error = int(e);
        return MSA_ERR_CUDA;
    }
    return MSA_OK;
}
// bf16 matrix of `rows` x `cols` (row stride = cols), box = box_cols x box_rows, 128B swizzle
msa_status_t make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                            uint32_t box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return MSA_ERR_CUDA;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error = int(r);
        return MSA_ERR_CUDA;
    }
    return MSA_OK;
}
msa_status_t make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                          uint32_t box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return MSA_ERR_CUDA;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error = int(r);
        return MSA_ERR_CUDA;
    }
    return MSA_OK;
}
// Key / value rows of every (sequence, group) as a 3-D bf16 tensor (64-column halves, rows,
// sequence x group) whose row extent is `rows_valid` of the `l_cap` rows each (sequence, group)
// holds: a 128-row box that reaches past the valid rows is zero-filled there by the copy.
msa_status_t make_tmap_kv3d(CUtensorMap* m, const void* base, uint64_t rows_valid, uint64_t l_cap, uint64_t nbg) {
    auto fn = encode_fn();
    if (fn == nullptr) return MSA_ERR_CUDA;
    cuuint64_t dims[3] = {uint64_t(kHeadDim), rows_valid, nbg};
    cuuint64_t strides[2] = {uint64_t(kHeadDim) * 2, l_cap * kHeadDim * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error = int(r);
        return MSA_ERR_CUDA;
    }
    return MSA_OK;
}
msa_status_t make_tmap_qidx(CUtensorMap* m, const void* base, int G, uint64_t rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return MSA_ERR_CUDA;
    cuuint64_t dims[3] = {uint64_t(kIndexDim), uint64_t(G), rows};
    cuuint64_t strides[2] = {uint64_t(kIndexDim) * 2, uint64_t(G) * kIndexDim * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error = int(r);
        return MSA_ERR_CUDA;
    }
    return MSA_OK;
}
msa_status_t make_tmap_split(CUtensorMap* m, const void* base, uint64_t nbp, uint64_t nbg3) {
    auto fn = encode_fn();
    if (fn == nullptr) return MSA_ERR_CUDA;
    cuuint64_t dims[3] = {uint64_t(kIndexDim), nbp, nbg3};
    cuuint64_t strides[2] = {uint64_t(kIndexDim) * 2, nbp * kIndexDim * 2};
    cuuint32_t box[3] = {64, 32, 3};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error = int(r);
        return MSA_ERR_CUDA;
    }
    return MSA_OK;
}
msa_status_t make_tmap_q_rows(CUtensorMap* m, const void* base, uint64_t rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return MSA_ERR_CUDA;
    cuuint64_t dims[3] = {64, rows, 2};
    cuuint64_t strides[2] = {uint64_t(kHeadDim) * 2, 128};      // bytes: next row, next d half
    cuuint32_t box[3] = {64, 8, 2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        g_last_cuda_error = int(r);
        return MSA_ERR_CUDA;
    }
    return MSA_OK;
}
}  // namespace msa

using namespace msa;

namespace {

constexpr int64_t kMaxPos = kMaxDecodePos;

#define MSA_TRY(x)                            \
    do {                                      \
        msa_status_t _s = (x);                \
        if (_s != MSA_OK) return _s;          \
    } while (0)

#define MSA_REQ(cond, code)                   \
    do {                                      \
        if (!(cond)) return (code);           \
    } while (0)

size_t header_only() { return sizeof(WsHeader); }

size_t ws_size(const msa_shape_t* s, int32_t op, int64_t n) {
    if (check_shape(s) != MSA_OK || n < 0) return 0;
    const int hg = s->n_q_heads / s->n_kv_groups;
    switch (op) {
        case MSA_OP_INDEX_SELECT_PREFILL:
            if (n < 1) return 0;
            return select_prefill_ws_bytes(s->batch, s->n_kv_groups, n);
        case MSA_OP_INDEX_SELECT_DECODE:
            if (n > kMaxPos) return 0;
            return decode_select_ws_bytes(s->batch, s->n_kv_groups, n);
        case MSA_OP_ATTN_PREFILL:
            if (n < 1) return 0;
            return prefill_attn_ws_bytes(s->batch, n, s->n_kv_groups, hg, 0);
        case MSA_OP_ATTN_DECODE: return decode_attn_ws_bytes(s->batch, s->n_kv_groups, hg);
        case MSA_OP_ATTN_PREFILL_BACKWARD:
            if (n < 1) return 0;
            return backward_ws_bytes(s->batch, n, s->n_kv_groups, hg);
        default: return 0;
    }
}

// Argument checks shared by the decode entry points and msa_decode_step (shape already checked).
msa_status_t check_select_decode(const msa_shape_t* shape, int64_t max_pos, int64_t nb_cap, const void* workspace,
                                 size_t workspace_bytes) {
    MSA_REQ(max_pos <= kMaxPos, MSA_ERR_UNSUPPORTED);
    MSA_REQ(nb_cap >= max_pos / kBlock, MSA_ERR_INVALID_ARGUMENT);
    const size_t need = ws_size(shape, MSA_OP_INDEX_SELECT_DECODE, max_pos);
    MSA_REQ(workspace != nullptr && aligned16(workspace) && workspace_bytes >= need, MSA_ERR_WORKSPACE);
    return MSA_OK;
}

msa_status_t check_append(const void* k_idx_new, const void* k_new, const void* v_new, const int32_t* ctx_len,
                          const void* k_cache, const void* v_cache, int64_t l_cap, const float* tail_sum,
                          const float* pooled, int64_t nb_cap, const void* workspace, size_t workspace_bytes) {
    MSA_REQ(k_idx_new && aligned16(k_idx_new) && ctx_len && tail_sum && aligned16(tail_sum) && pooled &&
                aligned16(pooled),
            MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ((k_new == nullptr) == (v_new == nullptr), MSA_ERR_INVALID_ARGUMENT);
    if (k_new != nullptr)
        MSA_REQ(aligned16(k_new) && aligned16(v_new) && k_cache && v_cache && aligned16(k_cache) &&
                    aligned16(v_cache) && l_cap >= 1,
                MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(nb_cap >= 1, MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(workspace != nullptr && workspace_bytes >= header_only(), MSA_ERR_WORKSPACE);
    return MSA_OK;
}

msa_status_t check_attn_decode(const msa_shape_t* shape, const void* q, const void* k_cache, const void* v_cache,
                               int64_t l_cap, const int32_t* q_pos, int64_t max_pos, const int32_t* sel,
                               const void* out, const float* lse, const void* workspace, size_t workspace_bytes) {
    MSA_REQ(q && k_cache && v_cache && q_pos && sel && out && aligned16(q) && aligned16(k_cache) &&
                aligned16(v_cache) && aligned16(sel) && aligned16(out) &&
                (lse == nullptr || (reinterpret_cast<uintptr_t>(lse) & 3u) == 0),
            MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(l_cap >= 1 && max_pos >= 0 && max_pos < l_cap, MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(int64_t(shape->batch) * shape->n_kv_groups * l_cap + kBlock < (int64_t(1) << 31), MSA_ERR_UNSUPPORTED);
    const size_t need = ws_size(shape, MSA_OP_ATTN_DECODE, max_pos);
    MSA_REQ(workspace != nullptr && aligned16(workspace) && workspace_bytes >= need, MSA_ERR_WORKSPACE);
    return MSA_OK;
}

}  // namespace

extern "C" {

int32_t msa_abi_version(void) { return 1; }

const char* msa_status_string(msa_status_t s) {
    switch (s) {
        case MSA_OK: return "ok";
        case MSA_ERR_INVALID_ARGUMENT: return "invalid argument";
        case MSA_ERR_UNSUPPORTED: return "unsupported shape or constant";
        case MSA_ERR_WORKSPACE: return "workspace missing or too small";
        case MSA_ERR_CUDA: return "CUDA error";
        case MSA_ERR_TIMEOUT: return "device wait timed out";
        case MSA_ERR_DEVICE_BOUNDS: return "device index out of bounds";
        default: return "unknown status";
    }
}

int32_t msa_last_cuda_error(void) { return g_last_cuda_error; }

uint64_t msa_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int32_t msa_kernel_timing_enable(int32_t on) { return g_timing.exchange(on != 0) ? 1 : 0; }

int32_t msa_kernel_timing_read(int32_t* kernel, float* ms, int32_t cap) {
    std::lock_guard<std::mutex> lk(g_timing_mu);
    int32_t n = 0;
    bool failed = false;
    for (const TimingRec& r : g_timing_recs) {
        if (!failed && n < cap && kernel != nullptr && ms != nullptr) {
            float t = 0.f;
            if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
                failed = true;
            } else {
                kernel[n] = r.kid;
                ms[n] = t;
                ++n;
            }
        }
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    g_timing_recs.clear();
    return failed ? -1 : n;
}

size_t msa_workspace_size(const msa_shape_t* shape, int32_t op, int64_t n) { return ws_size(shape, op, n); }

msa_status_t msa_pool_index_keys(const msa_shape_t* shape, const void* k_idx, int64_t n_tokens, float* pooled,
                                 int64_t nb_cap, float* tail_sum, msa_stream_t stream) {
    MSA_CALL_RANGE();
    MSA_TRY(check_shape(shape));
    MSA_REQ(n_tokens >= 0 && n_tokens < (int64_t(1) << 31), MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(n_tokens == 0 || (k_idx != nullptr && aligned16(k_idx)), MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(nb_cap >= n_tokens / kBlock && nb_cap >= 0, MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(n_tokens < kBlock || (pooled != nullptr && aligned16(pooled)), MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(tail_sum == nullptr || aligned16(tail_sum), MSA_ERR_INVALID_ARGUMENT);
    launch_pool(k_idx, shape->batch, shape->n_kv_groups, n_tokens, pooled, nb_cap, tail_sum,
                reinterpret_cast<cudaStream_t>(stream));
    return cuda_status();
}

msa_status_t msa_index_select(const msa_shape_t* shape, const void* q_idx, int64_t n_queries, const int32_t* q_pos,
                              int64_t max_pos, const float* pooled, int64_t nb_cap, int32_t* sel, void* workspace,
                              size_t workspace_bytes, msa_stream_t stream) {
    MSA_CALL_RANGE();
    MSA_TRY(check_shape(shape));
    MSA_REQ(q_idx != nullptr && aligned16(q_idx) && sel != nullptr && aligned16(sel), MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(pooled == nullptr ? max_pos < kBlock : aligned16(pooled), MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(n_queries >= 1 && n_queries < (int64_t(1) << 31), MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(max_pos >= 0 && nb_cap >= 0, MSA_ERR_INVALID_ARGUMENT);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int B = shape->batch, G = shape->n_kv_groups;
    if (q_pos == nullptr) {                        // prefill: positions 0..n_queries-1
        MSA_REQ(max_pos >= n_queries - 1, MSA_ERR_INVALID_ARGUMENT);
        MSA_REQ(nb_cap >= (n_queries - 1) / kBlock, MSA_ERR_INVALID_ARGUMENT);
        const size_t need = ws_size(shape, MSA_OP_INDEX_SELECT_PREFILL, n_queries);
        MSA_REQ(workspace != nullptr && aligned16(workspace) && need > 0 && workspace_bytes >= need, MSA_ERR_WORKSPACE);
        MSA_TRY(launch_select_prefill_tc(q_idx, B, G, n_queries, 0, pooled, nb_cap, sel, workspace, st));
    } else {                                       // decode: one query per sequence at q_pos[b]
        MSA_REQ(n_queries == 1, MSA_ERR_INVALID_ARGUMENT);
        MSA_TRY(check_select_decode(shape, max_pos, nb_cap, workspace, workspace_bytes));
        launch_select_decode(q_idx, q_pos, max_pos, B, G, pooled, nb_cap, sel, workspace, st);
    }
    return cuda_status();
}

}  // extern "C"

namespace {
// Main Branch prefill for the n queries at positions P .. P + n - 1 against k, v [B, G, l_cap, d]
// (P = 0, l_cap = n: a whole prefill).
msa_status_t attn_prefill_impl(const msa_shape_t* shape, const void* q, const void* k, const void* v, int64_t l_cap,
                               int64_t P, int64_t n_tokens, const int32_t* sel, void* out, float* lse,
                               void* workspace, size_t workspace_bytes, msa_stream_t stream) {
    MSA_TRY(check_shape(shape));
    MSA_REQ(n_tokens >= 1 && n_tokens < (int64_t(1) << 31) && P >= 0 && P + n_tokens <= l_cap, MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(q && k && v && sel && out && aligned16(q) && aligned16(k) && aligned16(v) && aligned16(sel) &&
                aligned16(out) && (lse == nullptr || (reinterpret_cast<uintptr_t>(lse) & 3u) == 0),
            MSA_ERR_INVALID_ARGUMENT);
    const int B = shape->batch, G = shape->n_kv_groups, Hq = shape->n_q_heads, hg = Hq / G;
    // int32 device indexing: list entries, TMA row coordinates (query rows, key/value rows, and
    // the partial rows: one per token, query head and selected block), per-block histogram in
    // shared memory
    MSA_REQ(int64_t(B) * n_tokens * G * (kTopK - 1) < (int64_t(1) << 31) &&
                int64_t(B) * n_tokens * Hq * kTopK < (int64_t(1) << 31) &&
                int64_t(B) * G * l_cap + kBlock < (int64_t(1) << 31) &&
                (P + n_tokens + kBlock - 1) / kBlock <= 48 * 1024,
            MSA_ERR_UNSUPPORTED);
    const size_t need = prefill_attn_ws_bytes(B, n_tokens, G, hg, P);
    MSA_REQ(workspace != nullptr && aligned16(workspace) && need > 0 && workspace_bytes >= need, MSA_ERR_WORKSPACE);
    CUtensorMap tmQ, tmK, tmV;
    MSA_TRY(make_tmap_bf16(&tmQ, q, uint64_t(B) * n_tokens * Hq, kHeadDim, 64, uint32_t(hg)));
    // rows past P + n_tokens (the chunk's last position) read as zeros
    MSA_TRY(make_tmap_kv3d(&tmK, k, uint64_t(P + n_tokens), uint64_t(l_cap), uint64_t(B) * G));
    MSA_TRY(make_tmap_kv3d(&tmV, v, uint64_t(P + n_tokens), uint64_t(l_cap), uint64_t(B) * G));
    MSA_TRY(launch_attn_prefill_tc(q, tmQ, tmK, tmV, n_tokens, P, B, G, hg, sel, out, lse, workspace,
                                   reinterpret_cast<cudaStream_t>(stream)));
    return cuda_status();
}
}  // namespace

extern "C" {

msa_status_t msa_sparse_attn_prefill(const msa_shape_t* shape, const void* q, const void* k, const void* v,
                                     int64_t n_tokens, const int32_t* sel, void* out, float* lse, void* workspace,
                                     size_t workspace_bytes, msa_stream_t stream) {
    MSA_CALL_RANGE();
    return attn_prefill_impl(shape, q, k, v, n_tokens, 0, n_tokens, sel, out, lse, workspace, workspace_bytes,
                             stream);
}

msa_status_t msa_sparse_attn_prefill_backward(const msa_shape_t* shape, const void* q, const void* k, const void* v,
                                              int64_t n_tokens, const int32_t* sel, const void* out, const float* lse,
                                              const void* d_out, float* dq, float* dk, float* dv, void* workspace,
                                              size_t workspace_bytes, msa_stream_t stream) {
    MSA_CALL_RANGE();
    MSA_TRY(check_shape(shape));
    MSA_REQ(n_tokens >= 1 && n_tokens < (int64_t(1) << 31), MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(q && k && v && sel && out && lse && d_out && dq && dk && dv && aligned16(q) && aligned16(k) &&
                aligned16(v) && aligned16(sel) && aligned16(out) && aligned16(d_out) && aligned16(dq) &&
                aligned16(dk) && aligned16(dv) && (reinterpret_cast<uintptr_t>(lse) & 3u) == 0,
            MSA_ERR_INVALID_ARGUMENT);
    const int B = shape->batch, G = shape->n_kv_groups, Hq = shape->n_q_heads, hg = Hq / G;
    MSA_REQ(int64_t(B) * n_tokens * G * (kTopK - 1) < (int64_t(1) << 31) &&
                int64_t(B) * n_tokens * Hq * kTopK < (int64_t(1) << 31) &&
                (n_tokens + kBlock - 1) / kBlock <= 48 * 1024,
            MSA_ERR_UNSUPPORTED);
    const size_t need = backward_ws_bytes(B, n_tokens, G, hg);
    MSA_REQ(workspace != nullptr && aligned16(workspace) && workspace_bytes >= need, MSA_ERR_WORKSPACE);
    MSA_TRY(launch_attn_backward(q, k, v, n_tokens, B, G, hg, sel, out, lse, d_out, dq, dk, dv, workspace,
                                 reinterpret_cast<cudaStream_t>(stream)));
    return cuda_status();
}

size_t msa_prefill_chunk_workspace_size(const msa_shape_t* shape, int64_t q_start, int64_t n_queries) {
    if (check_shape(shape) != MSA_OK || q_start < 0 || n_queries < 1) return 0;
    return prefill_attn_ws_bytes(shape->batch, n_queries, shape->n_kv_groups, shape->n_q_heads / shape->n_kv_groups,
                                 q_start);
}

msa_status_t msa_pool_index_keys_chunk(const msa_shape_t* shape, const void* k_idx, int64_t q_start, int64_t n,
                                       float* pooled, int64_t nb_cap, float* tail_sum, msa_stream_t stream) {
    MSA_CALL_RANGE();
    MSA_TRY(check_shape(shape));
    MSA_REQ(n >= 1 && q_start >= 0 && q_start + n < (int64_t(1) << 31), MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(k_idx && aligned16(k_idx) && tail_sum && aligned16(tail_sum), MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(nb_cap >= (q_start + n) / kBlock && (q_start + n < kBlock * (q_start / kBlock + 1) ||
                                                 (pooled != nullptr && aligned16(pooled))),
            MSA_ERR_INVALID_ARGUMENT);
    launch_pool_chunk(k_idx, shape->batch, shape->n_kv_groups, n, q_start, pooled, nb_cap, tail_sum,
                      reinterpret_cast<cudaStream_t>(stream));
    return cuda_status();
}

msa_status_t msa_index_select_chunk(const msa_shape_t* shape, const void* q_idx, int64_t q_start, int64_t n,
                                    const float* pooled, int64_t nb_cap, int32_t* sel, void* workspace,
                                    size_t workspace_bytes, msa_stream_t stream) {
    MSA_CALL_RANGE();
    MSA_TRY(check_shape(shape));
    MSA_REQ(q_idx && aligned16(q_idx) && sel && aligned16(sel), MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(n >= 1 && q_start >= 0 && q_start + n < (int64_t(1) << 31), MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(nb_cap >= (q_start + n - 1) / kBlock, MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(pooled == nullptr ? q_start + n - 1 < kBlock : aligned16(pooled), MSA_ERR_INVALID_ARGUMENT);
    const size_t need = ws_size(shape, MSA_OP_INDEX_SELECT_PREFILL, q_start + n);
    MSA_REQ(workspace != nullptr && aligned16(workspace) && need > 0 && workspace_bytes >= need, MSA_ERR_WORKSPACE);
    MSA_TRY(launch_select_prefill_tc(q_idx, shape->batch, shape->n_kv_groups, n, q_start, pooled, nb_cap, sel,
                                     workspace, reinterpret_cast<cudaStream_t>(stream)));
    return cuda_status();
}

msa_status_t msa_sparse_attn_prefill_chunk(const msa_shape_t* shape, const void* q, const void* k_cache,
                                           const void* v_cache, int64_t l_cap, int64_t q_start, int64_t n,
                                           const int32_t* sel, void* out, float* lse, void* workspace,
                                           size_t workspace_bytes, msa_stream_t stream) {
    MSA_CALL_RANGE();
    return attn_prefill_impl(shape, q, k_cache, v_cache, l_cap, q_start, n, sel, out, lse, workspace,
                             workspace_bytes, stream);
}

msa_status_t msa_pooled_keys_append(const msa_shape_t* shape, const void* k_idx_new, const void* k_new,
                                    const void* v_new, const int32_t* ctx_len, void* k_cache, void* v_cache,
                                    int64_t l_cap, float* tail_sum, float* pooled, int64_t nb_cap, void* workspace,
                                    size_t workspace_bytes, msa_stream_t stream) {
    MSA_CALL_RANGE();
    MSA_TRY(check_shape(shape));
    MSA_TRY(check_append(k_idx_new, k_new, v_new, ctx_len, k_cache, v_cache, l_cap, tail_sum, pooled, nb_cap,
                         workspace, workspace_bytes));
    launch_append(k_idx_new, k_new, v_new, ctx_len, shape->batch, shape->n_kv_groups, k_cache, v_cache,
                  k_new ? l_cap : int64_t(1) << 62, tail_sum, pooled, nb_cap, workspace,
                  reinterpret_cast<cudaStream_t>(stream));
    return cuda_status();
}

msa_status_t msa_sparse_attn_decode(const msa_shape_t* shape, const void* q, const void* k_cache,
                                    const void* v_cache, int64_t l_cap, const int32_t* q_pos, int64_t max_pos,
                                    const int32_t* sel, void* out, float* lse, void* workspace,
                                    size_t workspace_bytes, msa_stream_t stream) {
    MSA_CALL_RANGE();
    MSA_TRY(check_shape(shape));
    MSA_TRY(check_attn_decode(shape, q, k_cache, v_cache, l_cap, q_pos, max_pos, sel, out, lse, workspace,
                              workspace_bytes));
    const int B = shape->batch, G = shape->n_kv_groups;
    MSA_TRY(launch_attn_decode(k_cache, v_cache, q, l_cap, q_pos, max_pos, sel, B, G, shape->n_q_heads / G, out, lse,
                               workspace, reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr, nullptr, nullptr,
                               0));
    return cuda_status();
}

msa_status_t msa_decode_step(const msa_shape_t* shape, const void* q, const void* q_idx, const void* k_idx_new,
                             const void* k_new, const void* v_new, const int32_t* ctx_len, void* k_cache,
                             void* v_cache, int64_t l_cap, float* tail_sum, float* pooled, int64_t nb_cap,
                             int64_t max_pos, int32_t* sel, void* out, float* lse, void* ws_select,
                             size_t ws_select_bytes, void* ws_append, size_t ws_append_bytes, void* ws_attn,
                             size_t ws_attn_bytes, msa_stream_t stream) {
    MSA_CALL_RANGE();
    MSA_TRY(check_shape(shape));
    // every argument of the three steps is checked before the first launch
    MSA_REQ(q_idx != nullptr && aligned16(q_idx) && sel != nullptr && aligned16(sel) && aligned16(pooled),
            MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(k_new != nullptr && max_pos >= 0 && nb_cap >= 0, MSA_ERR_INVALID_ARGUMENT);
    MSA_TRY(check_select_decode(shape, max_pos, nb_cap, ws_select, ws_select_bytes));
    MSA_TRY(check_append(k_idx_new, k_new, v_new, ctx_len, k_cache, v_cache, l_cap, tail_sum, pooled, nb_cap,
                         ws_append, ws_append_bytes));
    MSA_TRY(check_attn_decode(shape, q, k_cache, v_cache, l_cap, ctx_len, max_pos, sel, out, lse, ws_attn,
                              ws_attn_bytes));
    const int B = shape->batch, G = shape->n_kv_groups, Hg = shape->n_q_heads / G;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    launch_select_decode(q_idx, ctx_len, max_pos, B, G, pooled, nb_cap, sel, ws_select, st);
    launch_append(k_idx_new, k_new, v_new, ctx_len, B, G, k_cache, v_cache, l_cap, tail_sum, pooled, nb_cap, ws_append,
                  st);
    MSA_TRY(launch_attn_decode(k_cache, v_cache, q, l_cap, ctx_len, max_pos, sel, B, G, Hg, out, lse, ws_attn, st,
                               nullptr, nullptr, nullptr, nullptr, 0));
    return cuda_status();
}

msa_status_t msa_fp8_quantize_blocks(const msa_shape_t* shape, const void* k_cache, const void* v_cache, int64_t l_cap,
                                     int64_t n_tokens, void* k_codes, void* v_codes, float* k_scale, float* v_scale,
                                     int64_t nb_cap, msa_stream_t stream) {
    MSA_CALL_RANGE();
    MSA_TRY(check_shape(shape));
    MSA_REQ(n_tokens >= 0 && l_cap >= n_tokens && l_cap >= 1, MSA_ERR_INVALID_ARGUMENT);
    const int64_t nblk = n_tokens / kBlock;
    MSA_REQ(nb_cap >= nblk && nblk <= 65535, MSA_ERR_INVALID_ARGUMENT);
    if (nblk == 0) return MSA_OK;
    MSA_REQ(k_cache && v_cache && k_codes && v_codes && k_scale && v_scale && aligned16(k_cache) &&
                aligned16(v_cache) && aligned16(k_codes) && aligned16(v_codes) &&
                (reinterpret_cast<uintptr_t>(k_scale) & 3u) == 0 && (reinterpret_cast<uintptr_t>(v_scale) & 3u) == 0,
            MSA_ERR_INVALID_ARGUMENT);
    launch_fp8_quantize(k_cache, v_cache, l_cap, nblk, shape->batch, shape->n_kv_groups, k_codes, v_codes, k_scale,
                        v_scale, nb_cap, reinterpret_cast<cudaStream_t>(stream));
    return cuda_status();
}

msa_status_t msa_fp8_close_blocks(const msa_shape_t* shape, const int32_t* ctx_len, const void* k_cache,
                                  const void* v_cache, int64_t l_cap, void* k_codes, void* v_codes, float* k_scale,
                                  float* v_scale, int64_t nb_cap, void* workspace, size_t workspace_bytes,
                                  msa_stream_t stream) {
    MSA_CALL_RANGE();
    MSA_TRY(check_shape(shape));
    MSA_REQ(ctx_len && k_cache && v_cache && k_codes && v_codes && k_scale && v_scale && aligned16(k_cache) &&
                aligned16(v_cache) && aligned16(k_codes) && aligned16(v_codes) &&
                (reinterpret_cast<uintptr_t>(k_scale) & 3u) == 0 && (reinterpret_cast<uintptr_t>(v_scale) & 3u) == 0,
            MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(l_cap >= kBlock && nb_cap >= 1, MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(workspace != nullptr && workspace_bytes >= header_only(), MSA_ERR_WORKSPACE);
    launch_fp8_close(k_cache, v_cache, l_cap, ctx_len, shape->batch, shape->n_kv_groups, k_codes, v_codes, k_scale,
                     v_scale, nb_cap, workspace, reinterpret_cast<cudaStream_t>(stream));
    return cuda_status();
}

msa_status_t msa_sparse_attn_decode_fp8(const msa_shape_t* shape, const void* q, const void* k_codes,
                                        const void* v_codes, const float* k_scale, const float* v_scale,
                                        int64_t nb_cap, const void* k_cache, const void* v_cache, int64_t l_cap,
                                        const int32_t* q_pos, int64_t max_pos, const int32_t* sel, void* out,
                                        float* lse, void* workspace, size_t workspace_bytes, msa_stream_t stream) {
    MSA_CALL_RANGE();
    MSA_TRY(check_shape(shape));
    MSA_REQ(q && k_codes && v_codes && k_scale && v_scale && k_cache && v_cache && q_pos && sel && out &&
                aligned16(q) && aligned16(k_codes) && aligned16(v_codes) && aligned16(k_cache) &&
                aligned16(v_cache) && aligned16(sel) && aligned16(out) &&
                (reinterpret_cast<uintptr_t>(k_scale) & 3u) == 0 && (reinterpret_cast<uintptr_t>(v_scale) & 3u) == 0 &&
                (lse == nullptr || (reinterpret_cast<uintptr_t>(lse) & 3u) == 0),
            MSA_ERR_INVALID_ARGUMENT);
    MSA_REQ(l_cap >= 1 && max_pos >= 0 && max_pos < l_cap && nb_cap >= max_pos / kBlock, MSA_ERR_INVALID_ARGUMENT);
    const int B = shape->batch, G = shape->n_kv_groups;
    MSA_REQ(int64_t(B) * G * l_cap + kBlock < (int64_t(1) << 31), MSA_ERR_UNSUPPORTED);
    const size_t need = ws_size(shape, MSA_OP_ATTN_DECODE, max_pos);
    MSA_REQ(workspace != nullptr && aligned16(workspace) && workspace_bytes >= need, MSA_ERR_WORKSPACE);
    MSA_TRY(launch_attn_decode(k_cache, v_cache, q, l_cap, q_pos, max_pos, sel, B, G, shape->n_q_heads / G, out, lse,
                               workspace, reinterpret_cast<cudaStream_t>(stream), k_codes, v_codes, k_scale, v_scale,
                               nb_cap));
    return cuda_status();
}

msa_status_t msa_get_device_status(void* workspace, int32_t* info, msa_stream_t stream) {
    MSA_REQ(workspace != nullptr, MSA_ERR_INVALID_ARGUMENT);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    WsHeader h;
    if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return cuda_status();
    if (info) std::memcpy(info, h.info, sizeof(h.info));
    if (h.err != 0) {
        if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
            return cuda_status();
    }
    return static_cast<msa_status_t>(h.err);
}

}  // extern "C"

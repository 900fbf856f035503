// select.cu -- Index Branch scoring and exp-free top-k block selection.
//
// Sources: youmind article "MiniMax M3 sparse attention agents", paragraph "The mechanism
// that changes this" (score the context in blocks, keep the most relevant per query and
// GQA group) and bullet "Predictable cost at every length" (k = 16); KuCoin flash "MiniMax
// launches MSA sparse attention method and MiniMax-M3 model", summary (exp-free top-k).
//
// Decode: one query per (sequence, group). Every score is s_j = q_I . kbar_j in fp32 (the
// 1/sqrt(d_I) factor is an exact power of two and cannot change the order, so it is not
// applied). Ranking uses only compares of order-preserving keys (score, then the inverted block
// id, so equal scores rank the lower block first). The query's own block is added and the ids
// are written ascending. (The prefill selection is in select_tc.cu.)
#include <cooperative_groups.h>

#include "msa_common.cuh"

namespace msa {

constexpr int kKeep = kTopK - 1;   // best fully-past blocks kept besides the diagonal one

__device__ __forceinline__ void write_all_blocks(int32_t* out, int c) {
    int4* o = reinterpret_cast<int4*>(out);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        int4 v;
        v.x = (4 * q + 0 <= c) ? 4 * q + 0 : -1;
        v.y = (4 * q + 1 <= c) ? 4 * q + 1 : -1;
        v.z = (4 * q + 2 <= c) ? 4 * q + 2 : -1;
        v.w = (4 * q + 3 <= c) ? 4 * q + 3 : -1;
        o[q] = v;
    }
}

// ------------------------------------------------------------------ decode, split + merge
// One query per (sequence, group); its candidates [0, c) are split over 8 k CTAs that form k
// thread-block clusters of 8. A CTA of 4 warps scores its span 128 candidates per pass (each
// warp instruction reads two whole 256-byte pooled rows; 16 loads per lane are in flight), and
// every warp keeps a running best-16 list: the pass's 32 keys are sorted in registers
// (bitonic) and merged into the list (a bitonic merge). The CTA's 4 lists are merged into one
// in shared memory; after a cluster barrier the cluster's first CTA reads the 8 lists over
// distributed shared memory and merges them (3 rounds of pairwise merges). With one cluster
// per (sequence, group) -- the case whenever the batch fills the GPU -- that CTA writes the
// selection; with several, each cluster leaves its best 15 in the workspace and the cluster
// that arrives last merges those lists the same way (the arrival counter wraps to zero by
// itself, so the workspace is ready for the next call). No step depends on the data.
int num_sms();

constexpr int kSelThreads = 128;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelCluster = 8;                    // CTAs per cluster
constexpr int kSelMaxClusters = 64;               // clusters per (sequence, group)

// warp: the best 16 of two descending lists a, b of 16 (lanes 0-15 of the result)
__device__ __forceinline__ unsigned long long merge2(const unsigned long long* a, const unsigned long long* b, int lane) {
    return warp_merge_desc(lane < 16 ? a[lane] : b[31 - lane], lane);
}

// warp 0: write the 15 best ids of `best` and the diagonal block c in ascending order
__device__ __forceinline__ void write_selection(const unsigned long long* best, int32_t* out, int c) {
    const int lane = threadIdx.x;
    const int my_id = lane < kKeep ? key_block(best[lane]) : c;
    int rank = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int o = __shfl_sync(0xffffffffu, my_id, i);
        rank += (o < my_id);
    }
    if (lane < 16) out[rank] = my_id;
}

// Merge n <= 8 descending lists of 16 in `l` (n rows of 16) into l[0] with the CTA's warps.
__device__ __forceinline__ void merge8(unsigned long long (*l)[16], int n) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    while (n > 1) {
        const int npairs = n >> 1;
        unsigned long long x = 0ull;
        if (wid < npairs) x = merge2(l[2 * wid], l[2 * wid + 1], lane);
        __syncthreads();
        if (wid < npairs && lane < 16) l[wid][lane] = x;
        if ((n & 1) && wid == kSelWarps - 1 && lane < 16) l[npairs][lane] = l[n - 1][lane];
        __syncthreads();
        n = (n + 1) >> 1;
    }
}

__global__ void __launch_bounds__(kSelThreads, 8) select_decode_kernel(
    const uint16_t* __restrict__ q_idx, const int32_t* __restrict__ q_pos, int64_t max_pos, int G,
    const float* __restrict__ pooled, int64_t nb_cap, int32_t* __restrict__ sel,
    unsigned long long* __restrict__ cand, unsigned int* __restrict__ ctr, WsHeader* hdr) {
    __shared__ __align__(16) float qs[kIndexDim];
    __shared__ float sc[kSelThreads];
    __shared__ unsigned long long lists[kSelCluster][16];     // rank 0 of the cluster uses all 8
    __shared__ int last;
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    grid_dep_launch();                 // the attention kernel may start its prologue
    const int split = blockIdx.x, nsplit = gridDim.x, g = blockIdx.y, b = blockIdx.z;
    const int rank = int(cluster.block_rank()), cl = split / kSelCluster, ncl = nsplit / kSelCluster;
    const int bg = b * G + g;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    // the query row does not depend on the position: load both at once
    const float qx = tid < kIndexDim ? bf16_to_f32(q_idx[size_t(bg) * kIndexDim + tid]) : 0.f;
    const int pos = q_pos[b];
    // every CTA of a cluster belongs to the same (sequence, group): the early exits below are
    // taken by the whole cluster, before its barriers
    // (the writes of these exits wait for the preceding kernel like every other write of sel
    // and of the error word below, whatever that kernel is)
    if (pos < 0 || pos > max_pos || int64_t(pos / kBlock) > nb_cap) {
        grid_dep_wait();
        if (split == 0 && tid == 0) record_error(hdr, MSA_ERR_DEVICE_BOUNDS, KID_SELECT_DECODE, bg, 0, pos);
        return;
    }
    const int c = pos / kBlock;
    int32_t* out = sel + size_t(bg) * kTopK;
    if (c + 1 <= kTopK) {
        grid_dep_wait();
        if (split == 0 && tid == 0) write_all_blocks(out, c);
        return;
    }
    const int span = ((c + nsplit - 1) / nsplit + 31) / 32 * 32;
    const int lo = min(c, split * span), hi = min(c, lo + span);   // may be empty

    if (tid < kIndexDim) qs[tid] = qx;
    __syncthreads();
    const int part = lane & 15, half = lane >> 4;
    const float4 qv = *reinterpret_cast<const float4*>(&qs[4 * part]);
    const float4* rows = reinterpret_cast<const float4*>(pooled + size_t(bg) * nb_cap * kIndexDim);
    unsigned long long best = 0ull;                      // lanes 0-15: this warp's best 16
    for (int base = lo; base < hi; base += kSelThreads) {
        const int r0 = base + wid * 32;                  // this warp's 32 rows
        // the lane's 16 rows in two halves of 8: each half's loads go out back to back and are
        // scored before the next half is loaded (64 registers, so that eight CTAs fit on an SM
        // and a whole decode batch runs in one wave); in the span's last pass rows past the span
        // read its last row and are ignored
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
            float4 v[8];
            if (base + kSelThreads <= hi) {
                ld_nc_f4x8_s512(rows + size_t(r0 + 16 * hb + half) * (kIndexDim / 4) + part, v);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = r0 + 16 * hb + 2 * i + half;
                    v[i] = ld_nc_f4(rows + size_t(r < hi ? r : hi - 1) * (kIndexDim / 4) + part);
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                // fixed order: x, y, z, w, then a butterfly over the 16 lanes of this half-warp
                float d = fmaf(qv.x, v[i].x, 0.f);
                d = fmaf(qv.y, v[i].y, d);
                d = fmaf(qv.z, v[i].z, d);
                d = fmaf(qv.w, v[i].w, d);
#pragma unroll
                for (int off = 8; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
                if (part == 0) sc[wid * 32 + 16 * hb + 2 * i + half] = d;
            }
        }
        __syncwarp();
        const int j = r0 + lane;
        unsigned long long key = j < hi ? sel_key(sc[wid * 32 + lane], j) : 0ull;
        __syncwarp();
        key = warp_sort_desc(key, lane);
        const unsigned long long top16 = __shfl_sync(0xffffffffu, key, 31 - lane);   // lanes 16-31: ascending
        best = warp_merge_desc(lane < 16 ? best : top16, lane);
    }
    if (lane < 16) lists[wid][lane] = best;
    __syncthreads();
    merge8(lists, kSelWarps);                            // this CTA's best 16 in lists[0]
    cluster.sync();                                      // every CTA's list is ready
    if (rank == 0) {
        if (wid == 0) {
            for (int r = 1; r < kSelCluster; ++r) {
                const unsigned long long* rl = cluster.map_shared_rank(&lists[0][0], r);
                if (lane < 16) lists[r][lane] = rl[lane];
            }
        }
        __syncthreads();
        merge8(lists, kSelCluster);                      // the cluster's best 16 in lists[0]
    }
    cluster.sync();                                      // the other CTAs' lists have been read
    grid_dep_wait();
    // The selection does not read what the preceding append writes (only fully-past pooled
    // rows), so it waits for that kernel only before finishing: the attention kernel that waits
    // for this grid then also sees the appended token.
    if (rank != 0) return;
    if (ncl == 1) {                                      // the whole pair in this cluster
        if (wid == 0) write_selection(lists[0], out, c);
        return;
    }
    unsigned long long* mine = cand + (size_t(bg) * ncl + cl) * kKeep;
    if (tid < kKeep) mine[tid] = lists[0][tid];
    __threadfence();
    __syncthreads();
    if (tid == 0) last = (atomicInc(ctr + bg, unsigned(ncl - 1)) == unsigned(ncl - 1));
    __syncthreads();
    if (!last) return;
    __threadfence();
    // merge the ncl cluster lists, 8 at a time, keeping a running best 16 in lists[0]
    const unsigned long long* glists = cand + size_t(bg) * ncl * kKeep;
    for (int l0 = 0; l0 < ncl; l0 += kSelCluster - 1) {
        const int n = min(kSelCluster - 1, ncl - l0);
        for (int i = tid; i < n * 16; i += kSelThreads) {
            const int l = i >> 4, e = i & 15;
            lists[1 + l][e] = e < kKeep ? __ldcg(glists + (l0 + l) * kKeep + e) : 0ull;
        }
        if (l0 == 0 && tid < 16) lists[0][tid] = 0ull;
        __syncthreads();
        merge8(lists, 1 + n);
    }
    if (wid == 0) write_selection(lists[0], out, c);
}

// Clusters per (sequence, group): enough CTAs for about 7 per SM when the batch is small, at
// most one CTA per 128 candidates.
int decode_select_clusters(int B, int G, int64_t max_pos) {
    const int64_t cmax = max_pos / kBlock;
    const int64_t nbg = int64_t(B) * G;
    int64_t n = (int64_t(num_sms()) * 7 + nbg * kSelCluster - 1) / (nbg * kSelCluster);
    const int64_t cap = (cmax + kSelCluster * 128 - 1) / (kSelCluster * 128);
    if (n > cap) n = cap;
    if (n > kSelMaxClusters) n = kSelMaxClusters;
    return int(n < 1 ? 1 : n);
}

// workspace bound, independent of the device: one list per cluster at most
int decode_select_chunks(int64_t max_pos) {
    const int64_t cmax = max_pos / kBlock;
    const int64_t n = cmax <= 0 ? 1 : (cmax + kSelCluster * 128 - 1) / (kSelCluster * 128);
    return int(n < kSelMaxClusters ? (n < 1 ? 1 : n) : kSelMaxClusters);
}

size_t decode_select_ws_bytes(int B, int G, int64_t max_pos) {
    const size_t nbg = size_t(B) * G;
    size_t bytes = sizeof(WsHeader);
    bytes += (nbg * sizeof(unsigned int) + 255) / 256 * 256;
    bytes += nbg * decode_select_chunks(max_pos) * kKeep * sizeof(unsigned long long);
    return bytes;
}

void launch_select_decode(const void* q_idx, const int32_t* q_pos, int64_t max_pos, int B, int G,
                          const float* pooled, int64_t nb_cap, int32_t* sel, void* ws, cudaStream_t st) {
    const size_t nbg = size_t(B) * G;
    char* p = static_cast<char*>(ws);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(p);
    unsigned int* ctr = reinterpret_cast<unsigned int*>(p + sizeof(WsHeader));
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(
        p + sizeof(WsHeader) + (nbg * sizeof(unsigned int) + 255) / 256 * 256);
    const int ncl = decode_select_clusters(B, G, max_pos);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ncl * kSelCluster), static_cast<unsigned>(G), static_cast<unsigned>(B));
    cfg.blockDim = dim3(kSelThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap with the append's tail
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = kSelCluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const KernelTimer kt(KID_SELECT_DECODE, st);
    cudaLaunchKernelEx(&cfg, select_decode_kernel, static_cast<const uint16_t*>(q_idx), q_pos, max_pos, G, pooled,
                       nb_cap, sel, cand, ctr, hdr);
}

}  // namespace msa

// ------------------------------------------------------------------ allocation-free variant
// Some callers cannot allocate device memory when they select blocks: a serving engine that
// hands all device memory to its own pool at start-up and forbids allocation per step, or a
// host thread that must not block on the allocator while the GPU runs. For them the decode
// selection can keep its scratch (the error word, the arrival counters and the per-cluster
// candidate lists of select_decode_kernel) in this file-scope device array instead of a
// caller workspace.
// Every GPU that loads libmsa holds the array until the process exits.
#include <mutex>

namespace msa {

constexpr size_t kNoAllocSelectScratch = size_t(2) << 20;   // 2 MiB per GPU
static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocSelectScratch];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// The device address of g_select_scratch on the current device. The host-side name of the
// array is only a stand-in, so the address is looked up once per device, with that device
// current, and cached.
msa_status_t scratch_on_current_device(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) { g_last_cuda_error = int(e); return MSA_ERR_CUDA; }
    if (dev < 0 || dev >= kMaxDevices) return MSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_select_scratch);
        if (e != cudaSuccess || p == nullptr) { g_last_cuda_error = int(e); return MSA_ERR_CUDA; }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MSA_OK;
}
}  // namespace
}  // namespace msa

extern "C" msa_status_t msa_index_select_decode_noalloc(const msa_shape_t* shape, const void* q_idx,
                                                        const int32_t* q_pos, int64_t max_pos,
                                                        const float* pooled, int64_t nb_cap, int32_t* sel,
                                                        msa_stream_t stream) {
    MSA_CALL_RANGE();
    using namespace msa;
    msa_status_t s = check_shape(shape);
    if (s != MSA_OK) return s;
    if (q_idx == nullptr || !aligned16(q_idx) || q_pos == nullptr || sel == nullptr || !aligned16(sel) ||
        pooled == nullptr || !aligned16(pooled) || max_pos < 0 || nb_cap < max_pos / kBlock)
        return MSA_ERR_INVALID_ARGUMENT;
    if (max_pos > kMaxDecodePos) return MSA_ERR_UNSUPPORTED;
    const int B = shape->batch, G = shape->n_kv_groups;
    if (decode_select_ws_bytes(B, G, max_pos) > kNoAllocSelectScratch) return MSA_ERR_WORKSPACE;
    void* scratch = nullptr;
    s = scratch_on_current_device(&scratch);
    if (s != MSA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: the error word and the arrival counters
    // must start at zero. Rows are preset to -1 so that a query whose position the device finds
    // out of range is left all -1 (this variant has no workspace to report it in).
    const size_t zero_bytes = sizeof(WsHeader) + (size_t(B) * G * sizeof(unsigned int) + 255) / 256 * 256;
    cudaError_t e = cudaMemsetAsync(scratch, 0, zero_bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(sel, 0xFF, size_t(B) * G * kTopK * sizeof(int32_t), st);
    if (e != cudaSuccess) { g_last_cuda_error = int(e); return MSA_ERR_CUDA; }
    launch_select_decode(q_idx, q_pos, max_pos, B, G, pooled, nb_cap, sel, scratch, st);
    return cuda_status();
}

// select.cu -- Index Branch scoring and exp-free top-k block selection.
//
// Sources: youmind article "MiniMax M3 sparse attention agents", paragraph "The mechanism
// that changes this" (score the context in blocks, keep the most relevant per query and
// GQA group) and bullet "Predictable cost at every length" (k = 16); KuCoin flash "MiniMax
// launches MSA sparse attention method and MiniMax-M3 model", summary (exp-free top-k).
//
// Every score is s_j = q_I . kbar_j in fp32 (the 1/sqrt(d_I) factor is an exact power of two
// and cannot change the order, so it is not applied). Ranking uses only compares: the
// running top-15 keeps the earlier (lower) block on equal scores, which is the order
// (score desc, id asc). The query's own block is added and the ids are written ascending.
#include <cooperative_groups.h>

#include "msa_common.cuh"

namespace msa {

constexpr int kKeep = kTopK - 1;   // best fully-past blocks kept besides the diagonal one

// Sort 16 ids ascending in registers (odd-even transposition network).
__device__ __forceinline__ void sort16(int (&x)[16]) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
#pragma unroll
        for (int i = (r & 1); i + 1 < 16; i += 2) {
            const int a = min(x[i], x[i + 1]), bb = max(x[i], x[i + 1]);
            x[i] = a; x[i + 1] = bb;
        }
    }
}

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

// ------------------------------------------------------------------ prefill, warp MMAs
// The same selection with the scores of a 128-token query block as one dense contraction
// S = Q_I (128 x 64, bf16) x Kbar^T (64 x c) on the tensor cores (mma.sync m16n8k16, fp32
// accumulation). Kbar is fp32; each value is split exactly into three bf16 terms
// (hi = bf16(x), mid = bf16(x - hi), lo = bf16(x - hi - mid): 24 significant bits), so the
// contraction keeps fp32 accuracy. Candidates go 32 per pass: the CTA stages the pass's split
// keys in shared memory, each warp computes the scores of its 32 queries, writes them to
// shared memory, and thread i ranks query i's 32 new scores into its running best 15 (only
// compares). Query blocks are taken heaviest first (block c = gridDim.x - 1 - blockIdx.x).
constexpr int kSelPass = 32;            // candidates per pass
constexpr int kKRow = 72;               // bf16 per staged candidate row (64 + 8: no bank conflicts)
constexpr int kSRow = kSelPass + 1;     // floats per staged score row (odd: conflict-free row reads)

__device__ __forceinline__ uint32_t split3_pack(float x0, float x1, int part) {
    const float h0 = __bfloat162float(__float2bfloat16_rn(x0)), h1 = __bfloat162float(__float2bfloat16_rn(x1));
    if (part == 0) return pack_bf16x2(h0, h1);
    const float r0 = x0 - h0, r1 = x1 - h1;
    const float m0 = __bfloat162float(__float2bfloat16_rn(r0)), m1 = __bfloat162float(__float2bfloat16_rn(r1));
    if (part == 1) return pack_bf16x2(m0, m1);
    return pack_bf16x2(r0 - m0, r1 - m1);
}

// Queries are the N tokens at positions P .. P + N - 1 (P = 0 for a whole prefill, P > 0 for a
// chunk against cached blocks); query row i of q_idx and sel is position P + i. One CTA per
// 128-token query block c that holds any of them.
__global__ void __launch_bounds__(128, 2) select_prefill_mma_kernel(const uint16_t* __restrict__ q_idx, int64_t N,
                                                                 int64_t P, int G, const float* __restrict__ pooled,
                                                                 int64_t nb_cap, int32_t* __restrict__ sel) {
    __shared__ __align__(16) uint16_t kst[3][kSelPass][kKRow];
    __shared__ float scs[128][kSRow];
    const int c = int(P / kBlock) + int(gridDim.x) - 1 - int(blockIdx.x), g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int64_t t = int64_t(c) * kBlock + tid;       // position
    const bool live = t >= P && t < P + N;
    int32_t* out = sel + ((size_t(b) * N + (live ? t - P : 0)) * G + g) * kTopK;
    if (c + 1 <= kTopK) {
        if (live) write_all_blocks(out, c);
        return;
    }
    // A fragments of this warp's 32 query rows (m-tile m: rows 16 m + gq and + 8); rows outside
    // the queries read a valid query row and are never written
    uint32_t qa[2][4][4];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        int64_t ra = int64_t(c) * kBlock + warp * 32 + m * 16 + gq, rb = ra + 8;
        ra = ra < P ? P : (ra < P + N ? ra : P + N - 1);
        rb = rb < P ? P : (rb < P + N ? rb : P + N - 1);
        const uint16_t* pa = q_idx + ((size_t(b) * N + (ra - P)) * G + g) * kIndexDim;
        const uint16_t* pb = q_idx + ((size_t(b) * N + (rb - P)) * G + g) * kIndexDim;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            qa[m][ks][0] = __ldg(reinterpret_cast<const uint32_t*>(pa + ks * 16 + 2 * tq));
            qa[m][ks][1] = __ldg(reinterpret_cast<const uint32_t*>(pb + ks * 16 + 2 * tq));
            qa[m][ks][2] = __ldg(reinterpret_cast<const uint32_t*>(pa + ks * 16 + 8 + 2 * tq));
            qa[m][ks][3] = __ldg(reinterpret_cast<const uint32_t*>(pb + ks * 16 + 8 + 2 * tq));
        }
    }
    float best[kKeep];
    int bid[kKeep];
#pragma unroll
    for (int k = 0; k < kKeep; ++k) { best[k] = -INFINITY; bid[k] = 0x7fffffff; }

    const float4* pk = reinterpret_cast<const float4*>(pooled + (size_t(b) * G + g) * nb_cap * kIndexDim);
    for (int j0 = 0; j0 < c; j0 += kSelPass) {
        const int nj = min(kSelPass, c - j0);
        __syncthreads();                                 // the previous pass's keys have been read
#pragma unroll
        for (int r = 0; r < kSelPass * 16 / 128; ++r) {  // 32 candidates x 16 float4, 4 per thread
            const int i = tid + 128 * r, cand = i >> 4, f4 = i & 15;
            const float4 v = cand < nj ? __ldg(pk + size_t(j0 + cand) * (kIndexDim / 4) + f4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int part = 0; part < 3; ++part) {
                uint2 w;
                w.x = split3_pack(v.x, v.y, part);
                w.y = split3_pack(v.z, v.w, part);
                *reinterpret_cast<uint2*>(&kst[part][cand][f4 * 4]) = w;
            }
        }
        __syncthreads();
        float acc[2][4][4];
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n) acc[m][n][0] = acc[m][n][1] = acc[m][n][2] = acc[m][n][3] = 0.f;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
#pragma unroll
            for (int part = 0; part < 3; ++part) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint16_t* kr = &kst[part][n * 8 + gq][ks * 16 + 2 * tq];
                    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(kr);
                    const uint32_t b1 = *reinterpret_cast<const uint32_t*>(kr + 8);
#pragma unroll
                    for (int m = 0; m < 2; ++m)
                        mma_bf16_16816(acc[m][n], qa[m][ks][0], qa[m][ks][1], qa[m][ks][2], qa[m][ks][3], b0, b1);
                }
            }
        }
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int r = warp * 32 + m * 16 + gq, col = n * 8 + 2 * tq;
                scs[r][col] = acc[m][n][0];
                scs[r][col + 1] = acc[m][n][1];
                scs[r + 8][col] = acc[m][n][2];
                scs[r + 8][col + 1] = acc[m][n][3];
            }
        __syncwarp();                                    // a warp's rows are its own lanes' queries
        // Mark the pass's candidates above the current 15th score (no branches), then insert
        // only those, in id order: the warp runs as many insertion rounds as its busiest lane.
        unsigned msk = 0u;
        {
            const float thr = best[kKeep - 1];
#pragma unroll
            for (int jj = 0; jj < kSelPass; ++jj)
                msk |= (jj < nj && scs[tid][jj] > thr) ? (1u << jj) : 0u;
        }
        while (msk != 0u) {
            const int jj = __ffs(msk) - 1;
            msk &= msk - 1u;
            const float sc = scs[tid][jj];
            if (sc > best[kKeep - 1]) {
                best[kKeep - 1] = sc; bid[kKeep - 1] = j0 + jj;
#pragma unroll
                for (int k = kKeep - 1; k > 0; --k) {
                    if (best[k] > best[k - 1]) {
                        float tv = best[k]; best[k] = best[k - 1]; best[k - 1] = tv;
                        int ti = bid[k]; bid[k] = bid[k - 1]; bid[k - 1] = ti;
                    }
                }
            }
        }
        __syncwarp();
    }
    if (!live) return;
    int ids[16];
#pragma unroll
    for (int k = 0; k < kKeep; ++k) ids[k] = bid[k];
    ids[15] = c;
    sort16(ids);
    int4* o = reinterpret_cast<int4*>(out);
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) o[q4] = make_int4(ids[4 * q4], ids[4 * q4 + 1], ids[4 * q4 + 2], ids[4 * q4 + 3]);
}

void launch_select_prefill_mma(const void* q_idx, int B, int G, int64_t N, int64_t P, const float* pooled,
                               int64_t nb_cap, int32_t* sel, cudaStream_t st) {
    const int64_t nqb = (P + N - 1) / kBlock - P / kBlock + 1;    // query blocks holding positions P .. P + N - 1
    dim3 grid(static_cast<unsigned>(nqb), static_cast<unsigned>(G), static_cast<unsigned>(B));
    count_launch();
    select_prefill_mma_kernel<<<grid, 128, 0, st>>>(static_cast<const uint16_t*>(q_idx), N, P, G, pooled, nb_cap, sel);
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

__global__ void __launch_bounds__(kSelThreads) select_decode_kernel(
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
        // all 16 loads of the lane go out before any is used; in the span's last pass rows past
        // the span read its last row and are ignored
        float4 v[16];
        if (base + kSelThreads <= hi) {
            ld_nc_f4x16_s512(rows + size_t(r0 + half) * (kIndexDim / 4) + part, v);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = r0 + 2 * i + half;
                v[i] = ld_nc_f4(rows + size_t(r < hi ? r : hi - 1) * (kIndexDim / 4) + part);
            }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            // fixed order: x, y, z, w, then a butterfly over the 16 lanes of this half-warp
            float d = fmaf(qv.x, v[i].x, 0.f);
            d = fmaf(qv.y, v[i].y, d);
            d = fmaf(qv.z, v[i].z, d);
            d = fmaf(qv.w, v[i].w, d);
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
            if (part == 0) sc[wid * 32 + 2 * i + half] = d;
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
    count_launch();
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

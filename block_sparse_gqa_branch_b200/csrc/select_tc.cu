// select_tc.cu -- Index Branch for prefill on the 5th-generation tensor cores: block scores as
// one dense contraction per 128-query tile, and the exp-free top-15 per query.
//
// Sources: youmind article "MiniMax M3 sparse attention agents", paragraph "The mechanism that
// changes this" (score the context in blocks, keep the most relevant per query and GQA group)
// and bullet "Predictable cost at every length" (k = 16 blocks of 128 tokens); KuCoin flash
// "MiniMax launches MSA sparse attention method and MiniMax-M3 model", summary (exp-free top-k).
//
// A pre-pass splits every pooled key (fp32) exactly into three bf16 terms (hi = bf16(x),
// mid = bf16(x - hi), lo = bf16(x - hi - mid): 24 significant bits) once, into the workspace.
// Then one CTA of 128 threads per (128-token query block c, group g, sequence b), heaviest
// blocks first. The tile's index queries Q_I (128 x 64 bf16) arrive by TMA. The fully-past
// candidates j < c go 64 per chunk: the threads copy the chunk's three terms into three K-major
// shared-memory operands (the loads of chunk k + 1 are in flight while chunk k is ranked); one
// thread issues the 12 tcgen05.mma (3 terms x 4 k-steps of 16) that accumulate
// S = Q_I x Kbar^T (128 x 64, fp32) into tensor memory. Scores are fp32-accurate (a single bf16 term would move selections
// beyond the near-tie rule). Two S buffers let chunk k + 1's MMAs run while chunk k is ranked;
// 64-candidate chunks keep the CTA at 65 KB of shared memory, three CTAs per SM.
// Thread i owns query row i (tensor-memory lane i): it reads its row's 64 scores with
// tcgen05.ld, marks without branches the candidates that beat its current 15th best, and
// inserts only those, in id order, into its running best 15 -- compares only, so equal scores
// keep the lower block id. The 1/sqrt(d_I) factor is an exact power of two and cannot change
// the order, so it is not applied.
#include <atomic>

#include "msa_common.cuh"

namespace msa {

constexpr int kTcRows = 128;       // queries per tile (MMA M)
constexpr int kTcCand = 64;        // candidates per chunk (MMA N)
constexpr int kTcKeep = kTopK - 1;

struct __align__(1024) SelTcSmem {
    uint8_t q[kTcRows * 128];               // Q_I tile [128 rows][64 bf16], 128B swizzle
    uint8_t kb[2][3][kTcCand * 128];        // split pooled keys [buf][hi, mid, lo][64 cand][64 bf16], 128B swizzle
    uint64_t q_full, mma_done[2];
    uint32_t tmem_base;
};

__device__ __forceinline__ void split3(float x, float& h, float& m, float& l) {
    h = __bfloat162float(__float2bfloat16_rn(x));
    const float r = x - h;
    m = __bfloat162float(__float2bfloat16_rn(r));
    l = r - m;
}

// Split pooled keys: [B G][3 terms][nbp][64] bf16, one 128-byte row per (term, block); rows of
// blocks j >= ncand are zero. The fp32 subtractions are exact (Sterbenz), so hi + mid + lo = x.
__global__ void __launch_bounds__(256) split_pooled_kernel(const float* __restrict__ pooled, int64_t nb_cap,
                                                           int64_t ncand, int64_t nbp, uint16_t* __restrict__ split) {
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;   // (block j, 8-dim chunk ch)
    if (i >= nbp * 8) return;
    const int64_t j = i >> 3;
    const int ch = int(i & 7), bg = blockIdx.y;
    float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
    if (j < ncand) {
        const float4* src = reinterpret_cast<const float4*>(pooled + (size_t(bg) * nb_cap + j) * kIndexDim) + 2 * ch;
        v0 = __ldg(src);
        v1 = __ldg(src + 1);
    }
    const float xs[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float hs[8], ms[8], ls[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) split3(xs[e], hs[e], ms[e], ls[e]);
    uint4* row = reinterpret_cast<uint4*>(split + ((size_t(bg) * 3) * nbp + j) * kIndexDim) + ch;
    const size_t term = size_t(nbp) * kIndexDim / 8;                       // uint4 per term
    row[0] = make_uint4(pack_bf16x2(hs[0], hs[1]), pack_bf16x2(hs[2], hs[3]), pack_bf16x2(hs[4], hs[5]),
                        pack_bf16x2(hs[6], hs[7]));
    row[term] = make_uint4(pack_bf16x2(ms[0], ms[1]), pack_bf16x2(ms[2], ms[3]), pack_bf16x2(ms[4], ms[5]),
                           pack_bf16x2(ms[6], ms[7]));
    row[2 * term] = make_uint4(pack_bf16x2(ls[0], ls[1]), pack_bf16x2(ls[2], ls[3]), pack_bf16x2(ls[4], ls[5]),
                               pack_bf16x2(ls[6], ls[7]));
}

// 64 contiguous bytes at each of three addresses (the three terms of one candidate's half
// row), issued back to back
__device__ __forceinline__ void ld_nc_64Bx3(const uint4* p0, const uint4* p1, const uint4* p2, uint4 (&v)[3][4]) {
    asm volatile(
        "ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%48];\n\tld.global.nc.v4.u32 {%4, %5, %6, %7}, [%48+16];\n\t"
        "ld.global.nc.v4.u32 {%8, %9, %10, %11}, [%48+32];\n\tld.global.nc.v4.u32 {%12, %13, %14, %15}, [%48+48];\n\t"
        "ld.global.nc.v4.u32 {%16, %17, %18, %19}, [%49];\n\tld.global.nc.v4.u32 {%20, %21, %22, %23}, [%49+16];\n\t"
        "ld.global.nc.v4.u32 {%24, %25, %26, %27}, [%49+32];\n\tld.global.nc.v4.u32 {%28, %29, %30, %31}, [%49+48];\n\t"
        "ld.global.nc.v4.u32 {%32, %33, %34, %35}, [%50];\n\tld.global.nc.v4.u32 {%36, %37, %38, %39}, [%50+16];\n\t"
        "ld.global.nc.v4.u32 {%40, %41, %42, %43}, [%50+32];\n\tld.global.nc.v4.u32 {%44, %45, %46, %47}, [%50+48];"
        : "=r"(v[0][0].x), "=r"(v[0][0].y), "=r"(v[0][0].z), "=r"(v[0][0].w), "=r"(v[0][1].x), "=r"(v[0][1].y),
          "=r"(v[0][1].z), "=r"(v[0][1].w), "=r"(v[0][2].x), "=r"(v[0][2].y), "=r"(v[0][2].z), "=r"(v[0][2].w),
          "=r"(v[0][3].x), "=r"(v[0][3].y), "=r"(v[0][3].z), "=r"(v[0][3].w), "=r"(v[1][0].x), "=r"(v[1][0].y),
          "=r"(v[1][0].z), "=r"(v[1][0].w), "=r"(v[1][1].x), "=r"(v[1][1].y), "=r"(v[1][1].z), "=r"(v[1][1].w),
          "=r"(v[1][2].x), "=r"(v[1][2].y), "=r"(v[1][2].z), "=r"(v[1][2].w), "=r"(v[1][3].x), "=r"(v[1][3].y),
          "=r"(v[1][3].z), "=r"(v[1][3].w), "=r"(v[2][0].x), "=r"(v[2][0].y), "=r"(v[2][0].z), "=r"(v[2][0].w),
          "=r"(v[2][1].x), "=r"(v[2][1].y), "=r"(v[2][1].z), "=r"(v[2][1].w), "=r"(v[2][2].x), "=r"(v[2][2].y),
          "=r"(v[2][2].z), "=r"(v[2][2].w), "=r"(v[2][3].x), "=r"(v[2][3].y), "=r"(v[2][3].z), "=r"(v[2][3].w)
        : "l"(p0), "l"(p1), "l"(p2));
}

__device__ __forceinline__ void sort16_ids(int (&x)[16]) {
#pragma unroll
    for (int r = 0; r < 16; ++r) {
#pragma unroll
        for (int i = (r & 1); i + 1 < 16; i += 2) {
            const int a = min(x[i], x[i + 1]), bb = max(x[i], x[i + 1]);
            x[i] = a; x[i + 1] = bb;
        }
    }
}

// Queries are the N tokens at positions P .. P + N - 1 (P = 0 for a whole prefill); query row i
// of q_idx and sel is position P + i.
__global__ void __launch_bounds__(128) select_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                int64_t N, int64_t P, int G,
                                                                const uint16_t* __restrict__ split, int64_t nbp,
                                                                int32_t* __restrict__ sel, WsHeader* hdr) {
    extern __shared__ uint8_t smem_raw[];
    SelTcSmem& sm = *reinterpret_cast<SelTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int c = int((P + N - 1) / kBlock) - int(blockIdx.x), g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int64_t t = int64_t(c) * kBlock + tid;            // this thread's query position
    const bool live = t >= P && t < P + N;
    int32_t* out = sel + ((size_t(b) * N + (live ? t - P : 0)) * G + g) * kTopK;
    if (c + 1 <= kTopK) {                                    // every block 0..c is taken
        if (live) {
            int4* o = reinterpret_cast<int4*>(out);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                o[q] = make_int4(4 * q <= c ? 4 * q : -1, 4 * q + 1 <= c ? 4 * q + 1 : -1,
                                 4 * q + 2 <= c ? 4 * q + 2 : -1, 4 * q + 3 <= c ? 4 * q + 3 : -1);
        }
        return;
    }
    if (tid == 0) {
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.mma_done[0], 1);
        mbar_init(&sm.mma_done[1], 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmQ);
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 2 * kTcCand);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    if (tid == 0) {
        // rows 128 c - P .. + 127 of this sequence's queries (rows outside the queries are read
        // as zeros or as a neighbour's rows and never written)
        mbar_arrive_expect_tx(&sm.q_full, kTcRows * 128);
        tma_load_3d(sm.q, &tmQ, 0, g, int(int64_t(b) * N + int64_t(c) * kBlock - P), &sm.q_full);
    }
    const int nchunks = (c + kTcCand - 1) / kTcCand;
    const uint16_t* sbase = split + size_t(b * G + g) * 3 * nbp * kIndexDim;
    const uint32_t idesc = idesc_bf16_f32(kTcRows, kTcCand, 0, 0);   // both operands K-major

    // threads 2 i and 2 i + 1 copy candidate j0 + i of a chunk, 32 dims (64 bytes) of each of the
    // three terms: loaded into registers one chunk ahead, stored into the swizzled operands
    uint4 pre[3][4];
    auto load_chunk = [&](int k) {
        const int r = tid >> 1, j = k * kTcCand + r;             // j < nbp: nbp is a multiple of 64
        const uint4* p = reinterpret_cast<const uint4*>(sbase + size_t(j) * kIndexDim) + 4 * (tid & 1);
        const size_t term = size_t(nbp) * kIndexDim / 8;
        ld_nc_64Bx3(p, p + term, p + 2 * term, pre);
    };
    auto store_chunk = [&](int k) {
        const int r = tid >> 1;
        uint8_t* dst = sm.kb[k & 1][0];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            const uint32_t off = sw128(uint32_t(r), uint32_t(4 * (tid & 1) + c4));
#pragma unroll
            for (int t = 0; t < 3; ++t) *reinterpret_cast<uint4*>(dst + t * kTcCand * 128 + off) = pre[t][c4];
        }
        fence_proxy_async();                                 // visible to the tensor cores
    };
    // one thread: S[buf] = sum over the three terms of Q_I x term^T
    auto issue = [&](int k) {
        const int buf = k & 1;
        const uint32_t qb = smem_u32(sm.q), kbase = smem_u32(sm.kb[buf][0]);
#pragma unroll
        for (int part = 0; part < 3; ++part)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc_mma_ss(tmem + buf * kTcCand, sdesc_sw128(qb + ks * 32, 16, 1024),
                          sdesc_sw128(kbase + part * kTcCand * 128 + ks * 32, 16, 1024), idesc,
                          (part | ks) != 0);
        tc_commit(&sm.mma_done[buf]);
    };

    float best[kTcKeep];
    int bid[kTcKeep];
#pragma unroll
    for (int i = 0; i < kTcKeep; ++i) { best[i] = -INFINITY; bid[i] = 0x7fffffff; }
    // Every wait is bounded. A wait that gives up makes its warp stop ranking; the whole CTA then
    // leaves the loop at the next barrier, and thread 0 waits (bounded) for the MMAs it issued
    // before the tensor memory is freed.
    bool ok = true;
    int issued = 0, waited = 0;                              // chunks whose MMAs were issued / waited for
    load_chunk(0);
    store_chunk(0);
    if (nchunks > 1) load_chunk(1);
    __syncthreads();
    if (tid == 0) {
        ok = mbar_wait(&sm.q_full, 0, hdr, KID_SELECT_PREFILL);
        if (ok) {
            tc_fence_after();
            issue(0);
            issued = 1;
        }
    }
    ok = __syncthreads_and(ok);
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    for (int k = 0; ok && k < nchunks; ++k) {
        __syncthreads();                                     // chunk k - 1's stashed scores all read
        if (k + 1 < nchunks) {
            store_chunk(k + 1);                              // its buffer's MMAs (chunk k - 1) are done
            if (k + 2 < nchunks) load_chunk(k + 2);          // in flight while chunk k is ranked
        }
        tc_fence_before();
        if (!__syncthreads_and(ok)) { ok = false; break; }   // stored; chunk k - 1's scores all read
        tc_fence_after();
        if (tid == 0 && k + 1 < nchunks) { issue(k + 1); issued = k + 2; }
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.mma_done[k & 1], (k >> 1) & 1, hdr, KID_SELECT_PREFILL));
        if (!ok) continue;                                   // the loop ends at the next barrier
        waited = k + 1;
        tc_fence_after();
        const int j0 = k * kTcCand;
        // the chunk's operand buffer is free once its MMAs are done: it stashes each thread's
        // 32 scores of a pass (row stride 33 floats: conflict-free), so that an insertion reads
        // its score with one shared-memory load
        float* stash = reinterpret_cast<float*>(sm.kb[k & 1][0]) + tid * 33;
#pragma unroll 1
        for (int q32 = 0; q32 < kTcCand / 32; ++q32) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_off + (k & 1) * kTcCand + q32 * 32, v);
            tmem_wait_ld();
            // mark the candidates that beat the current 15th score (no branches), then insert
            // only those, in id order: the warp runs as many rounds as its busiest lane
            unsigned msk = 0u;
            const float thr = best[kTcKeep - 1];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                msk |= (j0 + q32 * 32 + i < c && __uint_as_float(v[i]) > thr) ? (1u << i) : 0u;
            if (__any_sync(0xffffffffu, msk != 0u)) {
#pragma unroll
                for (int i = 0; i < 32; ++i) stash[i] = __uint_as_float(v[i]);
            }
            while (msk != 0u) {
                const int i = __ffs(msk) - 1;
                msk &= msk - 1u;
                const float sc = stash[i];
                if (sc > best[kTcKeep - 1]) {
                    best[kTcKeep - 1] = sc; bid[kTcKeep - 1] = j0 + q32 * 32 + i;
#pragma unroll
                    for (int r = kTcKeep - 1; r > 0; --r) {
                        if (best[r] > best[r - 1]) {
                            float tv = best[r]; best[r] = best[r - 1]; best[r - 1] = tv;
                            int ti = bid[r]; bid[r] = bid[r - 1]; bid[r - 1] = ti;
                        }
                    }
                }
            }
        }
    }
    if (tid == 0)                                            // MMAs issued but not waited for (failure path)
        for (int kk = waited; kk < issued; ++kk) mbar_wait(&sm.mma_done[kk & 1], (kk >> 1) & 1, hdr, KID_SELECT_PREFILL);
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kTcCand);
    }
    if (!ok || !live) return;
    int ids[16];
#pragma unroll
    for (int i = 0; i < kTcKeep; ++i) ids[i] = bid[i];
    ids[15] = c;
    sort16_ids(ids);
    int4* o = reinterpret_cast<int4*>(out);
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) o[q4] = make_int4(ids[4 * q4], ids[4 * q4 + 1], ids[4 * q4 + 2], ids[4 * q4 + 3]);
}

// Blocks of split pooled keys the selection for queries up to position n_end - 1 keeps in its
// workspace (the fully-past candidates of the last query, rounded up to whole 64-candidate
// chunks), and the workspace bytes that need.
int64_t select_split_blocks(int64_t n_end) {
    const int64_t ncand = n_end > 0 ? (n_end - 1) / kBlock : 0;
    const int64_t chunks = (ncand + kTcCand - 1) / kTcCand;
    return (chunks > 0 ? chunks : 1) * kTcCand;
}
size_t select_split_offset() { return (sizeof(WsHeader) + 255) / 256 * 256; }
size_t select_prefill_ws_bytes(int B, int G, int64_t n_end) {
    return select_split_offset() + size_t(B) * G * 3 * size_t(select_split_blocks(n_end)) * kIndexDim * 2;
}

msa_status_t launch_select_prefill_tc(const void* q_idx, int B, int G, int64_t N, int64_t P, const float* pooled,
                                      int64_t nb_cap, int32_t* sel, void* ws, cudaStream_t st) {
    CUtensorMap tmQ;
    msa_status_t e = make_tmap_qidx(&tmQ, q_idx, G, uint64_t(B) * N);
    if (e != MSA_OK) return e;
    const int64_t ncand = (P + N - 1) / kBlock, nbp = select_split_blocks(P + N);
    uint16_t* split = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + select_split_offset());
    {
        const int64_t threads = nbp * 8;
        const KernelTimer kt(KID_SPLIT, st);
        split_pooled_kernel<<<dim3(unsigned((threads + 255) / 256), unsigned(B * G)), 256, 0, st>>>(pooled, nb_cap, ncand,
                                                                                              nbp, split);
    }
    const int64_t nqb = (P + N - 1) / kBlock - P / kBlock + 1;   // query blocks holding positions P .. P + N - 1
    const int smem = int(sizeof(SelTcSmem)) + 1024;
    static std::atomic<bool> attr_set[64];      // per device; setting it twice is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaFuncSetAttribute(select_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        attr_set[dev].store(true, std::memory_order_relaxed);
    }
    dim3 grid(static_cast<unsigned>(nqb), static_cast<unsigned>(G), static_cast<unsigned>(B));
    const KernelTimer kt(KID_SELECT_PREFILL, st);
    select_prefill_tc_kernel<<<grid, 128, smem, st>>>(tmQ, N, P, G, split, nbp, sel, static_cast<WsHeader*>(ws));
    return MSA_OK;
}

}  // namespace msa

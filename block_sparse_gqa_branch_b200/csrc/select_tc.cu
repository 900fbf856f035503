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
// Then one CTA per (128-token query block c, group g, sequence b), heaviest blocks first: four
// ranking warps (thread i owns query row i, tensor-memory lane i) and one producer warp. The
// producer brings the tile's index queries Q_I (128 x 64 bf16) and, 32 fully-past candidates
// j < c per item, the three split terms by TMA into a 3-stage ring, and issues the item's 12
// tcgen05.mma (3 terms x 4 k-steps of 16) that accumulate S = Q_I x Kbar^T (128 x 32, fp32)
// into one of two tensor-memory buffers. Scores are fp32-accurate (a single bf16 term would
// move selections beyond the near-tie rule).
// The ranking runs in two passes over the candidates, exp-free and compare-only:
//  * pass A keeps only the 15 largest score VALUES per query: the first 32 through a sorting
//    network, then the candidates that beat the current 15th value, two per round, through a
//    branch-free min/max merge (no block ids to carry, no dependent chain);
//  * pass B recomputes the same scores (the same MMAs on the same operands: bit-identical) and
//    emits, in id order, every block above the 15th value and then the first blocks equal to
//    it until 15 are taken -- exactly "score descending, then lower block id", already sorted.
// The 1/sqrt(d_I) factor is an exact power of two and cannot change the order, so it is not
// applied.
#include <atomic>

#include "msa_common.cuh"

namespace msa {

constexpr int kTcRows = 128;       // queries per tile (MMA M)
constexpr int kTcCand = 32;        // candidates per item (MMA N)
constexpr int kTcStages = 3;       // operand stages in flight
constexpr int kTcThreads = 160;    // 4 ranking warps (one query row per thread) + 1 producer warp
constexpr int kStashStride = 36;   // floats per ranking thread's stash row (16-byte rows, conflict-free stores)
constexpr uint32_t kTcStageBytes = 3 * kTcCand * 128;

struct __align__(1024) SelTcSmem {
    uint8_t q[kTcRows * 128];                   // Q_I tile [128 rows][64 bf16], 128B swizzle
    uint8_t kb[kTcStages][3][kTcCand * 128];    // split pooled keys [stage][hi, mid, lo][32 cand][64 bf16], 128B swizzle
    float stash[kTcRows * kStashStride];        // each ranking thread's scores of the current item
    uint64_t q_full, kfull[kTcStages], kempty[kTcStages], sfull[2], sempty[2];
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

// compare-exchange: a takes the larger value, b the smaller
__device__ __forceinline__ void cx_desc(float& a, float& b) {
    const float hi = fmaxf(a, b);
    b = fminf(a, b);
    a = hi;
}

// bitonic sorting network on 16 values, descending
__device__ __forceinline__ void sort16_desc(float (&a)[16]) {
#pragma unroll
    for (int k = 2; k <= 16; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int p = i ^ j;
                if (p > i) {
                    if ((i & k) == 0) cx_desc(a[i], a[p]);
                    else cx_desc(a[p], a[i]);
                }
            }
}

// best = the 15 largest of v[0..31] (no NaN), descending: both halves sorted, the larger of
// a[i] and b[15 - i] (the top 16, as a bitonic sequence), then a bitonic merge
__device__ __forceinline__ void top15_of_32(const float (&v)[32], float (&best)[kTopK - 1]) {
    float a[16], b[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) { a[i] = v[i]; b[i] = v[16 + i]; }
    sort16_desc(a);
    sort16_desc(b);
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = fmaxf(a[i], b[15 - i]);
#pragma unroll
    for (int j = 8; j > 0; j >>= 1)
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if ((i ^ j) > i) cx_desc(a[i], a[i ^ j]);
#pragma unroll
    for (int i = 0; i < kTopK - 1; ++i) best[i] = a[i];
}

// Merges two values x1, x2 (no NaN; -inf for none) into the descending list b of 15: the
// r-th largest of the union of a sorted list and a sorted pair x >= y is
// max(b[r], min(b[r-1], x), min(b[r-2], y)) with b[-1] = b[-2] = +inf. Branch-free, and every
// entry is independent of the others.
__device__ __forceinline__ void merge2(float (&b)[kTopK - 1], float x1, float x2) {
    const float x = fmaxf(x1, x2), y = fminf(x1, x2);
    float nb[kTopK - 1];
    nb[0] = fmaxf(b[0], x);
    nb[1] = fmax3(b[1], fminf(b[0], x), y);
#pragma unroll
    for (int r = 2; r < kTopK - 1; ++r) nb[r] = fmax3(b[r], fminf(b[r - 1], x), fminf(b[r - 2], y));
#pragma unroll
    for (int r = 0; r < kTopK - 1; ++r) b[r] = nb[r];
}

// Queries are the N tokens at positions P .. P + N - 1 (P = 0 for a whole prefill); query row i
// of q_idx and sel is position P + i.
__global__ void __launch_bounds__(kTcThreads, 3) select_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                         const __grid_constant__ CUtensorMap tmS,
                                                                         int64_t N, int64_t P, int G,
                                                                         int32_t* __restrict__ sel, WsHeader* hdr) {
    extern __shared__ uint8_t smem_raw[];
    SelTcSmem& sm = *reinterpret_cast<SelTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int c = int((P + N - 1) / kBlock) - int(blockIdx.x), g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t t = int64_t(c) * kBlock + tid;            // a ranking thread's query position
    const bool live = warp < 4 && t >= P && t < P + N;
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
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&sm.kfull[s], 1);
            mbar_init(&sm.kempty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.sfull[i], 1);
            mbar_init(&sm.sempty[i], 4);
        }
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 2 * kTcCand);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int n = (c + kTcCand - 1) / kTcCand;               // items per pass
    const int items = 2 * n;                                  // pass A (values), pass B (block ids)
    bool ok = true;
    int ids[kTopK - 1];                                       // a ranking thread's emitted blocks
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < kTopK - 1; ++i) ids[i] = -1;

    if (warp == 4) {
        // producer: TMA of the queries and of each item's 32 candidates (three split terms), and
        // the 12 MMAs of an item once its operands are in and its score buffer has been read
        if (lane == 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmS);
            const int zb = (b * G + g) * 3;
            mbar_arrive_expect_tx(&sm.q_full, kTcRows * 128);
            tma_load_3d(sm.q, &tmQ, 0, g, int(int64_t(b) * N + int64_t(c) * kBlock - P), &sm.q_full);
            int loaded = 0, landed = 0, mmas = 0;             // items loaded / waited for / multiplied
            for (; loaded < items && loaded < kTcStages; ++loaded) {
                mbar_arrive_expect_tx(&sm.kfull[loaded], kTcStageBytes);
                tma_load_3d(sm.kb[loaded][0], &tmS, 0, kTcCand * (loaded % n), zb, &sm.kfull[loaded]);
            }
            ok = mbar_wait(&sm.q_full, 0, hdr, KID_SELECT_PREFILL);
            const uint32_t idesc = idesc_bf16_f32(kTcRows, kTcCand, 0, 0);   // both operands K-major
            const uint32_t qb = smem_u32(sm.q);
            for (int it = 0; ok && it < items; ++it) {
                const int s = it % kTcStages;
                ok = mbar_wait(&sm.kfull[s], (it / kTcStages) & 1, hdr, KID_SELECT_PREFILL);
                if (!ok) break;
                landed = it + 1;
                if (it >= 2) ok = mbar_wait(&sm.sempty[it & 1], ((it >> 1) - 1) & 1, hdr, KID_SELECT_PREFILL);
                if (!ok) break;
                tc_fence_after();
                const uint32_t kbase = smem_u32(sm.kb[s][0]);
#pragma unroll
                for (int part = 0; part < 3; ++part)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        tc_mma_ss(tmem + (it & 1) * kTcCand, sdesc_sw128(qb + ks * 32, 16, 1024),
                                  sdesc_sw128(kbase + part * kTcCand * 128 + ks * 32, 16, 1024), idesc,
                                  (part | ks) != 0);
                tc_commit(&sm.sfull[it & 1]);
                tc_commit(&sm.kempty[s]);
                mmas = it + 1;
                // item it - 1's stage is free once its MMAs are done: load item it - 1 + stages
                if (it >= 1 && loaded < items) {
                    const int sp = (it - 1) % kTcStages;
                    ok = mbar_wait(&sm.kempty[sp], ((it - 1) / kTcStages) & 1, hdr, KID_SELECT_PREFILL);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&sm.kfull[sp], kTcStageBytes);
                    tma_load_3d(sm.kb[sp][0], &tmS, 0, kTcCand * (loaded % n), zb, &sm.kfull[sp]);
                    ++loaded;
                }
            }
            // nothing may still write this CTA's shared or tensor memory when it exits: wait
            // (bounded) for the last MMAs and for every copy not yet waited for
            if (mmas > 0) mbar_wait(&sm.kempty[(mmas - 1) % kTcStages], ((mmas - 1) / kTcStages) & 1, hdr,
                                    KID_SELECT_PREFILL);
            for (int it = landed; it < loaded; ++it)
                mbar_wait(&sm.kfull[it % kTcStages], (it / kTcStages) & 1, hdr, KID_SELECT_PREFILL);
        }
        __syncwarp();
    } else {
        // ranking thread: query row tid (tensor-memory lane tid). Pass A keeps the 15 largest
        // score values (compare-only min/max networks); pass B recomputes the same scores and
        // emits, in id order, every block above the 15th value and the first blocks equal to it.
        const uint32_t lane_off = uint32_t(warp * 32) << 16;
        float* stash = sm.stash + tid * kStashStride;
        float best[kTopK - 1];
        float thr = -INFINITY;
        int eq = 0, need_eq = 0;
#pragma unroll
        for (int i = 0; i < kTopK - 1; ++i) best[i] = -INFINITY;
        for (int it = 0; it < items; ++it) {
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.sfull[it & 1], (it >> 1) & 1, hdr, KID_SELECT_PREFILL));
            if (!ok) break;
            tc_fence_after();
            uint32_t v[32];
            tmem_ld32(tmem + lane_off + (it & 1) * kTcCand, v);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.sempty[it & 1]);
            const bool pass_a = it < n;
            const int j0 = (pass_a ? it : it - n) * kTcCand;
            const unsigned valid = c - j0 >= 32 ? 0xffffffffu : (1u << (c - j0)) - 1u;
            if (it == 0) {                                    // the first 32 candidates: a network
                float f[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float x = __uint_as_float(v[i]);
                    f[i] = ((valid >> i) & 1u) && x == x ? x : -INFINITY;
                }
                top15_of_32(f, best);
                continue;
            }
            if (it == n) {                                    // pass B starts: the 15th value decides
                thr = best[kTopK - 2];
                int gt = 0;
#pragma unroll
                for (int i = 0; i < kTopK - 1; ++i) gt += best[i] > thr ? 1 : 0;
                need_eq = kTopK - 1 - gt;
            }
            unsigned msk = 0u;
            if (pass_a) {
                const float th = best[kTopK - 2];
#pragma unroll
                for (int i = 0; i < 32; ++i) msk |= __uint_as_float(v[i]) > th ? (1u << i) : 0u;
            } else {
                if (!__any_sync(0xffffffffu, cnt < kTopK - 1)) continue;
#pragma unroll
                for (int i = 0; i < 32; ++i) msk |= __uint_as_float(v[i]) >= thr ? (1u << i) : 0u;
                if (cnt >= kTopK - 1) msk = 0u;
            }
            msk &= valid;
            if (msk != 0u) {
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4*>(stash + i) = make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                                                        __uint_as_float(v[i + 2]),
                                                                        __uint_as_float(v[i + 3]));
            }
            if (pass_a) {
                // two candidates per round; a round merges what beat the 15th value when the item
                // was read (a value that no longer does leaves the list unchanged)
                while (msk != 0u) {
                    const int i1 = __ffs(msk) - 1;
                    msk &= msk - 1u;
                    const float x1 = stash[i1];
                    const int i2 = msk != 0u ? __ffs(msk) - 1 : i1;
                    const float x2 = msk != 0u ? stash[i2] : -INFINITY;
                    msk &= msk - 1u;
                    merge2(best, x1, x2);
                }
            } else {
                while (msk != 0u) {
                    const int i = __ffs(msk) - 1;
                    msk &= msk - 1u;
                    const float x = stash[i];
                    const bool above = x > thr;
                    if (above || eq < need_eq) {
                        eq += above ? 0 : 1;
#pragma unroll
                        for (int r = 0; r < kTopK - 2; ++r) ids[r] = ids[r + 1];
                        ids[kTopK - 2] = j0 + i;
                        if (++cnt == kTopK - 1) msk = 0u;
                    }
                }
            }
        }
    }
    tc_fence_before();
    ok = __syncthreads_and(ok);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kTcCand);
    }
    if (!ok || !live) return;
    // ids[15 - cnt ..] hold the emitted blocks in ascending order (all 15 unless scores were NaN),
    // then the query's own block c (the largest id), then -1 padding
    int o16[kTopK];
    if (cnt == kTopK - 1) {
#pragma unroll
        for (int i = 0; i < kTopK - 1; ++i) o16[i] = ids[i];
        o16[kTopK - 1] = c;
    } else {
#pragma unroll
        for (int r = 0; r < kTopK; ++r) {
            int x = -1;
#pragma unroll
            for (int i = 0; i < kTopK - 1; ++i) x = (i == kTopK - 1 - cnt + r) ? ids[i] : x;
            o16[r] = r < cnt ? x : (r == cnt ? c : -1);
        }
    }
    int4* o = reinterpret_cast<int4*>(out);
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) o[q4] = make_int4(o16[4 * q4], o16[4 * q4 + 1], o16[4 * q4 + 2], o16[4 * q4 + 3]);
}

// Blocks of split pooled keys the selection for queries up to position n_end - 1 keeps in its
// workspace (the fully-past candidates of the last query, rounded up to whole 64-candidate
// chunks), and the workspace bytes that need.
int64_t select_split_blocks(int64_t n_end) {
    constexpr int64_t kRound = 64;                           // a multiple of the item size
    static_assert(kRound % kTcCand == 0, "whole items");
    const int64_t ncand = n_end > 0 ? (n_end - 1) / kBlock : 0;
    const int64_t chunks = (ncand + kRound - 1) / kRound;
    return (chunks > 0 ? chunks : 1) * kRound;
}
size_t select_split_offset() { return (sizeof(WsHeader) + 255) / 256 * 256; }
size_t select_prefill_ws_bytes(int B, int G, int64_t n_end) {
    return select_split_offset() + size_t(B) * G * 3 * size_t(select_split_blocks(n_end)) * kIndexDim * 2;
}

msa_status_t launch_select_prefill_tc(const void* q_idx, int B, int G, int64_t N, int64_t P, const float* pooled,
                                      int64_t nb_cap, int32_t* sel, void* ws, cudaStream_t st) {
    const int64_t ncand = (P + N - 1) / kBlock, nbp = select_split_blocks(P + N);
    uint16_t* split = reinterpret_cast<uint16_t*>(static_cast<char*>(ws) + select_split_offset());
    CUtensorMap tmQ, tmS;
    msa_status_t e = make_tmap_qidx(&tmQ, q_idx, G, uint64_t(B) * N);
    if (e == MSA_OK) e = make_tmap_split(&tmS, split, uint64_t(nbp), uint64_t(B) * G * 3);
    if (e != MSA_OK) return e;
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
    select_prefill_tc_kernel<<<grid, kTcThreads, smem, st>>>(tmQ, tmS, N, P, G, sel, static_cast<WsHeader*>(ws));
    return MSA_OK;
}

}  // namespace msa

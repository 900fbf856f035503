// attn_decode.cu -- Main Branch for one decode token per sequence: exact softmax attention
// over the k = 16 selected 128-token blocks of its GQA group, split across CTAs and merged by
// log-sum-exp.
//
// Sources: youmind article "MiniMax M3 sparse attention agents", figure 1 caption (the main
// branch attends only to the selected blocks) and paragraph "Why this comes now" (each block
// is read once with contiguous memory access); KuCoin flash "MiniMax launches MSA sparse
// attention method and MiniMax-M3 model", summary (exact softmax over the 16 blocks).
//
// Design (HBM-bound, 8 FLOP per byte read). The work items (sequence, group, selected block)
// are laid out in order and cut into one contiguous range per CTA (one persistent CTA per SM),
// so every CTA streams the same number of 64 KB K+V blocks. A loader warp walks the range and
// streams each item's K and V block -- two contiguous 32 KB ranges of the head-major cache --
// and the group's query rows with TMA into a 3-deep ring of stages, so several items' loads
// are in flight while the 8 compute warps work on another. For an item, warp w scores keys
// 16w..16w+15 for all Hg heads with warp MMAs; the row max is combined across warps in shared
// memory, P goes to shared memory as bf16, and warp w then accumulates output columns
// 16w..16w+15 over all 128 keys with an online softmax that runs across the items of one
// (sequence, group). A (sequence, group) whose items all lie in one CTA is written out
// directly; otherwise each CTA leaves an unnormalised partial (max, sum, o) and the last to
// finish merges them.
#include "msa_common.cuh"

namespace msa {

constexpr int kDecWarps = 8;           // compute warps; warp 8 loads
constexpr int kDecThreads = (kDecWarps + 1) * 32;
constexpr int kDecStages = 3;
constexpr int kDecDiagRows = 32;       // row granularity of the diagonal block's loads
constexpr int kPRow = 136;             // bf16 elements per P / Q row in shared memory (padded)

// A partial is [max: Hg][sum: Hg][pad to 4 floats][o: Hg x 128] fp32; o is 16-byte aligned.
__host__ __device__ inline int dec_part_ooff(int Hg) { return (2 * Hg + 3) / 4 * 4; }
__host__ __device__ inline int dec_part_stride(int Hg) { return dec_part_ooff(Hg) + Hg * kHeadDim; }

// address of bf16 element (row, col) in a K/V tile: two 64-column halves, each 128 rows x
// 128 B with the 128-byte swizzle
__device__ __forceinline__ uint32_t kv_off(int row, int col) {
    return uint32_t(col >> 6) * 16384u + sw128(uint32_t(row), uint32_t((col & 63) >> 3)) + uint32_t(col & 7) * 2u;
}

struct DecMaps {
    CUtensorMap k128, v128, k32, v32;   // boxes of 64 columns x 128 rows (full blocks) / 32 rows (diagonal)
};

struct __align__(1024) DecSmem {
    uint8_t kv[kDecStages][2][32768];           // [stage][K, V][d half][128 rows][128 B]
    uint16_t q[kDecStages][kMaxHg][kPRow];      // the item's query heads (rows padded)
    uint16_t p[kMaxHg][kPRow];                  // probabilities of the current item, bf16
    float red_m[kDecWarps][kMaxHg], red_l[kDecWarps][kMaxHg];
    float wts[kTopK][kMaxHg], ls[kTopK][kMaxHg], mrg_m[kMaxHg], mrg_l[kMaxHg];
    uint64_t full_k[kDecStages], full_v[kDecStages], empty[kDecStages];
    int meta_bg[kDecStages], meta_ntok[kDecStages], meta_fin[kDecStages], meta_nfrag[kDecStages],
        meta_frag[kDecStages];
    int ld_row[kTopK];                          // loader: selection row of the current group
    int is_last;
};

struct DecArgs {
    const uint16_t* q;
    int64_t l_cap, max_pos;
    const int32_t* q_pos;
    const int32_t* sel;
    int B, G, Hg;
    uint16_t* out;
    float* lse;
    float* part;
    unsigned int* ctr;
    WsHeader* hdr;
    float scale_log2;
};

// barrier among the compute warps only (the loader warp never joins it)
__device__ __forceinline__ void compute_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32) : "memory");
}

// the same barrier, returning whether any compute thread passed a nonzero flag
__device__ __forceinline__ bool compute_sync_or(bool flag) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}"
        : "=r"(r)
        : "r"(uint32_t(flag)), "n"(kDecWarps * 32)
        : "memory");
    return r != 0;
}

// first item of CTA c when n items are cut into `grid` contiguous ranges
__device__ __forceinline__ int64_t range_begin(int c, int64_t n, int grid) { return int64_t(c) * n / grid; }

// the CTA whose range holds item k
__device__ __forceinline__ int range_owner(int64_t k, int64_t n, int grid) {
    int c = int(k * grid / n);
    while (c + 1 < grid && range_begin(c + 1, n, grid) <= k) ++c;
    while (c > 0 && range_begin(c, n, grid) > k) --c;
    return c;
}

__global__ void __launch_bounds__(kDecThreads, 1) attn_decode_kernel(const __grid_constant__ DecMaps maps,
                                                                    const DecArgs a) {
    extern __shared__ uint8_t smem_raw[];
    DecSmem& sm = *reinterpret_cast<DecSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int Hg = a.Hg, G = a.G;
    const int stride = dec_part_stride(Hg), ooff = dec_part_ooff(Hg);

    if (tid == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(&sm.full_k[s], 1);
            mbar_init(&sm.full_v[s], 1);
            mbar_init(&sm.empty[s], kDecWarps);
        }
        fence_barrier_init();
    }
    for (int i = tid; i < kMaxHg * kPRow; i += kDecThreads) {      // rows >= Hg stay 0
        (&sm.p[0][0])[i] = 0;
        for (int s = 0; s < kDecStages; ++s) (&sm.q[s][0][0])[i] = 0;
    }
    __syncthreads();
    grid_dep_wait();                   // the selection and the appended token are ready from here on

    if (warp == kDecWarps) {
        // ---------------------------------------------------------------- loader warp (lane 0)
        // Streams the items of this CTA's range into the ring, skipping empty slots, and ends
        // with an end marker (bg = -1).
        if (lane != 0) return;
        const int64_t n_items = int64_t(a.B) * G * kTopK;
        const int64_t kend = range_begin(blockIdx.x + 1, n_items, gridDim.x);
        const uint64_t pol = l2_evict_first();               // K and V are read once
        const uint32_t qrow = kHeadDim * 2u;
        int cur_bg = -1, pos = 0, nsel = 0, nfrag = 1, frag = 0;
        int n = 0;
        bool ok = true;
        for (int64_t k = range_begin(blockIdx.x, n_items, gridDim.x); k < kend; ++k) {
            const int bg = int(k / kTopK), slot = int(k % kTopK);
            if (bg != cur_bg) {
                cur_bg = bg;
                nsel = 0;
                pos = a.q_pos[bg / G];
                if (pos < 0 || pos > a.max_pos || pos >= a.l_cap) {
                    if (slot == 0) record_error(a.hdr, MSA_ERR_DEVICE_BOUNDS, KID_ATTN_DECODE, bg, 0, pos);
                } else {
                    const int4* srow = reinterpret_cast<const int4*>(a.sel + size_t(bg) * kTopK);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int4 v = __ldcg(srow + q4);
                        sm.ld_row[4 * q4] = v.x; sm.ld_row[4 * q4 + 1] = v.y;
                        sm.ld_row[4 * q4 + 2] = v.z; sm.ld_row[4 * q4 + 3] = v.w;
                        nsel += (v.x >= 0) + (v.y >= 0) + (v.z >= 0) + (v.w >= 0);
                    }
                    if (nsel > 0) {
                        const int c0 = range_owner(int64_t(bg) * kTopK, n_items, gridDim.x);
                        const int c1 = range_owner(int64_t(bg) * kTopK + nsel - 1, n_items, gridDim.x);
                        nfrag = c1 - c0 + 1;
                        frag = int(blockIdx.x) - c0;
                    }
                }
            }
            if (slot >= nsel) {                               // the row's tail is empty
                k = int64_t(bg + 1) * kTopK - 1;
                continue;
            }
            const int stage = n % kDecStages;
            if (n >= kDecStages && !mbar_wait(&sm.empty[stage], ((n / kDecStages) - 1) & 1, a.hdr, KID_ATTN_DECODE)) {
                ok = false;
                break;
            }
            const int c = pos / kBlock;
            int j = sm.ld_row[slot];
            if (j > c || j < 0) {
                record_error(a.hdr, MSA_ERR_DEVICE_BOUNDS, KID_ATTN_DECODE, bg, slot, j);
                j = -1;
            }
            const int ntok = j < 0 ? 0 : (j == c ? pos - c * kBlock + 1 : kBlock);
            sm.meta_bg[stage] = bg;
            sm.meta_ntok[stage] = ntok;
            sm.meta_fin[stage] = (slot == nsel - 1 || k + 1 == kend);
            sm.meta_nfrag[stage] = nfrag;
            sm.meta_frag[stage] = frag;
            const bool full = ntok == kBlock;
            const int nload = full ? kBlock : (ntok + kDecDiagRows - 1) / kDecDiagRows * kDecDiagRows;
            mbar_arrive_expect_tx(&sm.full_k[stage], uint32_t(nload) * 256u + uint32_t(Hg) * qrow);
            mbar_arrive_expect_tx(&sm.full_v[stage], uint32_t(nload) * 256u);
            const uint16_t* qg = a.q + size_t(bg) * Hg * kHeadDim;
            for (int h = 0; h < Hg; ++h) bulk_load(sm.q[stage][h], qg + h * kHeadDim, qrow, &sm.full_k[stage]);
            const int row0 = int(int64_t(bg) * a.l_cap + int64_t(j < 0 ? 0 : j) * kBlock);
            uint8_t* ks = sm.kv[stage][0];
            uint8_t* vs = sm.kv[stage][1];
            if (full) {
                for (int h = 0; h < 2; ++h)
                    tma_load_2d_hint(ks + h * 16384, &maps.k128, h * 64, row0, &sm.full_k[stage], pol);
                for (int h = 0; h < 2; ++h)
                    tma_load_2d_hint(vs + h * 16384, &maps.v128, h * 64, row0, &sm.full_v[stage], pol);
            } else {
                for (int r0 = 0; r0 < nload; r0 += kDecDiagRows)
                    for (int h = 0; h < 2; ++h)
                        tma_load_2d_hint(ks + h * 16384 + r0 * 128, &maps.k32, h * 64, row0 + r0, &sm.full_k[stage], pol);
                for (int r0 = 0; r0 < nload; r0 += kDecDiagRows)
                    for (int h = 0; h < 2; ++h)
                        tma_load_2d_hint(vs + h * 16384 + r0 * 128, &maps.v32, h * 64, row0 + r0, &sm.full_v[stage], pol);
            }
            ++n;
        }
        // end marker; after a wait that gave up the compute warps stop on their own bounded waits
        const int stage = n % kDecStages;
        if (ok && n >= kDecStages) mbar_wait(&sm.empty[stage], ((n / kDecStages) - 1) & 1, a.hdr, KID_ATTN_DECODE);
        sm.meta_bg[stage] = -1;
        mbar_arrive(&sm.full_k[stage]);
        return;
    }

    // -------------------------------------------------------------------- compute warps
    const uint32_t psm = smem_u32(&sm.p[0][0]);
    float o[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};   // heads gq, gq + 8 x 4 columns
    float lsum0 = 0.f, lsum1 = 0.f;                                 // this thread's share of the sums
    float Mrun0 = -INFINITY, Mrun1 = -INFINITY;                      // running maxima (log2 units)
    for (int n = 0;; ++n) {
        const int stage = n % kDecStages;
        const uint32_t ph = (n / kDecStages) & 1;
        // A wait that gives up, or the loader's end marker, stops every compute warp at barrier
        // (A) below, so that no warp is left waiting at a barrier the others have left.
        const bool okk = mbar_wait(&sm.full_k[stage], ph, a.hdr, KID_ATTN_DECODE);
        const int bg = sm.meta_bg[stage];
        const bool stop = !okk || bg < 0;
        int ntok = stop ? 0 : sm.meta_ntok[stage];
        const int fin = sm.meta_fin[stage], nfrag = sm.meta_nfrag[stage], frag = sm.meta_frag[stage];
        const uint8_t* Ks = sm.kv[stage][0];
        // ---- scores of keys 16w .. 16w + 15 (two n-tiles) for all heads (rows of the MMA)
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const int kbase = warp * 16;
        if (kbase < ntok) {
            const uint16_t* q0 = sm.q[stage][gq];
            const uint16_t* q1 = sm.q[stage][gq + 8];
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int d0 = ks * 16 + 2 * tq;
                const uint32_t a0 = *reinterpret_cast<const uint32_t*>(q0 + d0);
                const uint32_t a1 = *reinterpret_cast<const uint32_t*>(q1 + d0);
                const uint32_t a2 = *reinterpret_cast<const uint32_t*>(q0 + d0 + 8);
                const uint32_t a3 = *reinterpret_cast<const uint32_t*>(q1 + d0 + 8);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int key = kbase + nt * 8 + gq;
                    const uint8_t* kr = Ks + (ks >> 2) * 16384 + 4 * tq;
                    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(kr + sw128(key, (ks & 3) * 2));
                    const uint32_t b1 = *reinterpret_cast<const uint32_t*>(kr + sw128(key, (ks & 3) * 2 + 1));
                    mma_bf16_16816(s[nt], a0, a1, a2, a3, b0, b1);
                }
            }
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const bool v = kbase + nt * 8 + 2 * tq + e < ntok;
                s[nt][e] = v ? s[nt][e] * a.scale_log2 : -INFINITY;
                s[nt][2 + e] = v ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
                mx0 = fmaxf(mx0, s[nt][e]);
                mx1 = fmaxf(mx1, s[nt][2 + e]);
            }
        }
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        if (tq == 0) {
            sm.red_m[warp][gq] = mx0;
            sm.red_m[warp][gq + 8] = mx1;
        }
        if (compute_sync_or(stop)) break;                 // (A) per-warp maxima visible
        float Mi0 = -INFINITY, Mi1 = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            Mi0 = fmaxf(Mi0, sm.red_m[w][gq]);
            Mi1 = fmaxf(Mi1, sm.red_m[w][gq + 8]);
        }
        const float Mn0 = fmaxf(Mrun0, Mi0), Mn1 = fmaxf(Mrun1, Mi1);
        const float base0 = Mn0 == -INFINITY ? 0.f : Mn0, base1 = Mn1 == -INFINITY ? 0.f : Mn1;
        const float al0 = Mrun0 == -INFINITY ? 0.f : fast_exp2(Mrun0 - Mn0);
        const float al1 = Mrun1 == -INFINITY ? 0.f : fast_exp2(Mrun1 - Mn1);
        Mrun0 = Mn0;
        Mrun1 = Mn1;
        float l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const float p0 = fast_exp2(s[nt][0] - base0), p1 = fast_exp2(s[nt][1] - base0);
            const float p2 = fast_exp2(s[nt][2] - base1), p3 = fast_exp2(s[nt][3] - base1);
            l0 += p0 + p1;
            l1 += p2 + p3;
            const int col = kbase + nt * 8 + 2 * tq;
            *reinterpret_cast<uint32_t*>(&sm.p[gq][col]) = pack_bf16x2(p0, p1);
            *reinterpret_cast<uint32_t*>(&sm.p[gq + 8][col]) = pack_bf16x2(p2, p3);
            o[nt][0] *= al0; o[nt][1] *= al0;
            o[nt][2] *= al1; o[nt][3] *= al1;
        }
        lsum0 = lsum0 * al0 + l0;
        lsum1 = lsum1 * al1 + l1;
        // ---- V (rows past the query in the diagonal block must be finite: zero them)
        if (ntok > 0 && !mbar_wait(&sm.full_v[stage], ph, a.hdr, KID_ATTN_DECODE)) ntok = 0;
        if (ntok < kBlock) {
            uint8_t* vw = sm.kv[stage][1];
            const int nload = (ntok + kDecDiagRows - 1) / kDecDiagRows * kDecDiagRows;
            for (int i = tid; i < (nload - ntok) * 16; i += kDecWarps * 32) {
                const int row = ntok + i / 16, ch = i % 16;
                *reinterpret_cast<uint4*>(vw + (ch >> 3) * 16384 + sw128(row, ch & 7)) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async();                          // ordered before the stage's next TMA fill
        }
        compute_sync();                                   // (B) P and zeroed V rows visible
        // ---- o[:, 16w .. 16w + 15] += P V over the block's keys
        const int nks = (ntok + 15) / 16;
        const uint32_t vsm = smem_u32(sm.kv[stage][1]);
        for (int kk = 0; kk < nks; ++kk) {
            uint32_t a0, a1, a2, a3;                      // P rows 0-15 x keys 16kk .. 16kk + 15
            {
                const int prow = lane & 15, pcol = kk * 16 + (lane >> 4) * 8;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                             : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                             : "r"(psm + uint32_t(prow * kPRow + pcol) * 2u));
            }
            uint32_t v0, v1, v2, v3;
            const int row = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int col = warp * 16 + (lane >> 4) * 8;
            ldsm_x4_trans(vsm + kv_off(row, col), v0, v1, v2, v3);
            mma_bf16_16816(o[0], a0, a1, a2, a3, v0, v1);
            mma_bf16_16816(o[1], a0, a1, a2, a3, v2, v3);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stage]);    // this warp is done with the stage
        if (!fin) continue;

        // ---- end of this CTA's share of (b, g): combine the warps' sums
        const int b = bg / G, g = bg % G;
        float L0 = lsum0, L1 = lsum1;
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
            L0 += __shfl_xor_sync(0xffffffffu, L0, off);
            L1 += __shfl_xor_sync(0xffffffffu, L1, off);
        }
        if (tq == 0) {
            sm.red_l[warp][gq] = L0;
            sm.red_l[warp][gq + 8] = L1;
        }
        compute_sync();                                   // (C)
        L0 = 0.f;
        L1 = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            L0 += sm.red_l[w][gq];
            L1 += sm.red_l[w][gq + 8];
        }
        const size_t orow = size_t(b) * G * Hg + size_t(g) * Hg;
        if (nfrag == 1) {
            const float inv0 = 1.f / L0, inv1 = 1.f / L1;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int col = warp * 16 + nt * 8 + 2 * tq;
                if (gq < Hg)
                    *reinterpret_cast<uint32_t*>(a.out + (orow + gq) * kHeadDim + col) =
                        pack_bf16x2(o[nt][0] * inv0, o[nt][1] * inv0);
                if (gq + 8 < Hg)
                    *reinterpret_cast<uint32_t*>(a.out + (orow + gq + 8) * kHeadDim + col) =
                        pack_bf16x2(o[nt][2] * inv1, o[nt][3] * inv1);
            }
            if (a.lse != nullptr && warp == 0 && tq == 0) {
                if (gq < Hg) a.lse[orow + gq] = (Mrun0 + log2f(L0)) * 0.69314718055994530942f;
                if (gq + 8 < Hg) a.lse[orow + gq + 8] = (Mrun1 + log2f(L1)) * 0.69314718055994530942f;
            }
        } else {
            float* mypart = a.part + (size_t(bg) * kTopK + frag) * stride;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int col = warp * 16 + nt * 8 + 2 * tq;
                if (gq < Hg) *reinterpret_cast<float2*>(mypart + ooff + gq * kHeadDim + col) = make_float2(o[nt][0], o[nt][1]);
                if (gq + 8 < Hg)
                    *reinterpret_cast<float2*>(mypart + ooff + (gq + 8) * kHeadDim + col) = make_float2(o[nt][2], o[nt][3]);
            }
            if (warp == 0 && tq == 0) {
                if (gq < Hg) { mypart[gq] = Mrun0; mypart[Hg + gq] = L0; }
                if (gq + 8 < Hg) { mypart[gq + 8] = Mrun1; mypart[Hg + gq + 8] = L1; }
            }
            __threadfence();
            compute_sync();                               // (D) the partial is written
            if (tid == 0) sm.is_last = (atomicInc(a.ctr + bg, unsigned(nfrag - 1)) == unsigned(nfrag - 1));
            compute_sync();                               // (E)
            if (sm.is_last) {
                __threadfence();
                // merge the nfrag partials: stage (max, sum) pairs, then thread t produces 8 columns
                const float* pbase = a.part + size_t(bg) * kTopK * stride;
                for (int i = tid; i < nfrag * Hg; i += kDecWarps * 32) {
                    const int f = i / Hg, h = i % Hg;
                    sm.wts[f][h] = __ldcg(pbase + f * stride + h);
                    sm.ls[f][h] = __ldcg(pbase + f * stride + Hg + h);
                }
                compute_sync();
                if (tid < Hg) {
                    float M = -INFINITY;
                    for (int f = 0; f < nfrag; ++f) M = fmaxf(M, sm.wts[f][tid]);
                    float L = 0.f;
                    for (int f = 0; f < nfrag; ++f) {
                        const float m = sm.wts[f][tid];
                        const float wf = (m == -INFINITY) ? 0.f : fast_exp2(m - M);
                        L += sm.ls[f][tid] * wf;
                        sm.wts[f][tid] = wf;
                    }
                    sm.mrg_m[tid] = M;
                    sm.mrg_l[tid] = L;
                }
                compute_sync();
                for (int base = tid * 8; base < Hg * kHeadDim; base += kDecWarps * 32 * 8) {
                    const int h = base / kHeadDim, col = base % kHeadDim;
                    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                    for (int f = 0; f < nfrag; ++f) {
                        const float4* src = reinterpret_cast<const float4*>(pbase + f * stride + ooff + h * kHeadDim + col);
                        const float4 x = __ldcg(src), y = __ldcg(src + 1);
                        const float wf = sm.wts[f][h];
                        acc[0] = fmaf(wf, x.x, acc[0]); acc[1] = fmaf(wf, x.y, acc[1]);
                        acc[2] = fmaf(wf, x.z, acc[2]); acc[3] = fmaf(wf, x.w, acc[3]);
                        acc[4] = fmaf(wf, y.x, acc[4]); acc[5] = fmaf(wf, y.y, acc[5]);
                        acc[6] = fmaf(wf, y.z, acc[6]); acc[7] = fmaf(wf, y.w, acc[7]);
                    }
                    const float inv = 1.f / sm.mrg_l[h];
                    uint4 ov;
                    ov.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
                    ov.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
                    ov.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
                    ov.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
                    *reinterpret_cast<uint4*>(a.out + (orow + h) * kHeadDim + col) = ov;
                    if (a.lse != nullptr && col == 0)
                        a.lse[orow + h] = (sm.mrg_m[h] + log2f(sm.mrg_l[h])) * 0.69314718055994530942f;
                }
                compute_sync();                           // merge buffers free for the next group
            }
        }
        o[0][0] = o[0][1] = o[0][2] = o[0][3] = 0.f;
        o[1][0] = o[1][1] = o[1][2] = o[1][3] = 0.f;
        lsum0 = lsum1 = 0.f;
        Mrun0 = Mrun1 = -INFINITY;
    }
}

size_t decode_attn_ws_bytes(int B, int G, int Hg) {
    const size_t nbg = size_t(B) * G;
    return sizeof(WsHeader) + (nbg * sizeof(unsigned int) + 255) / 256 * 256 +
           nbg * kTopK * dec_part_stride(Hg) * sizeof(float);
}

int num_sms();

msa_status_t launch_attn_decode(const void* k_cache, const void* v_cache, const void* q, int64_t l_cap,
                                const int32_t* q_pos, int64_t max_pos, const int32_t* sel, int B, int G, int Hg,
                                void* out, float* lse, void* ws, cudaStream_t st) {
    DecMaps maps;
    const uint64_t rows = uint64_t(B) * G * uint64_t(l_cap);
    msa_status_t e = make_tmap_bf16(&maps.k128, k_cache, rows, kHeadDim, 64, 128);
    if (e == MSA_OK) e = make_tmap_bf16(&maps.v128, v_cache, rows, kHeadDim, 64, 128);
    if (e == MSA_OK) e = make_tmap_bf16(&maps.k32, k_cache, rows, kHeadDim, 64, kDecDiagRows);
    if (e == MSA_OK) e = make_tmap_bf16(&maps.v32, v_cache, rows, kHeadDim, 64, kDecDiagRows);
    if (e != MSA_OK) return e;
    const size_t nbg = size_t(B) * G;
    char* p = static_cast<char*>(ws);
    DecArgs a;
    a.q = static_cast<const uint16_t*>(q);
    a.l_cap = l_cap; a.max_pos = max_pos; a.q_pos = q_pos; a.sel = sel;
    a.B = B; a.G = G; a.Hg = Hg;
    a.out = static_cast<uint16_t*>(out); a.lse = lse;
    a.hdr = reinterpret_cast<WsHeader*>(p);
    a.ctr = reinterpret_cast<unsigned int*>(p + sizeof(WsHeader));
    a.part = reinterpret_cast<float*>(p + sizeof(WsHeader) + (nbg * sizeof(unsigned int) + 255) / 256 * 256);
    a.scale_log2 = 1.4426950408889634f / sqrtf(float(kHeadDim));
    const int smem = int(sizeof(DecSmem)) + 1024;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        cudaFuncSetAttribute(attn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        attr_set[dev] = true;
    }
    const int64_t n_items = int64_t(B) * G * kTopK;
    const int grid = int(n_items < num_sms() ? n_items : num_sms());   // persistent: one CTA per SM
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap with the selection's tail
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launch();
    cudaLaunchKernelEx(&cfg, attn_decode_kernel, maps, a);
    return cuda_status();
}

}  // namespace msa

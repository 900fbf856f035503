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
// so every CTA streams the same number of 64 KB K+V blocks. Warp roles:
//   * loader (warp 8): streams each item's K and V block -- two contiguous 32 KB ranges of the
//     head-major cache -- and the group's query rows with TMA into a 3-deep ring of stages;
//   * compute (warps 0-7): warp w owns keys 16w..16w+15 of every block. It scores them for all
//     Hg heads with warp MMAs, turns them into probabilities in registers (the accumulator
//     layout of S is the A-operand layout of P) and accumulates all 128 output columns with
//     its own online softmax, so the warps never wait for one another. At the last item of a
//     group in this CTA each warp parks its state in its own 16 rows of the stage. When the
//     whole group ran in this CTA the 8 warps then fold the parked states together (warp w
//     the output columns 16w..16w+15) and write the output;
//   * epilogue (warp 9), for a group split across CTAs: folds the 8 parked states by
//     log-sum-exp, releases the stage, and deals with the other CTAs that hold parts of the
//     group: if all of them are in it merges their partials (max, sum, o) into its registers,
//     otherwise it leaves its own partial for the last one to arrive. None of this
//     global-memory traffic stalls the compute warps.
#include <atomic>

#include "msa_common.cuh"

namespace msa {

constexpr int kDecWarps = 8;           // compute warps; warp 8 loads, warp 9 finishes groups
constexpr int kDecLoader = kDecWarps, kDecEpi = kDecWarps + 1;
constexpr int kDecThreads = (kDecWarps + 2) * 32;
constexpr int kDecStages = 3;
constexpr int kDecDiagRows = 32;       // row granularity of the diagonal block's loads
constexpr int kQRow = 136;             // bf16 elements per query row in shared memory (padded)
constexpr int kRowCache = 8;           // selection rows the loader fetches per round trip

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
    CUtensorMap k8, v8;                 // FP8 variant: e4m3 codes, boxes of 128 bytes x 128 rows (full blocks)
};

struct __align__(1024) DecSmem {
    uint8_t kv[kDecStages][2][32768];           // [stage][K, V][d half][128 rows][128 B]
    uint16_t q[kDecStages][kMaxHg][kQRow];      // the item's query heads (rows padded)
    float pm[kDecStages][kDecWarps][kMaxHg];    // parked warp states: max and sum per head
    float pl[kDecStages][kDecWarps][kMaxHg];
    float4 ot[16][32];                          // epilogue: other CTAs' parts of its last group
    float om[kMaxHg], ol[kMaxHg];
    uint64_t full_k[kDecStages], full_v[kDecStages], empty[kDecStages];
    uint64_t parked[kDecStages];                // 8 warp states parked (queue of group ends)
    uint64_t fold;                              // 8 warp states parked for a fold by the compute warps
    int meta_bg[kDecStages], meta_ntok[kDecStages], meta_fin[kDecStages], meta_nfrag[kDecStages],
        meta_frag[kDecStages], meta_fp8[kDecStages];
    float meta_ks[kDecStages], meta_vs[kDecStages];   // FP8 variant: the block's key / value scales
    int park_stage[kDecStages];                 // stage holding the parked states (-1 = end)
    int row_sel[kRowCache][kTopK];              // loader: selection rows and positions
    int row_pos[kRowCache];
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
    double inv_grid, inv_items;                 // 1 / gridDim.x, 1 / (B G 16)
    const float* k_scale;                       // FP8 variant: [B, G, nb_cap] per-block scales
    const float* v_scale;
    int64_t nb_cap;
};

// FP8 variant: widen this warp's 16 rows (kbase..kbase+15) of an e4m3 value block, which TMA
// left as [128 rows][128 B] (128B swizzle) at the start of `buf`, in place into f16 in the
// 16-bit tile layout of the full blocks ([d half][128 rows][128 B], 128B swizzle), so that the
// P V step reads it like a bf16 block. The source bytes of a row lie inside the row's half-0
// destination, which only this warp writes, so every lane reads its codes before any lane
// writes.
__device__ __forceinline__ void widen_fp8_rows(uint8_t* buf, int kbase, int lane) {
    const int row = kbase + (lane >> 1), h = lane & 1;      // lane pair per row, one d half each
    uint4 c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int ch = 4 * h + i;                           // 16 codes: d = 16 ch .. 16 ch + 15
        c[i] = *reinterpret_cast<const uint4*>(buf + row * 128 + ((ch ^ (row & 7)) << 4));
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t w[4] = {c[i].x, c[i].y, c[i].z, c[i].w};
        uint32_t o[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            o[2 * e] = f16x2_from_e4m3x2(uint16_t(w[e] & 0xFFFFu));
            o[2 * e + 1] = f16x2_from_e4m3x2(uint16_t(w[e] >> 16));
        }
        // codes d = 64 h + 16 i .. +15 -> chunks (2 i) and (2 i + 1) of d half h
        *reinterpret_cast<uint4*>(buf + h * 16384 + sw128(row, 2 * i)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(buf + h * 16384 + sw128(row, 2 * i + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
    }
    __syncwarp();
}

// first item of CTA c when n items are cut into `grid` contiguous ranges: floor(c * n / grid)
__device__ __forceinline__ int range_begin(int c, int n, int grid, double inv_grid) {
    const long long t = (long long)c * n;
    int b = int(double(t) * inv_grid);
    while ((long long)(b + 1) * grid <= t) ++b;
    while ((long long)b * grid > t) --b;
    return b;
}

// the CTA whose range holds item k: the largest c with c * n < (k + 1) * grid
__device__ __forceinline__ int range_owner(int k, int n, int grid, double inv_n) {
    const long long t = (long long)(k + 1) * grid - 1;
    int c = int(double(t) * inv_n);
    while ((long long)(c + 1) * n <= t) ++c;
    while ((long long)c * n > t) --c;
    return c < grid - 1 ? c : grid - 1;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// raise the transaction count of the current phase without arriving
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive_n(uint64_t* bar, uint32_t n) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(n) : "memory");
}

// bounded wait by every lane of a warp, with one outcome for the whole warp
__device__ __forceinline__ bool warp_wait_all(uint64_t* bar, uint32_t parity, WsHeader* hdr) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, hdr, KID_ATTN_DECODE));
}

// log-sum-exp weights of two states with maxima m (own) and mo (other), log2 units
__device__ __forceinline__ void lse_weights(float m, float mo, float& mn, float& wa, float& wb) {
    mn = fmaxf(m, mo);
    wa = m == -INFINITY ? 0.f : fast_exp2(m - mn);
    wb = mo == -INFINITY ? 0.f : fast_exp2(mo - mn);
}

// A warp's part of an (unnormalised) attention state, in the accumulator layout of m16n8:
// rows (heads) gq and gq + 8, columns 8 nt + 2 tq + {0, 1}.
struct WarpState {
    float o[16][4];
    float m0, m1;        // maxima of rows gq, gq + 8 (log2 units)
    float l0, l1;        // sums
};

// Accumulators of a lane in groups of four: group g < 8 holds row gq, columns 16 g + 2 tq +
// {0, 1, 8, 9} (o[2g][0..1], o[2g+1][0..1]); group g >= 8 the same for row gq + 8.
__device__ __forceinline__ float4 acc_group(const WarpState& st, int g) {
    const int e = (g >> 3) << 1, nt = (g & 7) << 1;
    return make_float4(st.o[nt][e], st.o[nt][e + 1], st.o[nt + 1][e], st.o[nt + 1][e + 1]);
}
__device__ __forceinline__ void set_acc_group(WarpState& st, int g, float4 x) {
    const int e = (g >> 3) << 1, nt = (g & 7) << 1;
    st.o[nt][e] = x.x; st.o[nt][e + 1] = x.y; st.o[nt + 1][e] = x.z; st.o[nt + 1][e + 1] = x.w;
}

// Parked state of warp w in stage s: group g of lane l sits in the warp's own K rows (g < 8)
// or V rows (g >= 8), 512 B (32 lanes x 16 B) per group.
__device__ __forceinline__ float4* park_addr(DecSmem& sm, int s, int w, int g, int lane) {
    uint8_t* chunk = sm.kv[s][g >> 3] + ((g >> 2) & 1) * 16384 + w * 2048 + (g & 3) * 512;
    return reinterpret_cast<float4*>(chunk) + lane;
}

// Fold the partial of another CTA (max, sum, o of rows gq, gq + 8) into st.
// Every load of the partial goes out before any value is used (rows gq, gq + 8 past Hg read
// row 0 and are ignored).
__device__ __forceinline__ void merge_partial(WarpState& st, const float* pf, int Hg, int ooff, int gq, int tq) {
    const int r0 = gq < Hg ? gq : 0, r1 = gq + 8 < Hg ? gq + 8 : 0;
    const float2 ml0 = ld_cg_f2pair(pf + r0, pf + Hg + r0), ml1 = ld_cg_f2pair(pf + r1, pf + Hg + r1);
    const float m0 = ml0.x, l0 = ml0.y, m1 = ml1.x, l1 = ml1.y;
    float2 x0[16], x1[16];
    ld_cg_f2x16_s32(pf + ooff + r0 * kHeadDim + 2 * tq, x0);
    ld_cg_f2x16_s32(pf + ooff + r1 * kHeadDim + 2 * tq, x1);
    float wa0 = 1.f, wb0 = 0.f, wa1 = 1.f, wb1 = 0.f, mn;
    if (gq < Hg) {
        lse_weights(st.m0, m0, mn, wa0, wb0);
        st.l0 = st.l0 * wa0 + l0 * wb0;
        st.m0 = mn;
    }
    if (gq + 8 < Hg) {
        lse_weights(st.m1, m1, mn, wa1, wb1);
        st.l1 = st.l1 * wa1 + l1 * wb1;
        st.m1 = mn;
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
        if (gq < Hg) {
            st.o[nt][0] = st.o[nt][0] * wa0 + x0[nt].x * wb0;
            st.o[nt][1] = st.o[nt][1] * wa0 + x0[nt].y * wb0;
        }
        if (gq + 8 < Hg) {
            st.o[nt][2] = st.o[nt][2] * wa1 + x1[nt].x * wb1;
            st.o[nt][3] = st.o[nt][3] * wa1 + x1[nt].y * wb1;
        }
    }
}

// A group whose items all ran in this CTA is finished by the 8 compute warps together: once all
// have parked their states in the stage, warp w folds column group w (columns 16 w .. 16 w + 15;
// group w + 8 for rows gq + 8 when Hg > 8) of the 8 states by log-sum-exp and writes those
// output columns, so the fold runs 8 warps wide instead of on the epilogue warp alone.
__device__ __forceinline__ void fold_write_columns(DecSmem& sm, int stage, int warp, int lane, int Hg,
                                                   size_t orow, uint16_t* __restrict__ out, float* __restrict__ lse) {
    const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int row = gq + 8 * half;
        if (row >= Hg) continue;
        const int g = warp + 8 * half;
        float mw[kDecWarps];
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            mw[w] = sm.pm[stage][w][row];
            M = fmaxf(M, mw[w]);
        }
        float L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            const float wt = mw[w] == -INFINITY ? 0.f : fast_exp2(mw[w] - M);
            L += sm.pl[stage][w][row] * wt;
            const float4 x = *park_addr(sm, stage, w, g, lane);
            acc.x += x.x * wt; acc.y += x.y * wt; acc.z += x.z * wt; acc.w += x.w * wt;
        }
        const float inv = 1.f / L;
        uint16_t* o = out + (orow + row) * kHeadDim + 16 * warp + 2 * tq;
        *reinterpret_cast<uint32_t*>(o) = pack_bf16x2(acc.x * inv, acc.y * inv);
        *reinterpret_cast<uint32_t*>(o + 8) = pack_bf16x2(acc.z * inv, acc.w * inv);
        if (lse != nullptr && warp == 0 && tq == 0) lse[orow + row] = (M + log2f(L)) * 0.69314718055994530942f;
    }
}

__device__ __forceinline__ void clear_state(WarpState& st) {
#pragma unroll
    for (int i = 0; i < 16; ++i) st.o[i][0] = st.o[i][1] = st.o[i][2] = st.o[i][3] = 0.f;
    st.m0 = st.m1 = -INFINITY;
    st.l0 = st.l1 = 0.f;
}

template <bool kFp8>
__global__ void __launch_bounds__(kDecThreads, 1) attn_decode_kernel(const __grid_constant__ DecMaps maps,
                                                                    const DecArgs a) {
    extern __shared__ uint8_t smem_raw[];
    DecSmem& sm = *reinterpret_cast<DecSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int Hg = a.Hg, G = a.G;
    const int n_items = a.B * G * kTopK;

    if (tid == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(&sm.full_k[s], 1);
            mbar_init(&sm.full_v[s], 1);
            mbar_init(&sm.empty[s], kDecWarps);
            mbar_init(&sm.parked[s], kDecWarps);
        }
        mbar_init(&sm.fold, kDecWarps);
        fence_barrier_init();
    }
    for (int i = tid; i < kDecStages * kMaxHg * kQRow; i += kDecThreads) (&sm.q[0][0][0])[i] = 0;   // rows >= Hg stay 0
    __syncthreads();
    grid_dep_wait();                   // the selection and the appended token are ready from here on

    if (warp == kDecLoader) {
        // ---------------------------------------------------------------- loader warp
        // Streams the items of this CTA's range into the ring (lane 0 issues the copies),
        // skipping empty slots, and ends with an end marker (bg = -1).
        const int kbeg = range_begin(blockIdx.x, n_items, gridDim.x, a.inv_grid);
        const int kend = range_begin(blockIdx.x + 1, n_items, gridDim.x, a.inv_grid);
        const uint64_t pol = l2_evict_first();               // K and V are read once
        const uint32_t qrow = kHeadDim * 2u;
        int cache0 = 0, cachen = 0;                           // groups [cache0, cache0 + cachen) fetched
        int cur_bg = -1, pos = 0, nsel = 0, nfrag = 1, frag = 0;
        float ks_l = 1.f, vs_l = 1.f;                        // FP8: scales of the group's slot `lane`
        bool need_frag = false;
        int n = 0;
        bool ok = true;
        // The range is walked rotated: first the part of its last group (the next CTA finishes
        // that group last), then from its first item on. So this CTA ends with the tail of a
        // group whose head the previous CTA took first, and its epilogue warp has usually
        // merged that head before the tail arrives.
        const int kmid = max(kbeg, (kend - 1) / kTopK * kTopK);
        for (int idx = 0; idx < kend - kbeg; ++idx) {
            const bool first_seg = idx < kend - kmid;
            const int k = first_seg ? kmid + idx : kbeg + (idx - (kend - kmid));
            const int seg_end = first_seg ? kend : kmid;
            const int bg = k / kTopK, slot = k % kTopK;
            if (bg != cur_bg) {
                cur_bg = bg;
                if (bg < cache0 || bg >= cache0 + cachen) {   // fetch the next rows in one round trip
                    const int left = (seg_end - 1) / kTopK - bg + 1;
                    cache0 = bg;
                    cachen = left < kRowCache ? left : kRowCache;
                    __syncwarp();
                    if (lane < cachen * 4) {
                        const int4 v = __ldcg(reinterpret_cast<const int4*>(a.sel + size_t(bg) * kTopK) + lane);
                        int* d = &sm.row_sel[lane >> 2][(lane & 3) * 4];
                        d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
                    }
                    if (lane < cachen) sm.row_pos[lane] = __ldcg(a.q_pos + (bg + lane) / G);
                    __syncwarp();
                }
                const int r = bg - cache0;
                pos = sm.row_pos[r];
                nsel = 0;
#pragma unroll
                for (int i = 0; i < kTopK; ++i) nsel += sm.row_sel[r][i] >= 0;
                if (pos < 0 || pos > a.max_pos || pos >= a.l_cap) {
                    if (lane == 0 && slot == 0) record_error(a.hdr, MSA_ERR_DEVICE_BOUNDS, KID_ATTN_DECODE, bg, 0, pos);
                    nsel = 0;
                }
                need_frag = nsel > 0;
                if constexpr (kFp8) {
                    // the scales of all the group's closed blocks in one round trip (lane i: slot i),
                    // instead of one dependent load per item on the issuing lane
                    ks_l = vs_l = 1.f;
                    const int jl = lane < kTopK ? sm.row_sel[r][lane] : -1;
                    if (nsel > 0 && jl >= 0 && jl < pos / kBlock) {
                        const size_t si = size_t(bg) * a.nb_cap + jl;
                        ks_l = __ldg(a.k_scale + si);
                        vs_l = __ldg(a.v_scale + si);
                    }
                }
            }
            if (slot >= nsel) continue;                       // the row's tail is empty
            const int stage = n % kDecStages;
            if (n >= kDecStages) {
                bool w = true;
                if (lane == 0) w = mbar_wait(&sm.empty[stage], ((n / kDecStages) - 1) & 1, a.hdr, KID_ATTN_DECODE);
                if (!__shfl_sync(0xffffffffu, w, 0)) {
                    ok = false;
                    break;
                }
            }
            // The copies go out first; the item's description and the arrivals that complete the
            // stage follow (the phase cannot complete before those arrivals).
            float ksv = 1.f, vsv = 1.f;
            if constexpr (kFp8) {
                ksv = __shfl_sync(0xffffffffu, ks_l, slot);
                vsv = __shfl_sync(0xffffffffu, vs_l, slot);
            }
            int ntok = 0;
            if (lane == 0) {
                const int c = pos / kBlock;
                int j = sm.row_sel[bg - cache0][slot];
                if (j > c || j < 0) {
                    record_error(a.hdr, MSA_ERR_DEVICE_BOUNDS, KID_ATTN_DECODE, bg, slot, j);
                    j = -1;
                }
                ntok = j < 0 ? 0 : (j == c ? pos - c * kBlock + 1 : kBlock);
                const bool full = ntok == kBlock;
                const bool f8 = kFp8 && j >= 0 && j < c;          // a closed block: e4m3 codes
                const int nload = full ? kBlock : (ntok + kDecDiagRows - 1) / kDecDiagRows * kDecDiagRows;
                const uint32_t row_bytes = f8 ? 128u : 256u;
                mbar_expect_tx(&sm.full_k[stage], uint32_t(nload) * row_bytes + uint32_t(Hg) * qrow);
                mbar_expect_tx(&sm.full_v[stage], uint32_t(nload) * row_bytes);
                const int row0 = int(int64_t(bg) * a.l_cap + int64_t(j < 0 ? 0 : j) * kBlock);
                uint8_t* ks = sm.kv[stage][0];
                uint8_t* vs = sm.kv[stage][1];
                sm.meta_fp8[stage] = f8 ? 1 : 0;
                if (f8) {
                    tma_load_2d_hint(ks, &maps.k8, 0, row0, &sm.full_k[stage], pol);
                } else if (full) {
                    for (int h = 0; h < 2; ++h)
                        tma_load_2d_hint(ks + h * 16384, &maps.k128, h * 64, row0, &sm.full_k[stage], pol);
                } else {
                    for (int r0 = 0; r0 < nload; r0 += kDecDiagRows)
                        for (int h = 0; h < 2; ++h)
                            tma_load_2d_hint(ks + h * 16384 + r0 * 128, &maps.k32, h * 64, row0 + r0, &sm.full_k[stage], pol);
                }
                const uint16_t* qg = a.q + size_t(bg) * Hg * kHeadDim;
                for (int h = 0; h < Hg; ++h) bulk_load(sm.q[stage][h], qg + h * kHeadDim, qrow, &sm.full_k[stage]);
                if (f8) {
                    tma_load_2d_hint(vs, &maps.v8, 0, row0, &sm.full_v[stage], pol);
                    sm.meta_ks[stage] = ksv;
                    sm.meta_vs[stage] = vsv;
                } else if (full) {
                    for (int h = 0; h < 2; ++h)
                        tma_load_2d_hint(vs + h * 16384, &maps.v128, h * 64, row0, &sm.full_v[stage], pol);
                } else {
                    for (int r0 = 0; r0 < nload; r0 += kDecDiagRows)
                        for (int h = 0; h < 2; ++h)
                            tma_load_2d_hint(vs + h * 16384 + r0 * 128, &maps.v32, h * 64, row0 + r0, &sm.full_v[stage], pol);
                }
            }
            if (need_frag) {                                  // parts of this group in other CTAs
                const int c0 = range_owner(bg * kTopK, n_items, gridDim.x, a.inv_items);
                const int c1 = range_owner(bg * kTopK + nsel - 1, n_items, gridDim.x, a.inv_items);
                nfrag = c1 - c0 + 1;
                frag = int(blockIdx.x) - c0;
                need_frag = false;
            }
            if (lane == 0) {
                sm.meta_bg[stage] = bg;
                sm.meta_ntok[stage] = ntok;
                sm.meta_fin[stage] = (slot == nsel - 1 || k + 1 == seg_end);
                sm.meta_nfrag[stage] = nfrag;
                sm.meta_frag[stage] = frag;
                mbar_arrive(&sm.full_k[stage]);
                mbar_arrive(&sm.full_v[stage]);
            }
            __syncwarp();
            ++n;
        }
        if (lane == 0) {
            // end marker; after a wait that gave up the other warps stop on their own bounded waits
            const int stage = n % kDecStages;
            if (ok && n >= kDecStages) mbar_wait(&sm.empty[stage], ((n / kDecStages) - 1) & 1, a.hdr, KID_ATTN_DECODE);
            sm.meta_bg[stage] = -1;
            mbar_arrive(&sm.full_k[stage]);
        }
        return;
    }

    if (warp == kDecEpi) {
        // ---------------------------------------------------------------- epilogue warp
        const int stride = dec_part_stride(Hg), ooff = dec_part_ooff(Hg);
        const int ngroups = Hg > 8 ? 16 : 8;
        // The last group this CTA works on: when its other parts live in other CTAs (which reach
        // them first), merge those partials while the compute warps still work, so that the
        // group's output leaves without further global round trips.
        int tgt_bg = -1, tgt_nfrag = 1, tgt_frag = 0;
        {
            // the group the loader walks last (see the rotated walk above)
            const int kbeg = range_begin(blockIdx.x, n_items, gridDim.x, a.inv_grid);
            const int kend = range_begin(blockIdx.x + 1, n_items, gridDim.x, a.inv_grid);
            const int kmid = max(kbeg, (kend - 1) / kTopK * kTopK);
            const int bgl = kmid > kbeg ? (kmid - 1) / kTopK : (kend - 1) / kTopK;
            const int v = lane < kTopK ? __ldcg(a.sel + size_t(bgl) * kTopK + lane) : -1;
            const int nsel = __popc(__ballot_sync(0xffffffffu, v >= 0));
            const int pos = __ldcg(a.q_pos + bgl / G);
            if (!(pos < 0 || pos > a.max_pos || pos >= a.l_cap) && nsel > 0) {
                const int c0 = range_owner(bgl * kTopK, n_items, gridDim.x, a.inv_items);
                const int c1 = range_owner(bgl * kTopK + nsel - 1, n_items, gridDim.x, a.inv_items);
                if (int(blockIdx.x) >= c0 && int(blockIdx.x) <= c1 && c1 > c0) {
                    tgt_bg = bgl;
                    tgt_nfrag = c1 - c0 + 1;
                    tgt_frag = int(blockIdx.x) - c0;
                }
            }
        }
        int pre = tgt_bg >= 0 ? 1 : 0;                        // 1: others pending, 2: merged in ot
        WarpState st;
        for (int f = 0;; ++f) {
            const int qs = f % kDecStages;
            const uint32_t par = (f / kDecStages) & 1;
            bool got = false;
            const long long t0 = clock64();
            while (true) {
                got = __all_sync(0xffffffffu, mbar_try_wait(&sm.parked[qs], par));
                if (got) break;
                if (pre == 1) {
                    unsigned cnt = 0;
                    if (lane == 0) cnt = ld_acquire_gpu(a.ctr + tgt_bg);
                    if (__shfl_sync(0xffffffffu, cnt, 0) == unsigned(tgt_nfrag - 1)) {
                        clear_state(st);
                        for (int fo = 0; fo < tgt_nfrag; ++fo)
                            if (fo != tgt_frag)
                                merge_partial(st, a.part + (size_t(tgt_bg) * kTopK + fo) * stride, Hg, ooff, gq, tq);
#pragma unroll
                        for (int g = 0; g < 16; ++g)
                            if (g < ngroups) sm.ot[g][lane] = acc_group(st, g);
                        if (tq == 0) {
                            sm.om[gq] = st.m0; sm.om[gq + 8] = st.m1;
                            sm.ol[gq] = st.l0; sm.ol[gq + 8] = st.l1;
                        }
                        __syncwarp();
                        pre = 2;
                    } else {
                        __nanosleep(500);
                    }
                }
                if (clock64() - t0 > kWaitCycles) {
                    if (lane == 0) record_error(a.hdr, MSA_ERR_TIMEOUT, KID_ATTN_DECODE, blockIdx.x, threadIdx.x, int(par));
                    break;
                }
            }
            if (!got) break;
            const int stage = sm.park_stage[qs];
            if (stage < 0) break;
            const int bg = sm.meta_bg[stage], nfrag = sm.meta_nfrag[stage], frag = sm.meta_frag[stage];
            const bool premerged = pre == 2 && bg == tgt_bg;
            // fold the 8 parked warp states (and the pre-merged other parts)
            float mw0[kDecWarps + 1], mw1[kDecWarps + 1];
            st.m0 = st.m1 = -INFINITY;
#pragma unroll
            for (int w = 0; w < kDecWarps + 1; ++w) {
                mw0[w] = w < kDecWarps ? sm.pm[stage][w][gq] : (premerged ? sm.om[gq] : -INFINITY);
                mw1[w] = w < kDecWarps ? sm.pm[stage][w][gq + 8] : (premerged ? sm.om[gq + 8] : -INFINITY);
                st.m0 = fmaxf(st.m0, mw0[w]);
                st.m1 = fmaxf(st.m1, mw1[w]);
            }
            st.l0 = st.l1 = 0.f;
#pragma unroll
            for (int w = 0; w < kDecWarps + 1; ++w) {
                mw0[w] = mw0[w] == -INFINITY ? 0.f : fast_exp2(mw0[w] - st.m0);
                mw1[w] = mw1[w] == -INFINITY ? 0.f : fast_exp2(mw1[w] - st.m1);
                st.l0 += (w < kDecWarps ? sm.pl[stage][w][gq] : (premerged ? sm.ol[gq] : 0.f)) * mw0[w];
                st.l1 += (w < kDecWarps ? sm.pl[stage][w][gq + 8] : (premerged ? sm.ol[gq + 8] : 0.f)) * mw1[w];
            }
#pragma unroll
            for (int g = 0; g < 16; ++g) {
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                if (g < ngroups) {
#pragma unroll
                    for (int w = 0; w < kDecWarps; ++w) {
                        const float4 x = *park_addr(sm, stage, w, g, lane);
                        const float wt = g >= 8 ? mw1[w] : mw0[w];
                        acc.x += x.x * wt; acc.y += x.y * wt; acc.z += x.z * wt; acc.w += x.w * wt;
                    }
                    if (premerged) {
                        const float4 x = sm.ot[g][lane];
                        const float wt = g >= 8 ? mw1[kDecWarps] : mw0[kDecWarps];
                        acc.x += x.x * wt; acc.y += x.y * wt; acc.z += x.z * wt; acc.w += x.w * wt;
                    }
                }
                set_acc_group(st, g, acc);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_n(&sm.empty[stage], kDecWarps);   // the stage may be refilled

            const int b = bg / G, g = bg % G;
            const size_t orow = size_t(b) * G * Hg + size_t(g) * Hg;
            bool last = nfrag == 1 || premerged;
            if (premerged && lane == 0) *reinterpret_cast<volatile unsigned*>(a.ctr + bg) = 0u;   // ready for the next call
            if (!last) {
                // Parts of a split group: if all the others are in, merge them into these
                // registers; otherwise leave this one for the last to arrive.
                unsigned cnt = 0;
                if (lane == 0) cnt = ld_acquire_gpu(a.ctr + bg);
                cnt = __shfl_sync(0xffffffffu, cnt, 0);
                if (cnt == unsigned(nfrag - 1)) {
                    last = true;
                    if (lane == 0) *reinterpret_cast<volatile unsigned*>(a.ctr + bg) = 0u;
                } else {
                    float* mypart = a.part + (size_t(bg) * kTopK + frag) * stride;
                    if (tq == 0) {
                        if (gq < Hg) { mypart[gq] = st.m0; mypart[Hg + gq] = st.l0; }
                        if (gq + 8 < Hg) { mypart[gq + 8] = st.m1; mypart[Hg + gq + 8] = st.l1; }
                    }
#pragma unroll
                    for (int nt = 0; nt < 16; ++nt) {
                        const int col = nt * 8 + 2 * tq;
                        if (gq < Hg)
                            *reinterpret_cast<float2*>(mypart + ooff + gq * kHeadDim + col) = make_float2(st.o[nt][0], st.o[nt][1]);
                        if (gq + 8 < Hg)
                            *reinterpret_cast<float2*>(mypart + ooff + (gq + 8) * kHeadDim + col) =
                                make_float2(st.o[nt][2], st.o[nt][3]);
                    }
                    __syncwarp();
                    unsigned old = 0;
                    if (lane == 0) {
                        __threadfence();
                        old = atomicInc(a.ctr + bg, unsigned(nfrag - 1));
                    }
                    last = __shfl_sync(0xffffffffu, old, 0) == unsigned(nfrag - 1);
                }
                if (last) {
                    __threadfence();
                    for (int fo = 0; fo < nfrag; ++fo)
                        if (fo != frag) merge_partial(st, a.part + (size_t(bg) * kTopK + fo) * stride, Hg, ooff, gq, tq);
                }
            }
            if (last) {
                const float inv0 = 1.f / st.l0, inv1 = 1.f / st.l1;
#pragma unroll
                for (int nt = 0; nt < 16; ++nt) {
                    const int col = nt * 8 + 2 * tq;
                    if (gq < Hg)
                        *reinterpret_cast<uint32_t*>(a.out + (orow + gq) * kHeadDim + col) =
                            pack_bf16x2(st.o[nt][0] * inv0, st.o[nt][1] * inv0);
                    if (gq + 8 < Hg)
                        *reinterpret_cast<uint32_t*>(a.out + (orow + gq + 8) * kHeadDim + col) =
                            pack_bf16x2(st.o[nt][2] * inv1, st.o[nt][3] * inv1);
                }
                if (a.lse != nullptr && tq == 0) {
                    if (gq < Hg) a.lse[orow + gq] = (st.m0 + log2f(st.l0)) * 0.69314718055994530942f;
                    if (gq + 8 < Hg) a.lse[orow + gq + 8] = (st.m1 + log2f(st.l1)) * 0.69314718055994530942f;
                }
            }
        }
        return;
    }

    // -------------------------------------------------------------------- compute warps
    // Every wait below is bounded; a warp whose wait gives up leaves the loop, and the others
    // then give up at their next wait for it.
    const int kbase = warp * 16;
    WarpState st;
    clear_state(st);
    int nfin = 0;                                       // group ends parked so far
    int nfold = 0;                                      // groups folded by the compute warps so far
    for (int n = 0;; ++n) {
        const int stage = n % kDecStages;
        const uint32_t ph = (n / kDecStages) & 1;
        if (!warp_wait_all(&sm.full_k[stage], ph, a.hdr)) break;
        const int bg = sm.meta_bg[stage];
        if (bg < 0) {                                   // end: tell the epilogue warp
            const int qs = nfin % kDecStages;
            if (warp == 0 && lane == 0) sm.park_stage[qs] = -1;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.parked[qs]);
            break;
        }
        const int ntok = sm.meta_ntok[stage], fin = sm.meta_fin[stage];
        const bool active = kbase < ntok;
        const bool f8 = kFp8 && sm.meta_fp8[stage] != 0;   // e4m3 codes: scores and P take the scales
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        if (f8) {
            // FP8 block: f16 MMAs (every e4m3 code is exact in f16); the query rows go to f16 (exact
            // in f16's normal range) and the key codes straight from the e4m3 tile
            // ([128 rows][128 B], 128B swizzle) into B fragments
            const uint8_t* K8 = sm.kv[stage][0];
            const uint16_t* q0 = sm.q[stage][gq];
            const uint16_t* q1 = sm.q[stage][gq + 8];
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int d0 = ks * 16 + 2 * tq;
                const uint32_t a0 = f16x2_from_bf16x2(*reinterpret_cast<const uint32_t*>(q0 + d0));
                const uint32_t a1 = f16x2_from_bf16x2(*reinterpret_cast<const uint32_t*>(q1 + d0));
                const uint32_t a2 = f16x2_from_bf16x2(*reinterpret_cast<const uint32_t*>(q0 + d0 + 8));
                const uint32_t a3 = f16x2_from_bf16x2(*reinterpret_cast<const uint32_t*>(q1 + d0 + 8));
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int key = kbase + nt * 8 + gq;
                    const uint8_t* kr = K8 + key * 128 + ((ks ^ (key & 7)) << 4) + 2 * tq;
                    const uint32_t b0 = f16x2_from_e4m3x2(*reinterpret_cast<const uint16_t*>(kr));
                    const uint32_t b1 = f16x2_from_e4m3x2(*reinterpret_cast<const uint16_t*>(kr + 8));
                    mma_f16_16816(s[nt], a0, a1, a2, a3, b0, b1);
                }
            }
        } else if (active) {
            const uint8_t* Ks = sm.kv[stage][0];
            const uint16_t* q0 = sm.q[stage][gq];       // query rows gq, gq + 8 (A fragments)
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
        // ---- online softmax of this warp's 16 keys (rows gq, gq + 8 of the accumulators)
        float mx0 = -INFINITY, mx1 = -INFINITY;
        const float s_scale = f8 ? sm.meta_ks[stage] * a.scale_log2 : a.scale_log2;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const bool v = kbase + nt * 8 + 2 * tq + e < ntok;
                s[nt][e] = v ? s[nt][e] * s_scale : -INFINITY;
                s[nt][2 + e] = v ? s[nt][2 + e] * s_scale : -INFINITY;
                mx0 = fmaxf(mx0, s[nt][e]);
                mx1 = fmaxf(mx1, s[nt][2 + e]);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        float mn0, mn1, al0, al1, dummy;
        lse_weights(st.m0, mx0, mn0, al0, dummy);
        lse_weights(st.m1, mx1, mn1, al1, dummy);
        const float base0 = mn0 == -INFINITY ? 0.f : mn0, base1 = mn1 == -INFINITY ? 0.f : mn1;
        st.m0 = mn0;
        st.m1 = mn1;
        float p[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            p[nt][0] = fast_exp2(s[nt][0] - base0);
            p[nt][1] = fast_exp2(s[nt][1] - base0);
            p[nt][2] = fast_exp2(s[nt][2] - base1);
            p[nt][3] = fast_exp2(s[nt][3] - base1);
        }
        st.l0 = st.l0 * al0 + (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
        st.l1 = st.l1 * al1 + (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]);
        if (!__all_sync(0xffffffffu, al0 == 1.f && al1 == 1.f)) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                st.o[i][0] *= al0; st.o[i][1] *= al0;
                st.o[i][2] *= al1; st.o[i][3] *= al1;
            }
        }
        // ---- o += P V over this warp's 16 keys: the accumulator layout of S is the A layout of P
        if (active) {
            if (!warp_wait_all(&sm.full_v[stage], ph, a.hdr)) break;
            uint8_t* Vs = sm.kv[stage][1];
            if (f8) widen_fp8_rows(Vs, kbase, lane);
            if (ntok < kbase + 16) {                    // rows past the query must be finite: zero them
                const int r0 = ntok - kbase;             // 1 .. 15
                for (int i = lane; i < (16 - r0) * 16; i += 32) {
                    const int row = kbase + r0 + i / 16, ch = i % 16;
                    *reinterpret_cast<uint4*>(Vs + (ch >> 3) * 16384 + sw128(row, ch & 7)) = make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
            }
            const uint32_t vrow = smem_u32(Vs);
            const int row = kbase + (lane & 7) + ((lane >> 3) & 1) * 8;
            if (f8) {
                // the values are code x scale: P is weighted by the block's value scale, in f16
                const float vsc = sm.meta_vs[stage];
                const uint32_t pa0 = pack_f16x2(p[0][0] * vsc, p[0][1] * vsc), pa1 = pack_f16x2(p[0][2] * vsc, p[0][3] * vsc);
                const uint32_t pa2 = pack_f16x2(p[1][0] * vsc, p[1][1] * vsc), pa3 = pack_f16x2(p[1][2] * vsc, p[1][3] * vsc);
#pragma unroll
                for (int dn = 0; dn < 8; ++dn) {
                    uint32_t v0, v1, v2, v3;
                    ldsm_x4_trans(vrow + kv_off(row, dn * 16 + (lane >> 4) * 8), v0, v1, v2, v3);
                    mma_f16_16816(st.o[2 * dn], pa0, pa1, pa2, pa3, v0, v1);
                    mma_f16_16816(st.o[2 * dn + 1], pa0, pa1, pa2, pa3, v2, v3);
                }
            } else {
                const uint32_t pa0 = pack_bf16x2(p[0][0], p[0][1]), pa1 = pack_bf16x2(p[0][2], p[0][3]);
                const uint32_t pa2 = pack_bf16x2(p[1][0], p[1][1]), pa3 = pack_bf16x2(p[1][2], p[1][3]);
#pragma unroll
                for (int dn = 0; dn < 8; ++dn) {
                    uint32_t v0, v1, v2, v3;
                    ldsm_x4_trans(vrow + kv_off(row, dn * 16 + (lane >> 4) * 8), v0, v1, v2, v3);
                    mma_bf16_16816(st.o[2 * dn], pa0, pa1, pa2, pa3, v0, v1);
                    mma_bf16_16816(st.o[2 * dn + 1], pa0, pa1, pa2, pa3, v2, v3);
                }
            }
        }
        if (!fin) {
            if (f8 || (active && ntok < kbase + 16)) fence_proxy_async();   // rewritten rows before the next TMA fill
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);   // this warp is done with the stage
            continue;
        }
        // ---- end of this CTA's share of the group: park the state in this warp's own rows of
        // the stage (no other warp reads them) and hand the stage to the epilogue warp
        st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, 1);
        st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, 1);
        st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, 2);
        st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, 2);
        __syncwarp();                                   // every lane is done reading its rows
#pragma unroll
        for (int g = 0; g < 16; ++g)
            if (g < 8 || Hg > 8) *park_addr(sm, stage, warp, g, lane) = acc_group(st, g);
        if (tq == 0) {
            sm.pm[stage][warp][gq] = st.m0;
            sm.pm[stage][warp][gq + 8] = st.m1;
            sm.pl[stage][warp][gq] = st.l0;
            sm.pl[stage][warp][gq + 8] = st.l1;
        }
        fence_proxy_async();                            // smem writes before the stage's next TMA fill
        if (sm.meta_nfrag[stage] == 1) {
            // the whole group ran in this CTA: fold it here, 8 warps wide
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.fold);
            if (!warp_wait_all(&sm.fold, uint32_t(nfold & 1), a.hdr)) break;
            ++nfold;
            const size_t orow = size_t(bg / G) * G * Hg + size_t(bg % G) * Hg;
            fold_write_columns(sm, stage, warp, lane, Hg, orow, a.out, a.lse);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[stage]);   // this warp has read the parked states
            clear_state(st);
            continue;
        }
        const int qs = nfin % kDecStages;
        if (warp == 0 && lane == 0) sm.park_stage[qs] = stage;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.parked[qs]);
        ++nfin;
        clear_state(st);
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
                                void* out, float* lse, void* ws, cudaStream_t st, const void* k8, const void* v8,
                                const float* k_scale, const float* v_scale, int64_t nb_cap) {
    const bool fp8 = k8 != nullptr;
    DecMaps maps;
    const uint64_t rows = uint64_t(B) * G * uint64_t(l_cap);
    msa_status_t e = make_tmap_bf16(&maps.k128, k_cache, rows, kHeadDim, 64, 128);
    if (e == MSA_OK) e = make_tmap_bf16(&maps.v128, v_cache, rows, kHeadDim, 64, 128);
    if (e == MSA_OK) e = make_tmap_bf16(&maps.k32, k_cache, rows, kHeadDim, 64, kDecDiagRows);
    if (e == MSA_OK) e = make_tmap_bf16(&maps.v32, v_cache, rows, kHeadDim, 64, kDecDiagRows);
    if (fp8) {
        if (e == MSA_OK) e = make_tmap_u8(&maps.k8, k8, rows, kHeadDim, 128, 128);
        if (e == MSA_OK) e = make_tmap_u8(&maps.v8, v8, rows, kHeadDim, 128, 128);
    } else {
        maps.k8 = maps.k128;                         // unused by the bf16 variant
        maps.v8 = maps.v128;
    }
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
    a.k_scale = k_scale; a.v_scale = v_scale; a.nb_cap = nb_cap;
    const int smem = int(sizeof(DecSmem)) + 1024;
    auto kern = fp8 ? attn_decode_kernel<true> : attn_decode_kernel<false>;
    static std::atomic<bool> attr_set[2][64];       // per variant and device; setting it twice is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[fp8][dev].load(std::memory_order_relaxed)) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        attr_set[fp8][dev].store(true, std::memory_order_relaxed);
    }
    // Persistent CTAs over the (sequence, group, block) items, cut into even contiguous ranges.
    // When the groups fill at least half the SMs, one CTA per group: no group is split, so no
    // partial state crosses CTAs (merging split groups costs a few microseconds of tail);
    // otherwise one CTA per SM, splitting groups to spread the bytes.
    const int64_t n_items = int64_t(B) * G * kTopK;
    const int64_t n_groups = int64_t(B) * G;
    const int sms = num_sms();
    const int grid = int(2 * n_groups >= sms ? (n_groups < sms ? n_groups : sms) : (n_items < sms ? n_items : sms));
    a.inv_grid = 1.0 / double(grid);
    a.inv_items = 1.0 / double(n_items);
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
    const KernelTimer kt(KID_ATTN_DECODE, st);
    cudaLaunchKernelEx(&cfg, kern, maps, a);
    return cuda_status();
}

}  // namespace msa

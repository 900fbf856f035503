// attn_decode.cu -- Main Branch for one decode token per sequence: exact softmax attention
// over the k = 16 selected 128-token blocks of its GQA group, split across CTAs by block and
// merged by log-sum-exp.
//
// Sources: youmind article "MiniMax M3 sparse attention agents", figure 1 caption (the main
// branch attends only to the selected blocks) and paragraph "Why this comes now" (each block
// is read once with contiguous memory access); KuCoin flash "MiniMax launches MSA sparse
// attention method and MiniMax-M3 model", summary (exact softmax over the 16 blocks).
//
// Design (HBM-bound): one CTA per (sequence, group, selected block) reads the block's K and
// V rows -- each a contiguous 32 KB range of the head-major cache -- with TMA tile loads into
// 128B-swizzled shared memory, computes the Hg heads' scores and weighted values with warp
// MMAs (the contraction is tiny: 8 FLOP per byte read, so tensor throughput is not the
// bound), and leaves an unnormalised partial (max, sum, o) in the workspace. The CTA that
// arrives last for a (sequence, group) merges the partials and writes the bf16 output.
#include "msa_common.cuh"

namespace msa {

constexpr int kDecAttnThreads = 128;
constexpr int kDecRowsPerBox = 32;

__host__ __device__ inline int dec_part_stride(int Hg) { return (Hg * (kHeadDim + 2) + 3) / 4 * 4; }

// address of bf16 element (row, col) in a K/V tile: two 64-column halves, each 128 rows x
// 128 B with the 128-byte swizzle
__device__ __forceinline__ uint32_t kv_off(int row, int col) {
    return uint32_t(col >> 6) * 16384u + sw128(uint32_t(row), uint32_t((col & 63) >> 3)) + uint32_t(col & 7) * 2u;
}

__global__ void __launch_bounds__(kDecAttnThreads) attn_decode_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const uint16_t* __restrict__ q, int64_t l_cap, const int32_t* __restrict__ q_pos, int64_t max_pos,
    const int32_t* __restrict__ sel, int G, int Hg, uint16_t* __restrict__ out, float* __restrict__ lse,
    float* __restrict__ part, unsigned int* __restrict__ ctr, WsHeader* hdr, float scale_log2) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar;
    __shared__ float red_m[4][kMaxHg], red_l[4][kMaxHg];
    __shared__ int s_last, s_nsel, s_j;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Ks = smem;                // 32 KB
    uint8_t* Vs = smem + 32768;        // 32 KB
    float* Ored = reinterpret_cast<float*>(Ks);   // reused after the scores: [4][Hg][128]

    const int slot = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int bg = b * G + g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int pos = q_pos[b];
    if (pos < 0 || pos > max_pos || pos >= l_cap) {
        if (slot == 0 && tid == 0) record_error(hdr, MSA_ERR_DEVICE_BOUNDS, KID_ATTN_DECODE, bg, 0, pos);
        return;
    }
    const int c = pos / kBlock;
    const int32_t* srow = sel + size_t(bg) * kTopK;
    if (tid == 0) {
        int n = 0;
        while (n < kTopK && srow[n] >= 0) ++n;
        s_nsel = n;
        int j = slot < n ? srow[slot] : -1;
        if (slot < n && (j > c)) {
            record_error(hdr, MSA_ERR_DEVICE_BOUNDS, KID_ATTN_DECODE, bg, slot, j);
            j = -2;                                  // contributes nothing, still arrives
        }
        s_j = j;
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    const int nsel = s_nsel;
    if (slot >= nsel) return;
    const int j = s_j;
    const int ntok = (j < 0) ? 0 : (j == c ? pos - c * kBlock + 1 : kBlock);
    const int nload = (ntok + kDecRowsPerBox - 1) / kDecRowsPerBox * kDecRowsPerBox;

    if (tid == 0 && ntok > 0) {
        mbar_arrive_expect_tx(&bar, uint32_t(nload) * 128u * 4u);
        const int row0 = int((int64_t(bg) * l_cap) + int64_t(j) * kBlock);
        for (int r0 = 0; r0 < nload; r0 += kDecRowsPerBox) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                tma_load_2d(Ks + h * 16384 + r0 * 128, &tmK, h * 64, row0 + r0, &bar);
                tma_load_2d(Vs + h * 16384 + r0 * 128, &tmV, h * 64, row0 + r0, &bar);
            }
        }
    }
    // query fragments (A operand, rows = heads): a0/a2 rows gq, a1/a3 rows gq + 8
    uint32_t qa[8][4];
    {
        const uint32_t* q32 = reinterpret_cast<const uint32_t*>(q + (size_t(b) * G * Hg + size_t(g) * Hg) * kHeadDim);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const int d0 = ks * 16 + 2 * tq;
            qa[ks][0] = gq < Hg ? __ldg(q32 + (gq * kHeadDim + d0) / 2) : 0u;
            qa[ks][1] = gq + 8 < Hg ? __ldg(q32 + ((gq + 8) * kHeadDim + d0) / 2) : 0u;
            qa[ks][2] = gq < Hg ? __ldg(q32 + (gq * kHeadDim + d0 + 8) / 2) : 0u;
            qa[ks][3] = gq + 8 < Hg ? __ldg(q32 + ((gq + 8) * kHeadDim + d0 + 8) / 2) : 0u;
        }
    }
    bool ok = true;
    if (ntok > 0) ok = mbar_wait(&bar, 0, hdr, KID_ATTN_DECODE);
    const int nk = ok ? ntok : 0;
    // rows [nk, nload) hold cache positions past the query: zero V so 0-weights stay finite
    if (nk < kBlock) {
        for (int i = tid; i < (nload - nk) * 16; i += kDecAttnThreads) {
            const int row = nk + i / 16, ch = i % 16;
            *reinterpret_cast<uint4*>(Vs + (ch >> 3) * 16384 + sw128(row, ch & 7)) = make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();

    // ---- scores for this warp's 32 keys
    float s[4][4];
    const int kbase = warp * 32;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
        const int n0 = kbase + nt * 8;
        if (n0 < nk) {
            const int key = n0 + gq;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t b0 = *reinterpret_cast<const uint32_t*>(Ks + (ks >> 2) * 16384 + sw128(key, (ks & 3) * 2) + 4 * tq);
                const uint32_t b1 = *reinterpret_cast<const uint32_t*>(Ks + (ks >> 2) * 16384 + sw128(key, (ks & 3) * 2 + 1) + 4 * tq);
                mma_bf16_16816(s[nt], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
            }
        }
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int key = kbase + nt * 8 + 2 * tq + e;
            const bool v = key < nk;
            s[nt][e] = v ? s[nt][e] * scale_log2 : -INFINITY;
            s[nt][2 + e] = v ? s[nt][2 + e] * scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, s[nt][e]);
            mx1 = fmaxf(mx1, s[nt][2 + e]);
        }
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float base0 = mx0 == -INFINITY ? 0.f : mx0;
    const float base1 = mx1 == -INFINITY ? 0.f : mx1;
    float l0 = 0.f, l1 = 0.f;
    uint32_t pa[2][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const float p0 = fast_exp2(s[nt][0] - base0), p1 = fast_exp2(s[nt][1] - base0);
        const float p2 = fast_exp2(s[nt][2] - base1), p3 = fast_exp2(s[nt][3] - base1);
        l0 += p0 + p1;
        l1 += p2 + p3;
        const int kk = nt >> 1, hi = nt & 1;
        pa[kk][0 + 2 * hi] = pack_bf16x2(p0, p1);
        pa[kk][1 + 2 * hi] = pack_bf16x2(p2, p3);
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    // ---- o = p v for this warp's keys, all 128 columns
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        const int k0 = kbase + kk * 16;
        if (k0 < nk) {
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                const int col = nt * 8 + gq;
                const int r = k0 + 2 * tq;
                const uint32_t v0 = *reinterpret_cast<const uint16_t*>(Vs + kv_off(r, col));
                const uint32_t v1 = *reinterpret_cast<const uint16_t*>(Vs + kv_off(r + 1, col));
                const uint32_t v2 = *reinterpret_cast<const uint16_t*>(Vs + kv_off(r + 8, col));
                const uint32_t v3 = *reinterpret_cast<const uint16_t*>(Vs + kv_off(r + 9, col));
                mma_bf16_16816(o[nt], pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3], v0 | (v1 << 16), v2 | (v3 << 16));
            }
        }
    }
    // ---- merge the four warps
    if (tq == 0) {
        if (gq < Hg) { red_m[warp][gq] = mx0; red_l[warp][gq] = l0; }
        if (gq + 8 < Hg) { red_m[warp][gq + 8] = mx1; red_l[warp][gq + 8] = l1; }
    }
    __syncthreads();   // all warps are past their reads of Ks: Ored may overwrite it
    float f0 = 0.f, f1 = 0.f;
    {
        float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            if (gq < Hg) M0 = fmaxf(M0, red_m[w][gq]);
            if (gq + 8 < Hg) M1 = fmaxf(M1, red_m[w][gq + 8]);
        }
        f0 = (mx0 == -INFINITY) ? 0.f : fast_exp2(mx0 - M0);
        f1 = (mx1 == -INFINITY) ? 0.f : fast_exp2(mx1 - M1);
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
        const int col = nt * 8 + 2 * tq;
        if (gq < Hg)
            *reinterpret_cast<float2*>(Ored + (warp * Hg + gq) * kHeadDim + col) = make_float2(o[nt][0] * f0, o[nt][1] * f0);
        if (gq + 8 < Hg)
            *reinterpret_cast<float2*>(Ored + (warp * Hg + gq + 8) * kHeadDim + col) = make_float2(o[nt][2] * f1, o[nt][3] * f1);
    }
    __syncthreads();
    const int stride = dec_part_stride(Hg);
    float* mypart = part + (size_t(bg) * kTopK + slot) * stride;
    for (int h = 0; h < Hg; ++h) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) acc += Ored[(w * Hg + h) * kHeadDim + tid];
        mypart[2 * Hg + h * kHeadDim + tid] = acc;
    }
    if (tid < Hg) {
        float M = -INFINITY, L = 0.f;
        for (int w = 0; w < 4; ++w) M = fmaxf(M, red_m[w][tid]);
        for (int w = 0; w < 4; ++w)
            if (red_m[w][tid] != -INFINITY) L += red_l[w][tid] * fast_exp2(red_m[w][tid] - M);
        mypart[tid] = M;
        mypart[Hg + tid] = L;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicInc(ctr + bg, unsigned(nsel - 1)) == unsigned(nsel - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // ---- last CTA of this (sequence, group): merge the nsel partials
    const float* pbase = part + size_t(bg) * kTopK * stride;
    for (int h = 0; h < Hg; ++h) {
        float M = -INFINITY;
        for (int sl = 0; sl < nsel; ++sl) M = fmaxf(M, __ldcg(pbase + sl * stride + h));
        float L = 0.f, acc = 0.f;
        for (int sl = 0; sl < nsel; ++sl) {
            const float m = __ldcg(pbase + sl * stride + h);
            if (m == -INFINITY) continue;
            const float f = fast_exp2(m - M);
            L += __ldcg(pbase + sl * stride + Hg + h) * f;
            acc += __ldcg(pbase + sl * stride + 2 * Hg + h * kHeadDim + tid) * f;
        }
        const size_t orow = (size_t(b) * G * Hg + size_t(g) * Hg + h) * kHeadDim;
        out[orow + tid] = __bfloat16_as_ushort(__float2bfloat16_rn(acc / L));
        if (lse != nullptr && tid == 0) lse[size_t(b) * G * Hg + size_t(g) * Hg + h] = (M + log2f(L)) * 0.69314718055994530942f;
    }
}

size_t decode_attn_ws_bytes(int B, int G, int Hg) {
    const size_t nbg = size_t(B) * G;
    return sizeof(WsHeader) + (nbg * sizeof(unsigned int) + 255) / 256 * 256 +
           nbg * kTopK * dec_part_stride(Hg) * sizeof(float);
}

void launch_attn_decode(const CUtensorMap& tmK, const CUtensorMap& tmV, const void* q, int64_t l_cap,
                        const int32_t* q_pos, int64_t max_pos, const int32_t* sel, int B, int G, int Hg,
                        void* out, float* lse, void* ws, cudaStream_t st) {
    const size_t nbg = size_t(B) * G;
    char* p = static_cast<char*>(ws);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(p);
    unsigned int* ctr = reinterpret_cast<unsigned int*>(p + sizeof(WsHeader));
    float* part = reinterpret_cast<float*>(p + sizeof(WsHeader) + (nbg * sizeof(unsigned int) + 255) / 256 * 256);
    const int smem = 65536 + 1024;
    static bool attr_set = false;
    if (!attr_set) {
        cudaFuncSetAttribute(attn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        attr_set = true;
    }
    const float scale_log2 = 1.4426950408889634f / sqrtf(float(kHeadDim));
    dim3 grid(kTopK, unsigned(G), unsigned(B));
    count_launch();
    attn_decode_kernel<<<grid, kDecAttnThreads, smem, st>>>(tmK, tmV, static_cast<const uint16_t*>(q), l_cap, q_pos,
                                                            max_pos, sel, G, Hg, static_cast<uint16_t*>(out), lse,
                                                            part, ctr, hdr, scale_log2);
}

}  // namespace msa

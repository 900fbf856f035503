// attn_prefill_simt.cu -- query-major Main Branch on CUDA cores: one CTA per (sequence,
// token, group) walks its selected blocks with an online softmax. It is the plain GPU path
// the tensor-core kernel is checked against and the fallback for query-head counts the
// tensor-core tiling does not cover; it re-reads every selected block per token, so it is
// bound by L2/HBM traffic, not by arithmetic.
//
// Sources: youmind article "MiniMax M3 sparse attention agents", figure 1 caption; KuCoin
// flash "MiniMax launches MSA sparse attention method and MiniMax-M3 model", summary (exact
// softmax attention over the selected blocks, causal inside the query's own block).
#include "msa_common.cuh"

namespace msa {

__global__ void __launch_bounds__(128) attn_prefill_simt_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
    int64_t N, int G, int Hg, const int32_t* __restrict__ sel, uint16_t* __restrict__ out,
    float* __restrict__ lse, float scale_log2) {
    __shared__ float qs[kMaxHg][kHeadDim];
    __shared__ float ps[kMaxHg][kBlock];
    __shared__ float red[kMaxHg][4];
    const int64_t t = blockIdx.x;
    const int g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int Hq = G * Hg;
    for (int i = tid; i < Hg * kHeadDim; i += 128) {
        const int h = i / kHeadDim, d = i % kHeadDim;
        qs[h][d] = bf16_to_f32(q[((size_t(b) * N + t) * Hq + g * Hg + h) * kHeadDim + d]) * scale_log2;
    }
    float m[kMaxHg], l[kMaxHg], o[kMaxHg];
#pragma unroll
    for (int h = 0; h < kMaxHg; ++h) { m[h] = -INFINITY; l[h] = 0.f; o[h] = 0.f; }
    const int32_t* srow = sel + ((size_t(b) * N + t) * G + g) * kTopK;
    const uint16_t* kg = k + (size_t(b) * G + g) * N * kHeadDim;
    const uint16_t* vg = v + (size_t(b) * G + g) * N * kHeadDim;
    __syncthreads();
    for (int slot = 0; slot < kTopK; ++slot) {
        const int j = srow[slot];
        if (j < 0) break;
        const int64_t u = int64_t(j) * kBlock + tid;
        const bool valid = u <= t;
        float s[kMaxHg];
#pragma unroll
        for (int h = 0; h < kMaxHg; ++h) s[h] = 0.f;
        if (valid) {
            const uint4* kr = reinterpret_cast<const uint4*>(kg + u * kHeadDim);
            for (int c8 = 0; c8 < kHeadDim / 8; ++c8) {
                const uint4 w = __ldg(kr + c8);
                const float kx[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                                     bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
#pragma unroll
                for (int h = 0; h < kMaxHg; ++h) {
                    if (h < Hg) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) s[h] = fmaf(qs[h][c8 * 8 + e], kx[e], s[h]);
                    }
                }
            }
        }
        // block max per head
#pragma unroll
        for (int h = 0; h < kMaxHg; ++h) {
            if (h >= Hg) break;
            float x = valid ? s[h] : -INFINITY;
            for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
            if (lane == 0) red[h][warp] = x;
        }
        __syncthreads();
        float alpha[kMaxHg], mn[kMaxHg];
#pragma unroll
        for (int h = 0; h < kMaxHg; ++h) {
            if (h >= Hg) break;
            const float bm = fmaxf(fmaxf(red[h][0], red[h][1]), fmaxf(red[h][2], red[h][3]));
            mn[h] = fmaxf(m[h], bm);
            alpha[h] = (m[h] == -INFINITY) ? 0.f : exp2f(m[h] - mn[h]);
            ps[h][tid] = valid ? exp2f(s[h] - mn[h]) : 0.f;
        }
        __syncthreads();
        // thread tid now owns output column d = tid
        const int nvalid = int(t - int64_t(j) * kBlock + 1 < kBlock ? t - int64_t(j) * kBlock + 1 : int64_t(kBlock));
#pragma unroll
        for (int h = 0; h < kMaxHg; ++h) {
            if (h >= Hg) break;
            float acc = 0.f, ls = 0.f;
            for (int uu = 0; uu < nvalid; ++uu) {
                const float p = ps[h][uu];
                ls += p;
                acc = fmaf(p, bf16_to_f32(vg[(size_t(j) * kBlock + uu) * kHeadDim + tid]), acc);
            }
            o[h] = o[h] * alpha[h] + acc;
            l[h] = l[h] * alpha[h] + ls;
            m[h] = mn[h];
        }
        __syncthreads();
    }
#pragma unroll
    for (int h = 0; h < kMaxHg; ++h) {
        if (h >= Hg) break;
        const size_t row = (size_t(b) * N + t) * Hq + g * Hg + h;
        out[row * kHeadDim + tid] = __bfloat16_as_ushort(__float2bfloat16_rn(o[h] / l[h]));
        if (lse != nullptr && tid == 0) lse[row] = (m[h] + log2f(l[h])) * 0.69314718055994530942f;
    }
}

void launch_attn_prefill_simt(const void* q, const void* k, const void* v, int64_t N, int B, int G, int Hg,
                              const int32_t* sel, void* out, float* lse, cudaStream_t st) {
    const float scale_log2 = 1.4426950408889634f / sqrtf(float(kHeadDim));
    dim3 grid(static_cast<unsigned>(N), static_cast<unsigned>(G), static_cast<unsigned>(B));
    count_launch();
    attn_prefill_simt_kernel<<<grid, 128, 0, st>>>(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                                                   static_cast<const uint16_t*>(v), N, G, Hg, sel,
                                                   static_cast<uint16_t*>(out), lse, scale_log2);
}

}  // namespace msa

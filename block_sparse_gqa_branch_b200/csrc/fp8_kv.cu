// fp8_kv.cu -- the FP8 (e4m3) key-value cache of the decode variant: per-block quantisation.
//
// Source: KuCoin flash "MiniMax launches MSA sparse attention method and MiniMax-M3 model",
// "ME AI News" paragraph (the SM100 attention kernel also takes FP8 inputs). The pages give no
// format details; this library's reading:
//  * only closed blocks are stored in e4m3 -- the open block, which is always the newest
//    query's own block, stays in bf16 until it fills (a per-block scale would otherwise change
//    with every append);
//  * one fp32 scale per (sequence, group, block) for keys and one for values,
//    scale = amax / 448 in fp32 (1 for an all-zero block);
//  * code = e4m3(x / scale), the division in fp32 (correctly rounded), rounded to nearest with
//    ties to the even mantissa, saturating at +-448 (NaN stays NaN).
// Layouts: codes [B, G, l_cap, 128] uint8 (the bf16 cache's layout with one byte per value),
// scales [B, G, nb_cap] fp32.
#include "msa_common.cuh"

namespace msa {

// Two fp32 values -> two e4m3 codes (lo in the low byte): round to nearest even, saturating to
// the largest finite value.
__device__ __forceinline__ uint16_t e4m3x2_from_f32(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// One CTA of 256 threads quantises one 128 x 128 block of one tensor (K or V) of one
// (sequence, group): 64 values per thread, held in registers between the amax and the codes.
__device__ __forceinline__ void quantize_block(const uint16_t* __restrict__ src, uint8_t* __restrict__ dst,
                                               float* __restrict__ scale_out) {
    __shared__ float red[8];
    const int tid = threadIdx.x;
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __ldg(s4 + tid + 256 * i);    // 16 B = 8 values, coalesced
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e]))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    uint2* d2 = reinterpret_cast<uint2*>(dst);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        uint32_t packed[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint16_t c0 = e4m3x2_from_f32(__fdiv_rn(bf16_lo(w[2 * h]), scale), __fdiv_rn(bf16_hi(w[2 * h]), scale));
            const uint16_t c1 =
                e4m3x2_from_f32(__fdiv_rn(bf16_lo(w[2 * h + 1]), scale), __fdiv_rn(bf16_hi(w[2 * h + 1]), scale));
            packed[h] = uint32_t(c0) | (uint32_t(c1) << 16);
        }
        d2[tid + 256 * i] = make_uint2(packed[0], packed[1]);
    }
    if (tid == 0) *scale_out = scale;
}

struct Fp8Args {
    const uint16_t* k;            // bf16 caches [B, G, l_cap, 128]
    const uint16_t* v;
    uint8_t* k8;                  // codes [B, G, l_cap, 128]
    uint8_t* v8;
    float* ks;                    // scales [B, G, nb_cap]
    float* vs;
    int64_t l_cap, nb_cap;
    int G;
};

// grid (n_blocks, 2 G, B): block j of tensor (y & 1) of group y / 2 of sequence z
__global__ void __launch_bounds__(256) fp8_quantize_kernel(const Fp8Args a) {
    const int j = blockIdx.x, g = blockIdx.y >> 1, which = blockIdx.y & 1, b = blockIdx.z;
    const size_t row0 = (size_t(b) * a.G + g) * a.l_cap + size_t(j) * kBlock;
    const size_t sidx = (size_t(b) * a.G + g) * a.nb_cap + j;
    if (which == 0) quantize_block(a.k + row0 * kHeadDim, a.k8 + row0 * kHeadDim, a.ks + sidx);
    else quantize_block(a.v + row0 * kHeadDim, a.v8 + row0 * kHeadDim, a.vs + sidx);
}

// grid (1, 2 G, B): the block that the token at position ctx_len[b] completes, if it does
__global__ void __launch_bounds__(256) fp8_close_kernel(const Fp8Args a, const int32_t* __restrict__ ctx_len,
                                                        WsHeader* hdr) {
    grid_dep_launch();                     // the selection may start: it reads no code or scale
    grid_dep_wait();                       // the append that wrote the token has completed
    const int g = blockIdx.y >> 1, which = blockIdx.y & 1, b = blockIdx.z;
    const int pos = ctx_len[b];
    if (pos < 0 || pos >= a.l_cap) {
        if (threadIdx.x == 0 && blockIdx.y == 0) record_error(hdr, MSA_ERR_DEVICE_BOUNDS, KID_FP8, b, 0, pos);
        return;
    }
    if ((pos + 1) % kBlock != 0) return;
    const int64_t j = pos / kBlock;
    if (j >= a.nb_cap) {
        if (threadIdx.x == 0 && blockIdx.y == 0) record_error(hdr, MSA_ERR_DEVICE_BOUNDS, KID_FP8, b, 1, pos);
        return;
    }
    const size_t row0 = (size_t(b) * a.G + g) * a.l_cap + size_t(j) * kBlock;
    const size_t sidx = (size_t(b) * a.G + g) * a.nb_cap + j;
    if (which == 0) quantize_block(a.k + row0 * kHeadDim, a.k8 + row0 * kHeadDim, a.ks + sidx);
    else quantize_block(a.v + row0 * kHeadDim, a.v8 + row0 * kHeadDim, a.vs + sidx);
}

void launch_fp8_quantize(const void* k, const void* v, int64_t l_cap, int64_t n_blocks, int B, int G, void* k8,
                         void* v8, float* ks, float* vs, int64_t nb_cap, cudaStream_t st) {
    if (n_blocks <= 0) return;
    Fp8Args a{static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v), static_cast<uint8_t*>(k8),
              static_cast<uint8_t*>(v8), ks, vs, l_cap, nb_cap, G};
    const KernelTimer kt(KID_FP8, st);
    fp8_quantize_kernel<<<dim3(unsigned(n_blocks), unsigned(2 * G), unsigned(B)), 256, 0, st>>>(a);
}

void launch_fp8_close(const void* k, const void* v, int64_t l_cap, const int32_t* ctx_len, int B, int G, void* k8,
                      void* v8, float* ks, float* vs, int64_t nb_cap, void* ws, cudaStream_t st) {
    Fp8Args a{static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v), static_cast<uint8_t*>(k8),
              static_cast<uint8_t*>(v8), ks, vs, l_cap, nb_cap, G};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1u, unsigned(2 * G), unsigned(B));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap with the append's tail
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const KernelTimer kt(KID_FP8, st);
    cudaLaunchKernelEx(&cfg, fp8_close_kernel, a, ctx_len, static_cast<WsHeader*>(ws));
}

}  // namespace msa

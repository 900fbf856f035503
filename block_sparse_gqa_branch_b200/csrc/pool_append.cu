// pool_append.cu -- Index Branch block pooling (prefill) and the incremental pooled-key /
// KV-cache update of a decode step.
//
// Pooling: a block's pooled index key is the mean of its Bk = 128 index keys (youmind
// article "MiniMax M3 sparse attention agents", bullet "Predictable cost at every length"
// fixes Bk; the mean is this library's reading of the unspecified block summary).
// One CTA reads one 128-token block of all G groups: with G = 8 that is 128 contiguous
// 1 KB rows (128 KB), loaded as 16-byte vectors, so the kernel streams k_I once at HBM speed.
#include "msa_common.cuh"

namespace msa {

// grid (ceil(N / Bk), B), 256 threads.
__global__ void __launch_bounds__(256) pool_kernel(const uint16_t* __restrict__ k_idx, int64_t n_tokens,
                                                   int G, float* __restrict__ pooled, int64_t nb_cap,
                                                   float* __restrict__ tail_sum) {
    extern __shared__ float red[];                      // [nparts][G*dI]
    const int b = blockIdx.y;
    const int64_t blk = blockIdx.x;
    const int ncol = G * kIndexDim;                     // bf16 values per token row
    const int nchunk = ncol / 8;                        // 16-byte chunks per row
    const int nparts = nchunk >= 256 ? 1 : 256 / nchunk;
    const int64_t t0 = blk * kBlock;
    const int ntok = int((n_tokens - t0 < kBlock ? n_tokens - t0 : int64_t(kBlock)));
    const uint4* base = reinterpret_cast<const uint4*>(k_idx + (size_t(b) * n_tokens + t0) * ncol);

    for (int c0 = 0; c0 < nchunk; c0 += 256 / nparts) {
        const int chunk = c0 + (threadIdx.x % (256 / nparts));
        const int part = threadIdx.x / (256 / nparts);
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (chunk < nchunk && part < nparts) {
#pragma unroll 4
            for (int t = part; t < ntok; t += nparts) {
                uint4 v = __ldg(base + size_t(t) * nchunk + chunk);
                acc[0] += bf16_lo(v.x); acc[1] += bf16_hi(v.x);
                acc[2] += bf16_lo(v.y); acc[3] += bf16_hi(v.y);
                acc[4] += bf16_lo(v.z); acc[5] += bf16_hi(v.z);
                acc[6] += bf16_lo(v.w); acc[7] += bf16_hi(v.w);
            }
            float* r = red + (size_t(part) * nchunk + chunk) * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e) r[e] = acc[e];
        }
    }
    __syncthreads();
    const bool full = ntok == kBlock;
    for (int col = threadIdx.x; col < ncol; col += 256) {
        float s = 0.f;
        for (int p = 0; p < nparts; ++p) s += red[size_t(p) * ncol + col];
        const int g = col / kIndexDim, i = col % kIndexDim;
        if (full) {
            pooled[((size_t(b) * G + g) * nb_cap + blk) * kIndexDim + i] = s * (1.0f / kBlock);
        } else if (tail_sum) {
            tail_sum[(size_t(b) * G + g) * kIndexDim + i] = s;
        }
    }
}

__global__ void zero_kernel(float* p, int64_t n) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x)
        p[i] = 0.f;
}

void launch_pool(const void* k_idx, int B, int G, int64_t n_tokens, float* pooled, int64_t nb_cap,
                 float* tail_sum, cudaStream_t st) {
    if (tail_sum && n_tokens % kBlock == 0) {
        int64_t n = int64_t(B) * G * kIndexDim;
        const KernelTimer kt(KID_POOL, st);
        zero_kernel<<<int((n + 255) / 256), 256, 0, st>>>(tail_sum, n);
    }
    if (n_tokens == 0) return;
    const int nchunk = G * kIndexDim / 8;
    const int nparts = nchunk >= 256 ? 1 : 256 / nchunk;
    size_t smem = size_t(nparts) * G * kIndexDim * sizeof(float);
    if (smem > 48 * 1024) cudaFuncSetAttribute(pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    dim3 grid(unsigned((n_tokens + kBlock - 1) / kBlock), unsigned(B));
    const KernelTimer kt(KID_POOL, st);
    pool_kernel<<<grid, 256, smem, st>>>(static_cast<const uint16_t*>(k_idx), n_tokens, G, pooled,
                                          nb_cap, tail_sum);
}

// ---------------------------------------------------------------- chunk pooling
// Pooling for a chunk of n index-key rows at positions P .. P + n - 1 (k_idx [B, n, G, dI])
// appended to a sequence whose first P positions are already pooled: tail_sum holds the plain
// sum over the open block's cached positions Bk floor(P / Bk) .. P - 1. Two launches, in
// stream order: every block the chunk completes (the first one adds the cached running sum),
// then the new running sum of the trailing open block, which overwrites tail_sum only after
// the first launch has read it.
// grid (blocks, B), 256 threads; block j = j_first + blockIdx.x, positions max(Bk j, P) ..
// min(Bk (j + 1), P + n) - 1.
__global__ void __launch_bounds__(256) pool_chunk_kernel(const uint16_t* __restrict__ k_idx, int64_t n, int64_t P,
                                                         int G, float* __restrict__ pooled, int64_t nb_cap,
                                                         float* __restrict__ tail_sum, int64_t j_first,
                                                         int trailing) {
    extern __shared__ float red[];                      // [nparts][G*dI]
    const int b = blockIdx.y;
    const int64_t j = j_first + blockIdx.x;
    const int ncol = G * kIndexDim;
    const int nchunk = ncol / 8;
    const int nparts = nchunk >= 256 ? 1 : 256 / nchunk;
    const int64_t p0 = j * kBlock > P ? j * kBlock : P;
    const int64_t p1 = (j + 1) * kBlock < P + n ? (j + 1) * kBlock : P + n;
    const int ntok = int(p1 - p0);                      // >= 0
    const uint4* base = reinterpret_cast<const uint4*>(k_idx + (size_t(b) * n + (p0 - P)) * ncol);
    for (int c0 = 0; c0 < nchunk; c0 += 256 / nparts) {
        const int chunk = c0 + (threadIdx.x % (256 / nparts));
        const int part = threadIdx.x / (256 / nparts);
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (chunk < nchunk && part < nparts) {
#pragma unroll 4
            for (int t = part; t < ntok; t += nparts) {
                uint4 v = __ldg(base + size_t(t) * nchunk + chunk);
                acc[0] += bf16_lo(v.x); acc[1] += bf16_hi(v.x);
                acc[2] += bf16_lo(v.y); acc[3] += bf16_hi(v.y);
                acc[4] += bf16_lo(v.z); acc[5] += bf16_hi(v.z);
                acc[6] += bf16_lo(v.w); acc[7] += bf16_hi(v.w);
            }
            float* r = red + (size_t(part) * nchunk + chunk) * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e) r[e] = acc[e];
        }
    }
    __syncthreads();
    // the block's positions before P are the cached running sum (only the block holding P)
    const bool with_cached = P % kBlock != 0 && j == P / kBlock;
    for (int col = threadIdx.x; col < ncol; col += 256) {
        float s = 0.f;
        for (int q = 0; q < nparts; ++q) s += red[size_t(q) * ncol + col];
        const int g = col / kIndexDim, i = col % kIndexDim;
        float* ts = tail_sum + (size_t(b) * G + g) * kIndexDim + i;
        if (with_cached) s = *ts + s;
        if (trailing) *ts = s;
        else pooled[((size_t(b) * G + g) * nb_cap + j) * kIndexDim + i] = s * (1.0f / kBlock);
    }
}

void launch_pool_chunk(const void* k_idx, int B, int G, int64_t n, int64_t P, float* pooled, int64_t nb_cap,
                       float* tail_sum, cudaStream_t st) {
    const int nchunk = G * kIndexDim / 8;
    const int nparts = nchunk >= 256 ? 1 : 256 / nchunk;
    const size_t smem = size_t(nparts) * G * kIndexDim * sizeof(float);
    if (smem > 48 * 1024)
        cudaFuncSetAttribute(pool_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    const int64_t j0 = P / kBlock, jt = (P + n) / kBlock;      // blocks j0 .. jt - 1 complete in the chunk
    if (jt > j0) {
        const KernelTimer kt(KID_POOL, st);
        pool_chunk_kernel<<<dim3(unsigned(jt - j0), unsigned(B)), 256, smem, st>>>(
            static_cast<const uint16_t*>(k_idx), n, P, G, pooled, nb_cap, tail_sum, j0, 0);
    }
    const KernelTimer kt(KID_POOL, st);                          // the trailing open block (maybe empty)
    pool_chunk_kernel<<<dim3(1u, unsigned(B)), 256, smem, st>>>(static_cast<const uint16_t*>(k_idx), n, P, G, pooled,
                                                              nb_cap, tail_sum, jt, 1);
}

// ---------------------------------------------------------------- decode append
// grid B, block 256. Writes the new token's K/V rows into the caches at position L_b and
// folds its index keys into the open block's running sum; closes the block into `pooled`
// when it becomes full. Launched with programmatic dependent launch: it may run during the
// tail of the kernel before it in the stream (a decode step's selection, which reads only the
// pooled keys of blocks below the open one), and it completes only after that kernel has, so
// that a kernel waiting for this one also sees the one before.
__global__ void __launch_bounds__(256) append_kernel(const uint16_t* __restrict__ k_idx_new,
                                                     const uint16_t* __restrict__ k_new,
                                                     const uint16_t* __restrict__ v_new,
                                                     const int32_t* __restrict__ ctx_len, int G,
                                                     uint16_t* __restrict__ k_cache,
                                                     uint16_t* __restrict__ v_cache, int64_t l_cap,
                                                     float* __restrict__ tail_sum,
                                                     float* __restrict__ pooled, int64_t nb_cap,
                                                     WsHeader* hdr) {
    grid_dep_launch();                 // the next kernel may start its prologue
    const int b = blockIdx.x;
    // Every load goes out before the first use (one memory round trip: the selection streams
    // HBM at the same time, so each dependent round trip here would stretch the step).
    const int nvec = G * kHeadDim / 8;                     // 16-byte vectors per token and tensor
    const int nidx = G * kIndexDim;
    uint4 kv[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
    float xi[2] = {0.f, 0.f}, ts[2] = {0.f, 0.f};
    const int i0 = threadIdx.x;
    if (k_new != nullptr && i0 < nvec) {
        kv[0] = __ldg(reinterpret_cast<const uint4*>(k_new) + size_t(b) * nvec + i0);
        kv[1] = __ldg(reinterpret_cast<const uint4*>(v_new) + size_t(b) * nvec + i0);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int i = i0 + r * 256;
        if (i < nidx) {
            xi[r] = bf16_to_f32(__ldg(k_idx_new + size_t(b) * nidx + i));
            ts[r] = tail_sum[size_t(b) * nidx + i];
        }
    }
    const int pos = ctx_len[b];
    const int64_t j = pos / kBlock;
    const bool close = ((pos + 1) % kBlock) == 0;
    if (pos < 0 || pos >= l_cap || (close && j >= nb_cap)) {
        if (threadIdx.x == 0) record_error(hdr, MSA_ERR_DEVICE_BOUNDS, KID_APPEND, b, 0, pos);
        grid_dep_wait();
        return;
    }
    if (k_new != nullptr) {
        for (int i = i0; i < nvec; i += 256) {
            const int g = i / (kHeadDim / 8), c = i % (kHeadDim / 8);
            const uint4 kx = i == i0 ? kv[0] : __ldg(reinterpret_cast<const uint4*>(k_new) + size_t(b) * nvec + i);
            const uint4 vx = i == i0 ? kv[1] : __ldg(reinterpret_cast<const uint4*>(v_new) + size_t(b) * nvec + i);
            const size_t dst = ((size_t(b) * G + g) * l_cap + pos) * (kHeadDim / 8) + c;
            reinterpret_cast<uint4*>(k_cache)[dst] = kx;
            reinterpret_cast<uint4*>(v_cache)[dst] = vx;
        }
    }
    const bool fresh = (pos % kBlock) == 0;
    for (int i = i0; i < nidx; i += 256) {
        const int g = i / kIndexDim, e = i % kIndexDim;
        const size_t o = (size_t(b) * G + g) * kIndexDim + e;
        const int r = (i - i0) / 256;
        const float x = r < 2 ? xi[r] : bf16_to_f32(k_idx_new[o]);
        const float t = r < 2 ? ts[r] : tail_sum[o];
        const float sum = fresh ? x : t + x;
        tail_sum[o] = sum;
        if (close) pooled[((size_t(b) * G + g) * nb_cap + j) * kIndexDim + e] = sum * (1.0f / kBlock);
    }
    grid_dep_wait();                   // complete only after the kernel before this one
}

void launch_append(const void* k_idx_new, const void* k_new, const void* v_new, const int32_t* ctx_len,
                   int B, int G, void* k_cache, void* v_cache, int64_t l_cap, float* tail_sum,
                   float* pooled, int64_t nb_cap, void* ws, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(B));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const KernelTimer kt(KID_APPEND, st);
    cudaLaunchKernelEx(&cfg, append_kernel, static_cast<const uint16_t*>(k_idx_new),
                       static_cast<const uint16_t*>(k_new), static_cast<const uint16_t*>(v_new), ctx_len, G,
                       static_cast<uint16_t*>(k_cache), static_cast<uint16_t*>(v_cache), l_cap, tail_sum, pooled,
                       nb_cap, static_cast<WsHeader*>(ws));
}

}  // namespace msa

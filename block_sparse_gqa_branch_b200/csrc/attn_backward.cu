// attn_backward.cu -- Main Branch backward pass for prefill: dQ, dK, dV of the exact softmax
// attention over the selected blocks, the selection held fixed (it is a discrete choice).
//
// Sources: youmind article "MiniMax M3 sparse attention agents", bullet on MSA-CPT and KuCoin
// flash "MiniMax launches MSA sparse attention method and MiniMax-M3 model", "ME AI News"
// (MSA-PT): the model is trained through the sparse attention, which needs its gradient.
// With z_u = s q . k_u (s = 1/sqrt(d)), p = softmax(z), o = sum_u p_u v_u and the upstream dO:
//   D = dO . o,  dV_u += p_u dO,  dP_u = dO . v_u,  dS_u = p_u (dP_u - D),
//   dQ = s sum_u dS_u k_u,  dK_u += s dS_u q.
// p comes from the forward's log-sum-exp (p_u = exp(z_u - lse)), so no softmax is rebuilt.
//
// Key-value-major like the forward: the forward's inverted index gives, for every (sequence,
// group, 16K-token range, block j), the tokens that selected j. A persistent CTA of 8 warps takes
// an item, loads K_j and V_j once, and walks the item's query rows 32 at a time (32 / Hg tokens x
// Hg heads), double-buffered. Warp w owns keys 16 w .. 16 w + 15 of the block: it computes S^T and
// dP^T for its keys and the 32 rows with warp MMAs (m16n8k16, bf16, fp32 accumulation), turns
// them into P^T and dS^T in registers (the accumulator layout is the A-operand layout), and
// accumulates dV and dK of its keys over the whole item in registers. dQ needs every key of a
// row: the warps exchange dS through shared memory and warp w computes dQ columns 16 w .. 16 w +
// 15 of the 32 rows, added to the fp32 dQ with vector atomics (a row's 16 blocks are spread over
// items). At the end of an item dK and dV are added to the fp32 dK, dV the same way.
#include <atomic>

#include "msa_common.cuh"

namespace msa {

size_t inverted_index_bytes(int B, int64_t N, int G, int Hg);
IndexOffsets inverted_index_offsets(int B, int64_t N, int G, int Hg);
void launch_inverted_index(const int32_t* sel, int64_t N, int64_t P, int B, int G, int Hg, void* ws, cudaStream_t st);
int num_sms();

constexpr int kBwdWarps = 8;
constexpr int kBwdThreads = kBwdWarps * 32;
constexpr int kBwdRows = 32;          // query rows per step
constexpr int kPad = 136;             // bf16 per shared-memory row (128 + 8: conflict-free ldmatrix)
constexpr int kBwdSlots = 16;         // entries of the inverted index are token * 16 + slot
constexpr int kBwdDiagFlag = int(0x40000000);

struct BwdSmem {
    uint16_t k[kBlock][kPad];         // K_j, V_j: [key][d]
    uint16_t v[kBlock][kPad];
    uint16_t q[2][kBwdRows][kPad];    // the step's query rows and dO rows, double-buffered
    uint16_t go[2][kBwdRows][kPad];
    uint16_t ds[kBwdRows][kPad];      // dS of the step, [row][key]
    float lse2[2][kBwdRows];          // lse * log2(e) per row (+inf: no row)
    float dd[2][kBwdRows];            // D = dO . o per row
    int tok[2][kBwdRows];             // the row's token (-1: no row)
    int item;
};

struct BwdArgs {
    const uint16_t* q;                // [B, N, Hq, d]
    const uint16_t* k;                // [B, G, N, d]
    const uint16_t* v;
    const uint16_t* go;               // dO [B, N, Hq, d]
    const float* lse;                 // [B, N, Hq] natural log
    const float* dd;                  // D [B, N, Hq]
    float* dq;                        // [B, N, Hq, d]
    float* dk;                        // [B, G, N, d]
    float* dv;
    int* n_items;
    const int4* items;
    const int* list;
    int64_t N;
    int G, Hg, Hq;
    float scale, scale_log2;
};

__device__ __forceinline__ void cp_async16_zfill(uint32_t smem_dst, const void* gsrc, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_dst), "l"(gsrc), "r"(valid ? 16 : 0)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t saddr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(saddr));
}

__device__ __forceinline__ void red_add_v2(float* addr, float x, float y) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(addr), "f"(x), "f"(y) : "memory");
}

// D[row] = dO . o over d, in fp32: one warp per row.
__global__ void __launch_bounds__(256) bwd_dot_kernel(const uint16_t* __restrict__ go, const uint16_t* __restrict__ o,
                                                      float* __restrict__ dd, int64_t rows) {
    const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const uint2 a = __ldg(reinterpret_cast<const uint2*>(go + row * kHeadDim) + lane);
    const uint2 b = __ldg(reinterpret_cast<const uint2*>(o + row * kHeadDim) + lane);
    float acc = bf16_lo(a.x) * bf16_lo(b.x);
    acc = fmaf(bf16_hi(a.x), bf16_hi(b.x), acc);
    acc = fmaf(bf16_lo(a.y), bf16_lo(b.y), acc);
    acc = fmaf(bf16_hi(a.y), bf16_hi(b.y), acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) dd[row] = acc;
}

// Rows of step `step` of an item into buffer `buf`: row r is token r / Hg of the step, head r % Hg.
__device__ __forceinline__ void load_rows(BwdSmem& sm, const BwdArgs& a, int buf, int b, int g, bool diag, int first,
                                          int n, int step) {
    const int tid = threadIdx.x, Hg = a.Hg, tps = kBwdRows / Hg;
    // 32 rows x 2 tensors x 16 chunks of 16 B: 4 per thread
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int idx = tid + kBwdThreads * i;           // 0 .. 1023
        const int which = idx >> 9, r = (idx >> 4) & 31, ch = idx & 15;
        const int e = step * tps + r / Hg;
        int t = 0;
        const bool valid = e < n;
        if (valid) t = diag ? first + e : __ldg(a.list + first + e) / kBwdSlots;
        const size_t row = (size_t(b) * a.N + t) * a.Hq + size_t(g) * Hg + (r % Hg);
        const uint16_t* src = (which ? a.go : a.q) + row * kHeadDim + ch * 8;
        uint16_t* dst = which ? &sm.go[buf][r][ch * 8] : &sm.q[buf][r][ch * 8];
        cp_async16_zfill(smem_u32(dst), src, valid);
        if (which == 0 && ch == 0) {
            sm.tok[buf][r] = valid ? t : -1;
            sm.lse2[buf][r] = valid ? __ldg(a.lse + row) * 1.4426950408889634f : INFINITY;
            sm.dd[buf][r] = valid ? __ldg(a.dd + row) : 0.f;
        }
    }
    cp_async_commit();
}

__global__ void __launch_bounds__(kBwdThreads, 1) attn_backward_kernel(const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    BwdSmem& sm = *reinterpret_cast<BwdSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const int kw = warp * 16;                            // this warp's keys
    const int n_items = a.n_items[0];
    const int Hg = a.Hg, tps = kBwdRows / Hg;

    for (;;) {
        __syncthreads();                                 // the previous item's buffers are free
        if (tid == 0) sm.item = atomicAdd(a.n_items + 1, 1);
        __syncthreads();
        const int kidx = sm.item;
        if (kidx >= n_items) break;
        const int4 it = __ldg(a.items + kidx);
        const int bg = it.x, b = bg / a.G, g = bg % a.G;
        const bool diag = (it.y & kBwdDiagFlag) != 0;
        const int j = it.y & ~kBwdDiagFlag, first = it.z, n = it.w;
        const int nsteps = (n + tps - 1) / tps;
        // K_j, V_j (rows past the sequence are zeros)
        for (int idx = tid; idx < 2 * kBlock * 16; idx += kBwdThreads) {
            const int which = idx >> 11, r = (idx >> 4) & 127, ch = idx & 15;
            const int64_t u = int64_t(j) * kBlock + r;
            const uint16_t* src = (which ? a.v : a.k) + ((size_t(bg) * a.N + (u < a.N ? u : 0)) * kHeadDim + ch * 8);
            cp_async16_zfill(smem_u32(which ? &sm.v[r][ch * 8] : &sm.k[r][ch * 8]), src, u < a.N);
        }
        cp_async_commit();
        load_rows(sm, a, 0, b, g, diag, first, n, 0);

        float dk[16][4], dv[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i) dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;

        for (int st = 0; st < nsteps; ++st) {
            const int buf = st & 1;
            if (st + 1 < nsteps) {
                load_rows(sm, a, buf ^ 1, b, g, diag, first, n, st + 1);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncthreads();                             // K, V and this step's rows are in
            // ---- S^T and dP^T of this warp's 16 keys x the 32 rows
            float s[4][4], dp[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t ka0, ka1, ka2, ka3, va0, va1, va2, va3;
                ldsm_x4(smem_u32(&sm.k[kw + (lane & 15)][ks * 16 + (lane >> 4) * 8]), ka0, ka1, ka2, ka3);
                ldsm_x4(smem_u32(&sm.v[kw + (lane & 15)][ks * 16 + (lane >> 4) * 8]), va0, va1, va2, va3);
#pragma unroll
                for (int np = 0; np < 2; ++np) {         // two 8-row n-tiles per x4 load
                    uint32_t q0, q1, q2, q3, o0, o1, o2, o3;
                    const int rr = np * 16 + (lane & 7) + ((lane >> 4) << 3), cc = ks * 16 + ((lane >> 3) & 1) * 8;
                    ldsm_x4(smem_u32(&sm.q[buf][rr][cc]), q0, q1, q2, q3);
                    ldsm_x4(smem_u32(&sm.go[buf][rr][cc]), o0, o1, o2, o3);
                    mma_bf16_16816(s[2 * np], ka0, ka1, ka2, ka3, q0, q1);
                    mma_bf16_16816(s[2 * np + 1], ka0, ka1, ka2, ka3, q2, q3);
                    mma_bf16_16816(dp[2 * np], va0, va1, va2, va3, o0, o1);
                    mma_bf16_16816(dp[2 * np + 1], va0, va1, va2, va3, o2, o3);
                }
            }
            // ---- P^T and dS^T (rows gq / gq + 8 of the accumulators are keys, columns are rows)
            uint32_t pa[4][2], sa[4][2];                 // [n-tile][key half] packed bf16 pairs
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {         // hh = 0: key kw + gq, 1: key kw + gq + 8
                    const int64_t u = int64_t(j) * kBlock + kw + gq + 8 * hh;
                    float pv[2], dsv[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int r = nt * 8 + 2 * tq + e;
                        const int t = sm.tok[buf][r];
                        const bool ok = t >= 0 && (!diag || u <= t);
                        const float p = ok ? fast_exp2(s[nt][2 * hh + e] * a.scale_log2 - sm.lse2[buf][r]) : 0.f;
                        pv[e] = p;
                        dsv[e] = p * (dp[nt][2 * hh + e] - sm.dd[buf][r]);
                    }
                    pa[nt][hh] = pack_bf16x2(pv[0], pv[1]);
                    sa[nt][hh] = pack_bf16x2(dsv[0], dsv[1]);
                    // dS to shared memory as [row][key] for the dQ step
                    const int r0 = nt * 8 + 2 * tq;
                    sm.ds[r0][kw + gq + 8 * hh] = uint16_t(sa[nt][hh] & 0xFFFFu);
                    sm.ds[r0 + 1][kw + gq + 8 * hh] = uint16_t(sa[nt][hh] >> 16);
                }
            }
            // ---- dV += P^T dO and dK += dS^T Q over the 32 rows (two k-steps of 16 rows)
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const uint32_t a0 = pa[2 * kk][0], a1 = pa[2 * kk][1], a2 = pa[2 * kk + 1][0], a3 = pa[2 * kk + 1][1];
                const uint32_t c0 = sa[2 * kk][0], c1 = sa[2 * kk][1], c2 = sa[2 * kk + 1][0], c3 = sa[2 * kk + 1][1];
                const int rr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
                for (int dn = 0; dn < 8; ++dn) {
                    uint32_t o0, o1, o2, o3, q0, q1, q2, q3;
                    const int cc = dn * 16 + (lane >> 4) * 8;
                    ldsm_x4_trans(smem_u32(&sm.go[buf][rr][cc]), o0, o1, o2, o3);
                    ldsm_x4_trans(smem_u32(&sm.q[buf][rr][cc]), q0, q1, q2, q3);
                    mma_bf16_16816(dv[2 * dn], a0, a1, a2, a3, o0, o1);
                    mma_bf16_16816(dv[2 * dn + 1], a0, a1, a2, a3, o2, o3);
                    mma_bf16_16816(dk[2 * dn], c0, c1, c2, c3, q0, q1);
                    mma_bf16_16816(dk[2 * dn + 1], c0, c1, c2, c3, q2, q3);
                }
            }
            __syncthreads();                             // dS of every key is in
            // ---- dQ columns 16 w .. 16 w + 15 of the 32 rows: dS (32 x 128 keys) K (keys x 16)
            {
                float acc[2][2][4];
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int nn = 0; nn < 2; ++nn) acc[m][nn][0] = acc[m][nn][1] = acc[m][nn][2] = acc[m][nn][3] = 0.f;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    uint32_t k0, k1, k2, k3;
                    ldsm_x4_trans(smem_u32(&sm.k[ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8][kw + (lane >> 4) * 8]),
                                  k0, k1, k2, k3);
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        uint32_t d0, d1, d2, d3;
                        ldsm_x4(smem_u32(&sm.ds[m * 16 + (lane & 15)][ks * 16 + (lane >> 4) * 8]), d0, d1, d2, d3);
                        mma_bf16_16816(acc[m][0], d0, d1, d2, d3, k0, k1);
                        mma_bf16_16816(acc[m][1], d0, d1, d2, d3, k2, k3);
                    }
                }
#pragma unroll
                for (int m = 0; m < 2; ++m) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int r = m * 16 + gq + 8 * hh;
                        const int t = sm.tok[buf][r];
                        if (t < 0) continue;
                        float* dst = a.dq + ((size_t(b) * a.N + t) * a.Hq + size_t(g) * Hg + (r % Hg)) * kHeadDim + kw;
#pragma unroll
                        for (int nn = 0; nn < 2; ++nn)
                            red_add_v2(dst + nn * 8 + 2 * tq, acc[m][nn][2 * hh] * a.scale, acc[m][nn][2 * hh + 1] * a.scale);
                    }
                }
            }
            // the next step reuses this buffer's rows and dS only after every warp is done with them
            __syncthreads();
        }
        // ---- this item's dK (scaled) and dV of the warp's keys
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int64_t u = int64_t(j) * kBlock + kw + gq + 8 * hh;
            if (u >= a.N) continue;
            float* pk = a.dk + (size_t(bg) * a.N + u) * kHeadDim;
            float* pv = a.dv + (size_t(bg) * a.N + u) * kHeadDim;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                red_add_v2(pk + nt * 8 + 2 * tq, dk[nt][2 * hh] * a.scale, dk[nt][2 * hh + 1] * a.scale);
                red_add_v2(pv + nt * 8 + 2 * tq, dv[nt][2 * hh], dv[nt][2 * hh + 1]);
            }
        }
    }
}

size_t backward_ws_bytes(int B, int64_t N, int G, int Hg) {
    const size_t idx = inverted_index_bytes(B, N, G, Hg);
    return (idx + 255) / 256 * 256 + size_t(B) * N * G * Hg * sizeof(float);
}

msa_status_t launch_attn_backward(const void* q, const void* k, const void* v, int64_t N, int B, int G, int Hg,
                                  const int32_t* sel, const void* out, const float* lse, const void* d_out, float* dq,
                                  float* dk, float* dv, void* ws, cudaStream_t st) {
    const int Hq = G * Hg;
    char* base = static_cast<char*>(ws);
    const size_t idx = inverted_index_bytes(B, N, G, Hg);
    float* dd = reinterpret_cast<float*>(base + (idx + 255) / 256 * 256);
    launch_inverted_index(sel, N, 0, B, G, Hg, ws, st);   // the forward's layout, at the start of ws
    cudaMemsetAsync(dq, 0, size_t(B) * N * Hq * kHeadDim * sizeof(float), st);
    cudaMemsetAsync(dk, 0, size_t(B) * G * N * kHeadDim * sizeof(float), st);
    cudaMemsetAsync(dv, 0, size_t(B) * G * N * kHeadDim * sizeof(float), st);
    {
        const int64_t rows = int64_t(B) * N * Hq;
        const KernelTimer kt(KID_BWD_DOT, st);
        bwd_dot_kernel<<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, st>>>(
            static_cast<const uint16_t*>(d_out), static_cast<const uint16_t*>(out), dd, rows);
    }
    BwdArgs a;
    a.q = static_cast<const uint16_t*>(q);
    a.k = static_cast<const uint16_t*>(k);
    a.v = static_cast<const uint16_t*>(v);
    a.go = static_cast<const uint16_t*>(d_out);
    a.lse = lse;
    a.dd = dd;
    a.dq = dq; a.dk = dk; a.dv = dv;
    const IndexOffsets off = inverted_index_offsets(B, N, G, Hg);
    a.n_items = reinterpret_cast<int*>(base + off.nitems);
    a.items = reinterpret_cast<const int4*>(base + off.items);
    a.list = reinterpret_cast<const int*>(base + off.list);
    a.N = N; a.G = G; a.Hg = Hg; a.Hq = Hq;
    a.scale = 1.0f / sqrtf(float(kHeadDim));
    a.scale_log2 = a.scale * 1.4426950408889634f;
    const int smem = int(sizeof(BwdSmem)) + 128;
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_relaxed)) {
        cudaFuncSetAttribute(attn_backward_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        attr_set[dev].store(true, std::memory_order_relaxed);
    }
    const KernelTimer kt(KID_ATTN_BACKWARD, st);
    attn_backward_kernel<<<num_sms(), kBwdThreads, smem, st>>>(a);
    return MSA_OK;
}

}  // namespace msa

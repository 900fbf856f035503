// attn_prefill.cu -- Main Branch for prefill on the 5th-generation tensor cores (tcgen05).
//
// Sources: youmind article "MiniMax M3 sparse attention agents", figure 1 caption (the main
// branch attends only to the selected blocks), bullet "Predictable cost at every length"
// (16 blocks of 128 tokens per query and GQA group) and paragraph "Why this comes now"
// (each block read once, contiguously); KuCoin flash "MiniMax launches MSA sparse attention
// method and MiniMax-M3 model", summary (exact softmax attention over the selected blocks).
//
// Why key-value-major. Adjacent queries share almost none of their 15 fully-past blocks on
// unstructured data, so a tile of query rows that share a key block cannot be formed by
// query position. Instead, for every (sequence, group, block j) the tokens that selected j
// are listed (an inverted index), and one CTA loads K_j and V_j once (two contiguous 32 KB
// ranges, TMA) and runs 128-row tiles of those tokens' query rows against them: a tile is
// (128 / Hg) tokens x Hg heads, S = Q K_j^T and O = P V_j on tcgen05 with S, P and O in
// tensor memory. Each (token, head, block) row leaves a normalised partial (o in bf16, its
// log2-sum-exp in fp32); the query's own (diagonal) block is processed the same way with a
// causal mask, and a last pass merges each query's partials by log-sum-exp.
//
// Work order. Lists are keyed by (sequence, group, range of kRange query tokens, block), and
// the persistent CTAs walk the work in that order, so the query rows gathered at any moment
// come from one 16K-token range of one group (32 MB at Hg = 8) and stay in L2.
#include "msa_common.cuh"

namespace msa {

constexpr int kRange = 16384;           // query tokens per work range
constexpr int kCountChunk = 1024;       // tokens per CTA of the counting pass (divides kRange)
constexpr int kMaxTilesPerItem = 32;    // tiles per work item (K/V loaded once per item)
constexpr int kSlots = 16;              // partial slots per (token, group); slot 15 = diagonal block
constexpr int kDiagSlot = 15;
constexpr int kDiagFlag = int(0x40000000);
constexpr int kKvThreads = 384;         // warp 0 TMA, warp 1 MMA, warps 4-7 and 8-11 softmax/epilogue

static_assert(kRange % kCountChunk == 0 && kRange % kBlock == 0, "range must hold whole chunks and blocks");

// ------------------------------------------------------------------ workspace layout
struct PrefillLayout {
    int nb, nR, nbins_seg, tpt;
    size_t nbins, max_items, max_entries;
    size_t off_counts, off_offsets, off_nitems, off_items, off_list, off_lse, off_o, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline int64_t imin64(int64_t x, int64_t y) { return x < y ? x : y; }

PrefillLayout prefill_layout(int B, int64_t N, int G, int Hg) {
    PrefillLayout L{};
    L.nb = int((N + kBlock - 1) / kBlock);
    L.nR = int((N + kRange - 1) / kRange);
    L.nbins_seg = L.nb + 1;                                   // blocks + one bin for the diagonal items
    L.tpt = kBlock / Hg;
    L.nbins = size_t(B) * G * L.nR * L.nbins_seg;
    L.max_entries = size_t(B) * N * G * (kTopK - 1);
    L.max_items = L.max_entries / (size_t(L.tpt) * kMaxTilesPerItem) + 1 + size_t(B) * G * L.nR * L.nb +
                  size_t(B) * G * L.nb;
    size_t o = sizeof(WsHeader);
    L.off_counts = o;   o = align_up(o + L.nbins * 4, 256);
    L.off_offsets = o;  o = align_up(o + L.nbins * 4, 256);
    L.off_nitems = o;   o = align_up(o + 16, 256);
    L.off_items = o;    o = align_up(o + L.max_items * 16, 256);
    L.off_list = o;     o = align_up(o + L.max_entries * 4, 256);
    L.off_lse = o;      o = align_up(o + size_t(B) * N * G * kSlots * Hg * 4, 256);
    L.off_o = o;        o = align_up(o + size_t(B) * N * G * kSlots * Hg * kHeadDim * 2, 256);
    L.total = o;
    return L;
}

size_t prefill_attn_ws_bytes(int B, int64_t N, int G, int Hg) { return prefill_layout(B, N, G, Hg).total; }

// ------------------------------------------------------------------ CSR: count
// grid (ceil(N / 1024), G, B), 256 threads, dynamic smem nb ints.
__global__ void __launch_bounds__(256) csr_count_kernel(const int32_t* __restrict__ sel, int64_t N, int G, int nb,
                                                        int nR, int* __restrict__ counts, WsHeader* hdr) {
    extern __shared__ int hist[];
    const int g = blockIdx.y, b = blockIdx.z;
    const int64_t t0 = int64_t(blockIdx.x) * kCountChunk;
    const int64_t t1 = imin64(N, t0 + kCountChunk);
    const int R = int(t0 / kRange);
    for (int i = threadIdx.x; i < nb; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int64_t t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        const int4* row = reinterpret_cast<const int4*>(sel + ((size_t(b) * N + t) * G + g) * kTopK);
        const int c = int(t / kBlock);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int4 v = row[q];
            const int ids[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int id = ids[e];
                if (id >= 0 && id < c) atomicAdd(&hist[id], 1);
                else if (id > c) record_error(hdr, MSA_ERR_DEVICE_BOUNDS, KID_CSR, int(t), 4 * q + e, id);
            }
        }
    }
    __syncthreads();
    int* seg = counts + (size_t(b * G + g) * nR + R) * (nb + 1);
    for (int i = threadIdx.x; i < nb; i += blockDim.x)
        if (hist[i]) atomicAdd(seg + i, hist[i]);
}

// ------------------------------------------------------------------ CSR: scan + work items
// One CTA of 1024 threads. Bins are ordered (b, g, R, j) with j = nb the diagonal bin of the
// range. Writes entry offsets, resets the counts (they become fill cursors), and emits the
// work items in bin order: {b*G+g, j (| kDiagFlag), first entry (or first token), count}.
__global__ void __launch_bounds__(1024) csr_scan_kernel(int* __restrict__ counts, int* __restrict__ offsets,
                                                        int4* __restrict__ items, int* __restrict__ n_items,
                                                        int64_t nbins, int nb, int nR, int64_t N, int tpt) {
    __shared__ long long s_e[1024], s_i[1024];
    const int nbs = nb + 1;
    const int64_t per = (nbins + 1023) / 1024;
    const int64_t lo = imin64(nbins, int64_t(threadIdx.x) * per), hi = imin64(nbins, lo + per);
    const int items_per_max = kMaxTilesPerItem * tpt;
    auto diag_blocks = [&](int R, int& c0, int& c1) {
        c0 = R * (kRange / kBlock);
        c1 = min(nb, (R + 1) * (kRange / kBlock));
    };
    long long se = 0, si = 0;
    for (int64_t bin = lo; bin < hi; ++bin) {
        const int j = int(bin % nbs);
        if (j < nb) {
            const int cnt = counts[bin];
            se += cnt;
            if (cnt > 0) si += (cnt + items_per_max - 1) / items_per_max;
        } else {
            int c0, c1;
            diag_blocks(int((bin / nbs) % nR), c0, c1);
            si += max(0, c1 - c0);
        }
    }
    s_e[threadIdx.x] = se;
    s_i[threadIdx.x] = si;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {             // inclusive Hillis-Steele scan
        long long ae = 0, ai = 0;
        if (threadIdx.x >= off) { ae = s_e[threadIdx.x - off]; ai = s_i[threadIdx.x - off]; }
        __syncthreads();
        s_e[threadIdx.x] += ae;
        s_i[threadIdx.x] += ai;
        __syncthreads();
    }
    long long eoff = s_e[threadIdx.x] - se, ioff = s_i[threadIdx.x] - si;
    for (int64_t bin = lo; bin < hi; ++bin) {
        const int j = int(bin % nbs);
        const int64_t seg = bin / nbs;
        const int R = int(seg % nR);
        const int bg = int(seg / nR);
        if (j < nb) {
            const int cnt = counts[bin];
            offsets[bin] = int(eoff);
            counts[bin] = 0;
            for (int k0 = 0; k0 < cnt; k0 += items_per_max)
                items[ioff++] = make_int4(bg, j, int(eoff + k0), min(items_per_max, cnt - k0));
            eoff += cnt;
        } else {
            int c0, c1;
            diag_blocks(R, c0, c1);
            for (int c = c0; c < c1; ++c)
                items[ioff++] = make_int4(bg, c | kDiagFlag, c * kBlock, int(imin64(kBlock, N - int64_t(c) * kBlock)));
        }
    }
    if (threadIdx.x == 1023) n_items[0] = int(ioff);
}

// ------------------------------------------------------------------ CSR: fill
// one thread per (b, t, g): appends (t, slot) to the list of every fully-past selected block
__global__ void __launch_bounds__(256) csr_fill_kernel(const int32_t* __restrict__ sel, int64_t N, int G, int nb,
                                                       int nR, const int* __restrict__ offsets,
                                                       int* __restrict__ cursors, int* __restrict__ list,
                                                       int64_t total) {
    const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int g = int(idx % G);
    const int64_t t = (idx / G) % N;
    const int b = int(idx / (int64_t(G) * N));
    const int c = int(t / kBlock);
    const int R = int(t / kRange);
    const int4* row = reinterpret_cast<const int4*>(sel + size_t(idx) * kTopK);
    const size_t seg = (size_t(b * G + g) * nR + R) * (nb + 1);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int4 v = row[q];
        const int ids[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int id = ids[e];
            if (id >= 0 && id < c) {
                const int pos = offsets[seg + id] + atomicAdd(cursors + seg + id, 1);
                list[pos] = int(t) * kSlots + (4 * q + e);
            }
        }
    }
}

// ------------------------------------------------------------------ the tensor-core kernel
struct __align__(1024) KvSmem {
    uint8_t kv[2][2][32768];   // [K/V buffer][K, V][d half][128 rows][128 B], 128B swizzle
    uint8_t q[2][32768];       // [stage][d half][128 rows][128 B], 128B swizzle
    uint64_t kv_full[2], kv_empty[2], q_full[2], q_empty[2];
    uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
    uint32_t tmem_base;
    int abort_flag;
};

struct PrefillArgs {
    int64_t N;
    int G, Hg, Hq, tpt;
    const int* n_items;
    const int4* items;
    const int* list;
    float* part_lse;
    uint16_t* part_o;
    WsHeader* hdr;
    float scale_log2;
};

__global__ void __launch_bounds__(kKvThreads, 1) attn_kvmajor_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                     const __grid_constant__ CUtensorMap tmK,
                                                                     const __grid_constant__ CUtensorMap tmV,
                                                                     const PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    KvSmem& sm = *reinterpret_cast<KvSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = *a.n_items;
    const int tpt = a.tpt, Hg = a.Hg;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.kv_full[i], 1);
            mbar_init(&sm.kv_empty[i], 1);
            mbar_init(&sm.q_full[i], 1);
            mbar_init(&sm.q_empty[i], 1);
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_full[i], 128);
            mbar_init(&sm.o_full[i], 1);
            mbar_init(&sm.o_free[i], 128);
        }
        sm.abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        int it = 0, ic = 0;
        for (int k = blockIdx.x; k < n_items; k += gridDim.x, ++ic) {
            const int4 item = a.items[k];
            const int bg = item.x, b = bg / a.G, g = bg % a.G;
            const bool diag = (item.y & kDiagFlag) != 0;
            const int j = item.y & ~kDiagFlag;
            const int kvb = ic & 1;
            bool ok = true;
            if (lane == 0) {
                ok = mbar_wait(&sm.kv_empty[kvb], ((ic >> 1) & 1) ^ 1, a.hdr, KID_ATTN_PREFILL);
                if (ok) {
                    mbar_arrive_expect_tx(&sm.kv_full[kvb], 65536);
                    const int row0 = int(int64_t(bg) * a.N + int64_t(j) * kBlock);
                    for (int h = 0; h < 2; ++h) {
                        tma_load_2d(sm.kv[kvb][0] + h * 16384, &tmK, h * 64, row0, &sm.kv_full[kvb]);
                        tma_load_2d(sm.kv[kvb][1] + h * 16384, &tmV, h * 64, row0, &sm.kv_full[kvb]);
                    }
                }
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) { sm.abort_flag = 1; break; }
            const int n = item.w;
            const int ntiles = (n + tpt - 1) / tpt;
            for (int tt = 0; tt < ntiles; ++tt, ++it) {
                const int buf = it & 1;
                const int nv = min(tpt, n - tt * tpt);
                if (lane == 0) {
                    ok = mbar_wait(&sm.q_empty[buf], ((it >> 1) & 1) ^ 1, a.hdr, KID_ATTN_PREFILL);
                    if (ok) mbar_arrive_expect_tx(&sm.q_full[buf], uint32_t(nv) * Hg * 256u);
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) { sm.abort_flag = 1; break; }
                for (int r = lane; r < nv; r += 32) {
                    const int e = tt * tpt + r;
                    const int t = diag ? item.z + e : (a.list[item.z + e] / kSlots);
                    const int qrow = int((int64_t(b) * a.N + t) * a.Hq + int64_t(g) * Hg);
                    tma_load_2d(sm.q[buf] + r * Hg * 128, &tmQ, 0, qrow, &sm.q_full[buf]);
                    tma_load_2d(sm.q[buf] + 16384 + r * Hg * 128, &tmQ, 64, qrow, &sm.q_full[buf]);
                }
                __syncwarp();
            }
            if (sm.abort_flag) break;
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);   // Q (K-major) x K_j (K-major)
            const uint32_t idesc_o = idesc_bf16_f32(128, 128, 0, 1);   // P (TMEM) x V_j (MN-major)
            int it = 0, ic = 0;
            int prev_it = -1, prev_kvb = 0;
            bool prev_last = false, ok = true;
            auto issue_o = [&](int pit, int pkvb, bool plast) -> bool {
                const int pbuf = pit & 1;
                if (!mbar_wait(&sm.p_full[pbuf], (pit >> 1) & 1, a.hdr, KID_ATTN_PREFILL)) return false;
                if (!mbar_wait(&sm.o_free[pbuf], ((pit >> 1) & 1) ^ 1, a.hdr, KID_ATTN_PREFILL)) return false;
                tc_fence_after();
                const uint32_t tS = tmem + pbuf * 128, tO = tmem + 256 + pbuf * 128;
                const uint32_t vbase = smem_u32(sm.kv[pkvb][1]);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc_mma_ts(tO, tS + ks * 8, sdesc_sw128(vbase + ks * 2048, 16384, 1024), idesc_o, ks > 0);
                tc_commit(&sm.o_full[pbuf]);
                if (plast) tc_commit(&sm.kv_empty[pkvb]);
                return true;
            };
            for (int k = blockIdx.x; k < n_items && ok; k += gridDim.x, ++ic) {
                const int4 item = a.items[k];
                const int n = item.w;
                const int ntiles = (n + tpt - 1) / tpt;
                const int kvb = ic & 1;
                if (!mbar_wait(&sm.kv_full[kvb], (ic >> 1) & 1, a.hdr, KID_ATTN_PREFILL)) { ok = false; break; }
                tc_fence_after();
                const uint32_t kbase = smem_u32(sm.kv[kvb][0]);
                for (int tt = 0; tt < ntiles; ++tt, ++it) {
                    const int buf = it & 1;
                    if (!mbar_wait(&sm.q_full[buf], (it >> 1) & 1, a.hdr, KID_ATTN_PREFILL)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t qbase = smem_u32(sm.q[buf]);
                    const uint32_t tS = tmem + buf * 128;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                        tc_mma_ss(tS, sdesc_sw128(qbase + off, 16, 1024), sdesc_sw128(kbase + off, 16, 1024),
                                  idesc_s, ks > 0);
                    }
                    tc_commit(&sm.s_full[buf]);
                    tc_commit(&sm.q_empty[buf]);
                    if (prev_it >= 0 && !issue_o(prev_it, prev_kvb, prev_last)) { ok = false; break; }
                    prev_it = it;
                    prev_kvb = kvb;
                    prev_last = (tt == ntiles - 1);
                }
            }
            if (ok && prev_it >= 0) issue_o(prev_it, prev_kvb, prev_last);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- softmax + epilogue
        const int w = (warp - 4) >> 2;                      // warpgroup: tiles with it % 2 == w
        const int row = (warp & 3) * 32 + lane;             // TMEM lane = tile row
        const int r = row / Hg, h = row % Hg;
        const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + w * 128;
        const uint32_t tO = tmem + lane_off + 256 + w * 128;
        const float sl2 = a.scale_log2;
        int it = 0;
        for (int k = blockIdx.x; k < n_items; k += gridDim.x) {
            const int4 item = a.items[k];
            const int bg = item.x, b = bg / a.G, g = bg % a.G;
            const bool diag = (item.y & kDiagFlag) != 0;
            const int j = item.y & ~kDiagFlag;
            const int n = item.w;
            const int ntiles = (n + tpt - 1) / tpt;
            bool ok = true;
            for (int tt = 0; tt < ntiles; ++tt, ++it) {
                if ((it & 1) != w) continue;
                const int use = it >> 1;
                const int e = tt * tpt + r;
                const bool valid = e < n;
                int t = 0, slot = kDiagSlot;
                if (valid) {
                    if (diag) t = item.z + e;
                    else { const int v = a.list[item.z + e]; t = v / kSlots; slot = v % kSlots; }
                }
                const int lim = diag ? (t - j * kBlock) : (kBlock - 1);      // last visible key column
                if (!mbar_wait(&sm.s_full[w], use & 1, a.hdr, KID_ATTN_PREFILL)) { ok = false; break; }
                tc_fence_after();
                uint32_t v[32];
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    tmem_ld32(tS + c * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (c * 32 + i <= lim) mx = fmaxf(mx, __uint_as_float(v[i]));
                }
                const float ms = (mx == -INFINITY) ? 0.f : mx * sl2;
                float l = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    tmem_ld32(tS + c * 32, v);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int col = c * 32 + 2 * i;
                        const float p0 = col <= lim ? fast_exp2(fmaf(__uint_as_float(v[2 * i]), sl2, -ms)) : 0.f;
                        const float p1 = col + 1 <= lim ? fast_exp2(fmaf(__uint_as_float(v[2 * i + 1]), sl2, -ms)) : 0.f;
                        l += p0 + p1;
                        pk[i] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(tS + c * 16, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&sm.p_full[w]);

                if (!mbar_wait(&sm.o_full[w], use & 1, a.hdr, KID_ATTN_PREFILL)) { ok = false; break; }
                tc_fence_after();
                const float inv_l = 1.f / l;
                const size_t prow = ((((size_t(b) * a.N + t) * a.G + g) * kSlots + slot) * Hg + h);
                uint4* dst = reinterpret_cast<uint4*>(a.part_o + prow * kHeadDim);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    tmem_ld32(tO + c * 32, v);
                    tmem_wait_ld();
                    if (valid) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 o;
                            o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) * inv_l, __uint_as_float(v[8 * q + 1]) * inv_l);
                            o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) * inv_l, __uint_as_float(v[8 * q + 3]) * inv_l);
                            o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) * inv_l, __uint_as_float(v[8 * q + 5]) * inv_l);
                            o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) * inv_l, __uint_as_float(v[8 * q + 7]) * inv_l);
                            __stcs(dst + c * 4 + q, o);
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&sm.o_free[w]);
                if (valid) __stcs(a.part_lse + prow, ms + __log2f(l));
            }
            if (!ok || sm.abort_flag) { sm.abort_flag = 1; break; }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ combine
// One thread per (b, t, g, head, 32-column quarter): log-sum-exp merge of the query's
// partials (fully-past slots 0..n-2 and the diagonal slot 15).
__global__ void __launch_bounds__(256) combine_kernel(const int32_t* __restrict__ sel,
                                                      const float* __restrict__ part_lse,
                                                      const uint16_t* __restrict__ part_o, int64_t N, int G,
                                                      int Hg, uint16_t* __restrict__ out, float* __restrict__ lse,
                                                      int64_t total) {
    const int64_t gid = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gid >= total) return;
    const int q4 = int(gid & 3);
    const int h = int((gid >> 2) % Hg);
    const int64_t btg = (gid >> 2) / Hg;                   // (b * N + t) * G + g
    const int g = int(btg % G);
    const int64_t bt = btg / G;
    const int4* srow = reinterpret_cast<const int4*>(sel + size_t(btg) * kTopK);
    int nsel = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int4 v = __ldg(srow + q);
        nsel += (v.x >= 0) + (v.y >= 0) + (v.z >= 0) + (v.w >= 0);
    }
    const size_t pbase = size_t(btg) * kSlots;
    float lse_s[kSlots];
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < kSlots; ++s) {
        const bool use = (s == kDiagSlot) || (s < nsel - 1);
        lse_s[s] = use ? __ldcs(part_lse + (pbase + s) * Hg + h) : -INFINITY;
        M = fmaxf(M, lse_s[s]);
    }
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    float L = 0.f;
#pragma unroll 4
    for (int s = 0; s < kSlots; ++s) {
        if (lse_s[s] == -INFINITY) continue;
        const float wgt = fast_exp2(lse_s[s] - M);
        L += wgt;
        const uint4* src = reinterpret_cast<const uint4*>(part_o + ((pbase + s) * Hg + h) * kHeadDim + q4 * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 u = __ldcs(src + q);
            acc[8 * q + 0] = fmaf(wgt, bf16_lo(u.x), acc[8 * q + 0]);
            acc[8 * q + 1] = fmaf(wgt, bf16_hi(u.x), acc[8 * q + 1]);
            acc[8 * q + 2] = fmaf(wgt, bf16_lo(u.y), acc[8 * q + 2]);
            acc[8 * q + 3] = fmaf(wgt, bf16_hi(u.y), acc[8 * q + 3]);
            acc[8 * q + 4] = fmaf(wgt, bf16_lo(u.z), acc[8 * q + 4]);
            acc[8 * q + 5] = fmaf(wgt, bf16_hi(u.z), acc[8 * q + 5]);
            acc[8 * q + 6] = fmaf(wgt, bf16_lo(u.w), acc[8 * q + 6]);
            acc[8 * q + 7] = fmaf(wgt, bf16_hi(u.w), acc[8 * q + 7]);
        }
    }
    const float inv = 1.f / L;
    const int Hq = G * Hg;
    uint4* dst = reinterpret_cast<uint4*>(out + ((size_t(bt) * Hq + size_t(g) * Hg + h) * kHeadDim) + q4 * 32);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 o;
        o.x = pack_bf16x2(acc[8 * q + 0] * inv, acc[8 * q + 1] * inv);
        o.y = pack_bf16x2(acc[8 * q + 2] * inv, acc[8 * q + 3] * inv);
        o.z = pack_bf16x2(acc[8 * q + 4] * inv, acc[8 * q + 5] * inv);
        o.w = pack_bf16x2(acc[8 * q + 6] * inv, acc[8 * q + 7] * inv);
        dst[q] = o;
    }
    if (lse != nullptr && q4 == 0) lse[size_t(bt) * Hq + size_t(g) * Hg + h] = (M + __log2f(L)) * 0.69314718055994530942f;
}

// ------------------------------------------------------------------ host launcher
int num_sms() {
    static int n[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (n[dev] == 0) cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev);
    return n[dev] > 0 ? n[dev] : 148;
}

void launch_attn_prefill_tc(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, int64_t N,
                            int B, int G, int Hg, const int32_t* sel, void* out, float* lse, void* ws,
                            cudaStream_t st) {
    const PrefillLayout L = prefill_layout(B, N, G, Hg);
    char* base = static_cast<char*>(ws);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(base);
    int* counts = reinterpret_cast<int*>(base + L.off_counts);
    int* offsets = reinterpret_cast<int*>(base + L.off_offsets);
    int* nitems = reinterpret_cast<int*>(base + L.off_nitems);
    int4* items = reinterpret_cast<int4*>(base + L.off_items);
    int* list = reinterpret_cast<int*>(base + L.off_list);
    float* part_lse = reinterpret_cast<float*>(base + L.off_lse);
    uint16_t* part_o = reinterpret_cast<uint16_t*>(base + L.off_o);

    cudaMemsetAsync(counts, 0, L.nbins * sizeof(int), st);
    {
        dim3 grid(static_cast<unsigned>((N + kCountChunk - 1) / kCountChunk), static_cast<unsigned>(G),
                  static_cast<unsigned>(B));
        const size_t smem = size_t(L.nb) * sizeof(int);
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(csr_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        count_launch();
        csr_count_kernel<<<grid, 256, smem, st>>>(sel, N, G, L.nb, L.nR, counts, hdr);
    }
    count_launch();
    csr_scan_kernel<<<1, 1024, 0, st>>>(counts, offsets, items, nitems, int64_t(L.nbins), L.nb, L.nR, N, L.tpt);
    {
        const int64_t total = int64_t(B) * N * G;
        count_launch();
        csr_fill_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(sel, N, G, L.nb, L.nR, offsets,
                                                                                   counts, list, total);
    }
    {
        PrefillArgs a;
        a.N = N; a.G = G; a.Hg = Hg; a.Hq = G * Hg; a.tpt = L.tpt;
        a.n_items = nitems; a.items = items; a.list = list; a.part_lse = part_lse; a.part_o = part_o;
        a.hdr = hdr;
        a.scale_log2 = 1.4426950408889634f / sqrtf(float(kHeadDim));
        const int smem = int(sizeof(KvSmem)) + 1024;
        static bool attr_set[64] = {false};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev >= 0 && dev < 64 && !attr_set[dev]) {
            cudaFuncSetAttribute(attn_kvmajor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            attr_set[dev] = true;
        }
        count_launch();
        attn_kvmajor_kernel<<<num_sms(), kKvThreads, smem, st>>>(tmQ, tmK, tmV, a);
    }
    {
        const int64_t total = int64_t(B) * N * G * Hg * 4;
        count_launch();
        combine_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(sel, part_lse, part_o, N, G, Hg,
                                                                                  static_cast<uint16_t*>(out), lse,
                                                                                  total);
    }
}

}  // namespace msa

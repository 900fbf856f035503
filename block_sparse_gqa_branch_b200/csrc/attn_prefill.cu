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
#include <atomic>

#include "msa_common.cuh"

namespace msa {

constexpr int kRange = 16384;           // query tokens per work range
constexpr int kCountChunk = 1024;       // tokens per CTA of the counting pass (divides kRange)
constexpr int kMaxTilesPerItem = 32;    // tiles per work item (K/V loaded once per item)
constexpr int kSlots = 16;              // partial slots per (token, group); slot 15 = diagonal block
constexpr int kDiagSlot = 15;
constexpr int kDiagFlag = int(0x40000000);
constexpr int kKvThreads = 352;         // warps 0-7 softmax/epilogue, 8 Q loads, 9 MMA, 10 K/V loads

static_assert(kRange % kCountChunk == 0 && kRange % kBlock == 0, "range must hold whole chunks and blocks");

// ------------------------------------------------------------------ workspace layout
// Queries are the n tokens at positions P .. P + n - 1 of each sequence (P = 0 for a whole
// prefill; P > 0 for a chunk against a cache that holds positions 0 .. P + n - 1). Token
// indices inside the kernels are chunk-relative (i = t - P); block ids are absolute.
struct PrefillLayout {
    int nb, nR, nbins_seg, tpt;     // nb: key blocks that can be selected (ceil((P + n) / Bk))
    size_t nbins, max_items, max_entries;
    size_t off_counts, off_offsets, off_nitems, off_items, off_list, off_lse, off_o, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline int64_t imin64(int64_t x, int64_t y) { return x < y ? x : y; }

PrefillLayout prefill_layout(int B, int64_t N, int G, int Hg, int64_t P) {
    PrefillLayout L{};
    L.nb = int((P + N + kBlock - 1) / kBlock);
    L.nR = int((N + kRange - 1) / kRange);
    L.nbins_seg = L.nb + 1;                                   // blocks + one bin for the diagonal items
    L.tpt = kBlock / Hg;
    L.nbins = size_t(B) * G * L.nR * L.nbins_seg;
    L.max_entries = size_t(B) * N * G * (kTopK - 1);
    // list items: at most one per started run of kMaxTilesPerItem tiles plus one per bin;
    // diagonal items: one per (range, query block) overlap, at most (query blocks + ranges)
    const size_t nqb = size_t((P + N - 1) / kBlock - P / kBlock + 1);
    L.max_items = L.max_entries / (size_t(L.tpt) * kMaxTilesPerItem) + 1 + size_t(B) * G * L.nR * L.nb +
                  size_t(B) * G * (nqb + L.nR);
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

size_t prefill_attn_ws_bytes(int B, int64_t N, int G, int Hg, int64_t P) {
    return prefill_layout(B, N, G, Hg, P).total;
}

// ------------------------------------------------------------------ CSR: count
// grid (ceil(N / 1024), G, B), 256 threads, dynamic smem nb ints. N queries from position P.
__global__ void __launch_bounds__(256) csr_count_kernel(const int32_t* __restrict__ sel, int64_t N, int64_t P, int G,
                                                        int nb, int nR, int* __restrict__ counts, WsHeader* hdr) {
    extern __shared__ int hist[];
    const int g = blockIdx.y, b = blockIdx.z;
    const int64_t t0 = int64_t(blockIdx.x) * kCountChunk;
    const int64_t t1 = imin64(N, t0 + kCountChunk);
    const int R = int(t0 / kRange);
    for (int i = threadIdx.x; i < nb; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int64_t t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        const int4* row = reinterpret_cast<const int4*>(sel + ((size_t(b) * N + t) * G + g) * kTopK);
        const int c = int((P + t) / kBlock);
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
// The bins go 1,024 at a time, thread i taking bin 1024 k + i, so every load and store of a
// round is coalesced; a block-wide scan of (entries, items) per round plus the running totals
// gives each bin its offsets, and the next round's counts are loaded during the current one.
// Entry and item totals fit in int: the host bounds B N G (k - 1) below 2^31.
__device__ __forceinline__ void warp_scan2(int& x, int& y, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int ax = __shfl_up_sync(0xffffffffu, x, off), ay = __shfl_up_sync(0xffffffffu, y, off);
        if (lane >= off) { x += ax; y += ay; }
    }
}

__global__ void __launch_bounds__(1024) csr_scan_kernel(int* __restrict__ counts, int* __restrict__ offsets,
                                                        int4* __restrict__ items, int* __restrict__ n_items,
                                                        int64_t nbins, int nb, int nR, int64_t N, int64_t P, int tpt) {
    __shared__ int w_e[2][32], w_i[2][32];          // per-warp totals, one set per round parity
    const int nbs = nb + 1;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int items_per_max = kMaxTilesPerItem * tpt;
    int carry_e = 0, carry_i = 0;                    // entries and items of the earlier rounds
    int64_t bin = threadIdx.x;
    int cnt_next = bin < nbins ? counts[bin] : 0;
    for (int round = 0; int64_t(round) * 1024 < nbins; ++round, bin += 1024) {
        const int cnt = cnt_next;
        cnt_next = bin + 1024 < nbins ? counts[bin + 1024] : 0;
        const bool live = bin < nbins;
        const int j = int(bin % nbs);
        const int64_t seg = bin / nbs;
        const int R = int(seg % nR), bg = int(seg / nR);
        // diagonal bin: query blocks [c0, c1) that hold positions of range R
        const int64_t qa = int64_t(R) * kRange, qz = imin64(N, int64_t(R + 1) * kRange);
        const int c0 = int((P + qa) / kBlock), c1 = int((P + qz - 1) / kBlock) + 1;
        int ve = 0, vi = 0;
        if (live) {
            if (j < nb) { ve = cnt; vi = (cnt + items_per_max - 1) / items_per_max; }
            else vi = max(0, c1 - c0);
        }
        int se = ve, si = vi;
        warp_scan2(se, si, lane);
        const int buf = round & 1;
        if (lane == 31) { w_e[buf][wid] = se; w_i[buf][wid] = si; }
        __syncthreads();
        if (wid == 0) {
            int te = w_e[buf][lane], ti = w_i[buf][lane];
            warp_scan2(te, ti, lane);
            w_e[buf][lane] = te;
            w_i[buf][lane] = ti;
        }
        __syncthreads();
        const int eoff = carry_e + (wid > 0 ? w_e[buf][wid - 1] : 0) + se - ve;
        int ioff = carry_i + (wid > 0 ? w_i[buf][wid - 1] : 0) + si - vi;
        carry_e += w_e[buf][31];
        carry_i += w_i[buf][31];
        if (!live) continue;
        if (j < nb) {
            offsets[bin] = eoff;
            counts[bin] = 0;
            for (int k0 = 0; k0 < cnt; k0 += items_per_max)
                items[ioff++] = make_int4(bg, j, eoff + k0, min(items_per_max, cnt - k0));
        } else {
            // diagonal items: the range's queries inside block c, as (first query index, count)
            for (int c = c0; c < c1; ++c) {
                const int64_t f = int64_t(c) * kBlock - P > qa ? int64_t(c) * kBlock - P : qa;
                const int64_t e = imin64(qz, int64_t(c + 1) * kBlock - P);
                items[ioff++] = make_int4(bg, c | kDiagFlag, int(f), int(e - f));
            }
        }
    }
    if (threadIdx.x == 0) {
        n_items[0] = carry_i;
        n_items[1] = 0;                                   // work-item counter of the tensor-core kernel
    }
}

// ------------------------------------------------------------------ CSR: fill
// grid (ceil(N / 1024), G, B), 1024 threads (one query each), dynamic smem nb ints. Every
// fully-past selected block of the chunk's queries gets the entry (t, slot) in its list. The
// chunk lies in one range (kRange is a multiple of kCountChunk), so it reserves one run of
// each block's list with one global atomic: the queries number their entries per block in
// shared memory, the counts reserve the runs, and each entry goes to its run's base plus its
// number.
__global__ void __launch_bounds__(1024) csr_fill_kernel(const int32_t* __restrict__ sel, int64_t N, int64_t P, int G,
                                                        int nb, int nR, const int* __restrict__ offsets,
                                                        int* __restrict__ cursors, int* __restrict__ list) {
    extern __shared__ int runs[];                 // per block: entries of the chunk, then the run's base
    const int g = blockIdx.y, b = blockIdx.z;
    const int64_t t = int64_t(blockIdx.x) * kCountChunk + threadIdx.x;
    const int R = int((int64_t(blockIdx.x) * kCountChunk) / kRange);
    for (int i = threadIdx.x; i < nb; i += blockDim.x) runs[i] = 0;
    int ids[kTopK];
    if (t < N) {
        const int4* row = reinterpret_cast<const int4*>(sel + ((size_t(b) * N + t) * G + g) * kTopK);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int4 v = row[q];
            ids[4 * q] = v.x; ids[4 * q + 1] = v.y; ids[4 * q + 2] = v.z; ids[4 * q + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < kTopK; ++e) ids[e] = -1;
    }
    const int c = int((P + t) / kBlock);
    __syncthreads();
    int num[kTopK];
#pragma unroll
    for (int e = 0; e < kTopK; ++e) {
        const int id = ids[e];
        num[e] = (id >= 0 && id < c) ? atomicAdd(&runs[id], 1) : -1;
    }
    __syncthreads();
    const size_t seg = (size_t(b * G + g) * nR + R) * (nb + 1);
    for (int i = threadIdx.x; i < nb; i += blockDim.x) {
        const int n = runs[i];
        if (n > 0) runs[i] = offsets[seg + i] + atomicAdd(cursors + seg + i, n);
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kTopK; ++e)
        if (num[e] >= 0) list[runs[ids[e]] + num[e]] = int(t) * kSlots + e;
}

// ------------------------------------------------------------------ the tensor-core kernel
constexpr int kQStages = 3;
constexpr int kRing = 8;           // work items handed from the scheduler to the other roles
constexpr int kRingReaders = 10;   // Q warp, MMA thread, 8 softmax warps

struct __align__(1024) KvSmem {
    uint8_t k[2][32768];          // K_j, double-buffered: [d half][128 rows][128 B], 128B swizzle
    uint8_t v[32768];             // V_j: [d half][128 rows][128 B], 128B swizzle
    uint8_t q[kQStages][32768];   // gathered query rows: [d half][128 rows][128 B], 128B swizzle
    uint8_t o_stage[8][4096];     // per softmax warp, one d half at a time: [32 output rows][128 B] (bf16), 128B swizzle
    uint64_t k_full[2], k_empty[2], v_full, v_empty, q_full[kQStages], q_empty[kQStages];
    uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
    uint64_t item_full[kRing], item_empty[kRing];
    volatile int item_ring[kRing];
    uint32_t tmem_base;
    int abort_flag;
};

struct PrefillArgs {
    int64_t N;                     // queries per sequence (positions P .. P + N - 1)
    int64_t P;                     // position of the first query
    int G, Hg, Hq, tpt;
    int* n_items;                  // [0] = number of work items, [1] = next item to hand out
    const int4* items;
    const int* list;
    float* part_lse;
    uint16_t* part_o;
    const uint16_t* q;
    WsHeader* hdr;
    float scale_log2;
};

// packed fp32x2 arithmetic (one instruction for two lanes of data)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// Work-item decoding shared by every role: all roles walk items blockIdx.x, +gridDim.x, ...
struct Item {
    int bg, b, g, j, first, n, ntiles;
    bool diag;
};
__device__ __forceinline__ Item load_item(const PrefillArgs a, int k) {
    const int4 v = a.items[k];
    Item it;
    it.bg = v.x; it.b = v.x / a.G; it.g = v.x % a.G;
    it.diag = (v.y & kDiagFlag) != 0;
    it.j = v.y & ~kDiagFlag;
    it.first = v.z; it.n = v.w;
    it.ntiles = (v.w + a.tpt - 1) / a.tpt;
    return it;
}

// O = P V for a tile whose S was issued earlier (MMA-issuing thread only). The first tile of an
// item waits for the item's V; the last one releases V when its MMAs complete.
struct PendO { int it, ic; bool first, last; };
__device__ __forceinline__ bool issue_o(KvSmem& sm, const PrefillArgs a, uint32_t tmem, uint32_t vbase,
                                        uint32_t idesc_o, const PendO& p) {
    const int buf = p.it & 1;
    if (p.first && !mbar_wait(&sm.v_full, p.ic & 1, a.hdr, KID_ATTN_PREFILL)) return false;
    if (!mbar_wait(&sm.p_full[buf], (p.it >> 1) & 1, a.hdr, KID_ATTN_PREFILL)) return false;
    if (!mbar_wait(&sm.o_free[buf], ((p.it >> 1) & 1) ^ 1, a.hdr, KID_ATTN_PREFILL)) return false;
    tc_fence_after();
    const uint32_t tS = tmem + buf * 128, tO = tmem + 256 + buf * 128;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
        tc_mma_ts(tO, tS + 64 + ks * 8, sdesc_sw128(vbase + ks * 2048, 16384, 1024), idesc_o, ks > 0);
    tc_commit(&sm.o_full[buf]);
    if (p.last) tc_commit(&sm.v_empty);
    return true;
}

// A bounded wait by every lane of a warp whose outcome is the same for the whole warp (a lane
// that timed out makes all lanes fail), so the warp's collective instructions stay converged.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, WsHeader* hdr) {
    const bool ok = mbar_wait(bar, parity, hdr, KID_ATTN_PREFILL);
    return __all_sync(0xffffffffu, ok);
}

// Next work item of a role's sequence s (-1 = no more work, -2 = timeout). With whole_warp,
// every lane of the warp calls this, reads the slot, and lane 0 releases it after the warp has
// read it; otherwise a single thread calls it and releases the slot itself.
__device__ __forceinline__ int ring_take(KvSmem& sm, int s, WsHeader* hdr, bool whole_warp) {
    const int slot = s % kRing;
    const bool got = whole_warp ? warp_wait(&sm.item_full[slot], (s / kRing) & 1, hdr)
                                : mbar_wait(&sm.item_full[slot], (s / kRing) & 1, hdr, KID_ATTN_PREFILL);
    if (!got) return -2;
    const int k = sm.item_ring[slot];
    if (whole_warp) {
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(&sm.item_empty[slot]);
    } else {
        mbar_arrive(&sm.item_empty[slot]);
    }
    return k;
}

// token of row group r of tile tt of an item (0 when r is past the item's end)
__device__ __forceinline__ int fetch_token(const PrefillArgs a, const Item item, int tt, int r) {
    const int e = tt * a.tpt + r;
    if (r >= a.tpt || tt >= item.ntiles || e >= item.n) return 0;
    return item.diag ? item.first + e : (__ldg(a.list + item.first + e) / kSlots);
}

// Epilogue of a softmax warpgroup's tile: O from tensor memory, divided by the row sums, to
// bf16, staged per warp and stored with TMA, plus the rows' log2-sum-exp.
struct PendEpi {
    int use;                 // the tile's use of its S/O buffer pair (-1: none)
    size_t prow;             // partial row of this thread's (token, head)
    bool valid;
    float l, ms;             // row sum and scaled row max
};
__device__ __forceinline__ bool epilogue_tile(KvSmem& sm, const PrefillArgs& a, const CUtensorMap* tmO, uint32_t tO,
                                  uint8_t* stg, uint64_t stream, int w, int lane, int Hg, int h,
                                  const PendEpi& p) {
    uint32_t va[32], vb[32];
    if (!warp_wait(&sm.o_full[w], p.use & 1, a.hdr)) return false;
    tc_fence_after();
    const float inv_l = 1.f / p.l;
    const float2 il = make_float2(inv_l, inv_l);
    // this warp's 32 rows hold 32 / Hg whole tokens; lane i stores token i's Hg rows
    const int ntok_w = 32 / Hg;
    const int src_lane = (lane * Hg) & 31;
    const int tok_prow = __shfl_sync(0xffffffffu, int(p.prow - h), src_lane);   // row of head 0
    const bool tok_valid = __shfl_sync(0xffffffffu, p.valid, src_lane) && lane < ntok_w;
    // both d halves leave tensor memory first (packed to bf16 in registers), so the O buffer is
    // free for the next tile's P V before any staging or store
    uint32_t o[2][8][4];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        tmem_ld32(tO + half * 64, va);
        tmem_ld32(tO + half * 64 + 32, vb);
        tmem_wait_ld();
        if (half == 1) {
            tc_fence_before();
            mbar_arrive(&sm.o_free[w]);                // O of this buffer fully read
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                const int i0 = (8 * c + 2 * e2) & 31;
                const uint32_t x0 = c < 4 ? va[i0] : vb[i0];
                const uint32_t x1 = c < 4 ? va[i0 + 1] : vb[i0 + 1];
                const float2 y = fmul2(make_float2(__uint_as_float(x0), __uint_as_float(x1)), il);
                o[half][c][e2] = pack_bf16x2(y.x, y.y);
            }
        }
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        bulk_wait_read0();              // the staging's earlier stores have read it
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(stg + sw128(lane, c)) =
                make_uint4(o[half][c][0], o[half][c][1], o[half][c][2], o[half][c][3]);
        fence_proxy_async();
        __syncwarp();
        if (tok_valid) {
            tma_store_2d_hint(tmO, half * 64, tok_prow, stg + lane * Hg * 128, stream);
            bulk_commit();
        }
    }
    if (p.valid) __stcs(a.part_lse + p.prow, p.ms + __log2f(p.l));
    return true;
}

__global__ void __launch_bounds__(kKvThreads, 1) attn_kvmajor_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                     const __grid_constant__ CUtensorMap tmK,
                                                                     const __grid_constant__ CUtensorMap tmV,
                                                                     const __grid_constant__ CUtensorMap tmO,
                                                                     const PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    KvSmem& sm = *reinterpret_cast<KvSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = *a.n_items;
    const int tpt = a.tpt, Hg = a.Hg;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.k_full[i], 1);
            mbar_init(&sm.k_empty[i], 1);
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_full[i], 128);
            mbar_init(&sm.o_full[i], 1);
            mbar_init(&sm.o_free[i], 128);
        }
        for (int i = 0; i < kQStages; ++i) {
            mbar_init(&sm.q_full[i], 1);
            mbar_init(&sm.q_empty[i], 1);
        }
        mbar_init(&sm.v_full, 1);
        mbar_init(&sm.v_empty, 1);
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&sm.item_full[i], 1);
            mbar_init(&sm.item_empty[i], kRingReaders);
        }
        sm.abort_flag = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmO);
    }
    if (warp == 9) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 8) {
        // ---------------------------------------------------------------- Q gather (TMA)
        // Tile it goes to stage it % kQStages; lane r issues the copies of the tile's tokens r,
        // r + 32, ... For Hg >= 8 one 3-D box brings 8 head rows of a token with both d halves
        // (2 KB): the stage is laid out as 8-row groups of 2 KB ([half][8 rows][128 B], 128B
        // swizzle). For Hg < 8 a token's Hg rows come as two 2-D boxes into [half][128 rows][128 B].
        // List entries of the next tile are fetched ahead. One warp produces every stage, so each
        // stage's uses are waited for in order.
        const uint64_t keep = l2_evict_last();          // query rows are re-read ~15 times per range
        int it = 0;
        for (int sq = 0;; ++sq) {
            const int k = ring_take(sm, sq, a.hdr, true);
            if (k < 0) { if (k == -2) sm.abort_flag = 1; break; }
            const Item item = load_item(a, k);
            int tok[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) tok[i] = fetch_token(a, item, 0, lane + 32 * i);
            for (int tt = 0; tt < item.ntiles; ++tt, ++it) {
                const int stage = it % kQStages, use = it / kQStages;
                const int nv = min(tpt, item.n - tt * tpt);
                bool ok = true;
                if (lane == 0) {
                    ok = mbar_wait(&sm.q_empty[stage], (use & 1) ^ 1, a.hdr, KID_ATTN_PREFILL);
                    if (ok) mbar_arrive_expect_tx(&sm.q_full[stage], uint32_t(nv) * Hg * 256u);
                }
                if (!__shfl_sync(0xffffffffu, ok, 0)) { sm.abort_flag = 1; break; }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = lane + 32 * i;
                    if (r < nv) {
                        const int qrow = int((int64_t(item.b) * a.N + tok[i]) * a.Hq + int64_t(item.g) * Hg);
                        if (Hg >= 8) {
                            for (int h8 = 0; h8 < Hg; h8 += 8)
                                tma_load_3d_hint(sm.q[stage] + (r * Hg + h8) * 256, &tmQ, 0, qrow + h8, 0, &sm.q_full[stage], keep);
                        } else {
                            tma_load_2d_hint(sm.q[stage] + r * Hg * 128, &tmQ, 0, qrow, &sm.q_full[stage], keep);
                            tma_load_2d_hint(sm.q[stage] + 16384 + r * Hg * 128, &tmQ, 64, qrow, &sm.q_full[stage], keep);
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) tok[i] = fetch_token(a, item, tt + 1, lane + 32 * i);
                __syncwarp();
            }
            if (__any_sync(0xffffffffu, sm.abort_flag != 0)) break;
        }
    } else if (warp == 10) {
        // ---------------------------------------------------------------- scheduler + K/V loads (TMA)
        // Items are handed out in list order through a global counter, so all CTAs stay within a
        // narrow window of the work order (the window's query rows stay in L2).
        if (lane == 0) {
            const uint64_t stream = l2_evict_first();   // a key/value block serves one work item
            for (int ic = 0;; ++ic) {
                const int slot = ic % kRing;
                if (!mbar_wait(&sm.item_empty[slot], ((ic / kRing) & 1) ^ 1, a.hdr, KID_ATTN_PREFILL)) {
                    sm.abort_flag = 1;
                    break;
                }
                int k = atomicAdd(a.n_items + 1, 1);
                if (k >= n_items) k = -1;
                sm.item_ring[slot] = k;
                mbar_arrive(&sm.item_full[slot]);
                if (k < 0) break;
                const Item item = load_item(a, k);
                if (!item.diag) {                           // warm L2 with the item's list entries
                    const uint64_t lo = (uint64_t(reinterpret_cast<uintptr_t>(a.list + item.first))) & ~uint64_t(15);
                    const uint64_t hi = (uint64_t(reinterpret_cast<uintptr_t>(a.list + item.first + item.n)) + 15) & ~uint64_t(15);
                    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(lo), "r"(uint32_t(hi - lo)) : "memory");
                }
                // block j of (sequence, group) bg: rows past the last query position are zeros
                const int row0 = item.j * kBlock;
                const int kb = ic & 1;
                if (!mbar_wait(&sm.k_empty[kb], ((ic >> 1) & 1) ^ 1, a.hdr, KID_ATTN_PREFILL)) { sm.abort_flag = 1; break; }
                mbar_arrive_expect_tx(&sm.k_full[kb], 32768);
                tma_load_3d_hint(sm.k[kb], &tmK, 0, row0, item.bg, &sm.k_full[kb], stream);
                tma_load_3d_hint(sm.k[kb] + 16384, &tmK, 64, row0, item.bg, &sm.k_full[kb], stream);
                if (!mbar_wait(&sm.v_empty, (ic & 1) ^ 1, a.hdr, KID_ATTN_PREFILL)) { sm.abort_flag = 1; break; }
                mbar_arrive_expect_tx(&sm.v_full, 32768);
                tma_load_3d_hint(sm.v, &tmV, 0, row0, item.bg, &sm.v_full, stream);
                tma_load_3d_hint(sm.v + 16384, &tmV, 64, row0, item.bg, &sm.v_full, stream);
            }
        }
        __syncwarp();
    } else if (warp == 9) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);   // Q (K-major) x K_j (K-major)
            // Q stage layout (see the Q gather): d-half offset and 8-row-group stride
            const uint32_t q_half = Hg >= 8 ? 1024u : 16384u, q_sbo = Hg >= 8 ? 2048u : 1024u;
            const uint32_t idesc_o = idesc_bf16_f32(128, 128, 0, 1);   // P (TMEM) x V_j (MN-major)
            const uint32_t vbase = smem_u32(sm.v);
            PendO pend{-1, 0, false, false};
            bool ok = true;
            int it = 0;
            for (int ic = 0; ok; ++ic) {
                const int k = ring_take(sm, ic, a.hdr, false);
                if (k < 0) { ok = (k == -1); break; }
                const Item item = load_item(a, k);
                const int kb = ic & 1;
                // finish the previous item's last tile before waiting for this item's keys
                if (pend.it >= 0) {
                    if (!issue_o(sm, a, tmem, vbase, idesc_o, pend)) { ok = false; break; }
                    pend.it = -1;
                }
                if (!mbar_wait(&sm.k_full[kb], (ic >> 1) & 1, a.hdr, KID_ATTN_PREFILL)) { ok = false; break; }
                tc_fence_after();
                const uint32_t kbase = smem_u32(sm.k[kb]);
                for (int tt = 0; tt < item.ntiles; ++tt, ++it) {
                    const int buf = it & 1, stage = it % kQStages;
                    if (!mbar_wait(&sm.q_full[stage], (it / kQStages) & 1, a.hdr, KID_ATTN_PREFILL)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t qbase = smem_u32(sm.q[stage]);
                    const uint32_t tS = tmem + buf * 128;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                        const uint32_t qoff = (ks >> 2) * q_half + (ks & 3) * 32;
                        tc_mma_ss(tS, sdesc_sw128(qbase + qoff, 16, q_sbo), sdesc_sw128(kbase + koff, 16, 1024),
                                  idesc_s, ks > 0);
                    }
                    tc_commit(&sm.s_full[buf]);
                    tc_commit(&sm.q_empty[stage]);
                    if (tt == item.ntiles - 1) tc_commit(&sm.k_empty[kb]);
                    if (pend.it >= 0 && !issue_o(sm, a, tmem, vbase, idesc_o, pend)) { ok = false; break; }
                    pend = PendO{it, ic, tt == 0, tt == item.ntiles - 1};
                }
            }
            if (ok && pend.it >= 0) issue_o(sm, a, tmem, vbase, idesc_o, pend);
            if (!ok) sm.abort_flag = 1;
        }
        __syncwarp();
    } else if (warp < 8) {
        // ---------------------------------------------------------------- softmax + epilogue
        const int w = warp >> 2;                            // warpgroup w takes the tiles with it % 2 == w
        const int row = (warp & 3) * 32 + lane;             // TMEM lane = tile row
        const int r = row / Hg, h = row % Hg;
        const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + w * 128;
        const uint32_t tO = tmem + lane_off + 256 + w * 128;
        const float sl2 = a.scale_log2;
        const float2 sc = make_float2(sl2, sl2);
        uint8_t* stg = sm.o_stage[warp];
        const uint64_t stream = l2_evict_first();       // partial outputs are read once, much later
        PendEpi pend{-1, 0, false, 1.f, 0.f};
        int it = 0;
        bool ok = true;
        for (int si = 0; ok; ++si) {
            const int k = ring_take(sm, si, a.hdr, true);
            if (k < 0) { ok = (k == -1); break; }
            const Item item = load_item(a, k);
            for (int tt = 0; tt < item.ntiles; ++tt, ++it) {
                if ((it & 1) != w) continue;
                const int use = it >> 1;
                const int e = tt * tpt + r;
                const bool valid = e < item.n;
                int t = 0, slot = kDiagSlot;
                if (valid) {
                    if (item.diag) t = item.first + e;
                    else { const int v = __ldg(a.list + item.first + e); t = v / kSlots; slot = v % kSlots; }
                }
                // columns past lim are masked (causal mask of the diagonal block; t is the
                // query index, P + t its position)
                const int lim = item.diag ? int(a.P + t - int64_t(item.j) * kBlock) : kBlock - 1;
                if (!warp_wait(&sm.s_full[w], use & 1, a.hdr)) { ok = false; break; }
                tc_fence_after();
                uint32_t va[32], vb[32];
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int p = 0; p < 2; ++p) {                       // row max, 64 columns per TMEM wait
                    tmem_ld32(tS + p * 64, va);
                    tmem_ld32(tS + p * 64 + 32, vb);
                    tmem_wait_ld();
                    if (!item.diag) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            m4[i & 3] = fmax3(m4[i & 3], __uint_as_float(va[i]), __uint_as_float(vb[i]));
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            if (p * 64 + i <= lim) m4[i & 3] = fmaxf(m4[i & 3], __uint_as_float(va[i]));
                            if (p * 64 + 32 + i <= lim) m4[i & 3] = fmaxf(m4[i & 3], __uint_as_float(vb[i]));
                        }
                    }
                }
                const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                const float ms = (mx == -INFINITY) ? 0.f : mx * sl2;
                const float2 nm = make_float2(-ms, -ms);
                float2 l2 = make_float2(0.f, 0.f);
                // p = 2^(s*scale - m) -> TMEM as bf16, into columns 64..127 of the S buffer (the
                // second half's S, already read): the second half first, from the registers the
                // max pass left it in, then the first half, read again
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {
                    const int p = 1 - pp;
                    if (p == 0) {
                        tmem_ld32(tS, va);
                        tmem_ld32(tS + 32, vb);
                        tmem_wait_ld();
                    }
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const uint32_t x0 = q == 0 ? va[2 * i] : vb[2 * i];
                            const uint32_t x1 = q == 0 ? va[2 * i + 1] : vb[2 * i + 1];
                            const float2 x = ffma2(make_float2(__uint_as_float(x0), __uint_as_float(x1)), sc, nm);
                            const int col = p * 64 + q * 32 + 2 * i;
                            float2 pv = make_float2(fast_exp2(x.x), fast_exp2(x.y));
                            if (item.diag) {
                                pv.x = col <= lim ? pv.x : 0.f;
                                pv.y = col + 1 <= lim ? pv.y : 0.f;
                            }
                            l2 = fadd2(l2, pv);
                            pk[i] = pack_bf16x2(pv.x, pv.y);
                        }
                        tmem_st16(tS + 64 + p * 32 + q * 16, pk);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&sm.p_full[w]);
                const float l = l2.x + l2.y;

                const size_t prow = ((((size_t(item.b) * a.N + t) * a.G + item.g) * kSlots + slot) * Hg + h);
                // the epilogue of this warpgroup's previous tile: its O was computed while this
                // tile's S and softmax ran, so nothing waits here for the tensor cores
                if (pend.use >= 0 && !epilogue_tile(sm, a, &tmO, tO, stg, stream, w, lane, Hg, h, pend)) {
                    ok = false;
                    break;
                }
                pend = PendEpi{use, prow, valid, l, ms};
            }
            if (__any_sync(0xffffffffu, sm.abort_flag != 0)) ok = false;
        }
        if (ok && pend.use >= 0) ok = epilogue_tile(sm, a, &tmO, tO, stg, stream, w, lane, Hg, h, pend);
        bulk_wait0();                               // this warp's stores are complete before exit
        __syncwarp();
        if (!ok) sm.abort_flag = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
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
    static std::atomic<int> n[64];                  // per device, filled on first use
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    int v = n[dev].load(std::memory_order_relaxed);
    if (v == 0 && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
        n[dev].store(v, std::memory_order_relaxed);
    return v > 0 ? v : 148;
}

// Bytes of the workspace's inverted index (header, counts, offsets, item list, entries): the
// part the backward pass shares with the forward; and where its parts start.
size_t inverted_index_bytes(int B, int64_t N, int G, int Hg) { return prefill_layout(B, N, G, Hg, 0).off_lse; }
IndexOffsets inverted_index_offsets(int B, int64_t N, int G, int Hg) {
    const PrefillLayout L = prefill_layout(B, N, G, Hg, 0);
    return IndexOffsets{L.off_nitems, L.off_items, L.off_list};
}

// The inverted index of a selection in `ws` (memset + count + scan + fill): work items
// {b G + g, block j (| kDiagFlag), first entry (or first query), count} in (b, g, range, j)
// order, their number in nitems[0] and a zeroed hand-out counter in nitems[1].
void launch_inverted_index(const int32_t* sel, int64_t N, int64_t P, int B, int G, int Hg, void* ws, cudaStream_t st) {
    const PrefillLayout L = prefill_layout(B, N, G, Hg, P);
    char* base = static_cast<char*>(ws);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(base);
    int* counts = reinterpret_cast<int*>(base + L.off_counts);
    int* offsets = reinterpret_cast<int*>(base + L.off_offsets);
    int* nitems = reinterpret_cast<int*>(base + L.off_nitems);
    int4* items = reinterpret_cast<int4*>(base + L.off_items);
    int* list = reinterpret_cast<int*>(base + L.off_list);
    cudaMemsetAsync(counts, 0, L.nbins * sizeof(int), st);
    {
        dim3 grid(static_cast<unsigned>((N + kCountChunk - 1) / kCountChunk), static_cast<unsigned>(G),
                  static_cast<unsigned>(B));
        const size_t smem = size_t(L.nb) * sizeof(int);
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(csr_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        const KernelTimer kt(KID_CSR, st);
        csr_count_kernel<<<grid, 256, smem, st>>>(sel, N, P, G, L.nb, L.nR, counts, hdr);
    }
    {
        const KernelTimer kt(KID_CSR, st);
        csr_scan_kernel<<<1, 1024, 0, st>>>(counts, offsets, items, nitems, int64_t(L.nbins), L.nb, L.nR, N, P, L.tpt);
    }
    {
        dim3 grid(static_cast<unsigned>((N + kCountChunk - 1) / kCountChunk), static_cast<unsigned>(G),
                  static_cast<unsigned>(B));
        const size_t smem = size_t(L.nb) * sizeof(int);
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(csr_fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        const KernelTimer kt(KID_CSR, st);
        csr_fill_kernel<<<grid, kCountChunk, smem, st>>>(sel, N, P, G, L.nb, L.nR, offsets, counts, list);
    }
}

msa_status_t launch_attn_prefill_tc(const void* q, const CUtensorMap& tmQ2, const CUtensorMap& tmK, const CUtensorMap& tmV, int64_t N,
                            int64_t P, int B, int G, int Hg, const int32_t* sel, void* out, float* lse,
                            void* ws, cudaStream_t st) {
    const PrefillLayout L = prefill_layout(B, N, G, Hg, P);
    char* base = static_cast<char*>(ws);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(base);
    int* nitems = reinterpret_cast<int*>(base + L.off_nitems);
    int4* items = reinterpret_cast<int4*>(base + L.off_items);
    int* list = reinterpret_cast<int*>(base + L.off_list);
    float* part_lse = reinterpret_cast<float*>(base + L.off_lse);
    uint16_t* part_o = reinterpret_cast<uint16_t*>(base + L.off_o);
    launch_inverted_index(sel, N, P, B, G, Hg, ws, st);
    {
        PrefillArgs a;
        a.N = N; a.P = P; a.G = G; a.Hg = Hg; a.Hq = G * Hg; a.tpt = L.tpt;
        a.n_items = nitems; a.items = items; a.list = list; a.part_lse = part_lse; a.part_o = part_o;
        a.q = static_cast<const uint16_t*>(q);
        a.hdr = hdr;
        a.scale_log2 = 1.4426950408889634f / sqrtf(float(kHeadDim));
        const int smem = int(sizeof(KvSmem)) + 1024;
        static std::atomic<bool> attr_set[64];      // per device; setting it twice is harmless
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_relaxed)) {
            cudaFuncSetAttribute(attn_kvmajor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            attr_set[dev].store(true, std::memory_order_relaxed);
        }
        CUtensorMap tmO, tmQ3;
        msa_status_t st_map = make_tmap_bf16(&tmO, part_o, uint64_t(B) * N * G * kSlots * Hg, kHeadDim, 64, uint32_t(Hg));
        if (st_map == MSA_OK && Hg >= 8) st_map = make_tmap_q_rows(&tmQ3, q, uint64_t(B) * N * G * Hg);
        if (st_map != MSA_OK) return st_map;
        const CUtensorMap& tmQ = Hg >= 8 ? tmQ3 : tmQ2;
        const KernelTimer kt(KID_ATTN_PREFILL, st);
        attn_kvmajor_kernel<<<num_sms(), kKvThreads, smem, st>>>(tmQ, tmK, tmV, tmO, a);
    }
    {
        const int64_t total = int64_t(B) * N * G * Hg * 4;
        const KernelTimer kt(KID_COMBINE, st);
        combine_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(sel, part_lse, part_o, N, G, Hg,
                                                                                  static_cast<uint16_t*>(out), lse,
                                                                                  total);
    }
    return MSA_OK;
}
}  // namespace msa

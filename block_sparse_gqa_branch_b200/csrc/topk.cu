// topk.cu -- exp-free top-k of every row of a score matrix: the Index Branch's selection on
// its own, for scores computed elsewhere.
//
// Sources: KuCoin flash "MiniMax launches MSA sparse attention method and MiniMax-M3 model",
// "ME AI News" paragraph (the index branch's top-k is exp-free and is compared with
// torch.topk at 128K context); youmind article "MiniMax M3 sparse attention agents", bullet
// "Fast in production" (the custom top-k measured against torch.topk).
//
// One warp per row. A score becomes an orderable 32-bit code (every NaN above +inf, -0 equal
// to +0, otherwise by value) and a candidate's key is (code, inverted column): keys are
// unique, and a larger key means a higher score or, at equal scores, a lower column. A row is
// read in chunks of 32 lanes x 32 values (eight 16-byte loads per lane in flight). In a chunk
// each lane takes the largest code of its values; the k-th largest of those 32 lane maxima
// belongs to k distinct values of the chunk, so it bounds from below the code of every chunk
// value that can be among the row's k best, and so does the code of the running k-th best.
// Only values at or above both bounds enter the exact merge: rounds of one value per lane,
// sorted across the warp (bitonic) and merged into the running best 16. On random scores
// about 20 of a chunk's 1,024 values pass, so a chunk costs its loads, a few integer
// instructions per value and two or three rounds. No exponential and no float arithmetic
// is used: only integer compares of the codes.
#include <type_traits>

#include "msa_common.cuh"

namespace msa {

int num_sms();

constexpr int kTopkThreads = 256;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkSteps = 8;                 // loads per lane and chunk
constexpr int kTopkMax = 16;                  // largest k
constexpr int64_t kTopkMaxCols = int64_t(1) << 30;

// orderable code of a score: every NaN above +inf, -0 equal to +0, otherwise by value
__device__ __forceinline__ uint32_t score_code(float x) {
    uint32_t u = __float_as_uint(x);
    const uint32_t a = u & 0x7fffffffu;
    u = (a > 0x7f800000u) ? 0x7fffffffu : (a == 0u ? 0u : u);
    return u ^ (uint32_t(int32_t(u) >> 31) | 0x80000000u);
}

// Bitonic sort of one 32-bit code per lane, descending across the warp's lanes.
__device__ __forceinline__ uint32_t warp_sort_desc32(uint32_t x, int lane) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
            x = (((lane & j) == 0) == ((lane & k) == 0)) ? max(x, y) : min(x, y);
        }
    }
    return x;
}

// the float at the bottom of the values whose code is >= c (c a code of a non-NaN value, or 0)
__device__ __forceinline__ float code_floor(uint32_t c) {
    if (c == 0u) return -INFINITY;                                   // below every real code
    return __uint_as_float((c & 0x80000000u) ? (c ^ 0x80000000u) : ~c);
}

constexpr int kStash = 36;                    // floats per lane in the staging rows (16-byte aligned, few conflicts)
constexpr int kList = 128;                    // passing values one chunk may hand to the merge rounds

// One round per value a lane still holds: the exact merge of the values in `pass` (codes in
// code[]) into the running best 16. Used for chunks the fast path does not take.
template <int VEC, int kPer>
__device__ __forceinline__ void merge_lanes(unsigned long long& best, uint32_t pass, const uint32_t (&code)[kPer],
                                            int base, int lane) {
    while (__any_sync(0xffffffffu, pass != 0u)) {
        unsigned long long key = 0ull;                  // below every real key
        if (pass != 0u) {
            const int p = __ffs(int(pass)) - 1;
            pass &= pass - 1u;
            uint32_t cp = 0u;
#pragma unroll
            for (int q = 0; q < kPer; ++q) cp = (q == p) ? code[q] : cp;
            const int col = base + ((p / VEC) * 32 + lane) * VEC + (p % VEC);
            key = (static_cast<unsigned long long>(cp) << 32) | uint32_t(~col);
        }
        key = warp_sort_desc(key, lane);
        const unsigned long long top16 = __shfl_sync(0xffffffffu, key, 31 - lane);   // lanes 16-31: ascending
        best = warp_merge_desc(lane < 16 ? best : top16, lane);
    }
}

// VEC = 4: rows start 16-byte aligned (n % 4 == 0) and are read as float4; VEC = 1 otherwise.
// Fast path of a chunk (no NaN in it, at most kList values passing): the lane maxima and the
// pass test are float compares against the bound's floor value (the same set as the codes'
// test: the code order is the float order once NaN is out, with -0 equal to +0); the passing
// values are compacted into the warp's list in shared memory, so that one 32-wide round of
// sort and merge takes 32 of them whatever lanes they came from.
template <int VEC>
__global__ void __launch_bounds__(kTopkThreads, 3) topk_rows_kernel(const float* __restrict__ scores, int64_t rows,
                                                                  int n, int k, int32_t* __restrict__ idx,
                                                                  float* __restrict__ val) {
    constexpr int kPer = kTopkSteps * VEC;    // values per lane and chunk
    constexpr int kChunk = 32 * kPer;
    __shared__ __align__(16) float stash[kTopkWarps][32 * kStash];
    __shared__ unsigned long long list[kTopkWarps][kList];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    float* my = &stash[wid][lane * kStash];
    unsigned long long* wl = list[wid];
    const int64_t nwarps = int64_t(gridDim.x) * kTopkWarps;
    for (int64_t row = int64_t(blockIdx.x) * kTopkWarps + wid; row < rows; row += nwarps) {
        const float* r = scores + row * n;
        unsigned long long best = 0ull;       // lanes 0-15: the best 16 keys so far, descending
        uint32_t floor_code = 0u;             // code of the running k-th best
        // one chunk; kFull: every column of the chunk is < n (no per-value validity tests)
        auto chunk = [&](int base, auto full_tag) {
            constexpr bool kFull = decltype(full_tag)::value;
            float v[kPer];
            uint32_t valid = kFull ? 0xffffffffu : 0u;   // bit p: this lane's value p is a column < n
#pragma unroll
            for (int i = 0; i < kTopkSteps; ++i) {
                const int c0 = base + (i * 32 + lane) * VEC;
                if constexpr (VEC == 4) {
                    float4 x = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
                    if (kFull || c0 < n) {
                        x = __ldcs(reinterpret_cast<const float4*>(r + c0));
                        if (!kFull) valid |= 0xfu << (4 * i);
                    }
                    v[4 * i + 0] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
                } else {
                    float x = -INFINITY;
                    if (kFull || c0 < n) {
                        x = __ldcs(r + c0);
                        if (!kFull) valid |= 1u << i;
                    }
                    v[i] = x;
                }
            }
            // lane maximum (a NaN is caught by the sums: it or inf - inf sends the chunk down the
            // exact path)
            float lm = -INFINITY, s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int p = 0; p + 1 < kPer; p += 2) lm = fmax3(lm, v[p], v[p + 1]);   // invalid values are -inf
            if constexpr (kPer % 2 == 1) lm = fmaxf(lm, v[kPer - 1]);
#pragma unroll
            for (int p = 0; p < kPer; ++p) {
                const float x = (kFull || ((valid >> p) & 1u)) ? v[p] : 0.f;
                if (p & 1) s1 += x;
                else s0 += x;
            }
            const bool nan_here = (s0 + s1) != (s0 + s1);
            const uint32_t lcode = (kFull || valid != 0u) ? score_code(lm) : 0u;
            const uint32_t kth_lane_max = __shfl_sync(0xffffffffu, warp_sort_desc32(lcode, lane), k - 1);
            const uint32_t bound = max(kth_lane_max, floor_code);
            const float bf = code_floor(bound);
            uint32_t pass = 0u;
#pragma unroll
            for (int p = 0; p < kPer; ++p)
                pass |= ((kFull || ((valid >> p) & 1u) != 0u) && v[p] >= bf) ? (1u << p) : 0u;
            const int cnt = __popc(pass);
            int incl = cnt;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += y;
            }
            const int total = __shfl_sync(0xffffffffu, incl, 31);
            if (__any_sync(0xffffffffu, nan_here) || total > kList) {
                // exact path: codes of every value, one round per value a lane holds
                uint32_t code[kPer];
                uint32_t pass_c = 0u;
#pragma unroll
                for (int p = 0; p < kPer; ++p) {
                    code[p] = ((valid >> p) & 1u) ? score_code(v[p]) : 0u;     // 0: below every real code
                    pass_c |= (((valid >> p) & 1u) != 0u && code[p] >= bound) ? (1u << p) : 0u;
                }
                merge_lanes<VEC, kPer>(best, pass_c, code, base, lane);
            } else if (total > 0) {
                if constexpr (VEC == 4) {
#pragma unroll
                    for (int i = 0; i < kTopkSteps; ++i)
                        *reinterpret_cast<float4*>(my + 4 * i) = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                } else {
#pragma unroll
                    for (int i = 0; i < kPer; ++i) my[i] = v[i];
                }
                __syncwarp();
                int o = incl - cnt;                      // this lane's first list slot; o + cnt <= total <= kList
                while (pass != 0u) {
                    const int p = __ffs(int(pass)) - 1;
                    pass &= pass - 1u;
                    const int col = base + ((p / VEC) * 32 + lane) * VEC + (p % VEC);
                    wl[o++] = (static_cast<unsigned long long>(score_code(my[p])) << 32) | uint32_t(~col);
                }
                __syncwarp();
                for (int r0 = 0; r0 < total; r0 += 32) {
                    unsigned long long key = r0 + lane < total ? wl[r0 + lane] : 0ull;
                    key = warp_sort_desc(key, lane);
                    const unsigned long long top16 = __shfl_sync(0xffffffffu, key, 31 - lane);
                    best = warp_merge_desc(lane < 16 ? best : top16, lane);
                }
                __syncwarp();                            // the list and the staging rows are free again
            }
        };
        for (int base = 0; base < n; base += kChunk) {
            if (base + kChunk <= n) chunk(base, std::true_type{});
            else chunk(base, std::false_type{});
            floor_code = uint32_t(__shfl_sync(0xffffffffu, best, k - 1) >> 32);
        }
        if (lane < k) {                       // n >= k: the first chunk alone passes k values
            const int col = int(~uint32_t(best));
            const bool ok = best != 0ull && col < n;
            idx[row * k + lane] = ok ? col : -1;
            if (val != nullptr) val[row * k + lane] = ok ? r[col] : __int_as_float(0x7fffffff);
        }
    }
}

}  // namespace msa

extern "C" msa_status_t msa_topk_rows(const float* scores, int64_t rows, int64_t n, int32_t k, int32_t* idx,
                                      float* val, msa_stream_t stream) {
    MSA_CALL_RANGE();
    using namespace msa;
    if (rows < 0 || k < 1 || k > kTopkMax || n < k || n > kTopkMaxCols) return MSA_ERR_INVALID_ARGUMENT;
    if (rows == 0) return MSA_OK;
    if (scores == nullptr || idx == nullptr || !aligned16(scores) || !aligned16(idx)) return MSA_ERR_INVALID_ARGUMENT;
    if (val != nullptr && !aligned16(val)) return MSA_ERR_INVALID_ARGUMENT;
    const int64_t want = (rows + kTopkWarps - 1) / kTopkWarps;
    const int blocks = int(want < int64_t(num_sms()) * 16 ? want : int64_t(num_sms()) * 16);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const KernelTimer kt(KID_TOPK, st);
    if (n % 4 == 0)
        topk_rows_kernel<4><<<blocks, kTopkThreads, 0, st>>>(scores, rows, int(n), k, idx, val);
    else
        topk_rows_kernel<1><<<blocks, kTopkThreads, 0, st>>>(scores, rows, int(n), k, idx, val);
    return cuda_status();
}

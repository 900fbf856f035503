// msa_common.cuh -- shared device helpers of libmsa (sm_100a): constants, the workspace
// error word, bf16 conversion, the exp-free selection key, and thin inline-PTX wrappers for
// mbarriers, TMA copies, warp-level MMA and the tcgen05 tensor-memory instructions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include "msa.h"

namespace msa {

// One NVTX range per C-ABI call, named for the entry point: a profiler attached to the process
// shows each call's kernels under it; without one, push and pop return at once.
struct CallRange {
    explicit CallRange(const char* name) { nvtxRangePushA(name); }
    ~CallRange() { nvtxRangePop(); }
    CallRange(const CallRange&) = delete;
    CallRange& operator=(const CallRange&) = delete;
};
#define MSA_CALL_RANGE() ::msa::CallRange msa_call_range_(__func__)

// host-side count of kernels enqueued by libmsa (see msa_kernel_launches)
void count_launch(unsigned n = 1);

// host-side argument checks shared by the entry points
extern thread_local int g_last_cuda_error;
bool aligned16(const void* p);
msa_status_t check_shape(const msa_shape_t* s);   // constants and head layout
msa_status_t cuda_status();                       // MSA_ERR_CUDA if the last launch failed
// 2-D bf16 TMA descriptor (rows x cols, row stride = cols), box box_cols x box_rows, 128B swizzle
msa_status_t make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                            uint32_t box_rows);
// 2-D uint8 TMA descriptor (rows x cols bytes, row stride = cols), box box_cols x box_rows, 128B swizzle
msa_status_t make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                          uint32_t box_rows);
// Key / value cache rows as a 3-D bf16 tensor {128 columns, rows_valid rows, nbg} with row stride
// 256 B and (sequence, group) stride l_cap rows; box {64, 128, 1}, 128B swizzle; rows at or past
// rows_valid are zero-filled by the copy.
msa_status_t make_tmap_kv3d(CUtensorMap* m, const void* base, uint64_t rows_valid, uint64_t l_cap, uint64_t nbg);
// Index queries q_idx [rows, G, 64] bf16 as a 3-D tensor {64, G, rows}; box {64, 1, 128}: 128
// rows of one group, [128 rows][128 B] with the 128B swizzle
msa_status_t make_tmap_qidx(CUtensorMap* m, const void* base, int G, uint64_t rows);
// Rows of 128 bf16 viewed as (64 columns, row, d half): box {64, 8, 2} lands 8 rows with both
// halves as [half][8 rows][128 B] (128B swizzle)
msa_status_t make_tmap_q_rows(CUtensorMap* m, const void* base, uint64_t rows);
// Split pooled keys [nbg3][nbp][64] bf16 as a 3-D tensor {64, nbp, nbg3}; box {64, 32, 3}: 32
// candidates of the three terms of one (sequence, group) as [term][32 rows][128 B] (128B swizzle)
msa_status_t make_tmap_split(CUtensorMap* m, const void* base, uint64_t nbp, uint64_t nbg3);

// byte offsets, inside a prefill workspace, of the inverted index's item count, items and entries
struct IndexOffsets { size_t nitems, items, list; };

// largest query position the decode path supports (bounds its workspaces and row indices)
constexpr int64_t kMaxDecodePos = (int64_t(1) << 24) - 1;

constexpr int kHeadDim = 128;   // d
constexpr int kIndexDim = 64;   // d_I
constexpr int kBlock = 128;     // Bk
constexpr int kTopK = 16;       // k
constexpr int kMaxHg = 16;      // query heads per group supported

// ---------------------------------------------------------------- workspace header
// Every workspace starts with this 256-byte header. err is the first device-detected
// status (0 = none); info holds (kernel id, block, index, value) of that event.
struct WsHeader {
    unsigned int err;
    int info[4];
    unsigned int pad[59];
};
static_assert(sizeof(WsHeader) == 256, "workspace header must be 256 bytes");

// kernel ids: the MSA_KERNEL_* values of msa.h (workspace error info[0], timing records)
enum KernelId : int {
    KID_POOL = MSA_KERNEL_POOL, KID_SELECT_PREFILL = MSA_KERNEL_SELECT_PREFILL,
    KID_SELECT_DECODE = MSA_KERNEL_SELECT_DECODE, KID_APPEND = MSA_KERNEL_APPEND,
    KID_ATTN_DECODE = MSA_KERNEL_ATTN_DECODE, KID_ATTN_PREFILL = MSA_KERNEL_ATTN_PREFILL,
    KID_CSR = MSA_KERNEL_INVERTED_INDEX, KID_COMBINE = MSA_KERNEL_COMBINE, KID_SELFTEST = MSA_KERNEL_SELFTEST,
    KID_FP8 = MSA_KERNEL_FP8, KID_SPLIT = MSA_KERNEL_SPLIT_KEYS, KID_ATTN_BACKWARD = MSA_KERNEL_ATTN_BACKWARD,
    KID_BWD_DOT = MSA_KERNEL_BACKWARD_DOT, KID_TOPK = MSA_KERNEL_TOPK
};

// Counts a launch (msa_kernel_launches) and, while kernel timing is on and the stream is not
// being captured, brackets it with two events on the stream (msa_kernel_timing_read). Declared
// in the scope that ends right after the launch.
class KernelTimer {
  public:
    KernelTimer(int kid, cudaStream_t st);
    ~KernelTimer();
    KernelTimer(const KernelTimer&) = delete;
    KernelTimer& operator=(const KernelTimer&) = delete;

  private:
    int kid_;
    cudaStream_t st_;
    cudaEvent_t a_ = nullptr, b_ = nullptr;
};

__device__ __forceinline__ void record_error(WsHeader* h, unsigned code, int kid, int blk,
                                             int idx, int val) {
    if (h == nullptr) return;
    if (atomicCAS(&h->err, 0u, code) == 0u) {
        h->info[0] = kid; h->info[1] = blk; h->info[2] = idx; h->info[3] = val;
        __threadfence();
    }
}

// max of three floats in one instruction (sm_100; used on finite scores)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// ---------------------------------------------------------------- bf16
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

// two floats -> packed bf16x2 (round to nearest even), lo in the low half
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------- selection key
// Exp-free ordering key of a block: larger key = better block. The high word maps the fp32
// score monotonically to an unsigned integer (after folding -0 into +0); the low word is the
// bitwise complement of the block id, so equal scores rank the lower id first.
__device__ __forceinline__ unsigned long long sel_key(float s, int j) {
    s = s + 0.0f;                                    // -0 -> +0
    uint32_t u = __float_as_uint(s);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (static_cast<unsigned long long>(u) << 32) | static_cast<uint32_t>(~j);
}
__device__ __forceinline__ int key_block(unsigned long long k) { return int(~uint32_t(k)); }

__device__ __forceinline__ unsigned long long umax64(unsigned long long x, unsigned long long y) { return x > y ? x : y; }
__device__ __forceinline__ unsigned long long umin64(unsigned long long x, unsigned long long y) { return x < y ? x : y; }

// Bitonic sort of one key per lane, descending across the warp's lanes.
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long x, int lane) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, j);
            x = (((lane & j) == 0) == ((lane & k) == 0)) ? umax64(x, y) : umin64(x, y);
        }
    }
    return x;
}

// Lanes 0-15 hold a descending list, lanes 16-31 another one in ascending order (a bitonic
// sequence): after the half-cleaners lanes 0-15 hold the 16 largest keys, descending.
__device__ __forceinline__ unsigned long long warp_merge_desc(unsigned long long x, int lane) {
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, j);
        x = ((lane & j) == 0) ? umax64(x, y) : umin64(x, y);
    }
    return x;
}

// ---------------------------------------------------------------- loads kept in flight
// Runs of global loads issued by ONE inline-asm statement: the whole run goes out back to back
// before any value is used (left to itself the compiler may interleave each load with its use
// to save registers, paying one memory round trip per load).
__device__ __forceinline__ float4 ld_nc_f4(const float4* p) {
    float4 v;
    asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
    return v;
}
// 8 float4 at p, p + 32, ..., p + 224 (a stride of 512 bytes)
__device__ __forceinline__ void ld_nc_f4x8_s512(const float4* p, float4 (&v)[8]) {
    asm volatile(
        "ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%32];\n\t"
        "ld.global.nc.v4.f32 {%4, %5, %6, %7}, [%32+512];\n\t"
        "ld.global.nc.v4.f32 {%8, %9, %10, %11}, [%32+1024];\n\t"
        "ld.global.nc.v4.f32 {%12, %13, %14, %15}, [%32+1536];\n\t"
        "ld.global.nc.v4.f32 {%16, %17, %18, %19}, [%32+2048];\n\t"
        "ld.global.nc.v4.f32 {%20, %21, %22, %23}, [%32+2560];\n\t"
        "ld.global.nc.v4.f32 {%24, %25, %26, %27}, [%32+3072];\n\t"
        "ld.global.nc.v4.f32 {%28, %29, %30, %31}, [%32+3584];"
        : "=f"(v[0].x), "=f"(v[0].y), "=f"(v[0].z), "=f"(v[0].w), "=f"(v[1].x), "=f"(v[1].y), "=f"(v[1].z), "=f"(v[1].w),
          "=f"(v[2].x), "=f"(v[2].y), "=f"(v[2].z), "=f"(v[2].w), "=f"(v[3].x), "=f"(v[3].y), "=f"(v[3].z), "=f"(v[3].w),
          "=f"(v[4].x), "=f"(v[4].y), "=f"(v[4].z), "=f"(v[4].w), "=f"(v[5].x), "=f"(v[5].y), "=f"(v[5].z), "=f"(v[5].w),
          "=f"(v[6].x), "=f"(v[6].y), "=f"(v[6].z), "=f"(v[6].w), "=f"(v[7].x), "=f"(v[7].y), "=f"(v[7].z), "=f"(v[7].w)
        : "l"(p));
}
// 16 float2 at p, p + 4, p + 8, ... (a stride of 32 bytes), from L2
__device__ __forceinline__ void ld_cg_f2x16_s32(const float* p, float2 (&v)[16]) {
    asm volatile(
        "ld.global.cg.v2.f32 {%0, %1}, [%32];\n\t"
        "ld.global.cg.v2.f32 {%2, %3}, [%32+32];\n\t"
        "ld.global.cg.v2.f32 {%4, %5}, [%32+64];\n\t"
        "ld.global.cg.v2.f32 {%6, %7}, [%32+96];\n\t"
        "ld.global.cg.v2.f32 {%8, %9}, [%32+128];\n\t"
        "ld.global.cg.v2.f32 {%10, %11}, [%32+160];\n\t"
        "ld.global.cg.v2.f32 {%12, %13}, [%32+192];\n\t"
        "ld.global.cg.v2.f32 {%14, %15}, [%32+224];\n\t"
        "ld.global.cg.v2.f32 {%16, %17}, [%32+256];\n\t"
        "ld.global.cg.v2.f32 {%18, %19}, [%32+288];\n\t"
        "ld.global.cg.v2.f32 {%20, %21}, [%32+320];\n\t"
        "ld.global.cg.v2.f32 {%22, %23}, [%32+352];\n\t"
        "ld.global.cg.v2.f32 {%24, %25}, [%32+384];\n\t"
        "ld.global.cg.v2.f32 {%26, %27}, [%32+416];\n\t"
        "ld.global.cg.v2.f32 {%28, %29}, [%32+448];\n\t"
        "ld.global.cg.v2.f32 {%30, %31}, [%32+480];"
        : "=f"(v[0].x), "=f"(v[0].y), "=f"(v[1].x), "=f"(v[1].y), "=f"(v[2].x), "=f"(v[2].y), "=f"(v[3].x), "=f"(v[3].y),
          "=f"(v[4].x), "=f"(v[4].y), "=f"(v[5].x), "=f"(v[5].y), "=f"(v[6].x), "=f"(v[6].y), "=f"(v[7].x), "=f"(v[7].y),
          "=f"(v[8].x), "=f"(v[8].y), "=f"(v[9].x), "=f"(v[9].y), "=f"(v[10].x), "=f"(v[10].y), "=f"(v[11].x),
          "=f"(v[11].y), "=f"(v[12].x), "=f"(v[12].y), "=f"(v[13].x), "=f"(v[13].y), "=f"(v[14].x), "=f"(v[14].y),
          "=f"(v[15].x), "=f"(v[15].y)
        : "l"(p));
}
__device__ __forceinline__ float2 ld_cg_f2pair(const float* p0, const float* p1) {
    float2 v;
    asm volatile("ld.global.cg.f32 %0, [%2];\n\tld.global.cg.f32 %1, [%3];" : "=f"(v.x), "=f"(v.y) : "l"(p0), "l"(p1));
    return v;
}

// ---------------------------------------------------------------- bounded waits
// A wait gives up after about 2 s of SM clocks (records MSA_ERR_TIMEOUT); callers then
// skip the rest of their work and still release what they hold.
constexpr long long kWaitCycles = 4000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
// Returns false on timeout (and records it).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, WsHeader* hdr, int kid) {
    if (mbar_try_wait(bar, parity)) return true;
    long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitCycles) {
            record_error(hdr, MSA_ERR_TIMEOUT, kid, blockIdx.x, threadIdx.x, int(parity));
            return false;
        }
    }
    return true;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// 3-D tiled load (coordinates x, y, z), completes on `bar`.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* m, int x, int y, int z,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z),
          "r"(smem_u32(bar)) : "memory");
}
// L2 eviction-priority policies for the cache-hinted copies below
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tma_load_2d_hint(void* smem_dst, const CUtensorMap* m, int x, int y, uint64_t* bar,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar)),
          "l"(policy) : "memory");
}
__device__ __forceinline__ void tma_load_3d_hint(void* smem_dst, const CUtensorMap* m, int x, int y, int z,
                                                 uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z),
          "r"(smem_u32(bar)), "l"(policy) : "memory");
}
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* m, int x, int y, const void* smem_src,
                                                  uint64_t policy) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%1, %2}], [%3], %4;"
                 ::"l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(smem_src)), "l"(policy)
                 : "memory");
}
// untiled bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16)
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a 128B-swizzled tile whose
// rows are 128 bytes (the layout TMA writes with CU_TENSOR_MAP_SWIZZLE_128B)
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// ---------------------------------------------------------------- warp MMA (m16n8k16 bf16)
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Programmatic dependent launch: wait for the preceding kernel's completion (a no-op when the
// kernel was launched without the attribute), and let the next kernel start launching.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ldmatrix x4 with transpose (four 8x8 b16 matrices; lane i addresses row i % 8 of matrix i / 8)
__device__ __forceinline__ void ldsm_x4_trans(uint32_t saddr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(saddr));
}

// Two e4m3 codes (lo in the low byte) -> two f16 values, exactly (every e4m3 value is a normal
// f16 value or zero), by the hardware conversion.
__device__ __forceinline__ uint32_t f16x2_from_e4m3x2(uint16_t codes) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(codes));
    return h;
}
// two floats -> packed f16x2 (round to nearest even), lo in the low half
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t h;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(hi), "f"(lo));
    return h;
}
// packed bf16x2 -> packed f16x2 (exact for values in the normal f16 range)
__device__ __forceinline__ uint32_t f16x2_from_bf16x2(uint32_t w) {
    return pack_f16x2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// warp MMA m16n8k16 with f16 operands and fp32 accumulators
__device__ __forceinline__ void mma_f16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace msa

// ---------------------------------------------------------------- tcgen05 (5th-gen tensor cores)
namespace msa {

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(smem_dst)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// mbarrier arrives once all tcgen05 operations issued so far by this thread have completed
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T  (kind::f16: bf16 inputs, fp32 accumulator)
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm100 format: start >> 4 in [0,14),
// leading byte offset >> 4 in [16,30), stride byte offset >> 4 in [32,46), version 1 at 46,
// layout type SWIZZLE_128B = 2 in [61,64)).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = uint64_t((saddr >> 4) & 0x3FFFu);
    d |= uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1) << 46;
    d |= uint64_t(2) << 61;
    return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and an fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn_major) << 15) | (uint32_t(b_mn_major) << 16) |
           (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// tcgen05.ld 32x32b.x32: thread i of the warp receives 32 consecutive 32-bit columns of TMEM
// lane (32 * (warp % 4) + i), starting at column taddr's column.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// tcgen05.st 32x32b.x16: thread i writes 16 consecutive 32-bit columns of its lane
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

}  // namespace msa

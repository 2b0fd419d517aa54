// Pieces shared by the grouped-FFN kernels (one CTA per tile job in
// ffn_tc.cu, CTA pairs sharing each MMA in ffn_pair.cu): the shared-memory
// budget, the job kinds, bounded waits on barriers, sentinels and counters,
// the element-wise helpers of the epilogue and the tensor-map builder.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {
namespace ffn {

constexpr int kThreads = 352;   // warps: 0 TMA, 1 MMA, 2-9 epilogue (two sets of four), 10 scheduler
constexpr int kEpiThreads = 256;
constexpr int kSchedWarp = 10;
constexpr int kUQ = 8;          // unit-queue depth
constexpr int kSlab = 128;      // K bytes per slab (one 128-byte swizzle row)
constexpr int kABytes = 128 * kSlab;   // 128 weight rows of one slab
constexpr int kMaxDynSmem = 232448;    // 227 KB per CTA
constexpr int kCtlBytes = 2048;        // barriers, job queue, flags, reductions
constexpr int kTileTabBytes = 4 * 1025 + 252;   // per-expert chunk table (E <= 1024)

enum : int { kKindGateUp = 0, kKindDown = 1, kKindEnd = 2, kKindAbort = 3 };
// weight formats: bf16 (kind::f16), e4m3 with fp32 128 x 128 block scales, and
// MX FP4 (e2m1, a UE8M0 scale per 32 along K) against e4m3 tokens, both
// kind::mxf8f6f4.block_scale
enum : int { kWBf16 = 0, kWE4m3 = 1, kWE2m1 = 2 };
// counter-set misc slots used by the FFN: calls completed on this dispatch,
// CTAs that left the current call, the next unit to hand out
enum : int { kFfnGen = 3, kFfnExit = 4, kFfnNext = 5 };

__device__ __forceinline__ int4 shfl_int4(int4 v) {
  v.x = __shfl_sync(0xffffffffu, v.x, 0);
  v.y = __shfl_sync(0xffffffffu, v.y, 0);
  v.z = __shfl_sync(0xffffffffu, v.z, 0);
  v.w = __shfl_sync(0xffffffffu, v.w, 0);
  return v;
}

// Bounded wait on an mbarrier phase; false on timeout (latched) or abort.
// kCl: the phase includes arrivals from the other CTA of a pair, whose writes
// the waiter then sees (acquire at cluster scope).
template <bool kCl = false>
__device__ __forceinline__ bool try_bar(uint64_t* bar, uint32_t parity) {
  if constexpr (kCl) return ptx::mbar_try_wait_cluster(bar, parity);
  else return ptx::mbar_try_wait(bar, parity);
}

template <bool kCl = false>
__device__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, Header* hdr,
                         uint32_t where) {
  if (try_bar<kCl>(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (try_bar<kCl>(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitBudgetNs) {
      latch_error(hdr, MOE_ERR_TIMEOUT, where);
      *abort_flag = 1;
      return false;
    }
  }
}

// Rows of global tile g once its sentinel carries this epoch.
static __device__ bool wait_tile(const Ws& ws, uint32_t epoch, int g, volatile int* abort_flag, int* rows) {
  const unsigned long long t0 = globaltimer();
  const uint32_t* sp = ws.sentinel + g;
  while (true) {
    const uint32_t s = ld_acquire(sp);
    if ((s >> 8) == (epoch & 0xFFFFFFu)) {
      *rows = (int)(s & 0xFF);
      if (*rows < 1 || *rows > kTileRows) {   // never published: a corrupt workspace
        latch_error(ws.hdr, MOE_ERR_INVALID_ARG, 0x22000000u | (uint32_t)g);
        *abort_flag = 1;
        return false;
      }
      return true;
    }
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitBudgetNs) {
      latch_error(ws.hdr, MOE_ERR_TIMEOUT, 0x23000000u | (uint32_t)g);
      *abort_flag = 1;
      return false;
    }
    __nanosleep(128);
  }
}

// Wait until `count` reaches `target` (acquire), bounded.
static __device__ bool wait_count(const uint32_t* count, uint32_t target, volatile int* abort_flag, Header* hdr,
                           uint32_t where) {
  const unsigned long long t0 = globaltimer();
  while (ld_acquire(count) < target) {
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitBudgetNs) {
      latch_error(hdr, MOE_ERR_TIMEOUT, where);
      *abort_flag = 1;
      return false;
    }
    __nanosleep(128);
  }
  return true;
}

__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.f + expf(-g)); }

// UE8M0 code of a power-of-two fp32 scale: its biased exponent.
__device__ __forceinline__ uint32_t ue8m0(float s) { return (__float_as_uint(s) >> 23) & 0xFFu; }

// A weight block scale the block-scaled MMA applies exactly: a positive,
// finite, normal power of two (sign and mantissa bits zero, exponent neither
// 0 nor 255). Any other value would lose its mantissa in ue8m0().
__device__ __forceinline__ bool pow2_scale_ok(float s) {
  const uint32_t b = __float_as_uint(s);
  const uint32_t e = (b >> 23) & 0xFFu;
  return (b & 0x807FFFFFu) == 0u && e != 0u && e != 0xFFu;
}

// ---- host side ----

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Element kinds of a tensor map: bf16, bytes (e4m3), and packed 4-bit codes
// that land 16 codes per 16 bytes in shared memory (8 bytes of codes, 8 of
// gap), the layout the block-scaled MMA reads 4-bit operands from.
enum TmapElem { kElBf16, kElU8, kElU4Spread };

// 2-D row-major [rows, cols] tensor (cols in elements), boxes of
// (box_cols x box_rows), 128-byte swizzle.
inline bool make_tmap(CUtensorMap* m, const void* base, TmapElem el, int64_t cols, int64_t rows, int box_cols,
               int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int64_t row_bytes = el == kElBf16 ? cols * 2 : (el == kElU8 ? cols : cols / 2);
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = el == kElBf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : (el == kElU8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B);
  CUresult r = fn(m, dt, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace ffn
}  // namespace moe

// Top-k weighted combine with the expert rows staged through shared memory
// by bulk copies (the TMA engine), for layers with many tokens.
//
// Pages: outputs are gathered directly from the expert windows, with no
// output-restoration buffer (Ascend report, abstract); combine is the third
// per-layer stage after dispatch and the grouped GEMM (GC-MoE feed item,
// "Key points").
//
//   out[t] = sum_{j < k} w[t, j] * y[pos[t*k + j]]    (fp32, slot order)
//
// rounded once to the output dtype; the same arithmetic, in the same order,
// as the register-gather kernel in combine.cu. A unit is (token, part of the
// row): one loader warp bulk-copies the unit's k row chunks (and, for e4m3
// identity rows, their scales) into a ring of shared-memory stages, so that
// two to three units' rows (~115-170 KB) are in flight per SM without
// holding them in registers; 16 compute warps (8 for fp32 rows) read the
// stage, form the weighted sums over the live slots (compacted by the
// loader) 8 or 16 values per thread and write the output coalesced. A
// persistent grid of one CTA per SM walks the units. Every wait is bounded:
// on expiry the kernel latches MOE_ERR_TIMEOUT, waits (bounded) for its
// copies and returns.
#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

// values per compute thread: one 16-byte shared-memory read per row (8 bf16,
// 16 e4m3; fp32 rows take four reads of 16 values), so that a warp's reads
// of a row are consecutive and free of bank conflicts
template <int kRowDt>
__host__ __device__ constexpr int vals_of() { return kRowDt == MOE_BF16 ? 8 : 16; }
// compute warps: 16, so that a unit's groups (V / vals_of) keep 14-16 warps
// busy; fp32 rows keep 8
template <int kRowDt>
__host__ __device__ constexpr int comp_warps() { return kRowDt == MOE_F32 ? 8 : 16; }
template <int kRowDt>
__host__ __device__ constexpr int threads_of() { return (comp_warps<kRowDt>() + 1) * 32; }   // + one loader warp
constexpr int kStages = 3;
constexpr int kRowCap = 64 * 1024;                // row-chunk bytes of one stage
constexpr int kMaxSlots = 32;
// a stage's slot list: the live slots (row copied, weight non-zero) in slot
// order, compacted by the loader: slot[32] | w[32] | row[32] | count
constexpr int kMetaBytes = 3 * kMaxSlots * 4 + 16;

struct Args {
  const int32_t* pos;
  const float* w;
  const uint8_t* rows;    // y rows, or xq rows for identity experts
  const float* xs;        // e4m3 identity rows: scales (else null)
  void* out;
  Header* hdr;
  int T, H, k;
  int elt;                // bytes per row element: 4, 2 or 1
  int nparts, V;          // parts per row, elements per part
  int scale_bulk;         // e4m3: the part's scales travel with the rows
  int off_scale, off_meta, stage_bytes;
};

template <int kRowDt>
__device__ __forceinline__ void fma_vals(const uint8_t* src, float s, float wj, float* acc) {
  if constexpr (kRowDt == MOE_BF16) {
    const uint4 r = *reinterpret_cast<const uint4*>(src);
    const uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(wj, __uint_as_float(u[i] << 16), acc[2 * i]);
      acc[2 * i + 1] = fmaf(wj, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
    }
  } else if constexpr (kRowDt == MOE_F32) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 r = reinterpret_cast<const uint4*>(src)[v];
      acc[4 * v] = fmaf(wj, __uint_as_float(r.x), acc[4 * v]);
      acc[4 * v + 1] = fmaf(wj, __uint_as_float(r.y), acc[4 * v + 1]);
      acc[4 * v + 2] = fmaf(wj, __uint_as_float(r.z), acc[4 * v + 2]);
      acc[4 * v + 3] = fmaf(wj, __uint_as_float(r.w), acc[4 * v + 3]);
    }
  } else {
    const uint4 r = *reinterpret_cast<const uint4*>(src);
    const uint32_t u[4] = {r.x, r.y, r.z, r.w};
    const float ws = wj * s;   // w_j * scale: exact scaling by a power of two
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(u[i / 2] >> (16 * (i % 2))), __NV_E4M3);
      const float2 f2 = __half22float2(__half2(h2));
      acc[2 * i] = fmaf(ws, f2.x, acc[2 * i]);
      acc[2 * i + 1] = fmaf(ws, f2.y, acc[2 * i + 1]);
    }
  }
}

// Bounded wait on an mbarrier phase by one lane; false on timeout (latched)
// or when another role gave up.
__device__ bool wait_phase(uint64_t* bar, uint32_t parity, volatile int* abort_flag, Header* hdr,
                           uint32_t where) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitBudgetNs) {
      latch_error(hdr, MOE_ERR_TIMEOUT, where);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

template <int kRowDt, int kOutDt>
__global__ void __launch_bounds__(threads_of<kRowDt>(), 1) combine_tma_kernel(const __grid_constant__ Args a) {
  constexpr int kCompWarps = comp_warps<kRowDt>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
  __shared__ uint64_t full[kStages], empty[kStages];
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(full + s, 1);
      ptx::mbar_init(empty + s, kCompWarps);
    }
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  const int64_t units = (int64_t)a.T * a.nparts;
  const int chunk_bytes = a.V * a.elt;
  const int nscales = a.V / kQBlock;

  if (warp == kCompWarps) {
    // ------------------------------------------------------------ loader
    uint32_t armed = 0, armed_parity = 0;
    // lane j's slot of a unit: its row and weight, loaded one unit ahead so
    // that the load's latency overlaps the wait for a free stage
    auto load_meta = [&](int64_t u, int* row, float* wj) {
      *row = -1;
      *wj = 0.f;
      if (u < units && lane < a.k) {
        const int64_t t = u / a.nparts;
        *row = __ldg(a.pos + t * a.k + lane);
        *wj = __ldg(a.w + t * a.k + lane);
      }
    };
    int row_next;
    float w_next;
    load_meta(blockIdx.x, &row_next, &w_next);
    for (int i = 0;; ++i) {
      const int64_t u = blockIdx.x + (int64_t)i * gridDim.x;
      if (u >= units) break;
      const int row = row_next;
      const float wj = w_next;
      load_meta(u + gridDim.x, &row_next, &w_next);
      const int s = i % kStages;
      int ok = 1;
      if (lane == 0 && i >= kStages)
        ok = wait_phase(empty + s, ((i / kStages) & 1) ^ 1, &abort_flag, a.hdr, 0xC1000000u | s);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const int part = (int)(u % a.nparts);
      uint8_t* st = smem + s * a.stage_bytes;
      const bool copy = lane < a.k && row >= 0 && wj != 0.f;
      const uint32_t live = __ballot_sync(0xffffffffu, copy);
      const uint32_t n = __popc(live);
      if (copy) {   // the live slots in slot order, so that the sums keep it
        const int c = __popc(live & ((1u << lane) - 1u));
        reinterpret_cast<int*>(st + a.off_meta)[c] = lane;
        reinterpret_cast<float*>(st + a.off_meta)[kMaxSlots + c] = wj;
        reinterpret_cast<int*>(st + a.off_meta)[2 * kMaxSlots + c] = row;
      }
      if (lane == 0) reinterpret_cast<int*>(st + a.off_meta)[3 * kMaxSlots] = (int)n;
      __syncwarp();   // the slot list is written before lane 0's arrive publishes it
      const uint32_t bytes = n * (uint32_t)(chunk_bytes + (a.scale_bulk ? nscales * 4 : 0));
      if (lane == 0) ptx::mbar_arrive_expect_tx(full + s, bytes);   // also publishes the meta words
      __syncwarp();
      if (copy) {
        ptx::bulk_load(st + lane * chunk_bytes, a.rows + ((int64_t)row * a.H + (int64_t)part * a.V) * a.elt,
                       (uint32_t)chunk_bytes, full + s);
        if (a.scale_bulk)
          ptx::bulk_load(st + a.off_scale + lane * nscales * 4,
                         a.xs + (int64_t)row * (a.H / kQBlock) + (int64_t)part * nscales, (uint32_t)(nscales * 4),
                         full + s);
      }
      __syncwarp();
      armed |= 1u << s;
      armed_parity = (armed_parity & ~(1u << s)) | ((uint32_t)((i / kStages) & 1) << s);
    }
    // every copy this warp started has landed before the CTA exits
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        if (!((armed >> s) & 1u)) continue;
        const unsigned long long t0 = globaltimer();
        while (!ptx::mbar_try_wait(full + s, (armed_parity >> s) & 1u)) {
          if (globaltimer() - t0 > kWaitBudgetNs) break;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute
    constexpr int kVals = vals_of<kRowDt>();
    const int ngroups = a.V / kVals;
    for (int i = 0;; ++i) {
      const int64_t u = blockIdx.x + (int64_t)i * gridDim.x;
      if (u >= units) break;
      const int s = i % kStages;
      int ok = 1;
      if (lane == 0) ok = wait_phase(full + s, (i / kStages) & 1, &abort_flag, a.hdr, 0xC2000000u | s);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const int t = (int)(u / a.nparts), part = (int)(u % a.nparts);
      const uint8_t* st = smem + s * a.stage_bytes;
      const int* sslot = reinterpret_cast<const int*>(st + a.off_meta);
      const float* sw = reinterpret_cast<const float*>(st + a.off_meta) + kMaxSlots;
      const int* srow = reinterpret_cast<const int*>(st + a.off_meta) + 2 * kMaxSlots;
      const int nlive = sslot[3 * kMaxSlots];
      for (int g = threadIdx.x; g < ngroups; g += kCompWarps * 32) {
        float acc[kVals];
#pragma unroll
        for (int v = 0; v < kVals; ++v) acc[v] = 0.f;
#pragma unroll 4
        for (int c = 0; c < nlive; ++c) {
          const int j = sslot[c];
          const float wj = sw[c];
          float sc = 0.f;
          if constexpr (kRowDt == MOE_E4M3) {
            const int blk = (g * kVals) / kQBlock;
            sc = a.scale_bulk ? reinterpret_cast<const float*>(st + a.off_scale)[j * nscales + blk]
                              : __ldg(a.xs + (int64_t)srow[c] * (a.H / kQBlock) + (int64_t)part * nscales + blk);
          }
          fma_vals<kRowDt>(st + j * chunk_bytes + g * kVals * a.elt, sc, wj, acc);
        }
        const int64_t off = (int64_t)t * a.H + (int64_t)part * a.V + g * kVals;
        if constexpr (kOutDt == MOE_BF16) {
          uint32_t wv[kVals / 2];
#pragma unroll
          for (int v = 0; v < kVals / 2; ++v) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * v], acc[2 * v + 1]);
            wv[v] = *reinterpret_cast<uint32_t*>(&b2);
          }
          uint4* p = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + off);
#pragma unroll
          for (int v = 0; v < kVals / 8; ++v) p[v] = make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]);
        } else {
          float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + off);
#pragma unroll
          for (int v = 0; v < kVals / 4; ++v) p[v] = make_float4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]);
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(empty + s);   // this warp is done with the stage
    }
  }
}

}  // namespace

// The staged combine when the shape suits it (returns false otherwise, and
// the caller uses the register-gather kernel): parts of the row whose k
// chunks fit one stage, e4m3 parts aligned to scale blocks.
bool launch_combine_tma(const Ctx& c, const moe_dispatch_bufs& b, const void* y, const float* topk_w, void* out,
                        cudaError_t* err) {
  const int T = (int)c.s.T, H = (int)c.s.H, k = (int)c.s.topk;
  const bool ident = c.s.identity_experts != 0;
  const int row_dt = ident ? c.s.xq_dtype : c.s.y_dtype;
  const int elt = row_dt == MOE_F32 ? 4 : (row_dt == MOE_BF16 ? 2 : 1);
  if (T == 0 || k > kMaxSlots || H % 16) return false;
  int nparts = 0, V = 0;
  for (int n = 1; n <= H / 16; ++n) {
    if (H % n) continue;
    const int v = H / n;
    if (v % 16 || (int64_t)k * v * elt > kRowCap) continue;
    if (row_dt == MOE_E4M3 && v % kQBlock) continue;
    nparts = n;
    V = v;
    break;
  }
  if (!nparts) return false;
  // enough units to fill the SMs with a few stages each; below that the
  // register-gather kernel's finer units win
  if ((int64_t)T * nparts < 6LL * c.num_sms) return false;
  Args a;
  a.pos = b.pos;
  a.w = topk_w;
  a.rows = reinterpret_cast<const uint8_t*>(ident ? b.xq : y);
  a.xs = ident && row_dt == MOE_E4M3 ? b.xs : nullptr;
  a.out = out;
  a.hdr = c.ws.hdr;
  a.T = T;
  a.H = H;
  a.k = k;
  a.elt = elt;
  a.nparts = nparts;
  a.V = V;
  const int nscales = V / kQBlock;
  a.scale_bulk = row_dt == MOE_E4M3 && (nscales * 4) % 16 == 0;
  const int row_bytes = k * V * elt;
  a.off_scale = row_bytes;
  const int scale_bytes = a.scale_bulk ? (k * nscales * 4 + 15) / 16 * 16 : 0;
  a.off_meta = row_bytes + scale_bytes;
  a.stage_bytes = (a.off_meta + kMetaBytes + 127) / 128 * 128;
  const int smem = kStages * a.stage_bytes + 128;
  const int grid = (int)std::min<int64_t>((int64_t)T * nparts, c.num_sms);
  const bool bf16_out = c.s.out_dtype == MOE_BF16;
  const int threads = row_dt == MOE_E4M3 ? threads_of<MOE_E4M3>()
                      : row_dt == MOE_BF16 ? threads_of<MOE_BF16>() : threads_of<MOE_F32>();
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) {
      kern<<<grid, threads, smem, c.stream>>>(a);
      e = cudaGetLastError();
    }
    *err = e;
  };
  if (row_dt == MOE_BF16) {
    if (bf16_out) go(combine_tma_kernel<MOE_BF16, MOE_BF16>);
    else go(combine_tma_kernel<MOE_BF16, MOE_F32>);
  } else if (row_dt == MOE_F32) {
    if (bf16_out) go(combine_tma_kernel<MOE_F32, MOE_BF16>);
    else go(combine_tma_kernel<MOE_F32, MOE_F32>);
  } else {
    if (bf16_out) go(combine_tma_kernel<MOE_E4M3, MOE_BF16>);
    else go(combine_tma_kernel<MOE_E4M3, MOE_F32>);
  }
  return true;
}

}  // namespace moe

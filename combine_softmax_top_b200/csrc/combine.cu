// Top-k weighted combine straight out of the expert windows.
//
// Pages: outputs are gathered directly from the expert windows, with no
// output-restoration buffer (Ascend report, abstract); combine is the third
// per-layer stage after dispatch and the grouped GEMM (GC-MoE feed item,
// "Key points").
//
//   out[t] = sum_{j < k} w[t, j] * y[pos[t*k + j]]    (fp32, slot order)
//
// rounded once to the output dtype. Work unit = (token, 512-value chunk of
// the row); each warp walks units grid-stride. Lanes j < k load pos/w of the
// token and broadcast them; every lane then owns 16 consecutive outputs and
// issues the k row loads (32 bytes each for bf16, 16 for e4m3) before any
// arithmetic, so a warp keeps k x 1 KB in flight per unit.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kVec = 16;                 // outputs per lane per unit
constexpr int kChunk = 32 * kVec;        // outputs per unit
constexpr int kBatch = 8;                // slots loaded together

struct Args {
  const int32_t* pos;
  const float* w;
  const void* rows;   // y rows, or xq rows for identity experts
  const float* xs;    // e4m3 identity rows: scales
  void* out;
  int T, H, k;
};

// Raw bytes of 16 consecutive values of one row (64 B f32, 32 B bf16, 16 B e4m3).
template <int kRowDt>
struct Raw16 {
  uint4 v[kRowDt == MOE_F32 ? 4 : (kRowDt == MOE_BF16 ? 2 : 1)];
};

template <int kRowDt>
__device__ __forceinline__ void load_raw(const Args& a, int row, int h0, Raw16<kRowDt>& r, float& s) {
  const int64_t off = (int64_t)row * a.H + h0;
  if constexpr (kRowDt == MOE_BF16) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.rows) + off);
    r.v[0] = __ldg(p);
    r.v[1] = __ldg(p + 1);
  } else if constexpr (kRowDt == MOE_F32) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(a.rows) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i) r.v[i] = __ldg(p + i);
  } else {
    r.v[0] = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(a.rows) + off));
    s = __ldg(a.xs + (int64_t)row * (a.H / kQBlock) + h0 / kQBlock);
  }
}

template <int kRowDt>
__device__ __forceinline__ void fma_raw(const Raw16<kRowDt>& r, float s, float wj, float* acc) {
  if constexpr (kRowDt == MOE_BF16) {
    const uint32_t u[8] = {r.v[0].x, r.v[0].y, r.v[0].z, r.v[0].w, r.v[1].x, r.v[1].y, r.v[1].z, r.v[1].w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      acc[2 * i] = fmaf(wj, __uint_as_float(u[i] << 16), acc[2 * i]);
      acc[2 * i + 1] = fmaf(wj, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
    }
  } else if constexpr (kRowDt == MOE_F32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[4 * i] = fmaf(wj, __uint_as_float(r.v[i].x), acc[4 * i]);
      acc[4 * i + 1] = fmaf(wj, __uint_as_float(r.v[i].y), acc[4 * i + 1]);
      acc[4 * i + 2] = fmaf(wj, __uint_as_float(r.v[i].z), acc[4 * i + 2]);
      acc[4 * i + 3] = fmaf(wj, __uint_as_float(r.v[i].w), acc[4 * i + 3]);
    }
  } else {
    const uint32_t u[4] = {r.v[0].x, r.v[0].y, r.v[0].z, r.v[0].w};
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

template <int kRowDt, int kOutDt>
__global__ void __launch_bounds__(kThreads) combine_kernel(Args a) {
  const int lane = threadIdx.x & 31;
  const int nch = (a.H + kChunk - 1) / kChunk;
  const int64_t units = (int64_t)a.T * nch;
  const int64_t nw = (int64_t)gridDim.x * kWarps;
  for (int64_t u = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); u < units; u += nw) {
    const int t = (int)(u / nch);
    const int h0 = (int)(u % nch) * kChunk + lane * kVec;
    const bool live = h0 < a.H;
    float acc[kVec];
#pragma unroll
    for (int i = 0; i < kVec; ++i) acc[i] = 0.f;
    for (int j0 = 0; j0 < a.k; j0 += 32) {
      // lanes j < k hold pos / w of slot j0 + j
      const int jl = j0 + lane;
      const int my_row = jl < a.k ? __ldg(a.pos + (int64_t)t * a.k + jl) : -1;
      const float my_w = jl < a.k ? __ldg(a.w + (int64_t)t * a.k + jl) : 0.f;
      const int nj = min(32, a.k - j0);
      for (int b0 = 0; b0 < nj; b0 += kBatch) {
        Raw16<kRowDt> r[kBatch];
        float sc[kBatch];
        float wj[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int row = __shfl_sync(0xffffffffu, my_row, (b0 + b) & 31);
          wj[b] = __shfl_sync(0xffffffffu, my_w, (b0 + b) & 31);
          sc[b] = 0.f;
          if (b0 + b < nj && row >= 0 && live) load_raw<kRowDt>(a, row, h0, r[b], sc[b]);
          else wj[b] = 0.f;
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b)
          if (wj[b] != 0.f) fma_raw<kRowDt>(r[b], sc[b], wj[b], acc);
      }
    }
    if (!live) continue;
    const int64_t off = (int64_t)t * a.H + h0;
    if constexpr (kOutDt == MOE_BF16) {
      uint32_t wv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        wv[i] = *reinterpret_cast<uint32_t*>(&b2);
      }
      uint4* p = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + off);
      p[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      p[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
    } else {
      float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + off);
#pragma unroll
      for (int i = 0; i < 4; ++i) p[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
    }
  }
}

}  // namespace

cudaError_t launch_combine(const Ctx& c, const moe_dispatch_bufs& b, const void* y,
                           const float* topk_w, void* out) {
  Args a;
  a.pos = b.pos;
  a.w = topk_w;
  a.T = (int)c.s.T;
  a.H = (int)c.s.H;
  a.k = (int)c.s.topk;
  a.out = out;
  int row_dt;
  if (c.s.identity_experts) {
    a.rows = b.xq;
    a.xs = b.xs;
    row_dt = c.s.xq_dtype;
  } else {
    a.rows = y;
    a.xs = nullptr;
    row_dt = c.s.y_dtype;
  }
  if (a.T == 0) return cudaSuccess;
  cudaError_t staged_err;
  if (launch_combine_tma(c, b, y, topk_w, out, &staged_err)) return staged_err;
  const int64_t units = (int64_t)a.T * ((a.H + kChunk - 1) / kChunk);
  const int64_t want = (units + kWarps - 1) / kWarps;
  const int grid = (int)std::min<int64_t>(want, (int64_t)c.num_sms * 4);
  const bool bf16_out = c.s.out_dtype == MOE_BF16;
  if (row_dt == MOE_BF16) {
    if (bf16_out) combine_kernel<MOE_BF16, MOE_BF16><<<grid, kThreads, 0, c.stream>>>(a);
    else combine_kernel<MOE_BF16, MOE_F32><<<grid, kThreads, 0, c.stream>>>(a);
  } else if (row_dt == MOE_F32) {
    if (bf16_out) combine_kernel<MOE_F32, MOE_BF16><<<grid, kThreads, 0, c.stream>>>(a);
    else combine_kernel<MOE_F32, MOE_F32><<<grid, kThreads, 0, c.stream>>>(a);
  } else {
    if (bf16_out) combine_kernel<MOE_E4M3, MOE_BF16><<<grid, kThreads, 0, c.stream>>>(a);
    else combine_kernel<MOE_E4M3, MOE_F32><<<grid, kThreads, 0, c.stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace moe

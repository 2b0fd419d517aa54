// Top-k weighted combine straight out of the expert windows.
//
// Pages: outputs are gathered directly from the expert windows, with no
// output-restoration buffer (Ascend report, abstract); combine is the third
// per-layer stage after dispatch and the grouped GEMM (GC-MoE feed item,
// "Key points").
//
//   out[t] = sum_{j < k} w[t, j] * y[pos[t*k + j]]    (fp32, slot order)
//
// rounded once to the output dtype. Grid (H chunks, tokens): each thread owns
// 8 consecutive outputs and issues the k gathers (16-byte loads for bf16 / 8
// for e4m3) before the FMAs so the loads overlap.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kVec = 8;  // outputs per thread

struct Args {
  const int32_t* pos;
  const float* w;
  const void* rows;   // y rows, or xq rows for identity experts
  const float* xs;    // e4m3 identity rows: scales
  void* out;
  int T, H, k;
  int row_dtype;      // MOE_F32 / MOE_BF16 / MOE_E4M3
  int out_dtype;
};

__device__ __forceinline__ void load_row8(const Args& a, int row, int h0, float* v) {
  const int64_t off = (int64_t)row * a.H + h0;
  if (a.row_dtype == MOE_BF16) {
    uint4 q = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.rows) + off));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else if (a.row_dtype == MOE_F32) {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.rows) + off);
    float4 q0 = __ldg(p), q1 = __ldg(p + 1);
    v[0] = q0.x; v[1] = q0.y; v[2] = q0.z; v[3] = q0.w;
    v[4] = q1.x; v[5] = q1.y; v[6] = q1.z; v[7] = q1.w;
  } else {
    uint2 q = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(a.rows) + off));
    const float s = __ldg(a.xs + (int64_t)row * (a.H / kQBlock) + h0 / kQBlock);
    const uint32_t w[2] = {q.x, q.y};
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = e4m3_to_f32((uint8_t)(w[i / 4] >> (8 * (i % 4)))) * s;
  }
}

__global__ void __launch_bounds__(kThreads) combine_kernel(Args a) {
  const int t = blockIdx.y;
  const int h0 = (blockIdx.x * kThreads + threadIdx.x) * kVec;
  if (h0 >= a.H) return;
  float acc[kVec];
#pragma unroll
  for (int i = 0; i < kVec; ++i) acc[i] = 0.f;
  constexpr int kBatch = 8;  // gathers in flight per thread
  for (int j0 = 0; j0 < a.k; j0 += kBatch) {
    float v[kBatch][kVec];
    float wj[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int j = j0 + b;
      const int row = j < a.k ? __ldg(a.pos + (int64_t)t * a.k + j) : -1;
      wj[b] = row >= 0 ? __ldg(a.w + (int64_t)t * a.k + j) : 0.f;
      if (row >= 0) load_row8(a, row, h0, v[b]);
      else {
#pragma unroll
        for (int i = 0; i < kVec; ++i) v[b][i] = 0.f;
      }
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
#pragma unroll
      for (int i = 0; i < kVec; ++i) acc[i] = fmaf(wj[b], v[b][i], acc[i]);
  }
  const int64_t off = (int64_t)t * a.H + h0;
  if (a.out_dtype == MOE_BF16) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&b2);
    }
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + off) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + off);
    p[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    p[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
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
  a.out_dtype = c.s.out_dtype;
  if (c.s.identity_experts) {
    a.rows = b.xq;
    a.xs = b.xs;
    a.row_dtype = c.s.xq_dtype;
  } else {
    a.rows = y;
    a.xs = nullptr;
    a.row_dtype = c.s.y_dtype;
  }
  if (a.T == 0) return cudaSuccess;
  dim3 grid((unsigned)((a.H + kThreads * kVec - 1) / (kThreads * kVec)), (unsigned)a.T);
  combine_kernel<<<grid, kThreads, 0, c.stream>>>(a);
  return cudaGetLastError();
}

}  // namespace moe

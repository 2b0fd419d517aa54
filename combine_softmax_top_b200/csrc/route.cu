// Routing: softmax over the router logits, then top-k.
//
// Reading of the pages: each token goes to the experts its gating result
// selects (GC-MoE explainer, "Why Expert Parallelism Is Inefficient in MoE
// Decoding"). Selection is done on the logits themselves (softmax is
// monotone), so it is exact and independent of how exp is evaluated; equal
// logits go to the lower expert index, slots are in descending logit order.
//
// One warp per token. The row of E logits is read with coalesced 16-byte
// loads (E % 4 == 0) into registers, k rounds of a warp-shuffle arg-max pick
// the experts, and the softmax denominator is a warp reduction.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWarpsPerBlock = 8;

struct Cand {
  float v;
  int i;
};

// a beats b: larger logit, or equal logit and lower index
__device__ __forceinline__ bool beats(float av, int ai, float bv, int bi) {
  return av > bv || (av == bv && ai < bi);
}

template <int NV>  // logits per lane (multiple of 4 when VEC)
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
route_kernel(const float* __restrict__ logits, int T, int E, int k, int renorm, int shared,
             int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, Header* hdr) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* row = logits + (int64_t)t * E;

  // element c of this lane is expert (c / 4) * 128 + lane * 4 + c % 4 when
  // E % 4 == 0 (16-byte loads), else lane + 32 * c.
  float v[NV];
  int ix[NV];
  const bool vec = (E & 3) == 0;
  if (vec) {
#pragma unroll
    for (int c4 = 0; c4 < NV / 4; ++c4) {
      const int base = c4 * 128 + lane * 4;
      float4 q = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      if (base < E) q = __ldg(reinterpret_cast<const float4*>(row + base));
      v[c4 * 4 + 0] = q.x; v[c4 * 4 + 1] = q.y; v[c4 * 4 + 2] = q.z; v[c4 * 4 + 3] = q.w;
#pragma unroll
      for (int j = 0; j < 4; ++j) ix[c4 * 4 + j] = base < E ? base + j : INT32_MAX;
    }
  } else {
#pragma unroll
    for (int c = 0; c < NV; ++c) {
      const int e = lane + 32 * c;
      v[c] = e < E ? __ldg(row + e) : -INFINITY;
      ix[c] = e < E ? e : INT32_MAX;
    }
  }

  bool bad = false;
#pragma unroll
  for (int c = 0; c < NV; ++c) bad |= (ix[c] != INT32_MAX) && !isfinite(v[c]);
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) latch_error(hdr, MOE_ERR_NONFINITE, (uint32_t)t);
    return;
  }

  unsigned taken = 0;  // bit c: element c already selected
  float sel_v = 0.f;   // lane j keeps slot j
  int sel_i = 0;
  float top = 0.f;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = INT32_MAX;
#pragma unroll
    for (int c = 0; c < NV; ++c) {
      if (!((taken >> c) & 1u) && beats(v[c], ix[c], bv, bi)) { bv = v[c]; bi = ix[c]; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (beats(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
#pragma unroll
    for (int c = 0; c < NV; ++c)
      if (ix[c] == bi) taken |= 1u << c;
    if (j == 0) top = bv;
    if (lane == j) { sel_v = bv; sel_i = bi; }
  }

  // softmax weights, max-subtracted
  float part = 0.f;
  if (renorm) {
    part = lane < k ? expf(sel_v - top) : 0.f;
  } else {
#pragma unroll
    for (int c = 0; c < NV; ++c)
      if (ix[c] != INT32_MAX) part += expf(v[c] - top);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
  // with a shared expert each token's row has k + 1 slots, the last being
  // the shared expert (index E) with weight 1
  const int ks = k + shared;
  if (lane < k) {
    topk_idx[(int64_t)t * ks + lane] = sel_i;
    topk_w[(int64_t)t * ks + lane] = expf(sel_v - top) / part;
  } else if (shared && lane == k) {
    topk_idx[(int64_t)t * ks + k] = E;
    topk_w[(int64_t)t * ks + k] = 1.f;
  }
}

template <int NV>
cudaError_t go(const Ctx& c, const float* logits, int32_t* idx, float* w) {
  const int T = (int)c.s.T;
  if (T == 0) return cudaSuccess;
  dim3 grid((T + kWarpsPerBlock - 1) / kWarpsPerBlock);
  route_kernel<NV><<<grid, kWarpsPerBlock * 32, 0, c.stream>>>(
      logits, T, (int)c.routed_E, (int)c.routed_k, c.s.renorm, c.shared, idx, w, c.ws.hdr);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route(const Ctx& c, const float* logits, int32_t* idx, float* w) {
  const int64_t E = c.routed_E;
  if (E <= 128) return go<4>(c, logits, idx, w);
  if (E <= 256) return go<8>(c, logits, idx, w);
  if (E <= 512) return go<16>(c, logits, idx, w);
  return go<32>(c, logits, idx, w);   // E <= 1024 (checked by the ABI)
}

}  // namespace moe

// Routing: softmax over the router logits, then top-k.
//
// Reading of the pages: each token goes to the experts its gating result
// selects (GC-MoE explainer, "Why Expert Parallelism Is Inefficient in MoE
// Decoding"). Selection is done on the logits themselves (softmax is
// monotone), so it is exact and independent of how exp is evaluated; equal
// logits go to the lower expert index, slots are in descending logit order.
//
// One warp per token. The row of E logits is read with coalesced 16-byte
// loads (E % 4 == 0) into registers. Each lane keeps the best of its own
// logits; each of the k rounds takes the warp's best with two reductions (the
// largest value as an order-preserving 32-bit key, then the lowest expert
// index among the lanes holding it), and only the lane that supplied the
// winner looks for its next best. The softmax denominator is a warp
// reduction.
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

// 32-bit key that orders like the float (no NaN; -0 already folded into +0)
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
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

  // fold -0 into +0 so that the keys compare like the logits (-0 == +0)
#pragma unroll
  for (int c = 0; c < NV; ++c) v[c] += 0.f;
  unsigned taken = 0;  // bit c: element c already selected
  float bv;            // this lane's best remaining logit and its expert
  int bi;
  auto local_best = [&]() {
    bv = -INFINITY;
    bi = INT32_MAX;
#pragma unroll
    for (int c = 0; c < NV; ++c)
      if (!((taken >> c) & 1u) && beats(v[c], ix[c], bv, bi)) { bv = v[c]; bi = ix[c]; }
  };
  local_best();
  float sel_v = 0.f;   // lane j keeps slot j
  int sel_i = 0;
  float top = 0.f;
  for (int j = 0; j < k; ++j) {
    const uint32_t key = bi == INT32_MAX ? 0u : order_key(bv);
    const uint32_t m = __reduce_max_sync(0xffffffffu, key);
    const uint32_t wi = __reduce_min_sync(0xffffffffu, key == m ? (uint32_t)bi : 0xFFFFFFFFu);
    const float wv = key_value(m);
    if (j == 0) top = wv;
    if (lane == j) { sel_v = wv; sel_i = (int)wi; }
    if ((uint32_t)bi == wi) {   // the winner came from this lane
#pragma unroll
      for (int c = 0; c < NV; ++c)
        if ((uint32_t)ix[c] == wi) taken |= 1u << c;
      local_best();
    }
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

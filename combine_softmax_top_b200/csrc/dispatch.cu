// One-pass dispatch into expert-major windows.
//
// Pages: tokens are pushed straight into the destination windows without a
// metadata exchange first, and the grouped GEMM reads them there in place
// (NVLinkOneSided abstract); a ready flag travels with the data (its
// "Sentinel" protocol); the producer bumps a counter per batch of filled ring
// blocks that the GEMM polls, and double-buffered counters remove the clean
// pass between calls (GC-MoE explainer, "Three-Node CUDA Graph and token-ring
// Handshake"). Only counts, offsets and sync metadata are kept (Ascend report,
// abstract).
//
// CTAs walk tokens; for each token:
//  1. lanes j < k claim row first(e) + atomicAdd(count[e], 1) for slot j (the
//     expert index loaded two tokens ahead, the atomic issued one token
//     ahead, so neither round trip stalls the CTA); first(e) = e * cap, or with
//     compact windows 128 * base[e] from the counting pass (plan_kernel);
//  2. all warps stream the token row once (16-byte loads) and write it to the
//     k claimed rows; E4M3 rows are quantised per 128 values with the
//     smallest power-of-two scale that keeps the block within +-448, and the
//     scale's exponent byte also goes to the tile's scale-factor atom read by
//     the block-scaled MMA;
//  3. each slot bumps its tile's fill counter; the bump that completes 128 rows
//     publishes the tile (sentinel + ring entry);
//  4. the last CTA to finish closes: it publishes the partial
//     last tile of each expert, writes counts/offsets and the tile total, and
//     advances the epoch.
// Every CTA first zeroes its share of the counter set the *next* dispatch will
// use, so no separate clean pass is needed.
//
// Compact windows (the NVLinkOneSided abstract's Fence protocol: the
// counts are settled before any row moves, here by stream order between two
// launches): plan_kernel histograms the expert indices and its last CTA
// lays the windows out back to back, each rounded up to whole 128-row tiles,
// so the buffers need T * k + 127 * E rows instead of E * cap.
#include <atomic>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxDevices = 64;   // per-device caches of launch parameters
constexpr int kElems = 16;  // values per lane per step

struct Args {
  const void* x;
  const int32_t* idx;
  int T, H, E, k, cap, tpe;
  int compact;         // windows at 128 * base[e] (set_base), sized by the counting pass
  int64_t tiles;
  int act, xq_dtype;
  moe_dispatch_bufs b;
  Ws ws;
  uint8_t* xsf;        // scale atoms for the block-scaled MMA (NULL: not written)
  int64_t set_words;
};

// Raw bytes of 16 consecutive values of x (bf16: 2 vectors, f32: 4).
template <int kAct>
struct Raw16 {
  uint4 r[kAct == MOE_BF16 ? 2 : 4];
};

template <int kAct>
__device__ __forceinline__ void load_raw(const void* x, int64_t off, Raw16<kAct>& v) {
  if constexpr (kAct == MOE_BF16) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(x) + off);
    v.r[0] = __ldg(p);
    v.r[1] = __ldg(p + 1);
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(x) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i) v.r[i] = __ldg(p + i);
  }
}

template <int kAct>
__device__ __forceinline__ void raw_to_f32(const Raw16<kAct>& v, float* f) {
  if constexpr (kAct == MOE_BF16) {
    const uint32_t w[8] = {v.r[0].x, v.r[0].y, v.r[0].z, v.r[0].w, v.r[1].x, v.r[1].y, v.r[1].z, v.r[1].w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[4 * i] = __uint_as_float(v.r[i].x);
      f[4 * i + 1] = __uint_as_float(v.r[i].y);
      f[4 * i + 2] = __uint_as_float(v.r[i].z);
      f[4 * i + 3] = __uint_as_float(v.r[i].w);
    }
  }
}

__device__ __forceinline__ void load16(const void* x, int act, int64_t off, float* v) {
  if (act == MOE_BF16) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(x) + off);
    uint4 a = __ldg(p), b = __ldg(p + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(x) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 q = __ldg(p + i);
      v[4 * i] = q.x; v[4 * i + 1] = q.y; v[4 * i + 2] = q.z; v[4 * i + 3] = q.w;
    }
  }
}

// Global tile g (rows 128 g ...) of expert e holds `rows` rows: set its
// sentinel and append it to the ring.
__device__ void publish_tile(const Args& a, uint32_t* set, uint32_t epoch, int e, int64_t g,
                             int rows) {
  st_release(a.ws.sentinel + g, (epoch << 8) | (uint32_t)rows);
  const uint32_t slot = atomicAdd(set_misc(set) + kRingHead, 1u);
  st_release64(a.ws.ring + slot, ring_entry(epoch, e, g));
}

// Row claims are pipelined over three tokens by the threads tid < k (slot
// tid): the expert index is loaded two tokens ahead, the atomicAdd on its
// count issued one token ahead, and its result used a whole token later, so
// neither round trip stalls the CTA.
__device__ __forceinline__ int load_expert(const Args& a, int t, int tid) {
  return t < a.T ? __ldg(a.idx + (int64_t)t * a.k + tid) : -1;
}

__device__ __forceinline__ uint32_t issue_claim(const Args& a, int t, int e, uint32_t* count) {
  return (t < a.T && e >= 0 && e < a.E) ? atomicAdd(count + e, 1u) : 0u;
}

// Token t's slot tid: the claimed row (or -1), recorded in pos/row_src/s_row.
// base: compact windows' first tiles (NULL: windows of cap rows).
__device__ __forceinline__ void finish_claim(const Args& a, const uint32_t* base, int t, int tid, int e,
                                             uint32_t p, int* s_row, int* s_e) {
  const int pair = t * a.k + tid;
  int row = -1;
  if (e >= 0 && e < a.E) {
    uint32_t first, room;
    if (base) {
      first = base[e] * (uint32_t)kTileRows;
      room = base[e + 1] * (uint32_t)kTileRows - first;
    } else {
      first = (uint32_t)e * (uint32_t)a.cap;
      room = (uint32_t)a.cap;
    }
    if (p < room) {
      row = (int)(first + p);
      a.b.row_src[row] = pair;
    } else {   // compact windows: only if idx changed after the counting pass
      latch_error(a.ws.hdr, MOE_ERR_CAPACITY, (uint32_t)e);
    }
  } else {
    latch_error(a.ws.hdr, MOE_ERR_INVALID_ARG, (uint32_t)pair);
  }
  a.b.pos[pair] = row;
  s_row[tid] = row;
  s_e[tid] = e;
}

// Write token t's row to its claimed rows (all threads; a lane group of 8
// covers one 128-value block). pre holds this thread's first kPre slices
// (loaded one token ahead); further slices (H > kPre * 4096) load here.
constexpr int kPre = 2;

// Quantise (or convert) one 16-value slice s of token t and store it to the
// token's k rows; all lanes of the warp take part (the 8-lane amax).
__device__ __forceinline__ void put_slice(const Args& a, int tid, const int* s_row, int s, bool live, const float* v) {
  {
    const int h0 = s * kElems;
    if (a.xq_dtype == MOE_E4M3) {
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < kElems; ++i) amax = fmaxf(amax, fabsf(v[i]));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
      if (!live) return;
      const int p = pow2_scale_exp(amax);
      const float inv = exp2i(-p > -126 ? -p : -126);  // 2^-p; p <= 120 for finite x
      uint32_t q[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint16_t lo = cvt_e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv);
        uint16_t hi = cvt_e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv);
        q[i] = (uint32_t)lo | ((uint32_t)hi << 16);
      }
      const uint4 qv = make_uint4(q[0], q[1], q[2], q[3]);
      const bool leader = (tid & 7) == 0;
      const int blk = h0 / kQBlock;
      for (int j = 0; j < a.k; ++j) {
        const int row = s_row[j];
        if (row < 0) continue;
        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(a.b.xq) + (int64_t)row * a.H + h0) = qv;
        if (leader) {
          a.b.xs[(int64_t)row * (a.H / kQBlock) + blk] = exp2i(p);
          if (a.xsf)   // global tile row / 128
            *sf_atom_byte(a.xsf, row / kTileRows, (a.H + 4 * kQBlock - 1) / (4 * kQBlock), blk,
                          row % kTileRows) = (uint8_t)(p + 127);
        }
      }
    } else if (live) {
      for (int j = 0; j < a.k; ++j) {
        const int row = s_row[j];
        if (row < 0) continue;
        const int64_t off = (int64_t)row * a.H + h0;
        if (a.xq_dtype == MOE_BF16) {
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&b2);
          }
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.b.xq) + off);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.b.xq) + off);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
    }
  }
}

template <int kAct>
__device__ __forceinline__ void stream_row(const Args& a, int t, int tid, const int* s_row, const Raw16<kAct>* pre) {
  const int steps = a.H / kElems;
  const int span = (steps + 31) / 32 * 32;   // whole warps take part in every pass
#pragma unroll
  for (int si = 0; si < kPre; ++si) {
    const int s = tid + si * kThreads;
    if (s >= span) break;
    float v[kElems];
    if (s < steps) raw_to_f32<kAct>(pre[si], v);
    else {
#pragma unroll
      for (int i = 0; i < kElems; ++i) v[i] = 0.f;
    }
    put_slice(a, tid, s_row, s, s < steps, v);
  }
  for (int s = tid + kPre * kThreads; s < span; s += kThreads) {
    float v[kElems];
    if (s < steps) load16(a.x, a.act, (int64_t)t * a.H + s * kElems, v);
    else {
#pragma unroll
      for (int i = 0; i < kElems; ++i) v[i] = 0.f;
    }
    put_slice(a, tid, s_row, s, s < steps, v);
  }
}

// bf16 activations: capped at 64 registers, four CTAs per SM (measured: the
// prefill dispatch 143 -> 136 us, the T = 4096 sweep 76.8 -> 74.6 us; five
// CTAs spill and are slower)
template <int kAct>
__global__ void __launch_bounds__(kThreads, kAct == MOE_BF16 ? 4 : 1) dispatch_kernel(Args a) {
  __shared__ int s_row[2][kMaxTopk];   // double-buffered: this token's rows, the next token's
  __shared__ int s_e[2][kMaxTopk];
  __shared__ uint32_t s_epoch;
  __shared__ int s_last;
  __shared__ uint32_t s_tiles;
  const int tid = threadIdx.x;
  if (tid == 0) s_epoch = a.ws.hdr->epoch_next;
  __syncthreads();
  const uint32_t epoch = s_epoch;
  uint32_t* set = a.ws.set[epoch & 1];
  uint32_t* next = a.ws.set[(epoch + 1) & 1];
  uint32_t* count = set_count(set);
  uint32_t* fill = set_fill(set, a.E);
  uint32_t* misc = set_misc(set);
  const uint32_t* base = a.compact ? set_base(set, a.E, a.tiles) : nullptr;

  // zero this CTA's share of the next counter set
  {
    const int64_t per = (a.set_words + gridDim.x - 1) / gridDim.x;
    const int64_t lo = per * blockIdx.x;
    const int64_t hi = min(lo + per, a.set_words);
    for (int64_t i = lo + tid; i < hi; i += kThreads) next[i] = 0u;
  }

  // Tokens blockIdx.x, + G, + 2G, ... (G = gridDim.x). The next token's row
  // slices are loaded while this token is written, and its row claims were
  // issued a token earlier still.
  const int G = gridDim.x;
  const int steps = a.H / kElems;
  int cur = 0;
  int t = blockIdx.x;
  Raw16<kAct> v0[kPre];
  int e1 = -1, e2 = -1;   // slot tid's expert for tokens t + G and t + 2G
  uint32_t p1 = 0;        // and the claim already issued for token t + G
  if (tid < a.k && t < a.T) {
    const int e0 = load_expert(a, t, tid);
    const uint32_t p0 = issue_claim(a, t, e0, count);
    e1 = load_expert(a, t + G, tid);
    p1 = issue_claim(a, t + G, e1, count);
    e2 = load_expert(a, t + 2 * G, tid);
    finish_claim(a, base, t, tid, e0, p0, s_row[0], s_e[0]);
  }
  if (t < a.T) {
#pragma unroll
    for (int i = 0; i < kPre; ++i)
      if (tid + i * kThreads < steps) load_raw<kAct>(a.x, (int64_t)t * a.H + (tid + i * kThreads) * kElems, v0[i]);
  }
  __syncthreads();
  for (; t < a.T; t += G) {
    const int tn = t + G;
    if (tid < a.k && tn < a.T) {
      finish_claim(a, base, tn, tid, e1, p1, s_row[cur ^ 1], s_e[cur ^ 1]);   // claimed a token ago
      p1 = issue_claim(a, tn + G, e2, count);
      e1 = e2;
      e2 = load_expert(a, tn + 2 * G, tid);
    }
    Raw16<kAct> vn[kPre];
    if (tn < a.T) {
#pragma unroll
      for (int i = 0; i < kPre; ++i)
        if (tid + i * kThreads < steps) load_raw<kAct>(a.x, (int64_t)tn * a.H + (tid + i * kThreads) * kElems, vn[i]);
    }
    stream_row<kAct>(a, t, tid, s_row[cur], v0);
    __threadfence();
    __syncthreads();
    // count the filled rows; the bump that completes a tile publishes it
    if (tid < a.k) {
      const int row = s_row[cur][tid];
      if (row >= 0) {
        const int g = row / kTileRows;   // windows start on tile boundaries
        const uint32_t old = atomicAdd(fill + g, 1u);
        if (old + 1 == (uint32_t)kTileRows) publish_tile(a, set, epoch, s_e[cur][tid], g, kTileRows);
      }
    }
#pragma unroll
    for (int i = 0; i < kPre; ++i) v0[i] = vn[i];
    cur ^= 1;
    __syncthreads();   // the next token's claims are visible; this token's rows are free
  }
  __threadfence();
  __syncthreads();

  // the last CTA closes
  if (tid == 0) s_last = atomicAdd(misc + kDone, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid == 0) s_tiles = 0;
  __syncthreads();
  for (int e = tid; e < a.E; e += kThreads) {
    const uint32_t c_raw = ld_acquire(count + e);
    const int first = base ? (int)base[e] : e * a.tpe;   // global tile
    const int c = (int)min(c_raw, base ? (base[e + 1] - base[e]) * (uint32_t)kTileRows : (uint32_t)a.cap);
    a.b.counts[e] = c;
    a.b.offsets[e] = first * kTileRows;
    const int full = c / kTileRows;
    const int rem = c % kTileRows;
    if (rem) publish_tile(a, set, epoch, e, first + full, rem);   // the partial last tile
    atomicAdd(&s_tiles, (uint32_t)(full + (rem ? 1 : 0)));
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    st_release(misc + kRingTotal, s_tiles);
    a.ws.hdr->epoch_cur = epoch;
    __threadfence();
    a.ws.hdr->epoch_next = epoch + 1;
  }
}

// ---- compact windows: the counting pass --------------------------------------

constexpr int kPlanThreads = 256;

struct PlanArgs {
  const int32_t* idx;
  int64_t pairs;   // T * k
  int E;
  int64_t tiles;   // set layout
  Ws ws;
};

// Count each expert's (token, slot) pairs into pre[], then (last CTA) lay
// the windows out: base[e] = sum over e' < e of ceil(pre[e'] / 128),
// base[E] = the total. Indices outside [0, E) are skipped here; the
// dispatch kernel reports them.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(PlanArgs a) {
  extern __shared__ uint32_t hist[];   // [E]
  __shared__ uint32_t s_last;
  __shared__ uint32_t s_warp[kPlanThreads / 32];
  const int tid = threadIdx.x;
  const uint32_t epoch = a.ws.hdr->epoch_next;
  if (blockIdx.x == 0 && tid == 0) a.ws.hdr->epoch_plan = epoch;
  uint32_t* set = a.ws.set[epoch & 1];
  uint32_t* pre = set_pre(set, a.E, a.tiles);
  uint32_t* base = set_base(set, a.E, a.tiles);
  for (int e = tid; e < a.E; e += kPlanThreads) hist[e] = 0u;
  __syncthreads();
  for (int64_t i = (int64_t)blockIdx.x * kPlanThreads + tid; i < a.pairs; i += (int64_t)gridDim.x * kPlanThreads) {
    const int e = __ldg(a.idx + i);
    if (e >= 0 && e < a.E) atomicAdd(hist + e, 1u);
  }
  __syncthreads();
  for (int e = tid; e < a.E; e += kPlanThreads)
    if (hist[e]) atomicAdd(pre + e, hist[e]);
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(set_misc(set) + kPlanDone, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // exclusive scan of the tile counts: thread tid owns experts
  // [tid * per, (tid + 1) * per)
  const int per = (a.E + kPlanThreads - 1) / kPlanThreads;
  const int e0 = min(a.E, tid * per), e1 = min(a.E, e0 + per);
  uint32_t own = 0;
  for (int e = e0; e < e1; ++e) own += (ld_acquire(pre + e) + kTileRows - 1) / kTileRows;
  uint32_t incl = own;
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  uint32_t run = incl - own;
  for (int w = 0; w < warp; ++w) run += s_warp[w];
  for (int e = e0; e < e1; ++e) {
    base[e] = run;
    run += (ld_acquire(pre + e) + kTileRows - 1) / kTileRows;
  }
  if (tid == kPlanThreads - 1) base[a.E] = run;   // the last thread's running total is the sum
}

}  // namespace

cudaError_t launch_plan(const Ctx& c, const int32_t* idx) {
  PlanArgs pa;
  pa.idx = idx;
  pa.pairs = c.s.T * c.s.topk;
  pa.E = (int)c.s.E;
  pa.tiles = c.L.tiles;
  pa.ws = c.ws;
  const int64_t want = (pa.pairs + 8 * kPlanThreads - 1) / (8 * kPlanThreads);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, c.num_sms));
  plan_kernel<<<grid, kPlanThreads, (size_t)pa.E * 4, c.stream>>>(pa);
  return cudaGetLastError();
}

cudaError_t launch_dispatch(const Ctx& c, const void* x, const int32_t* idx,
                            const moe_dispatch_bufs& b, bool write_sf, bool planned) {
  Args a;
  a.x = x;
  a.idx = idx;
  a.T = (int)c.s.T;
  a.H = (int)c.s.H;
  a.E = (int)c.s.E;
  a.k = (int)c.s.topk;
  a.cap = (int)c.L.cap;
  a.tpe = (int)c.L.tpe;
  a.compact = c.L.compact ? 1 : 0;
  a.tiles = c.L.tiles;
  a.act = c.s.act_dtype;
  a.xq_dtype = c.s.xq_dtype;
  a.b = b;
  a.ws = c.ws;
  a.xsf = write_sf && c.s.xq_dtype == MOE_E4M3 ? c.ws.xsf : nullptr;
  a.set_words = (int64_t)c.L.set_words;
  if (a.compact && !planned) {
    const cudaError_t err = launch_plan(c, idx);
    if (err != cudaSuccess) return err;
  }
  // one wave of resident CTAs on the SMs given (all, or a partition's),
  // each walking several tokens (fewer CTAs also means fewer arrivals on the
  // closing counter). The occupancy query is
  // cached per device and kernel; concurrent callers may both run it, and
  // they store the same value.
  auto go = [&](auto kern, std::atomic<int>* cache) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return;
    std::atomic<int>& slot = cache[dev >= 0 && dev < kMaxDevices ? dev : 0];
    int resident = (dev >= 0 && dev < kMaxDevices) ? slot.load(std::memory_order_relaxed) : 0;
    if (resident == 0) {
      int r = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r, kern, kThreads, 0) != cudaSuccess || r < 1) r = 1;
      resident = r;
      if (dev >= 0 && dev < kMaxDevices) slot.store(r, std::memory_order_relaxed);
    }
    const int grid = a.T > 0 ? std::min(a.T, c.num_sms * resident) : 1;
    kern<<<grid, kThreads, 0, c.stream>>>(a);
  };
  static std::atomic<int> resident_bf16[kMaxDevices], resident_f32[kMaxDevices];
  if (a.act == MOE_BF16) go(dispatch_kernel<MOE_BF16>, resident_bf16);
  else go(dispatch_kernel<MOE_F32>, resident_f32);
  return cudaGetLastError();
}

}  // namespace moe

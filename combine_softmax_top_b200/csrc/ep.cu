// Expert-parallel dispatch into rank-major windows, and the cross-rank flags
// of the Fence and Sentinel protocols.
//
// Pages: each source rank pushes its tokens, with no metadata exchanged
// first, into rank-major buffers on the ranks that own the experts, and the
// grouped GEMM reads them there in place; Fence suits throughput and Sentinel
// latency (NVLinkOneSided abstract). The combine reads expert outputs in
// place, with no relay buffer (Ascend report, abstract).
//
// Every rank d receives into V = E virtual experts v = el * R + src (local
// expert el, source rank src), so a source only ever claims rows in its own
// regions, with counters in its own workspace. A row goes to rank d's window
// row first(v) + p, p = the source's claim for global expert e:
//   Sentinel: first(v) = v * cap_src (regions of round_up(t_max, 128) rows)
//   Fence:    first(v) = 128 * base_d[v], base_d laid out by rank d from the
//             counts all sources wrote first (moe_ep_count / moe_ep_layout)
// Tiles of 128 rows are counted in the owner's fill counters (system-scope
// atomics) and the bump that completes one publishes its sentinel; the
// source's last CTA publishes its partial tiles, writes its region counts and
// tile totals into the owners' counter sets, and adds itself to each owner's
// count of closed sources, which the owner's grouped FFN waits for.
//
// Every store another rank reads is released at system scope; every wait is
// bounded (200 ms of %globaltimer, then MOE_ERR_TIMEOUT latched in this
// rank's workspace).
#include <algorithm>
#include <cstring>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kElems = 16;   // values per thread per slice

struct EpArgs {
  const void* x;
  const int32_t* idx;
  int32_t* pos;
  int T, H, k, E, R, rank, e_loc, protocol, act, xq_dtype;
  int64_t t_max, cap_src, tpe_src, rows, hgroups, tiles, set_words;
  uint8_t* xq_all;
  float* xs_all;
  int32_t* row_src_all;
  char* ws_all;
  int64_t ws_bytes;
  int64_t off_set0, off_set1, off_sentinel, off_xsf, src_off;
};

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ Header* hdr_of(const EpArgs& a, int d) {
  return reinterpret_cast<Header*>(a.ws_all + (int64_t)d * a.ws_bytes);
}

// rank d's counter set of `epoch`
__device__ __forceinline__ uint32_t* set_of(const EpArgs& a, int d, uint32_t epoch) {
  return reinterpret_cast<uint32_t*>(a.ws_all + (int64_t)d * a.ws_bytes + ((epoch & 1) ? a.off_set1 : a.off_set0));
}

__device__ __forceinline__ uint32_t* sentinel_of(const EpArgs& a, int d) {
  return reinterpret_cast<uint32_t*>(a.ws_all + (int64_t)d * a.ws_bytes + a.off_sentinel);
}

// this rank's claim counters (source role): [E] claims, then [8] misc
__device__ __forceinline__ uint32_t* claims_of(const EpArgs& a, uint32_t epoch) {
  return reinterpret_cast<uint32_t*>(a.ws_all + (int64_t)a.rank * a.ws_bytes + a.src_off) + (epoch & 1) * (a.E + 8);
}

// Bounded wait until *p == want (system scope); false (latched) on timeout.
__device__ bool wait_eq_sys(const EpArgs& a, const uint32_t* p, uint32_t want, uint32_t where) {
  const unsigned long long t0 = globaltimer();
  while (ld_acquire_sys(p) != want) {
    if (globaltimer() - t0 > kWaitBudgetNs) {
      latch_error(hdr_of(a, a.rank), MOE_ERR_TIMEOUT, where);
      return false;
    }
    __nanosleep(256);
  }
  return true;
}

// Region of virtual expert v in rank d's windows: first row and rows of room.
__device__ __forceinline__ void region(const EpArgs& a, int d, int v, uint32_t epoch, int64_t* first, int64_t* room) {
  if (a.protocol == MOE_EP_FENCE) {
    const uint32_t* base = set_base(set_of(a, d, epoch), a.E, a.tiles);
    *first = (int64_t)base[v] * kTileRows;
    // the layout never exceeds the windows for valid routing (distinct
    // experts per token); a region past their end gets no room
    *room = max((int64_t)0, min((int64_t)(base[v + 1] - base[v]) * kTileRows, a.rows - *first));
  } else {
    *first = (int64_t)v * a.cap_src;
    *room = a.cap_src;
  }
}

__device__ __forceinline__ void load16(const EpArgs& a, int64_t off, float* v) {
  if (a.act == MOE_BF16) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.x) + off);
    const uint4 q0 = __ldg(p), q1 = __ldg(p + 1);
    const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.x) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 q = __ldg(p + i);
      v[4 * i] = q.x; v[4 * i + 1] = q.y; v[4 * i + 2] = q.z; v[4 * i + 3] = q.w;
    }
  }
}

__global__ void __launch_bounds__(kThreads) ep_dispatch_kernel(EpArgs a) {
  __shared__ int s_row[kMaxTopk];   // row in the owner's windows, or -1
  __shared__ int s_d[kMaxTopk];     // the owner
  __shared__ uint32_t s_epoch;
  __shared__ int s_last;
  const int tid = threadIdx.x;
  if (tid == 0) s_epoch = hdr_of(a, a.rank)->epoch_next;
  __syncthreads();
  const uint32_t epoch = s_epoch;
  // this rank's counter set and claim counters of the next epoch: zeroed now
  // (every source of the next epoch comes after this rank's combine of this
  // one, which comes after this kernel)
  {
    uint32_t* nset = set_of(a, a.rank, epoch + 1);
    const int64_t per = (a.set_words + gridDim.x - 1) / gridDim.x;
    const int64_t lo = per * blockIdx.x, hi = min(lo + per, a.set_words);
    for (int64_t i = lo + tid; i < hi; i += kThreads) nset[i] = 0u;
    if (blockIdx.x == 0) {
      uint32_t* nclaims = claims_of(a, epoch + 1);
      for (int i = tid; i < a.E + 8; i += kThreads) nclaims[i] = 0u;
    }
  }
  uint32_t* claims = claims_of(a, epoch);
  if (a.protocol == MOE_EP_FENCE && tid < a.R)   // the owners' layouts of this epoch
    wait_eq_sys(a, &hdr_of(a, tid)->layout_ready, epoch, 0x41000000u | (uint32_t)tid);
  __syncthreads();

  const int steps = a.H / kElems;
  const int span = (steps + 31) / 32 * 32;   // whole warps in every pass (8-lane block max)
  const int64_t hs = a.H / kQBlock;
  for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
    if (tid < a.k) {
      const int pair = t * a.k + tid;
      const int e = __ldg(a.idx + pair);
      int row = -1, d = 0;
      if (e >= 0 && e < a.E) {
        const uint32_t p = atomicAdd(claims + e, 1u);
        d = e / a.e_loc;
        const int v = (e % a.e_loc) * a.R + a.rank;
        int64_t first, room;
        region(a, d, v, epoch, &first, &room);
        if ((int64_t)p < room) {
          row = (int)(first + p);
          a.row_src_all[(int64_t)d * a.rows + row] = (int32_t)((int64_t)a.rank * a.t_max * a.k + pair);
        } else {
          latch_error(hdr_of(a, a.rank), MOE_ERR_CAPACITY, (uint32_t)e);
        }
      } else {
        latch_error(hdr_of(a, a.rank), MOE_ERR_INVALID_ARG, (uint32_t)pair);
      }
      a.pos[pair] = row >= 0 ? (int32_t)((int64_t)d * a.rows + row) : -1;
      s_row[tid] = row;
      s_d[tid] = d;
    }
    __syncthreads();
    for (int s = tid; s < span; s += kThreads) {
      const bool live = s < steps;
      float v[kElems];
      if (live) load16(a, (int64_t)t * a.H + (int64_t)s * kElems, v);
      else {
#pragma unroll
        for (int i = 0; i < kElems; ++i) v[i] = 0.f;
      }
      const int h0 = s * kElems;
      if (a.xq_dtype == MOE_E4M3) {
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < kElems; ++i) amax = fmaxf(amax, fabsf(v[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        if (!live) continue;
        const int pe = pow2_scale_exp(amax);
        const float inv = exp2i(-pe > -126 ? -pe : -126);
        uint32_t q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          q[i] = (uint32_t)cvt_e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv) |
                 ((uint32_t)cvt_e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv) << 16);
        const uint4 qv = make_uint4(q[0], q[1], q[2], q[3]);
        const int blk = h0 / kQBlock;
        for (int j = 0; j < a.k; ++j) {
          const int row = s_row[j];
          if (row < 0) continue;
          const int64_t g = (int64_t)s_d[j] * a.rows + row;
          *reinterpret_cast<uint4*>(a.xq_all + g * a.H + h0) = qv;
          if ((tid & 7) == 0) {
            a.xs_all[g * hs + blk] = exp2i(pe);
            uint8_t* xsf = reinterpret_cast<uint8_t*>(a.ws_all + (int64_t)s_d[j] * a.ws_bytes + a.off_xsf);
            *sf_atom_byte(xsf, row / kTileRows, a.hgroups, blk, row % kTileRows) = (uint8_t)(pe + 127);
          }
        }
      } else if (live) {
        for (int j = 0; j < a.k; ++j) {
          const int row = s_row[j];
          if (row < 0) continue;
          const int64_t g = ((int64_t)s_d[j] * a.rows + row) * a.H + h0;
          if (a.xq_dtype == MOE_BF16) {
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
              w[i] = *reinterpret_cast<uint32_t*>(&b2);
            }
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.xq_all) + g);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          } else {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.xq_all) + g);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      }
    }
    __threadfence_system();
    __syncthreads();
    if (tid < a.k && s_row[tid] >= 0) {   // count the row; the bump completing a tile publishes it
      const int d = s_d[tid];
      const int g = s_row[tid] / kTileRows;
      const uint32_t old = atomicAdd_system(set_fill(set_of(a, d, epoch), a.E) + g, 1u);
      if (old + 1 == (uint32_t)kTileRows) st_release_sys(sentinel_of(a, d) + g, (epoch << 8) | (uint32_t)kTileRows);
    }
    __syncthreads();
  }
  __threadfence_system();
  __syncthreads();

  // the last CTA closes: partial tiles, region counts and tile totals into
  // the owners' sets, then this source counted as closed by every owner
  if (tid == 0) s_last = atomicAdd(claims + a.E, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence_system();
  for (int e = tid; e < a.E; e += kThreads) {
    const int d = e / a.e_loc;
    const int v = (e % a.e_loc) * a.R + a.rank;
    int64_t first, room;
    region(a, d, v, epoch, &first, &room);
    const int64_t c = min((int64_t)ld_acquire(claims + e), room);
    uint32_t* dset = set_of(a, d, epoch);
    set_count(dset)[v] = (uint32_t)c;
    const int64_t full = c / kTileRows, rem = c % kTileRows;
    const int64_t tile0 = first / kTileRows;
    if (rem) st_release_sys(sentinel_of(a, d) + tile0 + full, (epoch << 8) | (uint32_t)rem);
    if (full + (rem ? 1 : 0)) atomicAdd_system(set_misc(dset) + kRingTotal, (uint32_t)(full + (rem ? 1 : 0)));
  }
  __threadfence_system();
  __syncthreads();
  if (tid < a.R) atomicAdd_system(set_misc(set_of(a, tid, epoch)) + kSrcDone, 1u);
  if (tid == 0) {
    Header* h = hdr_of(a, a.rank);
    h->epoch_cur = epoch;
    __threadfence();
    h->epoch_next = epoch + 1;
  }
}

// Fence, step one: this source's pair count per expert, into the owners'
// sets (pre[v]), then counted by every owner. One CTA.
__global__ void __launch_bounds__(1024) ep_count_kernel(EpArgs a) {
  extern __shared__ uint32_t hist[];   // [E]
  const int tid = threadIdx.x;
  const uint32_t epoch = hdr_of(a, a.rank)->epoch_next;
  for (int e = tid; e < a.E; e += blockDim.x) hist[e] = 0u;
  __syncthreads();
  const int64_t pairs = (int64_t)a.T * a.k;
  for (int64_t i = tid; i < pairs; i += blockDim.x) {
    const int e = __ldg(a.idx + i);
    if (e >= 0 && e < a.E) atomicAdd(hist + e, 1u);
  }
  __syncthreads();
  for (int e = tid; e < a.E; e += blockDim.x) {
    const int d = e / a.e_loc;
    set_pre(set_of(a, d, epoch), a.E, a.tiles)[(e % a.e_loc) * a.R + a.rank] = hist[e];
  }
  __threadfence_system();
  __syncthreads();
  if (tid < a.R) atomicAdd_system(set_misc(set_of(a, tid, epoch)) + kSrcCounted, 1u);
}

// Fence, step two (the owner): once all R sources' counts are in, base[v] =
// the running sum of whole tiles over v' < v, then layout_ready = epoch.
__global__ void __launch_bounds__(kThreads) ep_layout_kernel(EpArgs a) {
  __shared__ uint32_t s_warp[kThreads / 32];
  __shared__ int s_ok;
  const int tid = threadIdx.x;
  Header* h = hdr_of(a, a.rank);
  const uint32_t epoch = h->epoch_next;
  uint32_t* set = set_of(a, a.rank, epoch);
  if (tid == 0) s_ok = wait_eq_sys(a, set_misc(set) + kSrcCounted, (uint32_t)a.R, 0x42000000u) ? 1 : 0;
  __syncthreads();
  if (!s_ok) return;
  const uint32_t* pre = set_pre(set, a.E, a.tiles);
  uint32_t* base = set_base(set, a.E, a.tiles);
  const int per = (a.E + kThreads - 1) / kThreads;
  const int e0 = min(a.E, tid * per), e1 = min(a.E, e0 + per);
  uint32_t own = 0;
  for (int v = e0; v < e1; ++v) own += (ld_acquire_sys(pre + v) + kTileRows - 1) / kTileRows;
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
  for (int v = e0; v < e1; ++v) {
    base[v] = run;
    run += (ld_acquire_sys(pre + v) + kTileRows - 1) / kTileRows;
  }
  if (tid == kThreads - 1) {
    base[a.E] = run;
    if ((int64_t)run > a.tiles) latch_error(h, MOE_ERR_CAPACITY, 0x43000000u | run);
  }
  __threadfence_system();
  __syncthreads();
  if (tid == 0) st_release_sys(&h->layout_ready, epoch);
}

// The owner's expert outputs of its current epoch are complete.
__global__ void ep_publish_y_kernel(Header* h) {
  __threadfence_system();
  st_release_sys(&h->y_ready, h->epoch_cur);
}

// Every owner has published y for this rank's current epoch (bounded).
__global__ void ep_wait_y_kernel(EpArgs a) {
  const int d = threadIdx.x;
  const uint32_t epoch = hdr_of(a, a.rank)->epoch_cur;
  if (d < a.R) wait_eq_sys(a, &hdr_of(a, d)->y_ready, epoch, 0x44000000u | (uint32_t)d);
}

EpArgs make_args(const Ctx& c, const EpGeom& g, const moe_ep_windows& all) {
  EpArgs a;
  memset(&a, 0, sizeof(a));
  a.T = (int)c.s.T;
  a.H = (int)c.s.H;
  a.k = (int)c.s.topk;
  a.E = (int)c.s.E;
  a.R = g.R;
  a.rank = g.rank;
  a.e_loc = g.e_loc;
  a.protocol = g.protocol;
  a.act = c.s.act_dtype;
  a.xq_dtype = c.s.xq_dtype;
  a.t_max = g.t_max;
  a.cap_src = g.cap_src;
  a.tpe_src = g.tpe_src;
  a.rows = g.rows;
  a.hgroups = g.RL.hgroups;
  a.tiles = g.RL.tiles;
  a.set_words = (int64_t)g.RL.set_words;
  a.xq_all = (uint8_t*)all.xq;
  a.xs_all = all.xs;
  a.row_src_all = all.row_src;
  a.ws_all = (char*)all.ws;
  a.ws_bytes = (int64_t)g.ws_bytes;
  a.off_set0 = (int64_t)g.RL.off_set[0];
  a.off_set1 = (int64_t)g.RL.off_set[1];
  a.off_sentinel = (int64_t)g.RL.off_sentinel;
  a.off_xsf = (int64_t)g.RL.off_xsf;
  a.src_off = (int64_t)g.src_off;
  return a;
}

}  // namespace

cudaError_t launch_ep_count(const Ctx& c, const EpGeom& g, const int32_t* idx, const moe_ep_windows& all) {
  EpArgs a = make_args(c, g, all);
  a.idx = idx;
  ep_count_kernel<<<1, 1024, (size_t)a.E * 4, c.stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ep_layout(const Ctx& c, const EpGeom& g, const moe_ep_windows& all) {
  ep_layout_kernel<<<1, kThreads, 0, c.stream>>>(make_args(c, g, all));
  return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const Ctx& c, const EpGeom& g, const void* x, const int32_t* idx,
                               const moe_ep_windows& all, int32_t* pos) {
  EpArgs a = make_args(c, g, all);
  a.x = x;
  a.idx = idx;
  a.pos = pos;
  // at least one CTA (the close runs even without tokens); a few per SM
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(a.T, (int64_t)c.num_sms * 4));
  ep_dispatch_kernel<<<grid, kThreads, 0, c.stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ep_publish_y(const Ctx& c) {
  ep_publish_y_kernel<<<1, 1, 0, c.stream>>>(c.ws.hdr);
  return cudaGetLastError();
}

cudaError_t launch_ep_wait_y(const Ctx& c, const EpGeom& g, const moe_ep_windows& all) {
  ep_wait_y_kernel<<<1, 64, 0, c.stream>>>(make_args(c, g, all));
  return cudaGetLastError();
}

}  // namespace moe

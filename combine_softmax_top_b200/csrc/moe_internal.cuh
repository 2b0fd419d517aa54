// Internal definitions shared by the kernels and the host ABI of libmoe.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "moe.h"   // include/moe.h (the C ABI)

namespace moe {

constexpr int kTileRows = 128;   // rows per expert-window tile (sentinel granularity)
constexpr int kQBlock = 128;     // quantisation block along H or I
constexpr int kSfAtomBytes = 512;  // one scale-factor atom: 128 rows x 4 blocks
constexpr int kMaxTopk = 32;

// Waits give up after this long (ns of %globaltimer) and latch MOE_ERR_TIMEOUT.
constexpr unsigned long long kWaitBudgetNs = 200ull * 1000ull * 1000ull;

// ---- workspace layout -------------------------------------------------------
//
// [header 256 B][counter set 0][counter set 1][sentinels][ring][xsf][hsf]
//
// header : epoch_next, epoch_cur, error, error_info, epoch_plan, layout_ready,
//          y_ready (u32 each); epoch_plan is the epoch the counting pass
//          planned, read by a grouped FFN that runs beside its dispatch (before
//          epoch_cur moves on); layout_ready / y_ready are the expert-parallel
//          flags other ranks poll
// set    : misc[8] (ring_head, done, ring_total, ...) | count[E] |
//          fill[tiles] | hdone[tiles] | pre[E] | base[E + 1]
//          two sets are used alternately by consecutive dispatches; each
//          dispatch zeroes the set the following dispatch will use.
//          hdone[g] counts the finished gate/up slices of global tile g;
//          pre / base: the counting pass's expert pair counts, taken before
//          dispatch (compact windows, or a grouped FFN run beside its
//          dispatch), and each expert's first global tile (compact windows).
// A global tile g covers rows 128 g .. 128 g + 127 of the expert buffers:
// expert e's tile i is g = e * tpe + i (windows of cap rows) or base[e] + i
// (compact windows); tiles = E * tpe or the compact bound.
// sentinel[tiles] u32 : (epoch << 8) | rows of a published tile
// ring[tiles] u64     : (epoch mod 2^24) << 40 | e << 24 | g, in publication order
// xsf / hsf           : UE8M0 scale atoms of xq / hq for the block-scaled MMA,
//                       [tile][group of four 128-value blocks][512 B]; row m of
//                       the tile owns the 32-bit word at (m % 32) * 16 +
//                       (m / 32) * 4, byte b holding block 4 * group + b
struct Header {
  uint32_t epoch_next;
  uint32_t epoch_cur;
  uint32_t error;
  uint32_t error_info;
  uint32_t epoch_plan;
  uint32_t layout_ready;   // expert parallelism, Fence: epoch whose window layout is laid out here
  uint32_t y_ready;        // expert parallelism: epoch whose expert outputs y are complete here
  uint32_t pad[57];
};
static_assert(sizeof(Header) == 256, "header size");

// misc slots of a counter set (3-5 belong to the grouped FFN); kSrcDone and
// kSrcCounted count the source ranks that closed their dispatch into this
// rank's windows / wrote their pair counts here (expert parallelism)
enum MiscSlot { kRingHead = 0, kDone = 1, kRingTotal = 2, kPlanDone = 6, kSrcDone = 8, kSrcCounted = 9,
                kMiscWords = 16 };

struct Layout {
  int64_t T, H, E, k, I, cap, tpe, tiles;   // tiles: E * tpe, or the compact bound
  bool compact;                             // windows packed at offsets[e] (MOE_FLAG_COMPACT)
  int64_t hgroups, igroups;                 // ceil(H/512), ceil(I/512): scale atoms per tile
  size_t set_words;                         // u32 words of one counter set
  size_t off_set[2], off_sentinel, off_ring, off_xsf, off_hsf, total;
};

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

inline int64_t default_cap(const moe_shape& s) {
  if (s.cap_rows > 0) return s.cap_rows;
  int64_t c = ceil_div(s.T, kTileRows) * kTileRows;
  return c < kTileRows ? kTileRows : c;
}

inline Layout make_layout(const moe_shape& s) {
  Layout L{};
  L.T = s.T; L.H = s.H; L.E = s.E; L.k = s.topk; L.I = s.I;
  L.compact = (s.flags & MOE_FLAG_COMPACT) != 0;
  if (L.compact) {
    // windows rounded up to whole tiles: the T * k rows plus at most one
    // partial tile per expert
    L.tiles = ceil_div(L.T * L.k, kTileRows) + L.E;
    L.cap = L.tiles * kTileRows;   // no per-expert limit
    L.tpe = L.tiles;
  } else {
    L.cap = default_cap(s);
    L.tpe = ceil_div(L.cap, kTileRows);
    L.tiles = L.E * L.tpe;
  }
  L.hgroups = ceil_div(L.H, 4 * kQBlock);
  L.igroups = ceil_div(L.I, 4 * kQBlock);
  L.set_words = (size_t)(kMiscWords + L.E + 2 * L.tiles + 2 * L.E + 1);
  size_t off = sizeof(Header);
  for (int i = 0; i < 2; ++i) {
    L.off_set[i] = off;
    off = align_up(off + L.set_words * 4, 256);
  }
  L.off_sentinel = off;
  off = align_up(off + (size_t)L.tiles * 4, 256);
  L.off_ring = off;
  off = align_up(off + (size_t)L.tiles * 8, 256);
  L.off_xsf = off;
  if (s.xq_dtype == MOE_E4M3) off = align_up(off + (size_t)L.tiles * L.hgroups * kSfAtomBytes, 256);
  L.off_hsf = off;
  if (s.h_dtype == MOE_E4M3 && !s.identity_experts)
    off = align_up(off + (size_t)L.tiles * L.igroups * kSfAtomBytes, 256);
  L.total = off;
  return L;
}

// Device view of the workspace.
struct Ws {
  Header* hdr;
  uint32_t* set[2];
  uint32_t* sentinel;
  unsigned long long* ring;
  uint8_t* xsf;
  uint8_t* hsf;
};

inline Ws ws_view(void* base, const Layout& L) {
  char* b = (char*)base;
  Ws w;
  w.hdr = (Header*)b;
  w.set[0] = (uint32_t*)(b + L.off_set[0]);
  w.set[1] = (uint32_t*)(b + L.off_set[1]);
  w.sentinel = (uint32_t*)(b + L.off_sentinel);
  w.ring = (unsigned long long*)(b + L.off_ring);
  w.xsf = (uint8_t*)(b + L.off_xsf);
  w.hsf = (uint8_t*)(b + L.off_hsf);
  return w;
}

// ---- device helpers -----------------------------------------------------------

__device__ __forceinline__ void latch_error(Header* h, uint32_t code, uint32_t info) {
  if (atomicCAS(&h->error, 0u, code) == 0u) atomicExch(&h->error_info, info);
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long ld_acquire64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_release64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Exponent p of the smallest power of two 2^p >= amax / 448, clamped to
// [-126, 127]; 0 for amax == 0. amax is a non-negative finite fp32 value.
// 448 = 1.75 * 2^8: with amax = m * 2^e (m in [1, 2)), p = e - 8 when
// m <= 1.75 and e - 7 otherwise. Exact integer work on the bit pattern.
__device__ __forceinline__ int pow2_scale_exp(float amax) {
  uint32_t b = __float_as_uint(amax);
  if (b == 0u) return 0;
  int e = (int)((b >> 23) & 0xFF);
  if (e == 0) return -126;                      // subnormal amax
  e -= 127;
  int p = ((b & 0x7FFFFFu) > 0x600000u) ? e - 7 : e - 8;
  return p < -126 ? -126 : (p > 127 ? 127 : p);
}

__device__ __forceinline__ float exp2i(int p) {  // 2^p for p in [-126, 127]
  return __uint_as_float((uint32_t)(p + 127) << 23);
}

// Two fp32 values -> two e4m3 bytes (lo first in memory), nearest-even, satfinite.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  __nv_fp8x2_storage_t r = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
  return (uint16_t)r;
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t q) {
  __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)q, __NV_E4M3);
  return __half2float(__half(hr));
}

// Byte offset of row m's 32-bit word inside one scale-factor atom of a
// 128-row tile: 32 lanes x 16 bytes, lane m % 32, word m / 32. Byte b of the
// word holds block b of the atom's group of four.
__device__ __forceinline__ int sf_atom_offset(int m) {
  return (m & 31) * 16 + (m >> 5) * 4;
}

// Scale atom (of xsf / hsf) of tile `tile` for 128-value block `blk`, and the
// byte of row m in it.
__device__ __forceinline__ uint8_t* sf_atom_byte(uint8_t* base, int64_t tile, int64_t groups, int blk, int m) {
  return base + (tile * groups + blk / 4) * kSfAtomBytes + sf_atom_offset(m) + (blk & 3);
}

// Counter-set views.
__device__ __forceinline__ uint32_t* set_misc(uint32_t* set) { return set; }
__device__ __forceinline__ uint32_t* set_count(uint32_t* set) { return set + kMiscWords; }
__device__ __forceinline__ uint32_t* set_fill(uint32_t* set, int E) { return set + kMiscWords + E; }
__device__ __forceinline__ uint32_t* set_hdone(uint32_t* set, int E, int64_t tiles) {
  return set + kMiscWords + E + tiles;
}
// compact windows: each expert's pair count, and its first global tile
// (entry E: the tiles of all windows), both written before dispatch
__device__ __forceinline__ uint32_t* set_pre(uint32_t* set, int E, int64_t tiles) {
  return set + kMiscWords + E + 2 * tiles;
}
__device__ __forceinline__ uint32_t* set_base(uint32_t* set, int E, int64_t tiles) {
  return set + kMiscWords + 2 * E + 2 * tiles;
}

// Ring entries: 24 bits of epoch (as the sentinels), expert, global tile.
__device__ __forceinline__ unsigned long long ring_entry(uint32_t epoch, int e, int64_t g) {
  return ((unsigned long long)(epoch & 0xFFFFFFu) << 40) | ((unsigned long long)e << 24) |
         (unsigned long long)g;
}

// ---- host-side argument checks (moe_api.cu) ---------------------------------

bool aligned16(const void* p);
moe_status check_shape(const moe_shape* s);
moe_status check_bufs(const moe_shape* s, const moe_dispatch_bufs* b, bool need_h);

// ---- launchers (host, internal) --------------------------------------------

// The shape the dispatch, grouped FFN and combine kernels work on: a shared
// expert is expert E of E + 1 and every token's slot k of k + 1 (weight 1).
inline moe_shape effective_shape(const moe_shape& s) {
  moe_shape e = s;
  if (s.flags & MOE_FLAG_SHARED_EXPERT) {
    e.E += 1;
    e.topk += 1;
  }
  return e;
}

struct Ctx {
  moe_shape s;        // effective shape (see effective_shape)
  int64_t routed_E;   // logits per token
  int64_t routed_k;   // experts chosen by the router
  int shared;         // 1: slot routed_k of every token is the shared expert
  Layout L;
  Ws ws;
  cudaStream_t stream;
  int num_sms;          // grid of the persistent kernels (all SMs, or a partition's share)
  bool streaming = false;   // grouped FFN launched beside its dispatch (counts from the counting pass)
  int ep_ranks = 0;     // grouped FFN of one rank under expert parallelism: windows of
                        // E_loc * R regions (one per local expert and source rank), R closes awaited
};

// ---- expert parallelism (ep.cu) ----------------------------------------------
//
// R ranks, rank d owning experts [d E_loc, (d + 1) E_loc), E_loc = E / R.
// Every rank receives into windows of V = E virtual experts, v = el * R + src
// (local expert el, source rank src): rank-major regions per source inside
// each expert's block, so that each source fills its own regions without
// asking anyone where (no metadata exchanged first). Sentinel protocol:
// regions of cap_src = round_up(t_max, 128) rows. Fence protocol: every
// source's pair counts are written to the receivers first, each receiver lays
// its regions out back to back in whole tiles (as compact windows), and
// sources place rows at exact offsets. All ranks' windows and workspaces are
// reached through rank-major address ranges (rank d's part at d * stride).
struct EpGeom {
  int R, rank, e_loc, protocol;
  int64_t t_max, cap_src, tpe_src, rows;   // rows of one rank's windows
  moe_shape rs;          // the receiver's shape: E = V virtual experts
  Layout RL;             // the receiver's workspace layout
  size_t src_off;        // the source's claim counters: [2][E + 8] u32 after RL.total
  size_t ws_bytes;       // one rank's workspace
};

inline EpGeom make_ep_geom(const moe_shape& s, const moe_ep& ep) {
  EpGeom g{};
  g.R = ep.ranks;
  g.rank = ep.rank;
  g.e_loc = (int)(s.E / ep.ranks);
  g.protocol = ep.protocol;
  g.t_max = ep.t_max;
  g.rs = s;
  g.rs.E = s.E;                                   // V = E_loc * R = E
  if (ep.protocol == MOE_EP_FENCE) {
    g.rs.flags = MOE_FLAG_COMPACT;
    g.rs.T = ep.t_max * ep.ranks;
    g.rs.topk = s.topk < g.e_loc ? s.topk : g.e_loc;   // pairs one token sends one rank
    g.rs.cap_rows = 0;
  } else {
    g.rs.flags = 0;
    g.rs.T = ep.t_max;
    g.rs.cap_rows = ceil_div(ep.t_max > 0 ? ep.t_max : 1, kTileRows) * kTileRows;
  }
  g.RL = make_layout(g.rs);
  g.cap_src = g.RL.cap;
  g.tpe_src = g.RL.tpe;
  g.rows = g.RL.tiles * kTileRows;
  g.src_off = align_up(g.RL.total, 256);
  g.ws_bytes = align_up(g.src_off + 2 * (size_t)(s.E + 8) * 4, 256);
  return g;
}

cudaError_t launch_route(const Ctx& c, const float* logits, int32_t* idx, float* w);
// write_sf: also write the e4m3 scale atoms the tensor-core FFN reads;
// planned: the counting pass already ran (launch_plan), else compact windows
// run it first
cudaError_t launch_dispatch(const Ctx& c, const void* x, const int32_t* idx,
                            const moe_dispatch_bufs& b, bool write_sf = true, bool planned = false);
// The counting pass: per-expert pair counts (and, with compact windows, the
// window layout) into the counter set of the next dispatch, and that
// dispatch's epoch into Header::epoch_plan.
cudaError_t launch_plan(const Ctx& c, const int32_t* idx);
// The shared-memory-staged combine for many-token layers; false when the
// shape does not suit it (nothing launched), else *err holds the launch result.
bool launch_combine_tma(const Ctx& c, const moe_dispatch_bufs& b, const void* y, const float* topk_w, void* out,
                        cudaError_t* err);
cudaError_t launch_combine(const Ctx& c, const moe_dispatch_bufs& b, const void* y,
                           const float* topk_w, void* out);
cudaError_t launch_ffn_simt(const Ctx& c, const moe_dispatch_bufs& b, const moe_weights& w,
                            void* y);
cudaError_t launch_ffn_tc(const Ctx& c, const moe_dispatch_bufs& b, const moe_weights& w,
                          void* y);
bool ffn_tc_supported(const moe_shape& s);
// The CTA-pair grouped FFN (e4m3 weights, many rows per expert).
bool ffn_pair_supported(const Ctx& c);
cudaError_t launch_ffn_pair(const Ctx& c, const moe_dispatch_bufs& b, const moe_weights& w, void* y);

// expert parallelism (ep.cu); g describes this rank, `all` the rank-major ranges
cudaError_t launch_ep_count(const Ctx& c, const EpGeom& g, const int32_t* idx, const moe_ep_windows& all);
cudaError_t launch_ep_layout(const Ctx& c, const EpGeom& g, const moe_ep_windows& all);
cudaError_t launch_ep_dispatch(const Ctx& c, const EpGeom& g, const void* x, const int32_t* idx,
                               const moe_ep_windows& all, int32_t* pos);
cudaError_t launch_ep_publish_y(const Ctx& c);
cudaError_t launch_ep_wait_y(const Ctx& c, const EpGeom& g, const moe_ep_windows& all);

}  // namespace moe

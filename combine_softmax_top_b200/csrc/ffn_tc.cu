// Grouped expert FFN on the 5th-generation tensor cores (tcgen05), one
// persistent kernel for gate/up + SwiGLU + requantisation and down.
//
// Pages: the compute partition runs operand-swapped tcgen05 block-scaled MMA
// with SwiGLU and requantisation fused (GC-MoE feed item, "Full text";
// explainer, "Two MMA Implementations in the Compute Partition"): the weights
// are the MMA's A operand (M = 128 output features) and the few tokens of an
// expert its N operand, which suits small per-expert token counts. The GEMM
// reads the dispatched rows in place (NVLinkOneSided abstract) and starts a
// tile once its sentinel is published (token-ring handshake, explainer,
// "Three-Node CUDA Graph and token-ring Handshake").
//
// Work units, processed in one fixed order by a persistent grid:
//   gate/up : (ring slot, 128-feature slice of I) -> h rows of that slice
//   down    : (ring slot, 128-feature slice of H) -> y rows of that slice
// All gate/up units come before all down units; a down unit waits until the
// I/128 gate/up units of its tile have stored h (per-slot counter).
//
// Per CTA (192 threads): warp 0 streams K slabs of 128 bytes into a 4-stage
// shared-memory ring with TMA (weights with an evict-first hint), and for
// e4m3 builds the weights' UE8M0 scale atoms and bulk-copies the tokens';
// warp 1 issues tcgen05.mma (kind::f16 for bf16, kind::mxf8f6f4.block_scale
// for e4m3) into tensor memory; warps 2-5 read the fp32 accumulators back with
// tcgen05.ld, apply SwiGLU and the per-128 requantisation (or round y to
// bf16) and store. Every wait is bounded: on expiry the kernel latches
// MOE_ERR_TIMEOUT, drains its copies and MMAs, frees tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kSlab = 128;                 // K bytes per stage (one 128-byte swizzle row)
constexpr int kABytes = 128 * kSlab;       // 128 weight rows
constexpr int kBBytes = 128 * kSlab;       // up to 128 token rows
constexpr int kOffA1 = kABytes;
constexpr int kOffB = 2 * kABytes;
constexpr int kOffSfa0 = 2 * kABytes + kBBytes;
constexpr int kOffSfa1 = kOffSfa0 + kSfAtomBytes;
constexpr int kOffSfb = kOffSfa1 + kSfAtomBytes;
constexpr int kStageStride = 51200;        // 50688 rounded up to 1024
static_assert(kOffSfb + kSfAtomBytes <= kStageStride, "stage layout");
constexpr int kBarOffset = kStages * kStageStride;
constexpr int kSmemBytes = kBarOffset + 1024 /* barriers, flags, reductions */ + 1024 /* alignment slack */;

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColG = 0, kColU = 128, kColSfa0 = 256, kColSfa1 = 260, kColSfb = 264;

struct TcParams {
  CUtensorMap tm_wg, tm_wu, tm_wd, tm_x, tm_h;
  const float* sg;
  const float* su;
  const float* sd;
  void* hq;
  float* hs;
  void* y;
  Ws ws;
  int H, I, E, cap, tpe;
  int n_islices, n_hslices;  // I/128, H/128
  int nk1, nk2;              // K slabs of gate/up (over H) and down (over I)
  int kelems;                // elements per slab
  int64_t tiles;
};

struct Unit {
  bool down;
  uint32_t slot;
  int slice;
};

__device__ __forceinline__ Unit unit_of(uint32_t u, uint32_t n1, int n_islices, int n_hslices) {
  Unit r;
  r.down = u >= n1;
  const uint32_t v = r.down ? u - n1 : u;
  const int ns = r.down ? n_hslices : n_islices;
  r.slot = v / ns;
  r.slice = (int)(v % ns);
  return r;
}

// Bounded wait on an mbarrier phase; false on timeout (latched) or abort.
__device__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, Header* hdr,
                         uint32_t where) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitBudgetNs) {
      latch_error(hdr, MOE_ERR_TIMEOUT, where);
      *abort_flag = 1;
      return false;
    }
  }
}

// The tile behind ring slot `slot` of this epoch: expert, tile index, rows.
__device__ bool fetch_tile(const TcParams& p, uint32_t epoch, uint32_t slot, volatile int* abort_flag,
                           int* e, int* tile, int* rows) {
  const unsigned long long t0 = globaltimer();
  unsigned long long ent;
  while (true) {
    ent = ld_acquire64(p.ws.ring + slot);
    if ((uint32_t)(ent >> 32) == epoch) break;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitBudgetNs) {
      latch_error(p.ws.hdr, MOE_ERR_TIMEOUT, 0x10000000u | slot);
      *abort_flag = 1;
      return false;
    }
    __nanosleep(128);
  }
  *e = (int)((ent >> 16) & 0xFFFF);
  *tile = (int)(ent & 0xFFFF);
  if (*e >= p.E || *tile >= p.tpe) {          // never published: a corrupt workspace
    latch_error(p.ws.hdr, MOE_ERR_INVALID_ARG, 0x11000000u | slot);
    *abort_flag = 1;
    return false;
  }
  const uint32_t* sp = p.ws.sentinel + (int64_t)(*e) * p.tpe + *tile;
  while (true) {
    const uint32_t s = ld_acquire(sp);
    if ((s >> 8) == (epoch & 0xFFFFFFu)) {
      *rows = (int)(s & 0xFF);
      if (*rows < 1 || *rows > kTileRows) {   // never published: a corrupt workspace
        latch_error(p.ws.hdr, MOE_ERR_INVALID_ARG, 0x21000000u | slot);
        *abort_flag = 1;
        return false;
      }
      return true;
    }
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitBudgetNs) {
      latch_error(p.ws.hdr, MOE_ERR_TIMEOUT, 0x20000000u | slot);
      *abort_flag = 1;
      return false;
    }
    __nanosleep(128);
  }
}

// Wait until `count` reaches `target` (acquire), bounded.
__device__ bool wait_count(const uint32_t* count, uint32_t target, volatile int* abort_flag, Header* hdr,
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

__device__ __forceinline__ float silu(float g) { return g / (1.f + expf(-g)); }

__device__ __forceinline__ uint32_t ue8m0_word(float s) {
  return ((__float_as_uint(s) >> 23) & 0xFFu) * 0x01010101u;
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1) ffn_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOffset);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* epi_info = reinterpret_cast<int*>(tmem_slot + 4);       // ok, e, tile, rows
  float* red = reinterpret_cast<float*>(tmem_slot + 8);        // [4 warps][16 tokens]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(full + s, 1);
      ptx::mbar_init(empty + s, 1);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(acc_empty, 1);
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const uint32_t epoch = p.ws.hdr->epoch_cur;
  uint32_t* set = p.ws.set[epoch & 1];
  const uint32_t ntiles = ld_acquire(set_misc(set) + kRingTotal);
  uint32_t* hdone = set_hdone(set, p.E, p.tiles);
  const uint32_t n1 = ntiles * (uint32_t)p.n_islices;
  const uint32_t total = n1 + ntiles * (uint32_t)p.n_hslices;
  Header* hdr = p.ws.hdr;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&p.tm_wg);
      ptx::prefetch_tmap(&p.tm_wu);
      ptx::prefetch_tmap(&p.tm_wd);
      ptx::prefetch_tmap(&p.tm_x);
      ptx::prefetch_tmap(&p.tm_h);
    }
    const uint64_t pol = ptx::policy_evict_first();
    uint32_t stage = 0, phase = 0;
    uint32_t armed = 0, armed_parity = 0;   // per stage: a load is outstanding / its phase parity
    bool ok = true;
    for (uint32_t u = blockIdx.x; ok && u < total; u += gridDim.x) {
      const Unit un = unit_of(u, n1, p.n_islices, p.n_hslices);
      int e = 0, tile = 0, rows = 0;
      int good = 1;
      if (lane == 0) {
        good = fetch_tile(p, epoch, un.slot, abort_flag, &e, &tile, &rows);
        if (good && un.down)
          good = wait_count(hdone + un.slot, (uint32_t)p.n_islices, abort_flag, hdr, 0x30000000u | un.slot);
        ptx::fence_proxy_async_global();   // rows written by other CTAs -> TMA reads
      }
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) { ok = false; break; }
      e = __shfl_sync(0xffffffffu, e, 0);
      tile = __shfl_sync(0xffffffffu, tile, 0);
      rows = __shfl_sync(0xffffffffu, rows, 0);
      const int N = (rows + 15) & ~15;
      const int nk = un.down ? p.nk2 : p.nk1;
      const int arow = e * (un.down ? p.H : p.I) + un.slice * 128;
      const int row0 = e * p.cap + tile * kTileRows;
      const int64_t tile_g = (int64_t)e * p.tpe + tile;
      const uint32_t tx = (un.down ? 1u : 2u) * kABytes + (uint32_t)N * kSlab + (kFp8 ? kSfAtomBytes : 0u);
      for (int kb = 0; kb < nk; ++kb) {
        int w_ok = 1;
        if (lane == 0) w_ok = wait_bar(empty + stage, phase ^ 1u, abort_flag, hdr, 0x40000000u | stage);
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        __syncwarp();
        uint8_t* st = smem + stage * kStageStride;
        if constexpr (kFp8) {
          // weight scale atoms: one scale for the whole 128 x 128 block
          if (un.down) {
            const float s0 = __ldg(p.sd + ((int64_t)e * p.n_hslices + un.slice) * (p.I / 128) + kb);
            const uint32_t w0 = ue8m0_word(s0);
            reinterpret_cast<uint4*>(st + kOffSfa0)[lane] = make_uint4(w0, w0, w0, w0);
          } else {
            const int64_t si = ((int64_t)e * p.n_islices + un.slice) * (p.H / 128) + kb;
            const uint32_t w0 = ue8m0_word(__ldg(p.sg + si));
            const uint32_t w1 = ue8m0_word(__ldg(p.su + si));
            reinterpret_cast<uint4*>(st + kOffSfa0)[lane] = make_uint4(w0, w0, w0, w0);
            reinterpret_cast<uint4*>(st + kOffSfa1)[lane] = make_uint4(w1, w1, w1, w1);
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(full + stage, tx);
          const int kx = kb * p.kelems;
          if (un.down) {
            ptx::tma_load_2d_hint(st, &p.tm_wd, full + stage, kx, arow, pol);
          } else {
            ptx::tma_load_2d_hint(st, &p.tm_wg, full + stage, kx, arow, pol);
            ptx::tma_load_2d_hint(st + kOffA1, &p.tm_wu, full + stage, kx, arow, pol);
          }
          const void* tmb = un.down ? (const void*)&p.tm_h : (const void*)&p.tm_x;
          for (int j = 0; j < N / 16; ++j) ptx::tma_load_2d(st + kOffB + j * 2048, tmb, full + stage, kx, row0 + 16 * j);
          if constexpr (kFp8) {
            const uint8_t* sf = un.down ? p.ws.hsf + (tile_g * (p.I / 128) + kb) * kSfAtomBytes
                                        : p.ws.xsf + (tile_g * (p.H / 128) + kb) * kSfAtomBytes;
            ptx::bulk_load(st + kOffSfb, sf, kSfAtomBytes, full + stage);
          }
        }
        __syncwarp();
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
    // drain: every load this warp started has landed before the CTA exits
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
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    uint32_t stage = 0, phase = 0, acc_phase = 0;
    bool ok = true;
    for (uint32_t u = blockIdx.x; ok && u < total; u += gridDim.x) {
      const Unit un = unit_of(u, n1, p.n_islices, p.n_hslices);
      int rows = 0, good = 1;
      if (lane == 0) {
        int e, tile;
        good = fetch_tile(p, epoch, un.slot, abort_flag, &e, &tile, &rows);
        if (good) good = wait_bar(acc_empty, acc_phase ^ 1u, abort_flag, hdr, 0x50000000u);
      }
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) { ok = false; break; }
      rows = __shfl_sync(0xffffffffu, rows, 0);
      ptx::tc_fence_after();
      const int N = (rows + 15) & ~15;
      const int nk = un.down ? p.nk2 : p.nk1;
      const uint32_t idesc = kFp8 ? ptx::idesc_mxf8(128, N, 0) : ptx::idesc_bf16(128, N);
      for (int kb = 0; kb < nk; ++kb) {
        int w_ok = 1;
        if (lane == 0) w_ok = wait_bar(full + stage, phase, abort_flag, hdr, 0x60000000u | stage);
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        ptx::tc_fence_after();
        if (lane == 0) {
          uint8_t* st = smem + stage * kStageStride;
          if constexpr (kFp8) {
            // 32 rows x 16 bytes, no swizzle: 8-row core matrices 128 bytes apart
            ptx::tmem_cp_32x128b_x4(tmem + kColSfa0, ptx::smem_desc(ptx::smem_u32(st + kOffSfa0), 16, 128, ptx::kLayoutNone));
            if (!un.down)
              ptx::tmem_cp_32x128b_x4(tmem + kColSfa1, ptx::smem_desc(ptx::smem_u32(st + kOffSfa1), 16, 128, ptx::kLayoutNone));
            ptx::tmem_cp_32x128b_x4(tmem + kColSfb, ptx::smem_desc(ptx::smem_u32(st + kOffSfb), 16, 128, ptx::kLayoutNone));
          }
          const uint64_t a0 = ptx::desc_kmajor_sw128(st);
          const uint64_t a1 = ptx::desc_kmajor_sw128(st + kOffA1);
          const uint64_t b = ptx::desc_kmajor_sw128(st + kOffB);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
            const uint64_t off = (uint64_t)(kk * 32) >> 4;   // 32 bytes of K per MMA
            if constexpr (kFp8) {
              ptx::mma_mxf8(tmem + kColG, a0 + off, b + off, idesc, tmem + kColSfa0, tmem + kColSfb, acc);
              if (!un.down)
                ptx::mma_mxf8(tmem + kColU, a1 + off, b + off, idesc, tmem + kColSfa1, tmem + kColSfb, acc);
            } else {
              ptx::mma_f16(tmem + kColG, a0 + off, b + off, idesc, acc);
              if (!un.down) ptx::mma_f16(tmem + kColU, a1 + off, b + off, idesc, acc);
            }
          }
          ptx::mma_commit(empty + stage);   // frees the stage once these MMAs are done
        }
        __syncwarp();
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (lane == 0) ptx::mma_commit(acc_full);
      __syncwarp();
      acc_phase ^= 1u;
    }
    // drain: all MMAs and copies issued by this warp are complete
    if (lane == 0) {
      ptx::mma_commit(drain);
      const unsigned long long t0 = globaltimer();
      while (!ptx::mbar_try_wait(drain, 0)) {
        if (globaltimer() - t0 > kWaitBudgetNs) break;
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int f = q * 32 + lane;            // output feature within the slice
    const int et = threadIdx.x - 64;        // 0..127
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint32_t acc_phase = 0;
    for (uint32_t u = blockIdx.x; u < total; u += gridDim.x) {
      const Unit un = unit_of(u, n1, p.n_islices, p.n_hslices);
      if (et == 0) {
        int e = 0, tile = 0, rows = 0;
        int good = fetch_tile(p, epoch, un.slot, abort_flag, &e, &tile, &rows);
        if (good) good = wait_bar(acc_full, acc_phase, abort_flag, hdr, 0x70000000u);
        epi_info[0] = good; epi_info[1] = e; epi_info[2] = tile; epi_info[3] = rows;
      }
      ptx::named_barrier(1, 128);
      const int good = epi_info[0], e = epi_info[1], tile = epi_info[2], rows = epi_info[3];
      ptx::named_barrier(1, 128);
      if (!good) break;
      while (!ptx::mbar_try_wait(acc_full, acc_phase)) {}   // completed: returns at once
      ptx::tc_fence_after();
      const int64_t row0 = (int64_t)e * p.cap + (int64_t)tile * kTileRows;
      const int64_t tile_g = (int64_t)e * p.tpe + tile;
      for (int n0 = 0; n0 < rows; n0 += 16) {
        uint32_t g[16], uu[16];
        ptx::tmem_ld_x16(tmem + lane_base + kColG + n0, g);
        if (!un.down) ptx::tmem_ld_x16(tmem + lane_base + kColU + n0, uu);
        ptx::tmem_wait_ld();
        const int nv = min(16, rows - n0);
        if (un.down) {
          __nv_bfloat16* yp = reinterpret_cast<__nv_bfloat16*>(p.y) + (row0 + n0) * p.H + un.slice * 128 + f;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < nv) yp[(int64_t)j * p.H] = __float2bfloat16_rn(__uint_as_float(g[j]));
          continue;
        }
        float h[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) h[j] = silu(__uint_as_float(g[j])) * __uint_as_float(uu[j]);
        if constexpr (kFp8) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float m = fabsf(h[j]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) red[q * 16 + j] = m;
          }
          ptx::named_barrier(1, 128);
          uint8_t* hp = reinterpret_cast<uint8_t*>(p.hq) + (row0 + n0) * p.I + un.slice * 128 + f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float amax = fmaxf(fmaxf(red[j], red[16 + j]), fmaxf(red[32 + j], red[48 + j]));
            const int pe = pow2_scale_exp(amax);
            if (j < nv) {
              const uint16_t b2 = cvt_e4m3x2(h[j] * exp2i(-pe > -126 ? -pe : -126), 0.f);
              hp[(int64_t)j * p.I] = (uint8_t)(b2 & 0xFF);
              if (f == 0) {
                const int64_t r = row0 + n0 + j;
                p.hs[r * (p.I / 128) + un.slice] = exp2i(pe);
                // scale atom of this tile and slice (row n0 + j of the tile)
                *reinterpret_cast<uint32_t*>(p.ws.hsf + (tile_g * (p.I / 128) + un.slice) * kSfAtomBytes +
                                             sf_atom_offset(n0 + j)) = (uint32_t)(pe + 127) * 0x01010101u;
              }
            }
          }
          ptx::named_barrier(1, 128);     // red[] is reused by the next chunk
        } else {
          __nv_bfloat16* hp = reinterpret_cast<__nv_bfloat16*>(p.hq) + (row0 + n0) * p.I + un.slice * 128 + f;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < nv) hp[(int64_t)j * p.I] = __float2bfloat16_rn(h[j]);
        }
      }
      // accumulators consumed: let the MMA warp start the next unit
      ptx::tc_fence_before();
      ptx::named_barrier(1, 128);
      if (et == 0) ptx::mbar_arrive(acc_empty);
      acc_phase ^= 1u;
      if (!un.down) {
        // publish this slice of h to the down units of the same tile
        __threadfence();
        ptx::named_barrier(1, 128);
        if (et == 0) atomicAdd(hdone + un.slot, 1u);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host side ------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2-D row-major [rows, cols] tensor, boxes of (box_cols x box_rows), 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, bool fp8, int64_t cols, int64_t rows, int box_cols,
               int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int elem = fp8 ? 1 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * elem)};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool kFp8>
cudaError_t launch_typed(const Ctx& c, const moe_dispatch_bufs& b, const moe_weights& w, void* y) {
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(ffn_tc_kernel<kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  TcParams p;
  memset(&p, 0, sizeof(p));
  const int64_t H = c.s.H, I = c.s.I, E = c.s.E, rows = E * c.L.cap;
  const int kel = kFp8 ? 128 : 64;
  if (!make_tmap(&p.tm_wg, w.w_gate, kFp8, H, E * I, kel, 128) ||
      !make_tmap(&p.tm_wu, w.w_up, kFp8, H, E * I, kel, 128) ||
      !make_tmap(&p.tm_wd, w.w_down, kFp8, I, E * H, kel, 128) ||
      !make_tmap(&p.tm_x, b.xq, kFp8, H, rows, kel, 16) ||
      !make_tmap(&p.tm_h, b.hq, kFp8, I, rows, kel, 16))
    return cudaErrorInvalidValue;
  p.sg = w.s_gate;
  p.su = w.s_up;
  p.sd = w.s_down;
  p.hq = b.hq;
  p.hs = b.hs;
  p.y = y;
  p.ws = c.ws;
  p.H = (int)H;
  p.I = (int)I;
  p.E = (int)E;
  p.cap = (int)c.L.cap;
  p.tpe = (int)c.L.tpe;
  p.n_islices = (int)(I / 128);
  p.n_hslices = (int)(H / 128);
  p.kelems = kel;
  p.nk1 = (int)(H / kel);
  p.nk2 = (int)(I / kel);
  p.tiles = c.L.tiles;
  ffn_tc_kernel<kFp8><<<c.num_sms, kThreads, kSmemBytes, c.stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

bool ffn_tc_supported(const moe_shape& s) {
  if (s.identity_experts) return false;
  const bool bf16 = s.xq_dtype == MOE_BF16 && s.weight_dtype == MOE_BF16 && s.h_dtype == MOE_BF16 &&
                    s.y_dtype == MOE_BF16;
  const bool fp8 = s.xq_dtype == MOE_E4M3 && s.weight_dtype == MOE_E4M3 && s.h_dtype == MOE_E4M3 &&
                   s.y_dtype == MOE_BF16;
  return (bf16 || fp8) && s.H % 128 == 0 && s.I % 128 == 0;
}

cudaError_t launch_ffn_tc(const Ctx& c, const moe_dispatch_bufs& b, const moe_weights& w, void* y) {
  return c.s.weight_dtype == MOE_E4M3 ? launch_typed<true>(c, b, w, y) : launch_typed<false>(c, b, w, y);
}

}  // namespace moe

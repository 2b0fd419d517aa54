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
//   gate/up : (token tile, 128-feature slice of I) -> h rows of that slice
//   down    : (token tile, 128-feature slice of H, or two slices sharing the
//             token tile) -> y rows
// All gate/up units come before all down units; a down unit waits until the
// I/128 gate/up units of its tile have stored h (per-tile counter).
//
// Per CTA (352 threads): warp 10 schedules jobs; warp 0 streams K slabs of
// 128 bytes into a 4-, 5- or 6-stage shared-memory ring with TMA (token tiles
// of up to 128, 64 or 16 rows), and for e4m3 weights builds their UE8M0 scale
// atoms, for MX FP4 weights bulk-copies theirs, and bulk-copies the tokens';
// warp 1 issues tcgen05.mma (kind::f16 for bf16, kind::mxf8f6f4.block_scale
// for e4m3 or E2M1 weights against e4m3 tokens) into tensor memory; warps 2-9
// read the fp32 accumulators back with tcgen05.ld, apply SwiGLU and the
// per-128 requantisation (or round y to bf16) and store. The producer and MMA
// warps run warp-uniform loops and one elected lane issues each copy, MMA and
// commit. Every wait is bounded: on expiry the kernel latches
// MOE_ERR_TIMEOUT, drains its copies and MMAs, frees tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "ffn_common.cuh"

namespace moe {
namespace {

using namespace ffn;

// With 128-row tiles, an expert's last tile of at most kTailMax rows joins
// the tile before it: one job of up to 128 + kTailMax rows.
constexpr int kTailMax = 32;

// Shared-memory stage for a variant whose token tiles hold up to kBRows rows:
// A0 | A1 | B (kBRows (+ kTailMax) x 128 B, or two slabs of N rows) | SFA0 |
// SFA1 | SFB0 | SFB1 (the joined tail's token scales).
template <int kBRows>
struct Stage {
  static constexpr int kBRowsMax = kBRows + (kBRows > 64 ? kTailMax : 0);
  static constexpr int kOffA1 = kABytes;
  static constexpr int kOffB = 2 * kABytes;
  static constexpr int kOffSfa0 = kOffB + kBRowsMax * kSlab;
  static constexpr int kOffSfa1 = kOffSfa0 + kSfAtomBytes;
  static constexpr int kOffSfb0 = kOffSfa1 + kSfAtomBytes;
  static constexpr int kOffSfb1 = kOffSfb0 + kSfAtomBytes;
  static constexpr int kStride = (kOffSfb1 + kSfAtomBytes + 1023) / 1024 * 1024;
  static constexpr int kStages = (kMaxDynSmem - kCtlBytes - kTileTabBytes - 1024) / kStride;
  static constexpr int kBarOffset = kStages * kStride;
  static constexpr int kSmemBytes = kBarOffset + kCtlBytes + kTileTabBytes + 1024 /* alignment slack */;
  static_assert(kStages >= 3, "pipeline depth");
  static_assert(kBRows <= 64 || kStages >= 4, "the joined tail keeps four stages");
};

constexpr uint32_t kTmemCols = 512;
// accumulators: two 128-column slots at columns 0 and 128 (a job with a joined
// tail: gate at 0, up at N, N <= 128 + kTailMax); scale factors from column
// 448, the tokens' over 8 columns (256 rows)
constexpr uint32_t kColSfa0 = 448, kColSfa1 = 452, kColSfb0 = 456;


struct TcParams {
  CUtensorMap tm_wg, tm_wu, tm_wd;
  CUtensorMap tm_x[4], tm_h[4];   // token rows in boxes of 16, 32, 64, 128 rows
  const void* sg;   // weight scales: fp32 per 128 x 128 block (e4m3) or UE8M0 atoms (e2m1)
  const void* su;
  const void* sd;
  void* hq;
  float* hs;
  void* y;
  Ws ws;
  int H, I, E, cap, tpe;
  int compact;               // expert windows start at base[e] tiles (set_base)
  int streaming;             // launched beside its dispatch: the counting pass's epoch and
                             // counts, no closed tile total
  int R;                     // windows per weight expert: 1, or the source ranks of expert
                             // parallelism (virtual expert v uses the weights of v / R)
  int ep_sources;            // expert parallelism: wait for this many closed sources (else 0)
  int n_islices, n_hslices;  // I/128, H/128
  int nk1, nk2;              // K slabs of gate/up (over H) and down (over I)
  int kelems;                // elements per slab
  int hgroups, igroups;      // scale atoms per tile along H and I (groups of 4 blocks)
  int64_t tiles;
};

// One queue entry: a chunk of <= kBRows rows of one tile, for one 128-feature
// slice, in one phase.
struct Job {
  int e, tile, slice, rows, row_off, kind, nslab, slot;
  int pair;   // down job over two 128-feature slices of H (slice, slice + 1)
  int wide;   // tile `tile` with the expert's short last tile joined (rows > 128)
};

__device__ __forceinline__ int4 pack_job(const Job& j) {
  return make_int4(j.e, j.tile | (j.slice << 16),
                   j.rows | (j.row_off << 8) | (j.kind << 16) | (j.nslab << 20) | (j.pair << 24) | (j.wide << 25),
                   j.slot);
}

__device__ __forceinline__ Job unpack_job(int4 v) {
  Job j;
  j.e = v.x;
  j.tile = v.y & 0xFFFF;
  j.slice = (v.y >> 16) & 0xFFFF;
  j.rows = v.z & 0xFF;
  j.row_off = (v.z >> 8) & 0xFF;
  j.kind = (v.z >> 16) & 0xF;
  j.nslab = (v.z >> 20) & 0xF;
  j.pair = (v.z >> 24) & 0x1;
  j.wide = (v.z >> 25) & 0x1;
  j.slot = v.w;
  return j;
}

template <int kW, int kBRows>
__global__ void __launch_bounds__(kThreads, 1) ffn_tc_kernel(const __grid_constant__ TcParams p) {
  constexpr bool kFp8 = kW != kWBf16;   // block-scaled MMA, e4m3 tokens
  constexpr bool kW4 = kW == kWE2m1;    // 4-bit weights
  using S = Stage<kBRows>;
  constexpr int kStages = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ctl = smem + S::kBarOffset;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;       // [2] per accumulator slot
  uint64_t* acc_empty = acc_full + 2;         // [2]
  uint64_t* drain = acc_empty + 2;
  uint64_t* uq_full = drain + 1;              // [kUQ] job queue
  uint64_t* uq_empty = uq_full + kUQ;         // [kUQ]
  static_assert((2 * kStages + 5 + 2 * kUQ) * 8 <= 320, "barriers fit before the job queue");
  int4* uq = reinterpret_cast<int4*>(ctl + 320);               // [kUQ] packed jobs
  int4* epi_job = reinterpret_cast<int4*>(ctl + 448);          // job broadcast to the epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 464);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 468);
  float* red = reinterpret_cast<float*>(ctl + 512);            // [2 sets][4 warps][32 tokens]
  float* sinv = reinterpret_cast<float*>(ctl + 1536);          // [2 sets][32 tokens] 1 / scale

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(full + s, 1);
      ptx::mbar_init(empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(acc_full + s, 1);
      ptx::mbar_init(acc_empty + s, 1);
    }
    ptx::mbar_init(drain, 1);
    for (int q = 0; q < kUQ; ++q) {
      ptx::mbar_init(uq_full + q, 1);
      ptx::mbar_init(uq_empty + q, 3);   // producer, MMA issuer, epilogue
    }
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

  // Beside its dispatch (streaming), the epoch is the one the counting pass
  // planned and the per-expert counts are its counts; tiles are taken as
  // their sentinels appear, before the dispatch has closed. After the
  // dispatch, the epoch it closed and its final counts and tile total.
  const uint32_t epoch = p.streaming ? p.ws.hdr->epoch_plan : p.ws.hdr->epoch_cur;
  uint32_t* set = p.ws.set[epoch & 1];
  uint32_t* misc = set_misc(set);
  const uint32_t ntiles_early = (p.streaming || p.ep_sources) ? 0u : ld_acquire(misc + kRingTotal);
  const uint32_t gen = ld_acquire(misc + kFfnGen);   // FFN calls already made on this dispatch
  uint32_t* hdone = set_hdone(set, p.E, p.tiles);
  // down units cover two slices of H each when tiles are large (the two share
  // the token tile, like gate and up)
  // (and with the 16-row variant, whose stage has room for one token slab
  // only: a pair keeps two weight tiles in every stage)
  const int dpair = ((kBRows > 64 || kBRows <= 16) && (p.n_hslices & 1) == 0) ? 2 : 1;
  Header* hdr = p.ws.hdr;

  // Take job i from the queue (one lane of a consumer role).
  auto take_job = [&](uint32_t i, Job* out) -> bool {
    const uint32_t q = i % kUQ, ph = (i / kUQ) & 1u;
    if (!wait_bar(uq_full + q, ph, abort_flag, hdr, 0x80000000u | q)) return false;
    *out = unpack_job(uq[q]);
    ptx::mbar_arrive(uq_empty + q);
    return true;
  };

  if (warp == kSchedWarp) {
    // ---------------------------------------------------------------- scheduler
    // Units, expert-major: for each expert, for each 128-feature slice, every
    // tile of that expert (all gate/up units before all down units), handed
    // out in that order from one global counter, so that CTAs that finish
    // early take more units. CTAs working at the same time thus hold the tiles
    // of one expert with the same weight slice and share it in L2.
    // For each unit the scheduler waits for the tile's sentinel (and a down
    // unit's h), splits the tile into chunks of <= kBRows rows and queues them.
    // Per expert, its first chunk (low 24 bits) and the rows of a joined tail
    // (high 8 bits). A chunk is one tile, except that with 128-row tiles an
    // expert's last tile of at most kTailMax rows joins the tile before it:
    // its weights are then not streamed again for a few tokens.
    int* chunk_tab = reinterpret_cast<int*>(ctl + kCtlBytes);   // [E + 1]
    if (p.ep_sources && lane == 0) {   // every source rank has closed its dispatch into these windows
      const unsigned long long t0 = globaltimer();
      uint32_t n;
      while (true) {
        asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(n) : "l"(misc + kSrcDone) : "memory");
        if (n >= (uint32_t)p.ep_sources || *abort_flag) break;
        if (globaltimer() - t0 > kWaitBudgetNs) {
          latch_error(hdr, MOE_ERR_TIMEOUT, 0x26000000u | n);
          *abort_flag = 1;
          break;
        }
        __nanosleep(256);
      }
    }
    __syncwarp();
    const uint32_t* base = p.compact ? set_base(set, p.E, p.tiles) : nullptr;
    int ntab = 0;   // tiles counted from the expert counts (lane 31)
    {
      const uint32_t* cnt = p.streaming ? set_pre(set, p.E, p.tiles) : set_count(set);
      const int per = (p.E + 31) / 32;
      auto tiles_of = [&](int e, int* tail) {
        const int c = (int)min(ld_acquire(cnt + e), (uint32_t)p.cap);
        const int nt = (c + kTileRows - 1) / kTileRows;
        const int last = c - (nt - 1) * kTileRows;
        *tail = (kBRows > 64 && nt >= 2 && last <= kTailMax) ? last : 0;
        return nt;
      };
      int lt = 0, lc = 0;
      for (int i = 0; i < per; ++i) {
        const int e = lane * per + i;
        if (e < p.E) {
          int tail;
          const int nt = tiles_of(e, &tail);
          lt += nt;
          lc += nt - (tail ? 1 : 0);
        }
      }
      int it = lt, ic = lc;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int vt = __shfl_up_sync(0xffffffffu, it, off);
        const int vc = __shfl_up_sync(0xffffffffu, ic, off);
        if (lane >= off) { it += vt; ic += vc; }
      }
      int rc = ic - lc;
      for (int i = 0; i < per; ++i) {
        const int e = lane * per + i;
        if (e < p.E) {
          int tail;
          const int nt = tiles_of(e, &tail);
          chunk_tab[e] = rc | (tail << 24);
          rc += nt - (tail ? 1 : 0);
        }
      }
      if (lane == 31) chunk_tab[p.E] = ic;
      ntab = __shfl_sync(0xffffffffu, it, 31);
      __syncwarp();
    }
    // (with expert parallelism the sources' tile totals are complete only now)
    const uint32_t ntiles = p.ep_sources ? ld_acquire(misc + kRingTotal) : ntiles_early;
    if (lane == 0) {
      uint32_t i = 0;
      bool good = true;
      auto push = [&](const Job& j) -> bool {
        const uint32_t q = i % kUQ, ph = (i / kUQ) & 1u;
        if (!wait_bar(uq_empty + q, ph ^ 1u, abort_flag, hdr, 0x90000000u | q)) return false;
        uq[q] = pack_job(j);
        ptx::mbar_arrive(uq_full + q);
        ++i;
        return true;
      };
      if (!p.streaming && (uint32_t)ntab != ntiles) {   // the published tile total disagrees with the counts
        latch_error(hdr, MOE_ERR_INVALID_ARG, 0x24000000u | (uint32_t)ntab);
        *abort_flag = 1;
        good = false;
      }
      const uint32_t nchunks = (uint32_t)(chunk_tab[p.E] & 0xFFFFFF);
      const uint32_t n1 = nchunks * (uint32_t)p.n_islices;                       // gate/up units
      const uint32_t total = n1 + nchunks * (uint32_t)(p.n_hslices / dpair);   // + down units
      // units are taken from one counter in increasing order (dynamic load
      // balance); every unit waits only on units earlier in that order
      while (good) {
        const uint32_t u = atomicAdd(misc + kFfnNext, 1u);
        if (u >= total) break;
        Job j;
        j.kind = u >= n1 ? kKindDown : kKindGateUp;
        const uint32_t v = j.kind == kKindDown ? u - n1 : u;
        const uint32_t ns = (uint32_t)(j.kind == kKindDown ? p.n_hslices / dpair : p.n_islices);
        // weight expert: the last we with first_chunk[we * R] * ns <= v (empty
        // ones never are); its units cover the chunks of its R windows
        // (consecutive in chunk_tab), slice-major, so that the windows sharing
        // a weight slice are worked on together
        const int R = p.R;
        int lo = 0, hi = p.E / R - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if ((uint32_t)(chunk_tab[mid * R] & 0xFFFFFF) * ns <= v) lo = mid;
          else hi = mid - 1;
        }
        const int c0 = chunk_tab[lo * R] & 0xFFFFFF;
        const uint32_t nc = (uint32_t)((chunk_tab[(lo + 1) * R] & 0xFFFFFF) - c0);
        const uint32_t w = v - (uint32_t)c0 * ns;
        const int cc = c0 + (int)(w % nc);   // the unit's chunk
        int ve = lo * R;                      // its window: the last with first chunk <= cc
        while (ve + 1 < (lo + 1) * R && (chunk_tab[ve + 1] & 0xFFFFFF) <= cc) ++ve;
        j.e = ve;
        const int tail = (int)((uint32_t)chunk_tab[ve] >> 24);
        const int ncv = (chunk_tab[ve + 1] & 0xFFFFFF) - (chunk_tab[ve] & 0xFFFFFF);
        j.pair = j.kind == kKindDown && dpair == 2;
        j.slice = (int)(w / nc) * (j.pair ? 2 : 1);
        j.tile = cc - (chunk_tab[ve] & 0xFFFFFF);
        // global tile: rows 128 * slot ..., the down units' counter
        j.slot = (base ? (int)base[j.e] : j.e * p.tpe) + j.tile;
        j.wide = tail && j.tile == ncv - 1;
        int rows = 0;
        good = wait_tile(p.ws, epoch, j.slot, abort_flag, &rows);
        if (good && j.wide) {   // the joined tail's sentinel too
          int rows2 = 0;
          good = wait_tile(p.ws, epoch, j.slot + 1, abort_flag, &rows2);
          rows += rows2;
        }
        if (!good) break;
        const int nch = j.wide ? 1 : (rows + kBRows - 1) / kBRows;
        if (j.kind == kKindDown)
          good = wait_count(hdone + j.slot, (uint32_t)(p.n_islices * nch) * (gen + 1u), abort_flag, hdr,
                            0x30000000u | (uint32_t)j.slot);
        for (int c = 0; good && c < nch; ++c) {
          j.row_off = c * kBRows;
          j.rows = j.wide ? rows : min(kBRows, rows - j.row_off);
          const int N = (j.rows + 15) & ~15;
          j.nslab = (j.kind == kKindDown && !j.pair && 2 * N <= kBRows && (p.nk2 & 1) == 0) ? 2 : 1;
          good = push(j);
        }
      }
      Job end;
      end.e = end.tile = end.slice = end.rows = end.row_off = end.slot = end.pair = end.wide = 0;
      end.nslab = 1;
      end.kind = good ? kKindEnd : kKindAbort;
      push(end);   // bounded; consumers also stop on the abort flag
    }
    __syncwarp();
  } else if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&p.tm_wg);
      ptx::prefetch_tmap(&p.tm_wu);
      ptx::prefetch_tmap(&p.tm_wd);
      for (int b = 0; b < 4; ++b) {
        ptx::prefetch_tmap(&p.tm_x[b]);
        ptx::prefetch_tmap(&p.tm_h[b]);
      }
    }
    // Weights: evict-first when each weight is read once (small tiles, one tile
    // per expert); the default policy when an expert's 2+ token tiles reuse the
    // same weight slices through L2. 4-bit weight rows are 64 bytes per K slab,
    // so one 256-byte L2 fill serves four slabs read on consecutive stages:
    // evict-first would drop some before their turn (measured: default
    // policy 1.183 ms vs 1.213 ms for the decode FFN with 4-bit weights).
    const uint64_t pol = kW4 ? ptx::policy_evict_normal() : ptx::policy_evict_first();
    uint32_t stage = 0, phase = 0;
    uint32_t armed = 0, armed_parity = 0;   // per stage: a load is outstanding / its phase parity
    for (uint32_t i = 0;; ++i) {
      int4 raw = make_int4(0, 0, kKindAbort << 16, 0);
      if (lane == 0) {
        Job jj;
        if (take_job(i, &jj)) raw = pack_job(jj);
        ptx::fence_proxy_async_global();   // rows written by other CTAs -> TMA reads
      }
      const Job j = unpack_job(shfl_int4(raw));
      if (j.kind >= kKindEnd) break;
      const bool down = j.kind == kKindDown;
      const int N = (j.rows + 15) & ~15;
      const int nsteps = down ? p.nk2 / j.nslab : p.nk1;
      const int we = j.e / p.R;   // the window's weight expert
      const int arow = we * (down ? p.H : p.I) + j.slice * 128;
      const int brow = j.slot * kTileRows + j.row_off;
      const int64_t tile_g = j.slot;
      const bool dual = !down || j.pair;   // two weight tiles share the token tile
      // a weight tile lands as 128 x 128 bytes; 4-bit weights travel as half
      // that (the copy spreads each 8 bytes of codes over 16 in shared memory)
      constexpr uint32_t kABytesIn = kW4 ? kABytes / 2 : kABytes;
      const uint32_t na = dual ? 2u : (uint32_t)j.nslab;   // weight tiles (and 4-bit scale atoms) per stage
      const uint32_t tx = na * kABytesIn + (uint32_t)(j.nslab * N * kSlab);
      // the job's weight scales, one per 128 x 128 block along K: lane l holds
      // the exponents of blocks l and l + 32 (gate/down in sa, up in sb), read
      // once per job
      uint32_t sa0 = 0, sa1 = 0, sb0 = 0, sb1 = 0;
      int sbase = 0;   // first K block held in sa*/sb*
      const int nkb = down ? p.I / 128 : p.H / 128;
      const float* pa = down ? (const float*)p.sd + ((int64_t)we * p.n_hslices + j.slice) * nkb
                             : (const float*)p.sg + ((int64_t)we * p.n_islices + j.slice) * nkb;
      const float* pb = down ? (const float*)p.sd + ((int64_t)we * p.n_hslices + j.slice + 1) * nkb
                             : (const float*)p.su + ((int64_t)we * p.n_islices + j.slice) * nkb;
      // 4-bit weights: the scale atoms of the job's weight tiles, one per
      // 128-value K block (row-major over [slice][K block])
      const uint8_t* atom_a = nullptr;
      const uint8_t* atom_b = nullptr;
      if constexpr (kW4) {
        const int n_out = down ? p.n_hslices : p.n_islices;
        atom_a = (const uint8_t*)(down ? p.sd : p.sg) + ((int64_t)we * n_out + j.slice) * nkb * kSfAtomBytes;
        atom_b = down ? atom_a + (int64_t)nkb * kSfAtomBytes
                      : (const uint8_t*)p.su + ((int64_t)we * n_out + j.slice) * nkb * kSfAtomBytes;
      }
      // A scale that is not a normal power of two latches
      // MOE_ERR_INVALID_ARG (info: 0x25, the matrix (0 gate / down, 1 up or
      // the second down slice) and the expert); the layer's outputs are then
      // unspecified. Every scale of every touched expert passes through here.
      auto load_scales = [&](int base) {
        bool bad = false;
        auto take = [&](const float* src, int kb) -> uint32_t {
          const float v = __ldg(src + kb);
          bad |= !pow2_scale_ok(v);
          return ue8m0(v);
        };
        if (lane + base < nkb) sa0 = take(pa, base + lane);
        if (lane + base + 32 < nkb) sa1 = take(pa, base + lane + 32);
        const bool bad_a = bad;
        if (dual) {
          if (lane + base < nkb) sb0 = take(pb, base + lane);
          if (lane + base + 32 < nkb) sb1 = take(pb, base + lane + 32);
        }
        const uint32_t which = __ballot_sync(0xffffffffu, bad_a) ? 0u : 1u;
        if (__ballot_sync(0xffffffffu, bad) != 0u && lane == 0)
          latch_error(hdr, MOE_ERR_INVALID_ARG, 0x25000000u | (which << 20) | (uint32_t)we);
      };
      // the four exponents of blocks kr .. kr+3 (relative to sbase), packed
      auto pack4 = [&](uint32_t r0, uint32_t r1, int kr) -> uint32_t {
        uint32_t w = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int kk = kr + b;
          const uint32_t v = __shfl_sync(0xffffffffu, kk < 32 ? r0 : r1, kk & 31);
          w |= (kk + sbase < nkb ? v : 0u) << (8 * b);
        }
        return w;
      };
      if constexpr (kW == kWE4m3) load_scales(0);
      bool ok = true;
      for (int st_i = 0; st_i < nsteps; ++st_i) {
        int w_ok = 1;
        if (lane == 0) w_ok = wait_bar(empty + stage, phase ^ 1u, abort_flag, hdr, 0x40000000u | stage);
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        __syncwarp();
        uint8_t* st = smem + stage * S::kStride;
        const int kb0 = st_i * j.nslab;   // first K slab of this stage
        // scale atoms cover four K blocks: they travel with the stage that
        // starts a group of four
        const bool sf_stage = kFp8 && (kb0 & 3) == 0;
        if constexpr (kW == kWE4m3) {
          if (sf_stage) {
            // weight scale atoms: one exponent per 128 x 128 block, the same
            // for all 128 rows; byte b = block kb0 + b
            if (kb0 + 3 >= sbase + 64) {   // next 64 blocks of scales (K > 8192)
              sbase = kb0;
              load_scales(sbase);
            }
            const int kr = kb0 - sbase;
            const uint32_t w0 = pack4(sa0, sa1, kr);
            reinterpret_cast<uint4*>(st + S::kOffSfa0)[lane] = make_uint4(w0, w0, w0, w0);
            if (dual) {
              const uint32_t w1 = pack4(sb0, sb1, kr);
              reinterpret_cast<uint4*>(st + S::kOffSfa1)[lane] = make_uint4(w1, w1, w1, w1);
            }
            ptx::fence_proxy_async_smem();
          }
          __syncwarp();
        }
        // one elected lane issues the copies; every operand is warp-uniform.
        // Each copy names its tensor map at a fixed parameter address: a map
        // chosen at run time costs about four times as much to issue.
        if (ptx::elect_one()) {
          uint64_t* fb = full + stage;
          ptx::mbar_arrive_expect_tx(fb, tx + (sf_stage ? (j.wide ? 2u : 1u) * (uint32_t)kSfAtomBytes : 0u) +
                                             (kW4 ? na * (uint32_t)kSfAtomBytes : 0u));
          const int kx0 = kb0 * p.kelems;
          if (down) {
            if constexpr (kBRows <= 64) {   // one slab of slices (slice, slice + 1), or nslab slabs of one slice
              if (j.pair) {
                ptx::tma_load_2d_hint(st, &p.tm_wd, fb, kx0, arow, pol);
                ptx::tma_load_2d_hint(st + S::kOffA1, &p.tm_wd, fb, kx0, arow + 128, pol);
              } else {
                for (int s = 0; s < j.nslab; ++s)
                  ptx::tma_load_2d_hint(st + s * S::kOffA1, &p.tm_wd, fb, kx0 + s * p.kelems, arow, pol);
              }
            } else {   // one slab of slices (slice, slice + 1), or nslab slabs of one slice
              if (j.pair) {
                ptx::tma_load_2d(st, &p.tm_wd, fb, kx0, arow);
                ptx::tma_load_2d(st + S::kOffA1, &p.tm_wd, fb, kx0, arow + 128);
              } else {
                for (int s = 0; s < j.nslab; ++s)
                  ptx::tma_load_2d(st + s * S::kOffA1, &p.tm_wd, fb, kx0 + s * p.kelems, arow);
              }
            }
          } else if constexpr (kBRows <= 64) {
            ptx::tma_load_2d_hint(st, &p.tm_wg, fb, kx0, arow, pol);
            ptx::tma_load_2d_hint(st + S::kOffA1, &p.tm_wu, fb, kx0, arow, pol);
          } else {   // default policy: an expert's token tiles reuse the slice through L2
            ptx::tma_load_2d(st, &p.tm_wg, fb, kx0, arow);
            ptx::tma_load_2d(st + S::kOffA1, &p.tm_wu, fb, kx0, arow);
          }
          // token rows: small tiles (decode) in 16-row boxes, large ones in
          // the fewest boxes of 128/64/32/16 rows; measured, each is the
          // faster choice for its variant
          for (int s = 0; s < j.nslab; ++s) {
            uint8_t* dst = st + S::kOffB + s * N * kSlab;
            const int kx = kx0 + s * p.kelems;
            if constexpr (kBRows <= 64) {
              if (down) {
                for (int r = 0; r < N / 16; ++r) ptx::tma_load_2d(dst + r * 2048, &p.tm_h[0], fb, kx, brow + 16 * r);
              } else {
                for (int r = 0; r < N / 16; ++r) ptx::tma_load_2d(dst + r * 2048, &p.tm_x[0], fb, kx, brow + 16 * r);
              }
            } else if (N == 128) {   // the common full tile: one box
              if (down) ptx::tma_load_2d(dst, &p.tm_h[3], fb, kx, brow);
              else ptx::tma_load_2d(dst, &p.tm_x[3], fb, kx, brow);
            } else if (down) {
              int r = 0;
              if (N - r >= 128) { ptx::tma_load_2d(dst + r * kSlab, &p.tm_h[3], fb, kx, brow + r); r += 128; }
              if (N - r >= 64) { ptx::tma_load_2d(dst + r * kSlab, &p.tm_h[2], fb, kx, brow + r); r += 64; }
              if (N - r >= 32) { ptx::tma_load_2d(dst + r * kSlab, &p.tm_h[1], fb, kx, brow + r); r += 32; }
              if (N - r >= 16) { ptx::tma_load_2d(dst + r * kSlab, &p.tm_h[0], fb, kx, brow + r); r += 16; }
            } else {
              int r = 0;
              if (N - r >= 128) { ptx::tma_load_2d(dst + r * kSlab, &p.tm_x[3], fb, kx, brow + r); r += 128; }
              if (N - r >= 64) { ptx::tma_load_2d(dst + r * kSlab, &p.tm_x[2], fb, kx, brow + r); r += 64; }
              if (N - r >= 32) { ptx::tma_load_2d(dst + r * kSlab, &p.tm_x[1], fb, kx, brow + r); r += 32; }
              if (N - r >= 16) { ptx::tma_load_2d(dst + r * kSlab, &p.tm_x[0], fb, kx, brow + r); r += 16; }
            }
          }
          if (sf_stage) {   // the tokens' scale atom(s) of this group of four blocks
            const uint8_t* sfb = down ? p.ws.hsf : p.ws.xsf;
            const int groups = down ? p.igroups : p.hgroups;
            ptx::bulk_load(st + S::kOffSfb0, sfb + (tile_g * groups + kb0 / 4) * kSfAtomBytes, kSfAtomBytes, fb);
            if (j.wide)   // the joined tail tile's atom
              ptx::bulk_load(st + S::kOffSfb1, sfb + ((tile_g + 1) * groups + kb0 / 4) * kSfAtomBytes, kSfAtomBytes,
                             fb);
          }
          if constexpr (kW4) {   // the weight tiles' scale atoms of this stage
            if (dual) {
              ptx::bulk_load(st + S::kOffSfa0, atom_a + (int64_t)kb0 * kSfAtomBytes, kSfAtomBytes, fb);
              ptx::bulk_load(st + S::kOffSfa1, atom_b + (int64_t)kb0 * kSfAtomBytes, kSfAtomBytes, fb);
            } else {
              for (int s = 0; s < j.nslab; ++s)
                ptx::bulk_load(st + (s ? S::kOffSfa1 : S::kOffSfa0), atom_a + (int64_t)(kb0 + s) * kSfAtomBytes,
                               kSfAtomBytes, fb);
            }
          }
        }
        __syncwarp();
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == (uint32_t)kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
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
    // Two 128-column accumulator slots: a job with N <= 64 (or a down job)
    // takes one (gate at +0, up at +64), a gate/up job with N > 64 takes both,
    // so the next job's MMAs overlap the previous job's epilogue. A job with
    // a joined tail (N <= 128 + kTailMax) takes both slots and the columns
    // after them: gate (or the down slice) at column 0, up (or the second
    // slice) at N.
    // The whole warp walks the loop with warp-uniform values (descriptors,
    // tensor-memory addresses); lane 0 polls the barriers and one elected
    // lane issues the copies, MMAs and commits.
    uint32_t stage = 0, phase = 0, acc_ph = 0 /* bit per slot */, next_slot = 0;
    for (uint32_t i = 0;; ++i) {
      int4 raw = make_int4(0, 0, kKindAbort << 16, 0);
      if (lane == 0) {
        Job jj;
        if (take_job(i, &jj)) raw = pack_job(jj);
      }
      const Job j = unpack_job(shfl_int4(raw));
      if (j.kind >= kKindEnd) break;
      const bool down = j.kind == kKindDown;
      const bool dual = !down || j.pair;   // two accumulators: gate/up or two slices of H
      const int N = (j.rows + 15) & ~15;
      const bool two = j.wide || (dual && N > 64);
      const uint32_t s0 = next_slot, s1 = next_slot ^ 1u;
      const uint32_t colG = j.wide ? 0u : 128u * s0;
      const uint32_t colU = j.wide ? (uint32_t)N : (two ? 128u * s1 : 128u * s0 + 64u);
      int ok = 1;
      if (lane == 0) {
        ok = wait_bar(acc_empty + s0, ((acc_ph >> s0) & 1u) ^ 1u, abort_flag, hdr, 0x50000000u | s0);
        if (ok && two) ok = wait_bar(acc_empty + s1, ((acc_ph >> s1) & 1u) ^ 1u, abort_flag, hdr, 0x50000000u | s1);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      ptx::tc_fence_after();
      const int nsteps = down ? p.nk2 / j.nslab : p.nk1;
      const uint32_t idesc = kFp8 ? ptx::idesc_mxf8(128, N, 0, kW4 ? ptx::kMxE2M1 : ptx::kMxE4M3)
                                  : ptx::idesc_bf16(128, N);
      // the token scale atom covers the whole 128-row tile (row m in TMEM
      // column m / 32, lane m % 32); a chunk starting at row_off (a multiple
      // of 64 with 64-row chunks) reads from column row_off / 32. A 16-row
      // chunk inside a tile gets its rows gathered into lanes 0-15 of a
      // scratch atom's first column instead (below).
      const bool sfb_gather = kFp8 && kBRows <= 16 && j.row_off != 0;
      const uint32_t sfb_off = kBRows <= 16 ? 0u : (uint32_t)j.row_off / 32u;
      for (int st_i = 0; st_i < nsteps; ++st_i) {
        int w_ok = 1;
        if (lane == 0) w_ok = wait_bar(full + stage, phase, abort_flag, hdr, 0x60000000u | stage);
        if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = 0; break; }
        ptx::tc_fence_after();
        uint8_t* st = smem + stage * S::kStride;
        const int kb0 = st_i * j.nslab;
        const uint64_t a0 = ptx::desc_kmajor_sw128(st);
        const uint64_t a1 = ptx::desc_kmajor_sw128(st + S::kOffA1);
        const uint64_t b0 = ptx::desc_kmajor_sw128(st + S::kOffB);
        // scale-factor byte of a K block inside its atom: in the instruction
        // descriptor and in the top two bits of the scale addresses
        auto sfid = [](int kb) -> uint32_t { return (uint32_t)(kb & 3); };
        if (sfb_gather && (kb0 & 3) == 0) {   // into the SFB1 slot, which 16-row stages leave unused
          const uint32_t* src = reinterpret_cast<const uint32_t*>(st + S::kOffSfb0);
          uint32_t* dst = reinterpret_cast<uint32_t*>(st + S::kOffSfb1);
          if (lane < 16) {
            const int m = j.row_off + lane;   // < 128: row_off <= 112
            dst[lane * 4] = src[(m % 32) * 4 + m / 32];
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
        }
        if (ptx::elect_one()) {
          if constexpr (kFp8) {
            // 32 rows x 16 bytes, no swizzle: 8-row core matrices 128 bytes apart
            auto sf_cp = [&](uint32_t col, int off) {
              ptx::tmem_cp_32x128b_x4(tmem + col, ptx::smem_desc(ptx::smem_u32(st + off), 16, 128, ptx::kLayoutNone));
            };
            if ((kb0 & 3) == 0) {   // a new group of four K blocks: the tokens' scale atoms
              sf_cp(kColSfb0, sfb_gather ? S::kOffSfb1 : S::kOffSfb0);
              if (j.wide) sf_cp(kColSfb0 + 4, S::kOffSfb1);   // the joined tail's rows 128.. read columns kColSfb0 + 4 ..
              if constexpr (kW == kWE4m3) {                   // and the weights' (one exponent per block)
                sf_cp(kColSfa0, S::kOffSfa0);
                if (dual) sf_cp(kColSfa1, S::kOffSfa1);
              }
            }
            if constexpr (kW4) {   // 4-bit weights: new scale atoms every K block
              sf_cp(kColSfa0, S::kOffSfa0);
              if (dual || j.nslab == 2) sf_cp(kColSfa1, S::kOffSfa1);
            }
          }
          // The weights' scale byte: the K block's (e4m3, one exponent per
          // 128 x 128 block) or, for 4-bit weights, the 32-value group's.
          if (dual) {
            const uint32_t id = sfid(kb0);
            const uint32_t sb = (tmem + kColSfb0 + sfb_off) | (id << 30);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t ida = kW4 ? (uint32_t)kk : id;
              const uint32_t idesc_k = idesc | (id << 4) | (ida << 29);
              const uint32_t sa0 = (tmem + kColSfa0) | (ida << 30), sa1 = (tmem + kColSfa1) | (ida << 30);
              const uint32_t acc = (st_i > 0 || kk > 0) ? 1u : 0u;
              const uint64_t off = (uint64_t)(kk * 32) >> 4;   // 32 bytes of K per MMA
              if constexpr (kFp8) {
                ptx::mma_mxf8(tmem + colG, a0 + off, b0 + off, idesc_k, sa0, sb, acc);
                ptx::mma_mxf8(tmem + colU, a1 + off, b0 + off, idesc_k, sa1, sb, acc);
              } else {
                ptx::mma_f16(tmem + colG, a0 + off, b0 + off, idesc, acc);
                ptx::mma_f16(tmem + colU, a1 + off, b0 + off, idesc, acc);
              }
            }
          } else {
            for (int sl = 0; sl < j.nslab; ++sl) {
              const uint64_t as = sl ? a1 : a0;
              const uint64_t bs = ptx::desc_kmajor_sw128(st + S::kOffB + sl * N * kSlab);
              const uint32_t id = sfid(kb0 + sl);
              const uint32_t sb = (tmem + kColSfb0 + sfb_off) | (id << 30);
              const uint32_t col_sa = (kW4 && sl) ? kColSfa1 : kColSfa0;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t ida = kW4 ? (uint32_t)kk : id;
                const uint32_t idesc_k = idesc | (id << 4) | (ida << 29);
                const uint32_t sa = (tmem + col_sa) | (ida << 30);
                const uint32_t acc = (st_i > 0 || sl > 0 || kk > 0) ? 1u : 0u;
                const uint64_t off = (uint64_t)(kk * 32) >> 4;
                if constexpr (kFp8) {
                  ptx::mma_mxf8(tmem + colG, as + off, bs + off, idesc_k, sa, sb, acc);
                } else {
                  ptx::mma_f16(tmem + colG, as + off, bs + off, idesc, acc);
                }
              }
            }
          }
          ptx::mma_commit(empty + stage);   // frees the stage once these MMAs are done
        }
        __syncwarp();
        if (++stage == (uint32_t)kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (ptx::elect_one()) {
        ptx::mma_commit(acc_full + s0);
        if (two) ptx::mma_commit(acc_full + s1);
      }
      __syncwarp();
      acc_ph ^= 1u << s0;
      if (two) acc_ph ^= 1u << s1;
      else next_slot ^= 1u;
    }
    // drain: all MMAs and copies issued by the elected lane are complete
    if (ptx::elect_one()) {
      ptx::mma_commit(drain);
      const unsigned long long t0 = globaltimer();
      while (!ptx::mbar_try_wait(drain, 0)) {
        if (globaltimer() - t0 > kWaitBudgetNs) break;
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    // Eight warps in two sets of four; warp w reads TMEM lanes 32 (w % 4) ..
    // +31 (output features), and set s takes the 32-token batches s, s + 2, ..
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int f = q * 32 + lane;            // output feature within the slice
    const int et = threadIdx.x - 64;        // 0..255
    const int set = et >> 7;                // 0 or 1
    const uint32_t set_bar = 2u + (uint32_t)set;   // named barrier of the set (128 threads)
    float* red_s = red + set * 128;
    float* sinv_s = sinv + set * 32;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint32_t acc_ph = 0, next_slot = 0;
    for (uint32_t i = 0;; ++i) {
      if (et == 0) {
        Job jj;
        int good = take_job(i, &jj);
        if (!good) jj.kind = kKindAbort;
        if (jj.kind < kKindEnd) {
          const int N = (jj.rows + 15) & ~15;
          const bool two = jj.wide || ((jj.kind == kKindGateUp || jj.pair) && N > 64);
          const uint32_t s0 = next_slot, s1 = next_slot ^ 1u;
          good = wait_bar(acc_full + s0, (acc_ph >> s0) & 1u, abort_flag, hdr, 0x70000000u | s0);
          if (good && two) good = wait_bar(acc_full + s1, (acc_ph >> s1) & 1u, abort_flag, hdr, 0x70000000u | s1);
          if (!good) jj.kind = kKindAbort;
        }
        *epi_job = pack_job(jj);
      }
      ptx::named_barrier(1, kEpiThreads);
      const Job j = unpack_job(*epi_job);
      ptx::named_barrier(1, kEpiThreads);
      if (j.kind >= kKindEnd) break;
      const bool down = j.kind == kKindDown;
      const bool dual = !down || j.pair;
      const int N = (j.rows + 15) & ~15;
      const bool two = j.wide || (dual && N > 64);
      const uint32_t s0 = next_slot, s1 = next_slot ^ 1u;
      const uint32_t colG = j.wide ? 0u : 128u * s0;
      const uint32_t colU = j.wide ? (uint32_t)N : (two ? 128u * s1 : 128u * s0 + 64u);
      while (!ptx::mbar_try_wait(acc_full + s0, (acc_ph >> s0) & 1u)) {}   // completed: returns at once
      if (two) while (!ptx::mbar_try_wait(acc_full + s1, (acc_ph >> s1) & 1u)) {}
      ptx::tc_fence_after();
      const int64_t row0 = (int64_t)j.slot * kTileRows + j.row_off;
      const int64_t tile_g = j.slot;
      // Set s owns the 32-token batches at columns 32 s and 32 s + 64 (a job
      // has at most 128 rows). Both are drained from TMEM into registers first
      // -- h = SwiGLU in fp32, or y already rounded to bf16 (two slices packed
      // per word) -- and the accumulators are released before any of the
      // slower per-token work, so the next job's MMAs overlap all of it.
      const int nA = max(0, min(32, j.rows - 32 * set));
      const int nB = max(0, min(32, j.rows - 32 * set - 64));
      uint32_t vA[32], vB[32];
      auto drain = [&](int n0, uint32_t (&v)[32]) {
#pragma unroll
        for (int hh = 0; hh < 32; hh += 16) {   // 16 columns at a time: fewer live registers
          uint32_t g[16], uu[16];
          ptx::tmem_ld_x16(tmem + lane_base + colG + n0 + hh, g);
          if (dual) ptx::tmem_ld_x16(tmem + lane_base + colU + n0 + hh, uu);
          ptx::tmem_wait_ld();
          if (down) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(g[jj]), dual ? __uint_as_float(uu[jj]) : 0.f);
              v[hh + jj] = *reinterpret_cast<uint32_t*>(&b2);
            }
          } else {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              v[hh + jj] = __float_as_uint(silu(__uint_as_float(g[jj])) * __uint_as_float(uu[jj]));
          }
        }
      };
      // accumulators consumed: let the MMA warp reuse the slot(s)
      auto release = [&]() {
        ptx::tc_fence_before();
        ptx::named_barrier(1, kEpiThreads);
        if (et == 0) {
          ptx::mbar_arrive(acc_empty + s0);
          if (two) ptx::mbar_arrive(acc_empty + s1);
        }
        acc_ph ^= 1u << s0;
        if (two) acc_ph ^= 1u << s1;
        else next_slot ^= 1u;
      };
      if (!j.wide) {
        if (nA > 0) drain(32 * set, vA);
        if (nB > 0) drain(32 * set + 64, vB);
        release();
      }
      // the per-token work on one drained batch: y stores, or the per-token
      // max over the 128 features (one redux per token per warp, the max over
      // the set's four warps and the scale once per token through shared
      // memory), requantisation and h stores
      auto finish = [&](int n0, int nv, const uint32_t (&v)[32]) {
        if (down) {
          __nv_bfloat16* yp = reinterpret_cast<__nv_bfloat16*>(p.y) + (row0 + n0) * p.H + j.slice * 128 + f;
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if (jj < nv) yp[(int64_t)jj * p.H] = __ushort_as_bfloat16((unsigned short)(v[jj] & 0xFFFFu));
          if (j.pair) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              if (jj < nv) yp[(int64_t)jj * p.H + 128] = __ushort_as_bfloat16((unsigned short)(v[jj] >> 16));
          }
          return;
        }
        if constexpr (kFp8) {
          // |h| bit patterns order like the values (non-negative floats)
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const uint32_t m = __reduce_max_sync(0xffffffffu, v[jj] & 0x7FFFFFFFu);
            if (lane == jj) red_s[q * 32 + jj] = __uint_as_float(m);
          }
          ptx::named_barrier(set_bar, 128);
          if (q == 0) {   // lane t: token n0 + t's scale over the 128 features
            const float amax = fmaxf(fmaxf(red_s[lane], red_s[32 + lane]), fmaxf(red_s[64 + lane], red_s[96 + lane]));
            const int pe = pow2_scale_exp(amax);
            sinv_s[lane] = exp2i(-pe > -126 ? -pe : -126);
            if (lane < nv) {
              const int64_t r = row0 + n0 + lane;
              p.hs[r * (p.I / 128) + j.slice] = exp2i(pe);
              // byte of this slice in its tile's scale atom (a joined tail's
              // rows past 128 belong to the next tile)
              const int rr = j.row_off + n0 + lane;
              *sf_atom_byte(p.ws.hsf, tile_g + rr / kTileRows, p.igroups, j.slice, rr % kTileRows) = (uint8_t)(pe + 127);
            }
          }
          ptx::named_barrier(set_bar, 128);
          uint8_t* hp = reinterpret_cast<uint8_t*>(p.hq) + (row0 + n0) * p.I + j.slice * 128 + f;
          const float4* sv = reinterpret_cast<const float4*>(sinv_s);
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 iv = sv[j4];
            const float inv[4] = {iv.x, iv.y, iv.z, iv.w};
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              const int jj = 4 * j4 + b;
              if (jj < nv) hp[(int64_t)jj * p.I] = (uint8_t)(cvt_e4m3x2(__uint_as_float(v[jj]) * inv[b], 0.f) & 0xFF);
            }
          }
          ptx::named_barrier(set_bar, 128);     // red / sinv are reused by the next batch
        } else {
          __nv_bfloat16* hp = reinterpret_cast<__nv_bfloat16*>(p.hq) + (row0 + n0) * p.I + j.slice * 128 + f;
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if (jj < nv) hp[(int64_t)jj * p.I] = __float2bfloat16_rn(__uint_as_float(v[jj]));
        }
      };
      if (!j.wide) {
        if (nA > 0) finish(32 * set, nA, vA);
        if (nB > 0) finish(32 * set + 64, nB, vB);
      } else {   // a joined tail: up to 5 batches, drained and finished one at a time
        for (int n0 = 32 * set; n0 < j.rows; n0 += 64) {
          drain(n0, vA);
          finish(n0, min(32, j.rows - n0), vA);
        }
        release();
      }
      if (!down) {
        // publish this chunk of this slice of h to the down jobs of the tile
        __threadfence();
        ptx::named_barrier(1, kEpiThreads);
        if (et == 0) atomicAdd(hdone + j.slot, 1u);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0) {
    // the last CTA out records that one more FFN call ran on this dispatch
    __threadfence();
    const uint32_t exits = atomicAdd(misc + kFfnExit, 1u) + 1u;
    if (exits == gridDim.x * (gen + 1u)) {   // every CTA is done with the unit counter
      misc[kFfnNext] = 0u;
      __threadfence();
      st_release(misc + kFfnGen, gen + 1u);
    }
  }
}

// ---- host side ------------------------------------------------------------

template <int kW, int kBRows>
cudaError_t launch_typed(const Ctx& c, const moe_dispatch_bufs& b, const moe_weights& w, void* y) {
  using S = Stage<kBRows>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(ffn_tc_kernel<kW, kBRows>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    S::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  TcParams p;
  memset(&p, 0, sizeof(p));
  const int64_t H = c.s.H, I = c.s.I, E = c.s.E, rows = c.L.tiles * kTileRows;
  constexpr bool kFp8 = kW != kWBf16;
  const int kel = kFp8 ? 128 : 64;   // elements per 128-byte slab row in shared memory
  const TmapElem wel = kW == kWE2m1 ? kElU4Spread : (kFp8 ? kElU8 : kElBf16);
  const TmapElem tel = kFp8 ? kElU8 : kElBf16;
  if (!make_tmap(&p.tm_wg, w.w_gate, wel, H, E * I, kel, 128) ||
      !make_tmap(&p.tm_wu, w.w_up, wel, H, E * I, kel, 128) ||
      !make_tmap(&p.tm_wd, w.w_down, wel, I, E * H, kel, 128))
    return cudaErrorInvalidValue;
  for (int bx = 0; bx < 4; ++bx) {
    if (!make_tmap(&p.tm_x[bx], b.xq, tel, H, rows, kel, 16 << bx) ||
        !make_tmap(&p.tm_h[bx], b.hq, tel, I, rows, kel, 16 << bx))
      return cudaErrorInvalidValue;
  }
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
  p.compact = c.L.compact ? 1 : 0;
  p.streaming = c.streaming ? 1 : 0;
  p.R = c.ep_ranks > 0 ? c.ep_ranks : 1;
  p.ep_sources = c.ep_ranks > 0 ? c.ep_ranks : 0;
  p.n_islices = (int)(I / 128);
  p.n_hslices = (int)(H / 128);
  p.kelems = kel;
  p.nk1 = (int)(H / kel);
  p.nk2 = (int)(I / kel);
  p.hgroups = (int)c.L.hgroups;
  p.igroups = (int)c.L.igroups;
  p.tiles = c.L.tiles;
  ffn_tc_kernel<kW, kBRows><<<c.num_sms, kThreads, S::kSmemBytes, c.stream>>>(p);
  return cudaGetLastError();
}

// Token tiles of up to 64 rows give a deeper pipeline (5 stages instead of 4),
// and of up to 16 rows 6 stages; they suit layers whose experts see few tokens
// each (decode). Bigger tiles are split into chunks of that many rows, which
// re-streams their weights, so layers with many tokens per expert use 128-row
// tiles.
template <int kW>
cudaError_t launch_by_rows(const Ctx& c, const moe_dispatch_bufs& b, const moe_weights& w, void* y) {
  const int64_t rows_per_expert = c.s.T * c.s.topk / c.s.E;
  // a few tokens per expert (decode): 16-row stages, six of them in flight.
  // A shared expert's window holds all T tokens, which 16-row chunks read as
  // T / 16 passes over its weights (from L2 after the first): measured at
  // decode with a shared expert, 1.075 vs 1.225 ms with 4-bit weights but
  // 1.736 vs 1.728 ms with e4m3 weights, so e4m3 keeps the 64-row tiles there.
  if (rows_per_expert <= 4 && (!c.shared || kW == kWE2m1)) return launch_typed<kW, 16>(c, b, w, y);
  if (rows_per_expert <= 32) return launch_typed<kW, 64>(c, b, w, y);
  // many rows per expert (prefill) with e4m3 weights: CTA pairs, one M = 256
  // MMA over both SMs, so that a job holds up to 256 + 64 of an expert's rows
  // and its weights are streamed once (ffn_pair.cu)
  if (kW == kWE4m3 && rows_per_expert >= 128 && ffn_pair_supported(c)) return launch_ffn_pair(c, b, w, y);
  return launch_typed<kW, 128>(c, b, w, y);
}

}  // namespace

bool ffn_tc_supported(const moe_shape& s) {
  if (s.identity_experts) return false;
  const bool bf16 = s.xq_dtype == MOE_BF16 && s.weight_dtype == MOE_BF16 && s.h_dtype == MOE_BF16 &&
                    s.y_dtype == MOE_BF16;
  const bool fp8 = s.xq_dtype == MOE_E4M3 && (s.weight_dtype == MOE_E4M3 || s.weight_dtype == MOE_E2M1) &&
                   s.h_dtype == MOE_E4M3 && s.y_dtype == MOE_BF16;
  return (bf16 || fp8) && s.H % 128 == 0 && s.I % 128 == 0;
}

cudaError_t launch_ffn_tc(const Ctx& c, const moe_dispatch_bufs& b, const moe_weights& w, void* y) {
  if (c.s.weight_dtype == MOE_E2M1) return launch_by_rows<kWE2m1>(c, b, w, y);
  return c.s.weight_dtype == MOE_E4M3 ? launch_by_rows<kWE4m3>(c, b, w, y) : launch_by_rows<kWBf16>(c, b, w, y);
}

}  // namespace moe

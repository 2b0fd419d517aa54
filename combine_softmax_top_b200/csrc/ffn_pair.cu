// Grouped expert FFN on CTA pairs, for layers whose experts see many tokens
// (prefill): every tcgen05 MMA has M = 256 and spans the two CTAs of a
// cluster (cta_group::2), e4m3 weights with 128 x 128 block scales against
// e4m3 tokens.
//
// Pages: as ffn_tc.cu, the operand-swapped block-scaled MMA with SwiGLU and
// requantisation fused (GC-MoE feed item, "Full text"; explainer, "Two MMA
// Implementations in the Compute Partition"), tiles read in place once
// published. What changes is the shape of a job. The one-CTA kernel holds
// gate and up of one 128-feature slice in one CTA, which caps a job at about
// 128 + 32 tokens (the accumulators of both fill tensor memory) and so
// streams an expert's weights once per 128 of its tokens. Here the slice's
// 256 weight rows form one M = 256 operand split over the pair, each CTA's
// tensor memory holds 128 rows of D, and a job takes up to 256 + kPTail of
// the expert's tokens: its weights are streamed once, and each CTA loads
// half of the token rows (the pair's MMA reads both halves).
//
// Work units, expert-major from one counter as in ffn_tc.cu, all gate/up
// before all down:
//   gate/up: (chunk, 128-feature slice s of I). CTA r holds features
//            64 r .. 64 r + 63 of the slice: their 64 gate rows, then their
//            64 up rows (one copy each), so that tensor-memory lane quarters
//            0-1 hold gate and 2-3 up of the same features; SwiGLU swaps half
//            of each 32-token batch between the two warps of a feature range
//            through shared memory. The per-128 requantisation takes each
//            token's max over both CTAs' 64 features, exchanged through
//            distributed shared memory.
//   down:    (chunk, slices 2 p and 2 p + 1 of H): CTA r's A = the 128 rows of
//            slice 2 p + r of W_down, and its D those 128 features of y.
// A chunk is two 128-row tiles of one expert, or one; an expert's last tile
// joins the chunk before it when it holds at most kPTail rows. Its token
// columns go to one MMA (N <= 256) or, with a joined tile, to two: the first
// tile (N1 = 128) and the rest (N2 <= 192).
//
// Roles per CTA (352 threads): warp 10 of the even CTA schedules jobs into
// both CTAs' queues; warp 0 of each CTA loads its half of every stage (the
// odd CTA's copies complete on the even CTA's barrier, whose expected bytes
// count both halves); warp 1 of the even CTA issues all MMAs and commits to both
// CTAs' barriers; warps 2-9 of each CTA drain their own tensor memory,
// consecutive jobs' accumulators sitting at opposite ends of it so that the
// next job's MMAs start once the overlapping columns are drained. Every
// wait is bounded; on expiry the kernel latches MOE_ERR_TIMEOUT, drains,
// meets its peer at a cluster barrier, frees tensor memory and exits.
#include "ffn_common.cuh"

namespace moe {
namespace {

using namespace ffn;

constexpr int kPTail = 64;                     // rows of a joined last tile
constexpr int kPMaxN = 256 + kPTail;           // token columns of one job
constexpr int kPBRows = kPMaxN / 2;            // token rows one CTA holds per stage
constexpr int kPBatches = kPMaxN / 64;         // 32-column batches per epilogue set
// stage: A (128 x 128 B) | B (kPBRows x 128 B) | SFA atom | SFB atoms (3)
constexpr int kPOffB = kABytes;
constexpr int kPOffSfa = kPOffB + kPBRows * kSlab;
constexpr int kPOffSfb = kPOffSfa + kSfAtomBytes;
constexpr int kPStride = (kPOffSfb + 3 * kSfAtomBytes + 1023) / 1024 * 1024;
// control: barriers | job queue | flags | reductions | token max exchange |
// inverse scales | SwiGLU swap buffers | weight scale atoms of three jobs
constexpr int kPSwapBytes = 2 * 2 * 2 * 16 * 32 * 4;   // [set][feature half][direction][16 columns][32 lanes]
constexpr int kPMaxGroups = 16;                         // K groups of four 128-value blocks (K <= 8192)
constexpr int kPTabRing = 3;                            // scale-atom tables in flight (built ahead by the scheduler)
constexpr int kPTabBytes = kPTabRing * kPMaxGroups * 128;   // [job % 3][group][8 rows x 16 B]
constexpr int kPCtlBytes = 9216 + kPSwapBytes + kPTabBytes;
constexpr int kPStages = (kMaxDynSmem - kPCtlBytes - kTileTabBytes - 1024) / kPStride;
constexpr int kPSmemBytes = kPStages * kPStride + kPCtlBytes + kTileTabBytes + 1024;
static_assert(kPStages >= 4 && kPStages <= 8, "pipeline depth");
static_assert(kPSmemBytes <= kMaxDynSmem, "shared memory");
// Tensor memory: the scale factors in the last 16 columns (one weight atom,
// up to three token atoms), accumulators below them. Consecutive jobs take
// opposite ends of the accumulator columns: job i from column 0 when i is
// even, else ending at kPAccEnd (its first column rounded down to 32), so
// that two jobs of up to kPMaxN columns overlap in at most 160 columns. The
// epilogue drains the columns the next job will write first and frees the
// accumulator then; the MMAs of the next job run while it drains the rest.
constexpr uint32_t kPColSfa = 496, kPColSfb = kPColSfa + 4;
constexpr int kPAccEnd = (int)kPColSfa;
constexpr int kPOddMin = (kPAccEnd - kPMaxN) / 32 * 32;   // lowest first column of an odd job
static_assert(kPColSfb + 12 <= 512 && kPOddMin >= 128, "tensor memory");
__device__ __forceinline__ int acc_base(uint32_t job, int ncol) {
  return (job & 1u) ? (kPAccEnd - ncol) / 32 * 32 : 0;
}

struct PairParams {
  CUtensorMap tm_wg, tm_wu;       // gate / up weights, boxes of 64 rows
  CUtensorMap tm_wd;              // down weights, boxes of 128 rows
  CUtensorMap tm_x[4], tm_h[4];   // token rows, boxes of 16, 32, 64, 128 rows
  CUtensorMap tm_xsf, tm_hsf;     // token scale atoms, one 512-byte atom per box
  const float* sg;
  const float* su;
  const float* sd;
  void* hq;
  float* hs;
  void* y;
  Ws ws;
  int H, I, E, cap, tpe;
  int compact, streaming, R, ep_sources;
  int n_islices, n_hslices, nk1, nk2, hgroups, igroups;
  int64_t tiles;
};

// One job: rows of one chunk (first global tile `slot`, `ntl` tiles) for one
// slice (gate/up) or slice pair (down).
struct PJob {
  int e, slice, rows, kind, ntl, slot;
};

__device__ __forceinline__ int4 pack(const PJob& j) {
  return make_int4(j.e, j.slice, j.rows | (j.kind << 12) | (j.ntl << 16), j.slot);
}

__device__ __forceinline__ PJob unpack(int4 v) {
  PJob j;
  j.e = v.x;
  j.slice = v.y;
  j.rows = v.z & 0xFFF;
  j.kind = (v.z >> 12) & 0xF;
  j.ntl = (v.z >> 16) & 0xF;
  j.slot = v.w;
  return j;
}

// Chunks of an expert with c rows (c <= 0: none): pairs of tiles, the last
// tile joining the pair before it when it holds at most kPTail rows.
__device__ __forceinline__ int chunks_of(int c) {
  if (c <= 0) return 0;
  const int nt = (c + kTileRows - 1) / kTileRows;
  const int last = c - (nt - 1) * kTileRows;
  return (nt & 1) && nt >= 3 && last <= kPTail ? nt / 2 : (nt + 1) / 2;
}

// Token columns of the MMAs of a job of `rows` rows (multiples of 32, so that
// each CTA's half is a whole number of 16-row boxes): one MMA up to 256, else
// the first tile (128) and the rest (at most 192). An MMA's time has a floor
// of about 80 cycles at small N and grows with N above it, so 128 + 192
// costs less than 256 plus a thin MMA of the joined tile's rows. The second
// MMA starts on a tile boundary, where its token scales start a scale atom.
__device__ __forceinline__ void split_n(int rows, int* n1, int* n2) {
  const int a = rows > 256 ? 128 : rows, b = rows - a;
  *n1 = (a + 31) & ~31;
  *n2 = b > 0 ? (b + 31) & ~31 : 0;
}

// Load `n` (a multiple of 16) token rows starting at global row `row` into
// dst, in the fewest boxes of 128/64/32/16 rows (each map at a fixed address).
__device__ __forceinline__ void load_rows(const CUtensorMap* tm, uint8_t* dst, uint32_t bar, int kx, int row, int n) {
  int r = 0;
  while (n - r >= 128) { ptx::tma_load_2d_pair(dst + r * kSlab, &tm[3], bar, kx, row + r); r += 128; }
  if (n - r >= 64) { ptx::tma_load_2d_pair(dst + r * kSlab, &tm[2], bar, kx, row + r); r += 64; }
  if (n - r >= 32) { ptx::tma_load_2d_pair(dst + r * kSlab, &tm[1], bar, kx, row + r); r += 32; }
  if (n - r >= 16) { ptx::tma_load_2d_pair(dst + r * kSlab, &tm[0], bar, kx, row + r); r += 16; }
}

__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.f + expf(-g)); }

template <int kUnused>
__global__ void __launch_bounds__(kThreads, 1) ffn_pair_kernel(const __grid_constant__ PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ctl = smem + kPStages * kPStride;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);   // [kPStages] even CTA: both halves landed
  uint64_t* empty = full + kPStages;                   // [kPStages] each CTA: the stage's MMAs are done
  uint64_t* acc_full = empty + kPStages;               // each CTA: the job's accumulators are complete
  uint64_t* acc_empty = acc_full + 1;                  // even CTA: both epilogues drained them
  uint64_t* drain = acc_empty + 1;
  uint64_t* xchg = drain + 1;                          // [2] each CTA: the peer's token maxima are here
  uint64_t* uq_full = xchg + 2;                        // [kUQ]
  uint64_t* uq_empty = uq_full + kUQ;                  // [kUQ] even CTA: all five consumers took the job
  uint64_t* tab_free = uq_empty + kUQ;                 // [3] even CTA: a job's scale-atom copies are done
  static_assert((2 * kPStages + 5 + kPTabRing + 2 * kUQ) * 8 <= 512, "barriers fit");
  int4* uq = reinterpret_cast<int4*>(ctl + 512);       // [kUQ]
  int4* epi_job = reinterpret_cast<int4*>(ctl + 640);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 656);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 660);
  float* red = reinterpret_cast<float*>(ctl + 1024);          // [2 sets][4 quarters][32]
  float* amax_loc = reinterpret_cast<float*>(ctl + 2048);     // [2][kPMaxN] this CTA's token maxima
  float* amax_peer = reinterpret_cast<float*>(ctl + 4608);    // [2][kPMaxN] written by the peer
  float* sinv = reinterpret_cast<float*>(ctl + 7168);         // [kPMaxN] 1 / scale per token
  float* swap = reinterpret_cast<float*>(ctl + 9216);         // SwiGLU swap buffers
  uint8_t* sfa_tab = ctl + 9216 + kPSwapBytes;                 // [kPTabRing][kPMaxGroups][128 B]
  static_assert(7168 + kPMaxN * 4 <= 9216, "control bytes");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();   // 0: issues the MMAs and schedules
  const uint32_t peer = rank ^ 1u;
  auto remote = [&](const void* local, uint32_t r) { return ptx::mapa_shared(ptx::smem_u32(local), r); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      ptx::mbar_init(full + s, 1);        // the even CTA's arm, expecting the bytes of both halves
      ptx::mbar_init(empty + s, 1);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(acc_empty, 2);
    ptx::mbar_init(drain, 1);
    ptx::mbar_init(xchg, 1);
    ptx::mbar_init(xchg + 1, 1);
    for (int q = 0; q < kUQ; ++q) {
      ptx::mbar_init(uq_full + q, 1);
      ptx::mbar_init(uq_empty + q, 5);   // producer, MMA issuer, epilogue (even) + producer, epilogue (odd)
    }
    for (int t = 0; t < kPTabRing; ++t) ptx::mbar_init(tab_free + t, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, 512);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();   // both CTAs' barriers and tensor memory exist before any remote use
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const uint32_t epoch = p.streaming ? p.ws.hdr->epoch_plan : p.ws.hdr->epoch_cur;
  uint32_t* set = p.ws.set[epoch & 1];
  uint32_t* misc = set_misc(set);
  const uint32_t gen = ld_acquire(misc + kFfnGen);
  uint32_t* hdone = set_hdone(set, p.E, p.tiles);
  Header* hdr = p.ws.hdr;

  // Take job i from this CTA's queue (one lane of a consumer role); the odd
  // CTA's consumers free the slot on the even CTA's barrier.
  auto take_job = [&](uint32_t i, PJob* out) -> bool {
    const uint32_t q = i % kUQ, ph = (i / kUQ) & 1u;
    if (!wait_bar<true>(uq_full + q, ph, abort_flag, hdr, 0x81000000u | q)) return false;
    *out = unpack(uq[q]);
    if (rank == 0) ptx::mbar_arrive(uq_empty + q);
    else ptx::mbar_arrive_cluster(remote(uq_empty + q, 0));
    return true;
  };

  if (warp == kSchedWarp) {
    // ---------------------------------------------------------------- scheduler (even CTA)
    if (rank == 0) {
      int* chunk_tab = reinterpret_cast<int*>(ctl + kPCtlBytes);   // [E + 1] first chunk of each window
      if (p.ep_sources && lane == 0) {   // expert parallelism: every source closed its dispatch here
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
      const uint32_t* cnt = p.streaming ? set_pre(set, p.E, p.tiles) : set_count(set);
      const uint32_t* base = p.compact ? set_base(set, p.E, p.tiles) : nullptr;
      int ntab = 0;
      {
        const int per = (p.E + 31) / 32;
        int lt = 0, lc = 0;
        for (int i = 0; i < per; ++i) {
          const int e = lane * per + i;
          if (e < p.E) {
            const int c = (int)min(ld_acquire(cnt + e), (uint32_t)p.cap);
            lt += (c + kTileRows - 1) / kTileRows;
            lc += chunks_of(c);
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
            chunk_tab[e] = rc;
            rc += chunks_of((int)min(ld_acquire(cnt + e), (uint32_t)p.cap));
          }
        }
        if (lane == 31) chunk_tab[p.E] = ic;
        ntab = __shfl_sync(0xffffffffu, it, 31);
        __syncwarp();
      }
      const uint32_t ntiles = p.streaming ? 0u : ld_acquire(misc + kRingTotal);
      uint32_t i = 0;   // jobs pushed so far (the queue index; every lane keeps it)
      auto push = [&](const PJob& j) -> bool {   // lane 0
        const uint32_t q = i % kUQ, ph = (i / kUQ) & 1u;
        if (!wait_bar<true>(uq_empty + q, ph ^ 1u, abort_flag, hdr, 0x91000000u | q)) return false;
        const int4 v = pack(j);
        uq[q] = v;
        ptx::st_cluster_v4(remote(uq + q, 1), v);
        ptx::mbar_arrive(uq_full + q);
        ptx::mbar_arrive_cluster(remote(uq_full + q, 1));
        return true;
      };
      // The weight scale atoms of job i, for both CTAs (warp-wide): e4m3
      // weights have one scale per 128 x 128 block, so an atom's 32 rows are
      // identical and a K group of four blocks is 8 rows of 16 bytes (the
      // copy reads them with a zero stride between its four 8-row core
      // matrices). Row m of A is lane m % 32, column m / 32 of an atom:
      // gate/up rows 0-63 are gate and 64-127 up (columns 0-1 gate, 2-3 up);
      // a down job's even CTA holds slice 2 p, the odd one 2 p + 1. Built a
      // few jobs ahead in a ring of three tables, each rewritten only after
      // the copies of the job three before it are done, so that neither the
      // loads nor the MMAs wait for it.
      auto build_table = [&](const PJob& j) -> bool {
        const bool down = j.kind == kKindDown;
        const int we = j.e / p.R;
        const int nkb = down ? p.I / 128 : p.H / 128;
        const float* pa = down ? p.sd + ((int64_t)we * p.n_hslices + 2 * j.slice) * nkb
                               : p.sg + ((int64_t)we * p.n_islices + j.slice) * nkb;
        const float* pb = down ? pa + nkb : p.su + ((int64_t)we * p.n_islices + j.slice) * nkb;
        const uint32_t ts = i % kPTabRing;
        int t_ok = 1;
        if (i >= (uint32_t)kPTabRing && lane == 0)
          t_ok = wait_bar(tab_free + ts, (i / kPTabRing - 1u) & 1u, abort_flag, hdr, 0x43000000u | ts);
        if (!__shfl_sync(0xffffffffu, t_ok, 0)) return false;
        bool bad = false;
        auto take = [&](const float* src, int kb) -> uint32_t {
          const float v = __ldg(src + kb);
          bad |= !pow2_scale_ok(v);
          return ue8m0(v);
        };
        uint32_t sa0 = 0, sa1 = 0, sb0 = 0, sb1 = 0;   // exponents of blocks lane and lane + 32
        if (lane < nkb) { sa0 = take(pa, lane); sb0 = take(pb, lane); }
        if (lane + 32 < nkb) { sa1 = take(pa, lane + 32); sb1 = take(pb, lane + 32); }
        if (__ballot_sync(0xffffffffu, bad) != 0u && lane == 0)
          latch_error(hdr, MOE_ERR_INVALID_ARG, 0x25000000u | (uint32_t)we);
        auto pack4 = [&](uint32_t r0, uint32_t r1, int kr) -> uint32_t {
          uint32_t w = 0;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int kk = kr + b;
            const uint32_t v = __shfl_sync(0xffffffffu, kk < 32 ? r0 : r1, kk & 31);
            w |= (kk < nkb ? v : 0u) << (8 * b);
          }
          return w;
        };
        uint8_t* tab = sfa_tab + ts * (kPMaxGroups * 128);
        for (int g = 0; g < (nkb + 3) / 4; ++g) {
          const uint32_t wa = pack4(sa0, sa1, 4 * g);
          const uint32_t wb = pack4(sb0, sb1, 4 * g);
          const uint4 own = down ? make_uint4(wa, wa, wa, wa) : make_uint4(wa, wa, wb, wb);
          const uint4 odd = down ? make_uint4(wb, wb, wb, wb) : own;
          if (lane < 8) reinterpret_cast<uint4*>(tab + g * 128)[lane] = own;
          else if (lane < 16)
            ptx::st_cluster_v4(remote(tab + g * 128, 1) + (uint32_t)(lane - 8) * 16u,
                               make_int4((int)odd.x, (int)odd.y, (int)odd.z, (int)odd.w));
        }
        ptx::fence_proxy_async_cluster();   // both tables -> the pair's copies
        __syncwarp();
        return true;
      };
      bool good = !*abort_flag;
      {
        int ok = 1;
        if (lane == 0 && good && !p.streaming && (uint32_t)ntab != ntiles) {
          latch_error(hdr, MOE_ERR_INVALID_ARG, 0x24000000u | (uint32_t)ntab);
          *abort_flag = 1;
          ok = 0;
        }
        good = good && __shfl_sync(0xffffffffu, ok, 0);
      }
      const uint32_t nchunks = (uint32_t)chunk_tab[p.E];
      const uint32_t npairs = (uint32_t)(p.n_hslices / 2);
      const uint32_t n1 = nchunks * (uint32_t)p.n_islices;
      const uint32_t total = n1 + nchunks * npairs;
      while (good) {
        // lane 0 resolves the next unit (1: a job, 0: none left, -1: a wait failed)
        int state = 0;
        int4 jv = make_int4(0, 0, 0, 0);
        if (lane == 0) {
          const uint32_t u = atomicAdd(misc + kFfnNext, 1u);
          if (u < total) {
            PJob j;
            j.kind = u >= n1 ? kKindDown : kKindGateUp;
            const uint32_t v = j.kind == kKindDown ? u - n1 : u;
            const uint32_t ns = j.kind == kKindDown ? npairs : (uint32_t)p.n_islices;
            // weight expert (R windows each, expert parallelism), then slice-major
            const int R = p.R;
            int lo = 0, hi = p.E / R - 1;
            while (lo < hi) {
              const int mid = (lo + hi + 1) >> 1;
              if ((uint32_t)chunk_tab[mid * R] * ns <= v) lo = mid;
              else hi = mid - 1;
            }
            const int c0 = chunk_tab[lo * R];
            const uint32_t nc = (uint32_t)(chunk_tab[(lo + 1) * R] - c0);
            const uint32_t w = v - (uint32_t)c0 * ns;
            const int cc = c0 + (int)(w % nc);
            int ve = lo * R;
            while (ve + 1 < (lo + 1) * R && chunk_tab[ve + 1] <= cc) ++ve;
            j.e = ve;
            j.slice = (int)(w / nc);
            const int ci = cc - chunk_tab[ve];                       // chunk within the window
            const int nchv = chunk_tab[ve + 1] - chunk_tab[ve];
            const int c = (int)min(ld_acquire(cnt + ve), (uint32_t)p.cap);
            const int nt = (c + kTileRows - 1) / kTileRows;
            j.ntl = ci == nchv - 1 ? nt - 2 * ci : 2;
            j.slot = (base ? (int)base[ve] : ve * p.tpe) + 2 * ci;
            bool ok = true;
            int rows = 0;
            for (int t = 0; ok && t < j.ntl; ++t) {
              int r = 0;
              ok = wait_tile(p.ws, epoch, j.slot + t, abort_flag, &r);
              rows += r;
            }
            j.rows = rows;
            if (ok && j.kind == kKindDown)   // both CTAs of every gate/up job of this chunk stored their h
              ok = wait_count(hdone + j.slot, 2u * (uint32_t)p.n_islices * (gen + 1u), abort_flag, hdr,
                              0x31000000u | (uint32_t)j.slot);
            state = ok ? 1 : -1;
            jv = pack(j);
          }
        }
        state = __shfl_sync(0xffffffffu, state, 0);
        if (state <= 0) {
          good = state == 0;
          break;
        }
        const PJob j = unpack(shfl_int4(jv));
        if (!build_table(j)) { good = false; break; }
        int pok = 1;
        if (lane == 0) pok = push(j);
        if (!__shfl_sync(0xffffffffu, pok, 0)) { good = false; break; }
        ++i;
      }
      if (lane == 0) {
        PJob end;
        end.e = end.slice = end.rows = end.ntl = end.slot = 0;
        end.kind = good ? kKindEnd : kKindAbort;
        push(end);
      }
      __syncwarp();
    }
  } else if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      ptx::prefetch_tmap(&p.tm_wg);
      ptx::prefetch_tmap(&p.tm_wu);
      ptx::prefetch_tmap(&p.tm_wd);
      ptx::prefetch_tmap(&p.tm_xsf);
      ptx::prefetch_tmap(&p.tm_hsf);
    }
    const uint32_t bar0 = remote(full, 0);   // the even CTA's full barriers (cluster addresses)
    uint32_t stage = 0, phase = 0;
    uint32_t armed_mask = 0, armed_parity = 0;   // even CTA: stages it armed, and their phase
    for (uint32_t i = 0;; ++i) {
      int4 raw = make_int4(0, 0, kKindAbort << 12, 0);
      if (lane == 0) {
        PJob jj;
        if (take_job(i, &jj)) raw = pack(jj);
        ptx::fence_proxy_async_global();   // rows and atoms written by other CTAs -> TMA reads
      }
      const PJob j = unpack(shfl_int4(raw));
      if (j.kind >= kKindEnd) break;
      const bool down = j.kind == kKindDown;
      int n1, n2;
      split_n(j.rows, &n1, &n2);
      const int h1 = n1 / 2, h2 = n2 / 2;
      const int nsteps = down ? p.nk2 : p.nk1;
      const int we = j.e / p.R;
      const int nkb = down ? p.I / 128 : p.H / 128;
      const int slice_w = down ? 2 * j.slice + (int)rank : j.slice;   // down: this CTA's slice of H
      const int arow_g = we * p.I + j.slice * 128 + 64 * (int)rank;    // gate/up: this CTA's 64 features
      const int arow_d = we * p.H + slice_w * 128;                       // down: this CTA's slice
      const int brow = j.slot * kTileRows;
      const CUtensorMap* tmt = down ? p.tm_h : p.tm_x;
      const CUtensorMap* tmsf = down ? &p.tm_hsf : &p.tm_xsf;
      const int groups = down ? p.igroups : p.hgroups;
      bool ok = true;
      for (int st_i = 0; st_i < nsteps; ++st_i) {
        int w_ok = 1;
        if (lane == 0) w_ok = wait_bar(empty + stage, phase ^ 1u, abort_flag, hdr, 0x41000000u | stage);
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        uint8_t* st = smem + stage * kPStride;
        const int kb0 = st_i;   // one 128-value K block per stage
        const bool sf_stage = (kb0 & 3) == 0;
        __syncwarp();
        if (ptx::elect_one()) {
          const uint32_t tx = (uint32_t)(kABytes + (h1 + h2) * kSlab + (sf_stage ? j.ntl * kSfAtomBytes : 0));
          if (rank == 0) ptx::mbar_arrive_expect_tx(full + stage, 2u * tx);   // both halves' bytes
          const uint32_t fb = bar0 + (uint32_t)(stage * 8);
          const int kx = kb0 * 128;
          if (down) {
            ptx::tma_load_2d_pair(st, &p.tm_wd, fb, kx, arow_d);
          } else {
            ptx::tma_load_2d_pair(st, &p.tm_wg, fb, kx, arow_g);
            ptx::tma_load_2d_pair(st + 64 * kSlab, &p.tm_wu, fb, kx, arow_g);
          }
          // token rows: this CTA's half of each MMA's columns
          load_rows(tmt, st + kPOffB, fb, kx, brow + (int)rank * h1, h1);
          if (h2) load_rows(tmt, st + kPOffB + h1 * kSlab, fb, kx, brow + n1 + (int)rank * h2, h2);
          if (sf_stage) {   // the chunk's token scale atoms (the same in both CTAs)
            for (int t = 0; t < j.ntl; ++t)
              ptx::tma_load_2d_pair(st + kPOffSfb + t * kSfAtomBytes, tmsf, fb, 0,
                                    (j.slot + t) * groups + kb0 / 4);
          }
        }
        __syncwarp();
        if (rank == 0) {
          armed_mask |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        }
        if (++stage == (uint32_t)kPStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
    // drain (even CTA): every stage it armed has landed, the odd CTA's copies included
    if (rank == 0 && lane == 0) {
      for (int s = 0; s < kPStages; ++s) {
        if (!((armed_mask >> s) & 1u)) continue;
        const unsigned long long t0 = globaltimer();
        while (!ptx::mbar_try_wait(full + s, (armed_parity >> s) & 1u)) {
          if (globaltimer() - t0 > kWaitBudgetNs) break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (even CTA)
    if (rank == 0) {
      uint32_t stage = 0, phase = 0, acc_ph = 0;
      for (uint32_t i = 0;; ++i) {
        int4 raw = make_int4(0, 0, kKindAbort << 12, 0);
        if (lane == 0) {
          PJob jj;
          if (take_job(i, &jj)) raw = pack(jj);
        }
        const PJob j = unpack(shfl_int4(raw));
        if (j.kind >= kKindEnd) break;
        const bool down = j.kind == kKindDown;
        int n1, n2;
        split_n(j.rows, &n1, &n2);
        const int h1 = n1 / 2;
        int ok = 1;
        if (lane == 0) ok = wait_bar(acc_empty, acc_ph ^ 1u, abort_flag, hdr, 0x51000000u);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        ptx::tc_fence_after();
        const int nsteps = down ? p.nk2 : p.nk1;
        const uint32_t d1 = tmem + (uint32_t)acc_base(i, n1 + n2);   // this job's first accumulator column
        const uint32_t idesc1 = ptx::idesc_mxf8(256, n1, 0);
        const uint32_t idesc2 = ptx::idesc_mxf8(256, n2 > 0 ? n2 : 16, 0);
        for (int st_i = 0; st_i < nsteps; ++st_i) {
          int w_ok = 1;
          const int kb0 = st_i;
          if (lane == 0) w_ok = wait_bar(full + stage, phase, abort_flag, hdr, 0x61000000u | stage);
          if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = 0; break; }
          ptx::tc_fence_after();
          uint8_t* st = smem + stage * kPStride;
          if (ptx::elect_one()) {
            if ((kb0 & 3) == 0) {   // scale atoms into both CTAs' tensor memory
              auto sf_cp = [&](uint32_t col, int off) {
                ptx::tmem_cp_32x128b_x4_pair(tmem + col,
                                             ptx::smem_desc(ptx::smem_u32(st + off), 16, 128, ptx::kLayoutNone));
              };
              const uint8_t* ta = sfa_tab + ((i % kPTabRing) * kPMaxGroups + kb0 / 4) * 128;
              ptx::tmem_cp_32x128b_x4_pair(tmem + kPColSfa,
                                           ptx::smem_desc(ptx::smem_u32(ta), 16, 0, ptx::kLayoutNone));
              for (int t = 0; t < j.ntl; ++t) sf_cp(kPColSfb + 4 * t, kPOffSfb + t * kSfAtomBytes);
            }
            const uint32_t id = (uint32_t)(kb0 & 3);
            const uint64_t a = ptx::desc_kmajor_sw128(st);
            const uint64_t b1 = ptx::desc_kmajor_sw128(st + kPOffB);
            const uint64_t b2 = ptx::desc_kmajor_sw128(st + kPOffB + h1 * kSlab);
            const uint32_t sfa = (tmem + kPColSfa) | (id << 30);
            const uint32_t sfb1 = (tmem + kPColSfb) | (id << 30);
            const uint32_t sfb2 = (tmem + kPColSfb + 4u * (uint32_t)(n1 / 128)) | (id << 30);   // from its first tile's atom
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t off = (uint64_t)(kk * 32) >> 4;
              const uint32_t acc = (st_i > 0 || kk > 0) ? 1u : 0u;
              ptx::mma_mxf8_pair(d1, a + off, b1 + off, idesc1 | (id << 4) | (id << 29), sfa, sfb1, acc);
              if (n2)
                ptx::mma_mxf8_pair(d1 + (uint32_t)n1, a + off, b2 + off, idesc2 | (id << 4) | (id << 29), sfa, sfb2,
                                   acc);
            }
            // the stage is free in both CTAs once these MMAs are done
            ptx::mma_commit_pair(remote(empty + stage, 0));
            ptx::mma_commit_pair(remote(empty + stage, 1));
          }
          __syncwarp();
          if (++stage == (uint32_t)kPStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (ptx::elect_one()) {
          ptx::mma_commit_pair(remote(acc_full, 0));
          ptx::mma_commit_pair(remote(acc_full, 1));
          ptx::mma_commit_pair(remote(tab_free + i % kPTabRing, 0));   // this job's scale-atom table is free
        }
        __syncwarp();
        acc_ph ^= 1u;
      }
      if (ptx::elect_one()) {   // drain: all MMAs and copies issued here are complete
        ptx::mma_commit_pair(remote(drain, 0));
        const unsigned long long t0 = globaltimer();
        while (!ptx::mbar_try_wait(drain, 0)) {
          if (globaltimer() - t0 > kWaitBudgetNs) break;
        }
      }
      __syncwarp();
    }
  } else if (warp >= 2 && warp <= 9) {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    // warp w reads tensor-memory lanes 32 (w % 4) .. + 31; set s (warps 2-5,
    // 6-9) takes the 32-column batches s, s + 2, ... For gate/up, quarters
    // 0-1 hold the gate and 2-3 the up rows of features 32 (q % 2) + lane:
    // the gate warp keeps the even columns of a batch, the up warp the odd
    // ones, and each hands the other its half through shared memory.
    const int q = warp & 3;
    const int et = threadIdx.x - 64;
    const int eset = et >> 7;
    const uint32_t set_bar = 2u + (uint32_t)eset;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const bool up_warp = q >= 2;
    const int fq = q & 1;                                    // feature half: 32 fq .. 32 fq + 31
    const uint32_t pair_bar = 4u + 2u * (uint32_t)eset + (uint32_t)fq;   // the gate and up warp of a half
    float* sw_mine = swap + ((eset * 2 + fq) * 2 + (up_warp ? 1 : 0)) * 512;   // [16 columns][32 lanes]
    float* sw_theirs = swap + ((eset * 2 + fq) * 2 + (up_warp ? 0 : 1)) * 512;
    float* red_s = red + eset * 128;
    uint32_t acc_ph = 0, gu = 0;   // gate/up jobs done (the exchange buffers alternate)
    for (uint32_t i = 0;; ++i) {
      if (et == 0) {
        PJob jj;
        const bool good = take_job(i, &jj);
        if (!good) jj.kind = kKindAbort;
        if (jj.kind < kKindEnd && !wait_bar(acc_full, acc_ph, abort_flag, hdr, 0x71000000u))
          jj.kind = kKindAbort;
        *epi_job = pack(jj);
      }
      ptx::named_barrier(1, kEpiThreads);
      const PJob j = unpack(*epi_job);
      ptx::named_barrier(1, kEpiThreads);
      if (j.kind >= kKindEnd) break;
      while (!ptx::mbar_try_wait(acc_full, acc_ph)) {}   // completed: returns at once
      ptx::tc_fence_after();
      acc_ph ^= 1u;
      const bool down = j.kind == kKindDown;
      int n1, n2;
      split_n(j.rows, &n1, &n2);
      const int ncol = n1 + n2;   // column base + c holds chunk row c
      const int nb = ncol / 32;     // 32-column batches
      const int64_t row0 = (int64_t)j.slot * kTileRows;
      // The batches the next job's accumulator overlaps are drained first:
      // an even job's high ones (the next job starts at kPOddMin or above, so
      // the drain runs from the last batch down), an odd job's low ones (the
      // next starts at column 0 and ends below kPMaxN). The accumulator is
      // freed once each set has drained rel_bi batches.
      const bool odd = (i & 1u) != 0u;
      const uint32_t base = (uint32_t)acc_base(i, ncol);
      const int n_pre = odd ? min(nb, max(0, kPMaxN - (int)base + 31) / 32) : max(0, nb - kPOddMin / 32);
      const int rel_bi = (n_pre + 1) / 2;
      auto col_of = [&](int pos) { return 32 * (odd ? pos : nb - 1 - pos); };   // chunk row of a batch
      auto release = [&]() {   // 2. the overlapped columns are drained in both sets: free them
        ptx::tc_fence_before();
        ptx::named_barrier(1, kEpiThreads);
        if (et == 0) {
          if (rank == 0) ptx::mbar_arrive(acc_empty);
          else ptx::mbar_arrive_remote(remote(acc_empty, 0));
        }
      };
      // 1. drain into registers: h = SwiGLU (gate/up; this thread's feature,
      //    even columns in the gate warp, odd in the up warp) or y in bf16
      //    pairs (down)
      uint32_t v[kPBatches][16];
#pragma unroll
      for (int bi = 0; bi < kPBatches; ++bi) {
        if (bi == rel_bi) release();
        const int pos = eset + 2 * bi;
        if (pos >= nb) continue;   // every thread still reaches the release
        const int c0 = col_of(pos);
        uint32_t r[32];
        ptx::tmem_ld_x16(tmem + lane_base + base + (uint32_t)c0, *reinterpret_cast<uint32_t(*)[16]>(r));
        ptx::tmem_ld_x16(tmem + lane_base + base + (uint32_t)c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
        ptx::tmem_wait_ld();
        if (down) {
#pragma unroll
          for (int k2 = 0; k2 < 16; ++k2) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(r[2 * k2]), __uint_as_float(r[2 * k2 + 1]));
            v[bi][k2] = *reinterpret_cast<uint32_t*>(&b2);
          }
        } else {
#pragma unroll
          for (int k2 = 0; k2 < 16; ++k2)   // the gate warp hands over odd columns, the up warp even ones
            sw_mine[k2 * 32 + lane] = __uint_as_float(up_warp ? r[2 * k2] : r[2 * k2 + 1]);
          ptx::named_barrier(pair_bar, 64);
#pragma unroll
          for (int k2 = 0; k2 < 16; ++k2) {
            const float got = sw_theirs[k2 * 32 + lane];
            const float h = up_warp ? silu_f(got) * __uint_as_float(r[2 * k2 + 1])
                                    : silu_f(__uint_as_float(r[2 * k2])) * got;
            v[bi][k2] = __float_as_uint(h);
          }
          ptx::named_barrier(pair_bar, 64);   // both read: the buffers are free for the next batch
        }
      }
      if (rel_bi >= kPBatches) release();
      if (down) {
        // 3. y rows: lane = feature of this CTA's slice
        __nv_bfloat16* yp = reinterpret_cast<__nv_bfloat16*>(p.y) + row0 * p.H +
                            (2 * j.slice + (int)rank) * 128 + q * 32 + lane;
#pragma unroll
        for (int bi = 0; bi < kPBatches; ++bi) {
          const int pos = eset + 2 * bi;
          if (pos >= nb) break;
          const int c0 = col_of(pos);
#pragma unroll
          for (int k2 = 0; k2 < 16; ++k2) {
            const int c = c0 + 2 * k2;
            if (c < j.rows) yp[(int64_t)c * p.H] = __ushort_as_bfloat16((unsigned short)(v[bi][k2] & 0xFFFFu));
            if (c + 1 < j.rows) yp[(int64_t)(c + 1) * p.H] = __ushort_as_bfloat16((unsigned short)(v[bi][k2] >> 16));
          }
        }
        continue;
      }
      // 3. each token's max over this CTA's 64 features: over the warp's 32
      //    features, then over the two warps holding the column
      const uint32_t par = gu & 1u;
      float* aloc = amax_loc + par * kPMaxN;
      const uint32_t apeer_remote = remote(amax_peer + par * kPMaxN, peer);
#pragma unroll
      for (int bi = 0; bi < kPBatches; ++bi) {
        const int pos = eset + 2 * bi;
        if (pos >= nb) break;
        const int c0 = col_of(pos);
#pragma unroll
        for (int k2 = 0; k2 < 16; ++k2) {   // |h| bit patterns order like the values
          const uint32_t m = __reduce_max_sync(0xffffffffu, v[bi][k2] & 0x7FFFFFFFu);
          if (lane == k2) red_s[q * 32 + k2] = __uint_as_float(m);
        }
        ptx::named_barrier(set_bar, 128);
        if (q == 0) {   // column c0 + lane: even ones in the gate warps (quarters 0, 1), odd in the up warps
          const int hq2 = (lane & 1) ? 64 : 0, k2 = lane >> 1;
          const float a = fmaxf(red_s[hq2 + k2], red_s[hq2 + 32 + k2]);
          aloc[c0 + lane] = a;
          ptx::st_cluster_u32(apeer_remote + (uint32_t)(c0 + lane) * 4u, __float_as_uint(a));
        }
        ptx::named_barrier(set_bar, 128);
      }
      // 4. exchange with the peer: its maxima are here once its arrive lands
      ptx::named_barrier(1, kEpiThreads);
      if (et == 0) {
        ptx::mbar_arrive_cluster(remote(xchg + par, peer));
        if (!wait_bar<true>(xchg + par, (gu >> 1) & 1u, abort_flag, hdr, 0x72000000u)) {}
      }
      ptx::named_barrier(1, kEpiThreads);
      const float* apeer = amax_peer + par * kPMaxN;
      for (int c = et; c < j.rows; c += kEpiThreads) {
        const float amax = fmaxf(aloc[c], apeer[c]);
        const int pe = pow2_scale_exp(amax);
        sinv[c] = exp2i(-pe > -126 ? -pe : -126);
        if (rank == 0) {
          const int64_t r = row0 + c;
          p.hs[r * (p.I / 128) + j.slice] = exp2i(pe);
          *sf_atom_byte(p.ws.hsf, j.slot + c / kTileRows, p.igroups, j.slice, c % kTileRows) = (uint8_t)(pe + 127);
        }
      }
      ptx::named_barrier(1, kEpiThreads);
      // 5. requantised h: this thread's feature, its columns
      uint8_t* hp = reinterpret_cast<uint8_t*>(p.hq) + row0 * p.I + j.slice * 128 + 64 * (int)rank + 32 * fq + lane;
#pragma unroll
      for (int bi = 0; bi < kPBatches; ++bi) {
        const int pos = eset + 2 * bi;
        if (pos >= nb) break;
        const int c0 = col_of(pos);
#pragma unroll
        for (int k2 = 0; k2 < 16; ++k2) {
          const int c = c0 + 2 * k2 + (up_warp ? 1 : 0);
          if (c < j.rows)
            hp[(int64_t)c * p.I] = (uint8_t)(cvt_e4m3x2(__uint_as_float(v[bi][k2]) * sinv[c], 0.f) & 0xFF);
        }
      }
      ++gu;
      // 6. this CTA's half of the slice is stored: count it for the down jobs
      __threadfence();
      ptx::named_barrier(1, kEpiThreads);
      if (et == 0) atomicAdd(hdone + j.slot, 1u);
    }
  }
  // every role is done in both CTAs (and every copy, MMA and remote access
  // with them) before tensor memory is freed and either CTA exits
  ptx::tc_fence_before();
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, 512);
  }
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t exits = atomicAdd(misc + kFfnExit, 1u) + 1u;
    if (exits == gridDim.x * (gen + 1u)) {
      misc[kFfnNext] = 0u;
      __threadfence();
      st_release(misc + kFfnGen, gen + 1u);
    }
  }
}

// 2-D map over the scale atoms [tiles * groups, 512 B] as rows of 128 words,
// one atom per box.
bool make_atom_tmap(CUtensorMap* m, const void* base, int64_t atoms) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {128, (cuuint64_t)(atoms > 0 ? atoms : 1)};
  cuuint64_t strides[1] = {512};
  cuuint32_t box[2] = {128, 1};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool ffn_pair_supported(const Ctx& c) {
  const moe_shape& s = c.s;
  return s.weight_dtype == MOE_E4M3 && s.xq_dtype == MOE_E4M3 && s.h_dtype == MOE_E4M3 &&
         s.y_dtype == MOE_BF16 && !s.identity_experts && (s.H / 128) % 2 == 0 && s.H % 128 == 0 &&
         s.I % 128 == 0 && s.H <= 128 * 4 * kPMaxGroups && s.I <= 128 * 4 * kPMaxGroups && c.s.E <= 1024;
}

cudaError_t launch_ffn_pair(const Ctx& c, const moe_dispatch_bufs& b, const moe_weights& w, void* y) {
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(ffn_pair_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  PairParams p;
  memset(&p, 0, sizeof(p));
  const int64_t H = c.s.H, I = c.s.I, E = c.s.E, rows = c.L.tiles * kTileRows;
  const int64_t wexp = c.ep_ranks > 0 ? E / c.ep_ranks : E;   // experts with weights here
  if (!make_tmap(&p.tm_wg, w.w_gate, kElU8, H, wexp * I, 128, 64) ||
      !make_tmap(&p.tm_wu, w.w_up, kElU8, H, wexp * I, 128, 64) ||
      !make_tmap(&p.tm_wd, w.w_down, kElU8, I, wexp * H, 128, 128))
    return cudaErrorInvalidValue;
  for (int bx = 0; bx < 4; ++bx) {
    if (!make_tmap(&p.tm_x[bx], b.xq, kElU8, H, rows, 128, 16 << bx) ||
        !make_tmap(&p.tm_h[bx], b.hq, kElU8, I, rows, 128, 16 << bx))
      return cudaErrorInvalidValue;
  }
  if (!make_atom_tmap(&p.tm_xsf, c.ws.xsf, c.L.tiles * c.L.hgroups) ||
      !make_atom_tmap(&p.tm_hsf, c.ws.hsf, c.L.tiles * c.L.igroups))
    return cudaErrorInvalidValue;
  p.sg = (const float*)w.s_gate;
  p.su = (const float*)w.s_up;
  p.sd = (const float*)w.s_down;
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
  p.nk1 = (int)(H / 128);
  p.nk2 = (int)(I / 128);
  p.hgroups = (int)c.L.hgroups;
  p.igroups = (int)c.L.igroups;
  p.tiles = c.L.tiles;
  // one persistent pair per two SMs, as many as can be resident at once
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  const int pairs = std::max(1, c.num_sms / 2);   // at least one pair, even on a one-SM share
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kPSmemBytes;
  cfg.stream = c.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, ffn_pair_kernel<0>, &cfg) == cudaSuccess && clusters > 0)
    cfg.gridDim.x = (unsigned)(2 * std::min(clusters, pairs));
  (void)cudaGetLastError();   // a failed query is not the launch's error
  return cudaLaunchKernelEx(&cfg, ffn_pair_kernel<0>, p);
}

}  // namespace moe

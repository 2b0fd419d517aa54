// Grouped expert FFN on the CUDA cores (fp32 FFMA), for the fp32 layer.
//
// Same schedule as the tensor-core kernel, without tensor cores: work units
// are (published tile, 128-feature slice); each unit waits for its tile's
// sentinel, then computes G and U (gate/up pass) or y (down pass) for up to
// 128 rows in 32-row steps with shared-memory tiles of 32 along K.
// h = silu(G) * U (SwiGLU, GC-MoE feed item "Full text"), requantised per 128
// values when stored as e4m3.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kF = 128;   // features per unit
constexpr int kR = 32;    // rows per step
constexpr int kK = 32;    // K per shared-memory stage

struct Args {
  const void* xq;  const float* xs;     // gate/up input rows
  void* hq;        float* hs;           // SwiGLU output rows
  void* y;
  const void* wg;  const void* wu;  const void* wd;
  const float* sg; const float* su; const float* sd;
  int H, I, E;
  int64_t tiles;                        // global tiles in the expert buffers
  int xq_dt, w_dt, h_dt, y_dt;
  Ws ws;
  uint8_t* hsf;
};

__device__ __forceinline__ float ld_act(const void* p, int dt, int64_t i) {
  if (dt == MOE_F32) return reinterpret_cast<const float*>(p)[i];
  if (dt == MOE_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  return e4m3_to_f32(reinterpret_cast<const uint8_t*>(p)[i]);
}

// Find the global tile behind ring slot `slot` for the current epoch (bounded wait).
__device__ bool fetch_tile(const Args& a, uint32_t epoch, uint32_t slot, int* e, int* tile,
                           int* rows) {
  const unsigned long long t0 = globaltimer();
  unsigned long long ent;
  while (true) {
    ent = ld_acquire64(a.ws.ring + slot);
    if ((uint32_t)(ent >> 40) == (epoch & 0xFFFFFFu)) break;
    if (globaltimer() - t0 > kWaitBudgetNs) {
      latch_error(a.ws.hdr, MOE_ERR_TIMEOUT, slot);
      return false;
    }
    __nanosleep(256);
  }
  *e = (int)((ent >> 24) & 0xFFFF);
  *tile = (int)(ent & 0xFFFFFF);
  if (*e >= a.E || *tile >= a.tiles) {          // never published: a corrupt workspace
    latch_error(a.ws.hdr, MOE_ERR_INVALID_ARG, slot);
    return false;
  }
  const uint32_t* sp = a.ws.sentinel + *tile;
  while (true) {
    const uint32_t s = ld_acquire(sp);
    if ((s >> 8) == (epoch & 0xFFFFFFu)) {
      *rows = (int)(s & 0xFF);
      if (*rows < 1 || *rows > kTileRows) {
        latch_error(a.ws.hdr, MOE_ERR_INVALID_ARG, slot);
        return false;
      }
      return true;
    }
    if (globaltimer() - t0 > kWaitBudgetNs) {
      latch_error(a.ws.hdr, MOE_ERR_TIMEOUT, slot);
      return false;
    }
    __nanosleep(256);
  }
}

__device__ __forceinline__ float silu(float g) { return g / (1.f + expf(-g)); }

// DOWN = false: gate/up + SwiGLU; DOWN = true: y = h W_down^T
template <bool DOWN>
__global__ void __launch_bounds__(kThreads) ffn_simt_kernel(Args a) {
  __shared__ float sx[kR][kK + 1];
  __shared__ float sw0[kF][kK + 1];
  __shared__ float sw1[DOWN ? 1 : kF][kK + 1];
  __shared__ float samax[kR][4];
  __shared__ int s_info[4];

  const int tid = threadIdx.x;
  const int f = tid & (kF - 1);
  const int rh = tid >> 7;          // rows rh*16 .. rh*16+15 of a step
  const int K = DOWN ? a.I : a.H;
  const int NF = DOWN ? a.H : a.I;  // output features
  const int nslices = NF / kF;
  const uint32_t epoch = a.ws.hdr->epoch_cur;
  const uint32_t* misc = set_misc(a.ws.set[epoch & 1]);
  const uint32_t total = ld_acquire(misc + kRingTotal);
  const void* xin = DOWN ? a.hq : a.xq;
  const float* xsc = DOWN ? a.hs : a.xs;
  const int xdt = DOWN ? a.h_dt : a.xq_dt;

  for (uint32_t u = blockIdx.x; u < total * (uint32_t)nslices; u += gridDim.x) {
    const uint32_t slot = u / nslices;
    const int slice = (int)(u % nslices);
    if (tid == 0) {
      int e = 0, tile = 0, rows = 0;
      const bool ok = fetch_tile(a, epoch, slot, &e, &tile, &rows);
      s_info[0] = ok ? e : -1; s_info[1] = tile; s_info[2] = rows;
    }
    __syncthreads();
    const int e = s_info[0], tile = s_info[1], rows = s_info[2];
    __syncthreads();
    if (e < 0) continue;
    const int64_t row0 = (int64_t)tile * kTileRows;   // global tile
    const int f0 = slice * kF;
    const void* w0 = DOWN ? a.wd : a.wg;
    const void* w1 = a.wu;
    const float* s0 = DOWN ? a.sd : a.sg;
    const float* s1 = a.su;
    const int64_t wrow0 = (int64_t)e * NF + f0;   // first weight row of this unit

    for (int r0 = 0; r0 < rows; r0 += kR) {
      float g[16], uu[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) { g[i] = 0.f; uu[i] = 0.f; }
      // K steps software-pipelined: the next step's loads are issued before
      // this step's FMAs, so each step's global-load latency overlaps work
      constexpr int kXPer = kR * kK / kThreads;   // 4
      constexpr int kWPer = kF * kK / kThreads;   // 16
      float xv[kXPer], wv0[kWPer], wv1[kWPer], sc0 = 1.f, sc1 = 1.f;
      auto load_step = [&](int k0) {
#pragma unroll
        for (int i = 0; i < kXPer; ++i) {
          const int idx = tid + kThreads * i, r = idx / kK, kk = idx % kK;
          xv[i] = 0.f;
          if (r0 + r < rows) {
            const int64_t row = row0 + r0 + r;
            xv[i] = ld_act(xin, xdt, row * K + k0 + kk);
            if (xdt == MOE_E4M3) xv[i] *= xsc[row * (K / kQBlock) + (k0 + kk) / kQBlock];
          }
        }
        if (a.w_dt == MOE_E4M3) {
          const int64_t sidx = ((int64_t)e * (NF / kQBlock) + f0 / kQBlock) * (K / kQBlock) + k0 / kQBlock;
          sc0 = s0[sidx];
          if (!DOWN) sc1 = s1[sidx];
        }
#pragma unroll
        for (int i = 0; i < kWPer; ++i) {
          const int idx = tid + kThreads * i, ff = idx / kK, kk = idx % kK;
          const int64_t widx = (wrow0 + ff) * K + k0 + kk;
          wv0[i] = ld_act(w0, a.w_dt, widx);
          wv1[i] = DOWN ? 0.f : ld_act(w1, a.w_dt, widx);
        }
      };
      load_step(0);
      for (int k0 = 0; k0 < K; k0 += kK) {
#pragma unroll
        for (int i = 0; i < kXPer; ++i) {
          const int idx = tid + kThreads * i;
          sx[idx / kK][idx % kK] = xv[i];
        }
#pragma unroll
        for (int i = 0; i < kWPer; ++i) {
          const int idx = tid + kThreads * i;
          sw0[idx / kK][idx % kK] = wv0[i] * sc0;
          if (!DOWN) sw1[idx / kK][idx % kK] = wv1[i] * sc1;
        }
        __syncthreads();
        if (k0 + kK < K) load_step(k0 + kK);
#pragma unroll 4
        for (int kk = 0; kk < kK; ++kk) {
          const float b0 = sw0[f][kk];
          const float b1 = DOWN ? 0.f : sw1[f][kk];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float xv_ = sx[rh * 16 + i][kk];
            g[i] = fmaf(xv_, b0, g[i]);
            if (!DOWN) uu[i] = fmaf(xv_, b1, uu[i]);
          }
        }
        __syncthreads();
      }

      if (DOWN) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = r0 + rh * 16 + i;
          if (r >= rows) break;
          const int64_t o = (row0 + r) * a.H + f0 + f;
          if (a.y_dt == MOE_F32) reinterpret_cast<float*>(a.y)[o] = g[i];
          else reinterpret_cast<__nv_bfloat16*>(a.y)[o] = __float2bfloat16_rn(g[i]);
        }
        continue;
      }
      float h[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) h[i] = silu(g[i]) * uu[i];
      if (a.h_dt == MOE_E4M3) {
        const int warp = (tid >> 5) & 3;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float m = fabsf(h[i]);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
          if ((tid & 31) == 0) samax[rh * 16 + i][warp] = m;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int rr = rh * 16 + i;
          const int r = r0 + rr;
          const float m = fmaxf(fmaxf(samax[rr][0], samax[rr][1]), fmaxf(samax[rr][2], samax[rr][3]));
          const int p = pow2_scale_exp(m);
          if (r < rows) {
            const int64_t row = row0 + r;
            const float q = h[i] * exp2i(-p > -126 ? -p : -126);
            const uint16_t b2 = cvt_e4m3x2(q, 0.f);
            reinterpret_cast<uint8_t*>(a.hq)[row * a.I + f0 + f] = (uint8_t)(b2 & 0xFF);
            if (f == 0) {
              a.hs[row * (a.I / kQBlock) + slice] = exp2i(p);
              if (a.hsf)
                *sf_atom_byte(a.hsf, row / kTileRows, (a.I + 4 * kQBlock - 1) / (4 * kQBlock), slice,
                              (int)(row % kTileRows)) = (uint8_t)(p + 127);
            }
          }
        }
        __syncthreads();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = r0 + rh * 16 + i;
          if (r >= rows) break;
          const int64_t o = (row0 + r) * a.I + f0 + f;
          if (a.h_dt == MOE_F32) reinterpret_cast<float*>(a.hq)[o] = h[i];
          else reinterpret_cast<__nv_bfloat16*>(a.hq)[o] = __float2bfloat16_rn(h[i]);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_ffn_simt(const Ctx& c, const moe_dispatch_bufs& b, const moe_weights& w,
                            void* y) {
  Args a;
  a.xq = b.xq; a.xs = b.xs; a.hq = b.hq; a.hs = b.hs; a.y = y;
  a.wg = w.w_gate; a.wu = w.w_up; a.wd = w.w_down;
  a.sg = (const float*)w.s_gate; a.su = (const float*)w.s_up; a.sd = (const float*)w.s_down;
  a.H = (int)c.s.H; a.I = (int)c.s.I; a.E = (int)c.s.E;
  a.tiles = c.L.tiles;
  a.xq_dt = c.s.xq_dtype; a.w_dt = c.s.weight_dtype; a.h_dt = c.s.h_dtype; a.y_dt = c.s.y_dtype;
  a.ws = c.ws;
  a.hsf = c.s.h_dtype == MOE_E4M3 ? c.ws.hsf : nullptr;
  const int grid = c.num_sms * 4;
  ffn_simt_kernel<false><<<grid, kThreads, 0, c.stream>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  ffn_simt_kernel<true><<<grid, kThreads, 0, c.stream>>>(a);
  return cudaGetLastError();
}

}  // namespace moe

// Host side of the C ABI declared in include/moe.h: argument checks, the
// workspace, and the kernel launches of each stage.
#include <algorithm>
#include <cstring>

#include "moe_internal.cuh"

namespace moe {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

namespace {

// activation, row and output dtypes (E2M1 is a weight dtype only)
bool is_dtype(int32_t d) { return d == MOE_F32 || d == MOE_BF16 || d == MOE_E4M3; }

}  // namespace

// Shape and dtype checks shared by every entry point.
moe_status check_shape(const moe_shape* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->H <= 0 || s->E < 1 || s->E > 65535) return MOE_ERR_INVALID_ARG;
  if (s->topk < 1 || s->topk > s->E || s->topk > kMaxTopk) return MOE_ERR_INVALID_ARG;
  if (s->quant_block != kQBlock || (s->flags & ~(MOE_FLAG_SHARED_EXPERT | MOE_FLAG_COMPACT)) != 0)
    return MOE_ERR_INVALID_ARG;
  const bool shared = (s->flags & MOE_FLAG_SHARED_EXPERT) != 0;
  const bool compact = (s->flags & MOE_FLAG_COMPACT) != 0;
  if (shared && (s->identity_experts || s->topk + 1 > kMaxTopk || s->E + 1 > 65535 ||
                 (!compact && default_cap(*s) < s->T)))
    return MOE_ERR_INVALID_ARG;   // the shared expert takes every token
  if ((s->renorm != 0 && s->renorm != 1) || (s->identity_experts != 0 && s->identity_experts != 1))
    return MOE_ERR_INVALID_ARG;
  if (s->cap_rows < 0 || (s->cap_rows > 0 && s->cap_rows % kTileRows != 0)) return MOE_ERR_INVALID_ARG;
  if (s->E > 1024) return MOE_ERR_UNSUPPORTED;      // route keeps a row in registers
  if (s->H % 16 != 0 || s->H > (1 << 24)) return MOE_ERR_INVALID_ARG;
  if (!is_dtype(s->act_dtype) || !is_dtype(s->xq_dtype) || !is_dtype(s->out_dtype))
    return MOE_ERR_INVALID_ARG;
  if (s->act_dtype == MOE_E4M3 || s->out_dtype == MOE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (s->xq_dtype == MOE_E4M3 && s->H % kQBlock != 0) return MOE_ERR_INVALID_ARG;
  const int64_t ne = s->E + (shared ? 1 : 0), nk = s->topk + (shared ? 1 : 0);
  if (s->T * nk >= (int64_t)INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (compact) {
    // windows sized by the counting pass; tile ids fit 16 bits per expert
    if (s->cap_rows != 0 || ceil_div(s->T * nk, kTileRows) + ne > 65535) return MOE_ERR_INVALID_ARG;
  } else {
    const int64_t cap = default_cap(*s);
    if (cap / kTileRows > 65535 || ne * cap >= (int64_t)INT32_MAX) return MOE_ERR_INVALID_ARG;
  }
  if (s->identity_experts) return MOE_OK;
  if (s->I <= 0 || s->I > (1 << 24) || s->I % 16 != 0) return MOE_ERR_INVALID_ARG;
  if ((!is_dtype(s->weight_dtype) && s->weight_dtype != MOE_E2M1) || !is_dtype(s->h_dtype) ||
      !is_dtype(s->y_dtype))
    return MOE_ERR_INVALID_ARG;
  if (s->y_dtype == MOE_E4M3) return MOE_ERR_UNSUPPORTED;
  const bool f32 = s->act_dtype == MOE_F32 && s->xq_dtype == MOE_F32 && s->weight_dtype == MOE_F32 &&
                   s->h_dtype == MOE_F32 && s->y_dtype == MOE_F32 && s->out_dtype == MOE_F32;
  const bool bf16 = s->act_dtype == MOE_BF16 && s->xq_dtype == MOE_BF16 &&
                    s->weight_dtype == MOE_BF16 && s->h_dtype == MOE_BF16 &&
                    s->y_dtype == MOE_BF16 && s->out_dtype == MOE_BF16;
  const bool fp8 = s->act_dtype == MOE_BF16 && s->xq_dtype == MOE_E4M3 &&
                   s->weight_dtype == MOE_E4M3 && s->h_dtype == MOE_E4M3 &&
                   s->y_dtype == MOE_BF16 && s->out_dtype == MOE_BF16;
  // MX FP4 weights with e4m3 tokens (block-scaled MMA of mixed operand types)
  const bool fp4w = s->act_dtype == MOE_BF16 && s->xq_dtype == MOE_E4M3 &&
                    s->weight_dtype == MOE_E2M1 && s->h_dtype == MOE_E4M3 &&
                    s->y_dtype == MOE_BF16 && s->out_dtype == MOE_BF16;
  if (!f32 && !bf16 && !fp8 && !fp4w) return MOE_ERR_UNSUPPORTED;
  // the expert FFN kernels work on 128-feature slices
  if (s->H % kQBlock != 0 || s->I % kQBlock != 0) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

namespace {

moe_status make_ctx(const moe_shape* s, void* ws, moe_stream_t stream, Ctx* c) {
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  if (!ws || ((uintptr_t)ws & 255u) != 0) return MOE_ERR_INVALID_ARG;
  c->s = effective_shape(*s);
  c->routed_E = s->E;
  c->routed_k = s->topk;
  c->shared = (s->flags & MOE_FLAG_SHARED_EXPERT) ? 1 : 0;
  c->L = make_layout(c->s);
  c->ws = ws_view(ws, c->L);
  c->stream = (cudaStream_t)stream;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// The intermediates moe_layer keeps in its workspace, after the stage
// workspace (Layout::total): topk_idx, topk_w, the dispatch buffers and y,
// each 256-byte aligned. rows = E * cap (or the compact bound) of the
// effective shape.
struct LayerState {
  size_t off_idx, off_w, off_xq, off_xs, off_counts, off_offsets, off_row_src, off_pos, off_hq, off_hs, off_y;
  size_t total;
};

size_t dtype_bytes(int32_t d) { return d == MOE_F32 ? 4 : (d == MOE_BF16 ? 2 : 1); }

LayerState layer_state(const moe_shape& s, const Layout& L) {
  LayerState st{};
  const size_t rows = (size_t)L.tiles * kTileRows;
  const size_t pairs = (size_t)s.T * (size_t)s.topk;
  size_t off = L.total;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  st.off_idx = take(pairs * 4);
  st.off_w = take(pairs * 4);
  st.off_xq = take(rows * (size_t)s.H * dtype_bytes(s.xq_dtype));
  st.off_xs = take(s.xq_dtype == MOE_E4M3 ? rows * (size_t)(s.H / kQBlock) * 4 : 0);
  st.off_counts = take((size_t)s.E * 4);
  st.off_offsets = take((size_t)s.E * 4);
  st.off_row_src = take(rows * 4);
  st.off_pos = take(pairs * 4);
  const bool ffn = !s.identity_experts;
  st.off_hq = take(ffn ? rows * (size_t)s.I * dtype_bytes(s.h_dtype) : 0);
  st.off_hs = take(ffn && s.h_dtype == MOE_E4M3 ? rows * (size_t)(s.I / kQBlock) * 4 : 0);
  st.off_y = take(ffn ? rows * (size_t)s.H * dtype_bytes(s.y_dtype) : 0);
  st.total = off;
  return st;
}

}  // namespace

moe_status check_bufs(const moe_shape* s, const moe_dispatch_bufs* b, bool need_h) {
  if (!b) return MOE_ERR_INVALID_ARG;
  if (!b->xq || !b->counts || !b->offsets || !b->row_src) return MOE_ERR_INVALID_ARG;
  if (!b->pos && s->T > 0) return MOE_ERR_INVALID_ARG;   // [T*topk]: may be NULL when T == 0
  if (!aligned16(b->xq)) return MOE_ERR_INVALID_ARG;
  if (s->xq_dtype == MOE_E4M3 && (!b->xs || !aligned16(b->xs))) return MOE_ERR_INVALID_ARG;
  if (need_h && !s->identity_experts) {
    if (!b->hq || !aligned16(b->hq)) return MOE_ERR_INVALID_ARG;
    if (s->h_dtype == MOE_E4M3 && (!b->hs || !aligned16(b->hs))) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

namespace {

moe_status check_weights(const moe_shape* s, const moe_weights* w) {
  if (!w || !w->w_gate || !w->w_up || !w->w_down) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->w_gate) || !aligned16(w->w_up) || !aligned16(w->w_down)) return MOE_ERR_INVALID_ARG;
  if (s->weight_dtype == MOE_E4M3 && (!w->s_gate || !w->s_up || !w->s_down)) return MOE_ERR_INVALID_ARG;
  if (s->weight_dtype == MOE_E2M1) {
    // packed 4-bit rows are copied by the tensor-memory-access unit, which
    // wants 32-byte aligned bases for them; scale atoms move in 16-byte units
    auto a32 = [](const void* p) { return ((uintptr_t)p & 31u) == 0; };
    if (!w->s_gate || !w->s_up || !w->s_down) return MOE_ERR_INVALID_ARG;
    if (!a32(w->w_gate) || !a32(w->w_up) || !a32(w->w_down)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w->s_gate) || !aligned16(w->s_up) || !aligned16(w->s_down)) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

__global__ void init_ws_kernel(uint32_t* words, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    words[i] = 0u;
  if (blockIdx.x == 0 && threadIdx.x == 0) words[0] = 1u;   // Header::epoch_next
}

// Token-sized arrays may be NULL when there are no tokens.
bool tok_ok(const Ctx& c, const void* p) { return c.s.T == 0 || p != nullptr; }

moe_status do_route(const Ctx& c, const float* logits, int32_t* idx, float* w) {
  if (!tok_ok(c, logits) || !tok_ok(c, idx) || !tok_ok(c, w) || !aligned16(logits)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_route(c, logits, idx, w));
}

moe_status do_dispatch(const Ctx& c, const void* x, const int32_t* idx, const moe_dispatch_bufs* b) {
  if (!tok_ok(c, x) || !tok_ok(c, idx) || !aligned16(x)) return MOE_ERR_INVALID_ARG;
  moe_status st = check_bufs(&c.s, b, false);
  if (st != MOE_OK) return st;
  return cuda_status(launch_dispatch(c, x, idx, *b));
}

moe_status do_ffn(const Ctx& c, const moe_dispatch_bufs* b, const moe_weights* w, void* y) {
  if (c.s.identity_experts) return MOE_OK;
  moe_status st = check_bufs(&c.s, b, true);
  if (st != MOE_OK) return st;
  st = check_weights(&c.s, w);
  if (st != MOE_OK) return st;
  if (!y || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if (ffn_tc_supported(c.s)) return cuda_status(launch_ffn_tc(c, *b, *w, y));
  return cuda_status(launch_ffn_simt(c, *b, *w, y));
}

moe_status do_combine(const Ctx& c, const moe_dispatch_bufs* b, const void* y, const float* topk_w,
                      void* out) {
  if (!b || !tok_ok(c, b->pos) || !tok_ok(c, topk_w) || !tok_ok(c, out) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if (c.s.identity_experts) {
    if (!b->xq || !aligned16(b->xq)) return MOE_ERR_INVALID_ARG;
    if (c.s.xq_dtype == MOE_E4M3 && !b->xs) return MOE_ERR_INVALID_ARG;
  } else if (!y || !aligned16(y)) {
    return MOE_ERR_INVALID_ARG;
  }
  return cuda_status(launch_combine(c, *b, y, topk_w, out));
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_workspace_bytes(const moe_shape* shape, size_t* bytes) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = make_layout(effective_shape(*shape)).total;
  return MOE_OK;
}

moe_status moe_workspace_init(const moe_shape* shape, void* ws, size_t bytes, moe_stream_t stream) {
  Ctx c;
  moe_status st = make_ctx(shape, ws, stream, &c);
  if (st != MOE_OK) return st;
  if (bytes < c.L.total) return MOE_ERR_INVALID_ARG;
  // header, both counter sets, sentinels and ring (everything before the scale atoms)
  const size_t words = c.L.off_xsf / 4;
  const int grid = (int)std::min<size_t>((words + 255) / 256, (size_t)c.num_sms * 8);
  init_ws_kernel<<<grid > 0 ? grid : 1, 256, 0, c.stream>>>((uint32_t*)ws, words);
  return cuda_status(cudaGetLastError());
}

moe_status moe_route(const moe_shape* shape, const float* logits, int32_t* topk_idx, float* topk_w,
                     void* ws, moe_stream_t stream) {
  Ctx c;
  moe_status st = make_ctx(shape, ws, stream, &c);
  return st != MOE_OK ? st : do_route(c, logits, topk_idx, topk_w);
}

moe_status moe_dispatch(const moe_shape* shape, const void* x, const int32_t* topk_idx, void* ws,
                        const moe_dispatch_bufs* bufs, moe_stream_t stream) {
  Ctx c;
  moe_status st = make_ctx(shape, ws, stream, &c);
  return st != MOE_OK ? st : do_dispatch(c, x, topk_idx, bufs);
}

moe_status moe_grouped_ffn(const moe_shape* shape, const moe_dispatch_bufs* bufs, const moe_weights* w,
                           void* ws, void* y, moe_stream_t stream) {
  Ctx c;
  moe_status st = make_ctx(shape, ws, stream, &c);
  return st != MOE_OK ? st : do_ffn(c, bufs, w, y);
}

moe_status moe_combine(const moe_shape* shape, const moe_dispatch_bufs* bufs, const void* y,
                       const float* topk_w, void* ws, void* out, moe_stream_t stream) {
  Ctx c;
  moe_status st = make_ctx(shape, ws, stream, &c);
  return st != MOE_OK ? st : do_combine(c, bufs, y, topk_w, out);
}

moe_status moe_layer_workspace_bytes(const moe_shape* shape, size_t* bytes) {
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  const moe_shape e = effective_shape(*shape);
  *bytes = layer_state(e, make_layout(e)).total;
  return MOE_OK;
}

namespace moe {
namespace {

// The layer's intermediates inside a workspace of moe_layer_workspace_bytes.
struct LayerPtrs {
  moe_dispatch_bufs bufs;
  int32_t* idx;
  float* w;
  void* y;
};

LayerPtrs layer_ptrs(const Ctx& c, void* ws) {
  const LayerState ls = layer_state(c.s, c.L);
  char* b = (char*)ws;
  LayerPtrs lp;
  lp.bufs.xq = b + ls.off_xq;
  lp.bufs.xs = c.s.xq_dtype == MOE_E4M3 ? (float*)(b + ls.off_xs) : nullptr;
  lp.bufs.counts = (int32_t*)(b + ls.off_counts);
  lp.bufs.offsets = (int32_t*)(b + ls.off_offsets);
  lp.bufs.row_src = (int32_t*)(b + ls.off_row_src);
  lp.bufs.pos = (int32_t*)(b + ls.off_pos);
  lp.bufs.hq = c.s.identity_experts ? nullptr : (void*)(b + ls.off_hq);
  lp.bufs.hs = (!c.s.identity_experts && c.s.h_dtype == MOE_E4M3) ? (float*)(b + ls.off_hs) : nullptr;
  lp.idx = (int32_t*)(b + ls.off_idx);
  lp.w = (float*)(b + ls.off_w);
  lp.y = c.s.identity_experts ? nullptr : (void*)(b + ls.off_y);
  return lp;
}

}  // namespace
}  // namespace moe

moe_status moe_layer(const moe_shape* shape, const void* x, const float* logits, const moe_weights* w,
                     void* ws, void* out, moe_stream_t stream) {
  Ctx c;
  moe_status st = make_ctx(shape, ws, stream, &c);
  if (st != MOE_OK) return st;
  LayerPtrs lp = layer_ptrs(c, ws);
  return moe_layer_bufs(shape, x, logits, w, lp.idx, lp.w, &lp.bufs, lp.y, ws, out, stream);
}

moe_status moe_layer_overlap(const moe_shape* shape, const void* x, const float* logits, const moe_weights* w,
                             void* ws, void* out, moe_stream_t stream, const moe_overlap* ov) {
  // the shape and the partition arguments are checked before any CUDA call
  moe_status st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!ov || !ov->dispatch_stream || !ov->fork_event || !ov->join_event || ov->dispatch_stream == stream ||
      ov->dispatch_sms < 1 || ov->ffn_sms < 0)
    return MOE_ERR_INVALID_ARG;
  Ctx c;
  if ((st = make_ctx(shape, ws, stream, &c)) != MOE_OK) return st;
  const int dsms = ov->dispatch_sms;
  const int fsms = ov->ffn_sms ? ov->ffn_sms : c.num_sms - dsms;
  if (dsms < 1 || dsms >= c.num_sms || fsms < 1 || fsms > c.num_sms - dsms) return MOE_ERR_INVALID_ARG;
  if (!ffn_tc_supported(c.s)) return MOE_ERR_UNSUPPORTED;
  LayerPtrs lp = layer_ptrs(c, ws);
  // every argument is checked before the first launch
  if (!tok_ok(c, logits) || !aligned16(logits) || !tok_ok(c, x) || !aligned16(x) || !tok_ok(c, out) ||
      !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_weights(&c.s, w)) != MOE_OK) return st;
  cudaEvent_t fork = (cudaEvent_t)ov->fork_event, join = (cudaEvent_t)ov->join_event;
  if ((st = do_route(c, logits, lp.idx, lp.w)) != MOE_OK) return st;
  if ((st = cuda_status(launch_plan(c, lp.idx))) != MOE_OK) return st;
  if (cudaEventRecord(fork, c.stream) != cudaSuccess ||
      cudaStreamWaitEvent((cudaStream_t)ov->dispatch_stream, fork, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  // the FFN first, so that its persistent CTAs hold their SMs and dispatch
  // takes the rest
  Ctx cf = c;
  cf.num_sms = fsms;
  cf.streaming = true;
  if ((st = cuda_status(launch_ffn_tc(cf, lp.bufs, *w, lp.y))) != MOE_OK) return st;
  Ctx cd = c;
  cd.num_sms = dsms;
  cd.stream = (cudaStream_t)ov->dispatch_stream;
  if ((st = cuda_status(launch_dispatch(cd, x, lp.idx, lp.bufs, true, true))) != MOE_OK) return st;
  if (cudaEventRecord(join, cd.stream) != cudaSuccess || cudaStreamWaitEvent(c.stream, join, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  return do_combine(c, &lp.bufs, lp.y, lp.w, out);
}

moe_status moe_layer_bufs(const moe_shape* shape, const void* x, const float* logits, const moe_weights* w,
                          int32_t* topk_idx, float* topk_w, const moe_dispatch_bufs* bufs, void* y,
                          void* ws, void* out, moe_stream_t stream) {
  Ctx c;
  moe_status st = make_ctx(shape, ws, stream, &c);
  if (st != MOE_OK) return st;
  // every argument is checked before the first launch
  if (!tok_ok(c, logits) || !tok_ok(c, topk_idx) || !tok_ok(c, topk_w) || !aligned16(logits) ||
      !tok_ok(c, x) || !aligned16(x) || !tok_ok(c, out) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  st = check_bufs(&c.s, bufs, true);
  if (st != MOE_OK) return st;
  if (!shape->identity_experts) {
    st = check_weights(&c.s, w);
    if (st != MOE_OK) return st;
    if (!y || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  }
  if ((st = do_route(c, logits, topk_idx, topk_w)) != MOE_OK) return st;
  if ((st = do_dispatch(c, x, topk_idx, bufs)) != MOE_OK) return st;
  if ((st = do_ffn(c, bufs, w, y)) != MOE_OK) return st;
  return do_combine(c, bufs, y, topk_w, out);
}

// ---- expert parallelism ------------------------------------------------------

namespace moe {
namespace {

// The global layer shape and the rank's place in it.
moe_status check_ep(const moe_shape* s, const moe_ep* ep) {
  moe_status st = check_shape(s);
  if (st != MOE_OK) return st;
  if (!ep || ep->ranks < 1 || ep->ranks > 64 || ep->rank < 0 || ep->rank >= ep->ranks || ep->reserved != 0 ||
      (ep->protocol != MOE_EP_SENTINEL && ep->protocol != MOE_EP_FENCE) || ep->t_max < s->T || ep->t_max < 0)
    return MOE_ERR_INVALID_ARG;
  if (s->E % ep->ranks != 0 || s->cap_rows != 0 || (s->flags & MOE_FLAG_COMPACT)) return MOE_ERR_INVALID_ARG;
  if (s->flags & MOE_FLAG_SHARED_EXPERT) return MOE_ERR_UNSUPPORTED;
  const EpGeom g = make_ep_geom(*s, *ep);
  if ((st = check_shape(&g.rs)) != MOE_OK) return st;   // the receivers' windows
  if ((int64_t)ep->ranks * g.rows >= (int64_t)INT32_MAX) return MOE_ERR_INVALID_ARG;   // pos is int32
  return MOE_OK;
}

moe_status ep_ctx(const moe_shape* s, const moe_ep* ep, const moe_ep_windows* all, moe_stream_t stream, Ctx* c,
                  EpGeom* g) {
  moe_status st = check_ep(s, ep);
  if (st != MOE_OK) return st;
  if (!all || !all->ws || ((uintptr_t)all->ws & 255u) != 0) return MOE_ERR_INVALID_ARG;
  *g = make_ep_geom(*s, *ep);
  if ((st = make_ctx(s, (char*)all->ws + (size_t)ep->rank * g->ws_bytes, stream, c)) != MOE_OK) return st;
  return MOE_OK;
}

size_t el_bytes(int32_t d) { return d == MOE_F32 ? 4 : (d == MOE_BF16 ? 2 : 1); }

}  // namespace
}  // namespace moe

moe_status moe_ep_sizes(const moe_shape* shape, const moe_ep* ep, int64_t* rows, size_t* ws_bytes) {
  moe_status st = check_ep(shape, ep);
  if (st != MOE_OK) return st;
  if (!rows || !ws_bytes) return MOE_ERR_INVALID_ARG;
  const EpGeom g = make_ep_geom(*shape, *ep);
  *rows = g.rows;
  *ws_bytes = g.ws_bytes;
  return MOE_OK;
}

moe_status moe_ep_workspace_init(const moe_shape* shape, const moe_ep* ep, const moe_ep_windows* all,
                                 moe_stream_t stream) {
  Ctx c;
  EpGeom g;
  moe_status st = ep_ctx(shape, ep, all, stream, &c, &g);
  if (st != MOE_OK) return st;
  const size_t words = g.ws_bytes / 4;
  const int grid = (int)std::min<size_t>((words + 255) / 256, (size_t)c.num_sms * 8);
  init_ws_kernel<<<grid > 0 ? grid : 1, 256, 0, c.stream>>>((uint32_t*)c.ws.hdr, words);
  return cuda_status(cudaGetLastError());
}

moe_status moe_ep_count(const moe_shape* shape, const moe_ep* ep, const int32_t* topk_idx,
                        const moe_ep_windows* all, moe_stream_t stream) {
  Ctx c;
  EpGeom g;
  moe_status st = ep_ctx(shape, ep, all, stream, &c, &g);
  if (st != MOE_OK) return st;
  if (ep->protocol != MOE_EP_FENCE || !tok_ok(c, topk_idx)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_ep_count(c, g, topk_idx, *all));
}

moe_status moe_ep_layout(const moe_shape* shape, const moe_ep* ep, const moe_ep_windows* all, moe_stream_t stream) {
  Ctx c;
  EpGeom g;
  moe_status st = ep_ctx(shape, ep, all, stream, &c, &g);
  if (st != MOE_OK) return st;
  if (ep->protocol != MOE_EP_FENCE) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_ep_layout(c, g, *all));
}

moe_status moe_ep_dispatch(const moe_shape* shape, const moe_ep* ep, const void* x, const int32_t* topk_idx,
                           const moe_ep_windows* all, int32_t* pos, moe_stream_t stream) {
  Ctx c;
  EpGeom g;
  moe_status st = ep_ctx(shape, ep, all, stream, &c, &g);
  if (st != MOE_OK) return st;
  if (!tok_ok(c, x) || !aligned16(x) || !tok_ok(c, topk_idx) || !tok_ok(c, pos)) return MOE_ERR_INVALID_ARG;
  if (!all->xq || !aligned16(all->xq) || !all->row_src || (c.s.xq_dtype == MOE_E4M3 && !all->xs))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_ep_dispatch(c, g, x, topk_idx, *all, pos));
}

moe_status moe_ep_grouped_ffn(const moe_shape* shape, const moe_ep* ep, const moe_weights* w,
                              const moe_ep_windows* all, moe_stream_t stream) {
  Ctx c;
  EpGeom g;
  moe_status st = ep_ctx(shape, ep, all, stream, &c, &g);
  if (st != MOE_OK) return st;
  if (shape->identity_experts) return MOE_OK;
  if (!ffn_tc_supported(g.rs)) return MOE_ERR_UNSUPPORTED;   // the tensor-core FFN's formats
  if ((st = check_weights(&g.rs, w)) != MOE_OK) return st;
  if (!all->xq || !all->hq || !all->y || (g.rs.xq_dtype == MOE_E4M3 && !all->xs) ||
      (g.rs.h_dtype == MOE_E4M3 && !all->hs))
    return MOE_ERR_INVALID_ARG;
  // this rank's part of the rank-major windows, as a receiver of V windows
  const int64_t r0 = (int64_t)ep->rank * g.rows;
  moe_dispatch_bufs b;
  memset(&b, 0, sizeof(b));
  b.xq = (char*)all->xq + r0 * g.rs.H * (int64_t)el_bytes(g.rs.xq_dtype);
  b.xs = all->xs ? all->xs + r0 * (g.rs.H / kQBlock) : nullptr;
  b.hq = (char*)all->hq + r0 * g.rs.I * (int64_t)el_bytes(g.rs.h_dtype);
  b.hs = all->hs ? all->hs + r0 * (g.rs.I / kQBlock) : nullptr;
  b.row_src = all->row_src ? all->row_src + r0 : nullptr;
  void* y = (char*)all->y + r0 * g.rs.H * (int64_t)el_bytes(g.rs.y_dtype);
  if (!aligned16(b.xq) || !aligned16(b.hq) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  Ctx cf = c;
  cf.s = g.rs;
  cf.L = g.RL;
  cf.ws = ws_view(c.ws.hdr, g.RL);
  cf.ep_ranks = g.R;
  if ((st = cuda_status(launch_ffn_tc(cf, b, *w, y))) != MOE_OK) return st;
  return cuda_status(launch_ep_publish_y(cf));
}

moe_status moe_ep_combine(const moe_shape* shape, const moe_ep* ep, const int32_t* pos, const float* topk_w,
                          const moe_ep_windows* all, void* out, moe_stream_t stream) {
  Ctx c;
  EpGeom g;
  moe_status st = ep_ctx(shape, ep, all, stream, &c, &g);
  if (st != MOE_OK) return st;
  if (!tok_ok(c, pos) || !tok_ok(c, topk_w) || !tok_ok(c, out) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  moe_dispatch_bufs b;
  memset(&b, 0, sizeof(b));
  b.pos = const_cast<int32_t*>(pos);
  if (shape->identity_experts) {   // the pushed tokens are complete once this rank's dispatch is
    if (!all->xq || !aligned16(all->xq) || (c.s.xq_dtype == MOE_E4M3 && !all->xs)) return MOE_ERR_INVALID_ARG;
    b.xq = all->xq;
    b.xs = all->xs;
    return cuda_status(launch_combine(c, b, nullptr, topk_w, out));
  }
  if (!all->y || !aligned16(all->y)) return MOE_ERR_INVALID_ARG;
  if ((st = cuda_status(launch_ep_wait_y(c, g, *all))) != MOE_OK) return st;
  return cuda_status(launch_combine(c, b, all->y, topk_w, out));
}

moe_status moe_poll_status(void* ws, moe_stream_t stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t err = 0;
  Header* h = (Header*)ws;
  if (cudaMemcpy(&err, &h->error, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (err != 0 && cudaMemset(&h->error, 0, 8) != cudaSuccess) return MOE_ERR_CUDA;
  return (moe_status)err;
}

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype combination";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_CAPACITY: return "an expert received more rows than cap_rows";
    case MOE_ERR_TIMEOUT: return "a device wait ran out of time";
    case MOE_ERR_NONFINITE: return "non-finite router logits";
  }
  return "unknown status";
}

}  // extern "C"

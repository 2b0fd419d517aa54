/*
 * moe.h - C ABI of the B200 (sm_100a) Mixture-of-Experts layer library.
 *
 * One MoE layer on one GPU, as four stages:
 *
 *   moe_route        router logits -> top-k experts and weights per token
 *   moe_dispatch     one pass: each (token, slot) pair claims a row of its
 *                    expert's window by atomic counter, quantises/copies the
 *                    token there and publishes per-tile sentinels
 *   moe_grouped_ffn  every expert's SwiGLU FFN over its rows, read in place
 *   moe_combine      top-k weighted gather-reduce back to token order
 *
 * and moe_layer, which enqueues all four; moe_layer_overlap, the same layer with
 * dispatch running beside the grouped FFN on a partition of the SMs; and the
 * expert-parallel calls moe_ep_* (experts split over ranks, tokens pushed into
 * the owners' rank-major windows). The stage split follows the pages:
 * an MoE layer is token dispatch, grouped GEMMs and a combine (GC-MoE feed
 * item, "Key points"; GC-MoE explainer, "Why Expert Parallelism Is
 * Inefficient in MoE Decoding"); dispatch pushes tokens into per-expert
 * windows without first exchanging counts, and the grouped GEMMs read them in
 * place rather than from a per-expert copy (NVLinkOneSided abstract); only
 * counts, offsets and synchronisation metadata are kept as control state
 * (Ascend relay-buffer-free report, abstract).
 *
 * Conventions for every entry point
 *  - Pointers marked "device" must be device memory of the current CUDA
 *    device; pointers marked "host" must be host memory. The caller owns all
 *    memory. The library allocates nothing and keeps no per-call global state:
 *    everything a call needs between kernels lives in the caller's workspace.
 *  - All work is enqueued asynchronously on `stream` (0 = legacy default
 *    stream). Calls on different workspaces may run concurrently.
 *  - Argument checks run on the host before anything is enqueued; on failure
 *    the call returns MOE_ERR_INVALID_ARG or MOE_ERR_UNSUPPORTED and enqueues
 *    nothing. A failing CUDA launch returns MOE_ERR_CUDA.
 *  - Errors found on the device (capacity overflow, non-finite logits, a wait
 *    that ran out of time) are latched into the workspace, first error wins,
 *    and read back by moe_poll_status. The library never traps, aborts or
 *    prints.
 *  - All device buffers must be 16-byte aligned; rows are dense (no padding).
 *    Arrays sized by T (x, logits, topk_idx, topk_w, pos, out) may be NULL
 *    when T == 0.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* moe_stream_t;

typedef enum moe_dtype {
  MOE_F32 = 0,   /* IEEE binary32 */
  MOE_BF16 = 1,  /* bfloat16 */
  MOE_E4M3 = 2,  /* OCP FP8 E4M3 with power-of-two fp32 block scales */
  MOE_E2M1 = 3   /* OCP MX FP4 E2M1, two per byte, UE8M0 scale per 32 (weights only) */
} moe_dtype;

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or workspace */
  MOE_ERR_UNSUPPORTED = 2,  /* valid but not implemented dtype combination */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  MOE_ERR_CAPACITY = 4,     /* an expert received more pairs than cap_rows */
  MOE_ERR_TIMEOUT = 5,      /* a bounded device wait gave up */
  MOE_ERR_NONFINITE = 6     /* router logits held NaN or Inf */
} moe_status;

/*
 * Problem description.
 *
 * T tokens of hidden size H, E experts of intermediate size I, top-k routing.
 * Supported dtype combinations (act, xq, weight, h, y, out):
 *   fp32 layer      F32,  F32,  F32,  F32,  F32,  F32
 *   bf16 layer      BF16, BF16, BF16, BF16, BF16, BF16
 *   fp8 layer       BF16, E4M3, E4M3, E4M3, BF16, BF16
 *   fp4-weight layer BF16, E4M3, E2M1, E4M3, BF16, BF16 (MX FP4 weights: the
 *                   GC-MoE explainer's "Two MMA Implementations" names 4-bit
 *                   weights whose 32-element blocks share one exponent)
 *   identity experts (identity_experts = 1): act BF16/F32, xq any, out BF16/F32;
 *                   weight/h/y ignored, moe_grouped_ffn is a no-op.
 * H must be a multiple of 16 (of quant_block = 128 when xq is E4M3); with
 * experts (identity_experts = 0) H and I must be multiples of 128. E <= 1024.
 * cap_rows, when given, must be a multiple of 128.
 * Routing weights are the softmax over all E logits of the selected experts,
 * renormalised over the k selected ones when renorm = 1.
 *
 * flags = MOE_FLAG_SHARED_EXPERT adds one shared expert that every token also
 * goes through, computed in the same grouped FFN launch and added to the
 * output with weight 1 (GC-MoE feed item: shared experts, when a model has
 * them, are fused into the compute partition; the weight-1 sum is this
 * library's reading).
 * E and topk stay the routed counts (logits are [T, E]); every per-expert and
 * per-pair array grows by one: the weight arrays hold E + 1 experts (the
 * shared one last, index E), topk_idx / topk_w have topk + 1 columns (moe_route
 * writes E and 1.0 into the last), the windows hold E + 1 experts
 * (counts / offsets [E + 1], rows (E + 1) * cap) and pos has T * (topk + 1)
 * entries. cap must cover all T tokens; topk + 1 <= 32; not with identity
 * experts.
 */
enum { MOE_FLAG_SHARED_EXPERT = 1 };

/*
 * flags |= MOE_FLAG_COMPACT packs the expert windows instead of giving every
 * expert cap rows: moe_dispatch first counts each expert's pairs (a fence:
 * the counts are complete before any row is placed, the NVLinkOneSided
 * abstract's Fence protocol), then expert e's window starts at offsets[e], the
 * 128-row-aligned running sum of the windows before it, and holds exactly
 * counts[e] rows (no capacity limit, no overflow). rows = 128 *
 * (ceil(T * slots / 128) + experts), slots = topk (+ 1 with a shared
 * expert), experts = E (+ 1); rows / 128 <= 65535. cap_rows must be 0.
 * moe_dispatch_noalloc returns MOE_ERR_UNSUPPORTED for it.
 */
enum { MOE_FLAG_COMPACT = 2 };

typedef struct moe_shape {
  int64_t T;              /* tokens, >= 0 */
  int64_t H;              /* hidden size */
  int64_t E;              /* experts, 1..65535 */
  int64_t topk;           /* experts per token, 1..min(E, 32) */
  int64_t I;              /* expert intermediate size */
  int32_t act_dtype;      /* dtype of x */
  int32_t xq_dtype;       /* dtype tokens are stored in inside expert windows */
  int32_t weight_dtype;   /* dtype of W_gate/W_up/W_down */
  int32_t h_dtype;        /* dtype of the SwiGLU output h */
  int32_t y_dtype;        /* dtype of expert outputs y */
  int32_t out_dtype;      /* dtype of the layer output */
  int32_t renorm;         /* 1: renormalise the k weights to sum to 1 */
  int32_t identity_experts; /* 1: every expert returns its input (no FFN) */
  int64_t cap_rows;       /* rows per expert window; 0 = round_up(T, 128) */
  int32_t quant_block;    /* must be 128 */
  int32_t flags;          /* 0 or MOE_FLAG_SHARED_EXPERT | MOE_FLAG_COMPACT */
} moe_shape;

/*
 * Expert-major buffers written by moe_dispatch and moe_grouped_ffn (all device,
 * caller-owned). cap = cap_rows (or its default); rows = E * cap. Expert e owns
 * rows [offsets[e], offsets[e] + counts[e]) (offsets[e] = e * cap, or packed
 * with MOE_FLAG_COMPACT, which also sets rows).
 *   xq      [rows, H]        tokens in xq_dtype
 *   xs      [rows, H/128]    fp32 power-of-two scales (E4M3 xq only, else NULL)
 *   counts  [E]   int32      rows filled per expert (bit-exact routing counts)
 *   offsets [E]   int32      first row of each expert window (e * cap, or packed)
 *   row_src [rows] int32     row -> pair id t*topk + j (rows past counts[e]
 *                            are left as they were)
 *   pos     [T*topk] int32   pair id -> row, or -1 if it was not placed
 *   hq      [rows, I]        SwiGLU output in h_dtype (NULL for identity experts)
 *   hs      [rows, I/128]    fp32 scales (E4M3 h only, else NULL)
 * The order of rows inside an expert window is not deterministic; the set of
 * pairs per expert is.
 */
typedef struct moe_dispatch_bufs {
  void* xq;
  float* xs;
  int32_t* counts;
  int32_t* offsets;
  int32_t* row_src;
  int32_t* pos;
  void* hq;
  float* hs;
} moe_dispatch_bufs;

/*
 * Expert weights (device, read only), row-major and K-major:
 *   w_gate, w_up [E, I, H]; w_down [E, H, I], in weight_dtype.
 *   E4M3 weights carry one fp32 scale per 128 x 128 block:
 *   s_gate, s_up [E, I/128, H/128]; s_down [E, H/128, I/128]. Scales must be
 *   positive, finite, normal powers of two (the tensor cores apply them as
 *   8-bit exponents): moe_grouped_ffn checks every scale it uses and latches
 *   MOE_ERR_INVALID_ARG for any other value (the outputs are then
 *   unspecified), rather than dropping its mantissa.
 *   E2M1 weights hold two 4-bit codes per byte, element 2i of a row in the
 *   low nibble of its byte i (w_gate, w_up [E, I, H/2] bytes; w_down
 *   [E, H, I/2]; each matrix 32-byte aligned), and one UE8M0 scale byte
 *   (value 2^(byte - 127), byte < 255) per 32 consecutive elements of a row,
 *   stored in the tensor cores' scale-atom order: s_gate, s_up
 *   [E, I/128, H/128, 512] bytes, s_down [E, H/128, I/128, 512]; inside the
 *   atom of a 128 x 128 block, row r's scale of elements 32 b .. 32 b + 31 of
 *   the block (b = 0..3) is byte (r % 32) * 16 + (r / 32) * 4 + b.
 *   NULL for unscaled weight dtypes.
 */
typedef struct moe_weights {
  const void* w_gate;
  const void* w_up;
  const void* w_down;
  const void* s_gate;
  const void* s_up;
  const void* s_down;
} moe_weights;

/* Workspace size in bytes for `shape` (host only, enqueues nothing). */
MOE_API moe_status moe_workspace_bytes(const moe_shape* shape, size_t* bytes);

/*
 * Prepare a workspace of at least moe_workspace_bytes bytes (device): zeroes
 * the counters, the sentinels and the error word, and starts the epoch at 1.
 * Must be called once before the first use of a workspace, and again before
 * reusing it for a different shape.
 */
MOE_API moe_status moe_workspace_init(const moe_shape* shape, void* ws, size_t bytes,
                              moe_stream_t stream);

/*
 * Routing (softmax then top-k). Reading of the pages: tokens are sent to
 * experts according to the gating result (GC-MoE explainer, "Why Expert
 * Parallelism Is Inefficient in MoE Decoding"); the rule itself is softmax
 * over the E router logits, top-k on the logits (the lower expert index wins
 * a tie), slots ordered by descending logit.
 *   logits   [T, E] fp32, device
 *   topk_idx [T, topk] int32, device (out)
 *   topk_w   [T, topk] fp32, device (out)
 *   ws       workspace (error word)
 * A non-finite logit latches MOE_ERR_NONFINITE; that token's outputs are
 * unspecified.
 */
MOE_API moe_status moe_route(const moe_shape* shape, const float* logits, int32_t* topk_idx,
                     float* topk_w, void* ws, moe_stream_t stream);

/*
 * One-pass dispatch (NVLinkOneSided abstract: tokens are pushed into the
 * destination windows with no metadata exchanged first; GC-MoE explainer,
 * "Three-Node CUDA Graph and token-ring Handshake": the producer publishes
 * filled ring blocks the consumer polls).
 *   x        [T, H] act_dtype, device
 *   topk_idx [T, topk] int32, device (experts must be in [0, E) and distinct
 *            per token)
 *   bufs     xq, xs, counts, offsets, row_src, pos are written
 * Each pair claims row offsets[e] + atomicAdd(count[e], 1); E4M3 rows are
 * quantised per 128 values with the smallest power-of-two scale that keeps
 * the block within +-448. A pair that finds its expert full is not placed,
 * pos = -1, and MOE_ERR_CAPACITY is latched. Every completed 128-row tile
 * (and, when the last token is done, every partial tile) gets a sentinel.
 */
MOE_API moe_status moe_dispatch(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                        void* ws, const moe_dispatch_bufs* bufs, moe_stream_t stream);

/*
 * Grouped expert FFN over the dispatched rows, read in place (NVLinkOneSided
 * abstract; GC-MoE feed item, "Full text": block-scaled tcgen05 MMA with fused
 * SwiGLU and requantisation). For every expert e and every filled row r:
 *   h = silu(xq_r W_gate[e]^T) * (xq_r W_up[e]^T), stored as h_dtype in bufs->hq
 *       (E4M3: requantised per 128 values like dispatch, scales in bufs->hs)
 *   y_r = h W_down[e]^T, stored as y_dtype.
 *   bufs  dispatch outputs (read) and hq/hs (written)
 *   w     expert weights
 *   y     [rows, H] y_dtype, device (out; rows past counts[e] untouched)
 * Work starts per tile as its sentinel is found set; waits are bounded and
 * latch MOE_ERR_TIMEOUT.
 */
MOE_API moe_status moe_grouped_ffn(const moe_shape* shape, const moe_dispatch_bufs* bufs,
                           const moe_weights* w, void* ws, void* y, moe_stream_t stream);

/*
 * Weighted combine (Ascend report abstract: outputs are read straight from
 * the expert windows, no output-restoration buffer):
 *   out[t] = sum_{j < topk} topk_w[t, j] * y[pos[t*topk + j]]
 * summed in slot order in fp32 and rounded once to out_dtype. With identity
 * experts the rows are the dispatched tokens themselves (xq, dequantised with
 * xs) and y may be NULL. Pairs with pos = -1 contribute nothing.
 *   bufs   pos (and xq/xs for identity experts)
 *   y      [rows, H] y_dtype, device
 *   topk_w [T, topk] fp32, device
 *   out    [T, H] out_dtype, device
 */
MOE_API moe_status moe_combine(const moe_shape* shape, const moe_dispatch_bufs* bufs, const void* y,
                       const float* topk_w, void* ws, void* out, moe_stream_t stream);

/*
 * Size in bytes of a workspace that moe_layer can use (host only): the stage
 * workspace of moe_workspace_bytes followed by room for the layer's
 * intermediates (topk_idx, topk_w, the expert-major buffers of
 * moe_dispatch_bufs and y, at the sizes given there; with MOE_FLAG_COMPACT
 * the buffers are the compact bound, about T * topk rows, else E * cap rows).
 */
MOE_API moe_status moe_layer_workspace_bytes(const moe_shape* shape, size_t* bytes);

/*
 * The whole layer (route, one-pass dispatch, grouped expert FFN, combine),
 * enqueued in that order on `stream`; the pages' problem statement in one
 * call (GC-MoE explainer, "Why Expert Parallelism Is Inefficient in MoE
 * Decoding": an MoE layer is gating, token dispatch, the experts' GEMMs and a
 * combine back to token order).
 *   x       [T, H] act_dtype, device
 *   logits  [T, E] fp32, device
 *   w       expert weights (as for moe_grouped_ffn; ignored with identity
 *           experts)
 *   ws      device workspace of at least moe_layer_workspace_bytes bytes,
 *           256-byte aligned and prepared by moe_workspace_init; every
 *           intermediate lives in it (the size cannot be checked here: a
 *           smaller buffer is the caller's error)
 *   out     [T, H] out_dtype, device
 * Errors as for the four stages; device errors latch into ws.
 */
MOE_API moe_status moe_layer(const moe_shape* shape, const void* x, const float* logits,
                     const moe_weights* w, void* ws, void* out, moe_stream_t stream);

/*
 * moe_layer with the intermediates in the caller's own buffers
 * (topk_idx/topk_w [T, topk], bufs, y, as for the stage calls), so that they
 * can be inspected or kept; ws needs only moe_workspace_bytes bytes.
 */
MOE_API moe_status moe_layer_bufs(const moe_shape* shape, const void* x, const float* logits,
                     const moe_weights* w, int32_t* topk_idx, float* topk_w,
                     const moe_dispatch_bufs* bufs, void* y, void* ws, void* out,
                     moe_stream_t stream);

/*
 * How moe_layer_overlap splits the device between dispatch and the grouped
 * FFN (all caller-owned; the library creates no stream or event).
 *   dispatch_stream  a second stream, not the legacy default stream, that
 *                    the dispatch kernel runs on. On two streams of one
 *                    context the split is by grid size: the grouped FFN's
 *                    persistent CTAs hold ffn_sms SMs and dispatch takes the
 *                    SMs they leave. For a split the device enforces, both
 *                    `stream` and dispatch_stream must belong to green
 *                    contexts over disjoint SM sets (ffn_sms at most the
 *                    former's SMs): a green context for dispatch alone does
 *                    not confine the FFN, whose CTAs may then occupy every
 *                    SM of dispatch's partition, so that its tile waits run
 *                    out (MOE_ERR_TIMEOUT)
 *   fork_event       cudaEvent_t (cudaEventDisableTiming is enough):
 *   join_event       recorded on `stream` / dispatch_stream to order the two
 *   dispatch_sms     SMs dispatch is sized for: its grid is one wave of
 *                    resident CTAs on that many SMs, 1 .. SMs - 1
 *   ffn_sms          the grouped FFN's persistent grid (one CTA per SM);
 *                    0 = the device's SMs minus dispatch_sms
 */
typedef struct moe_overlap {
  moe_stream_t dispatch_stream;
  void* fork_event;
  void* join_event;
  int32_t dispatch_sms;
  int32_t ffn_sms;
} moe_overlap;

/*
 * moe_layer with dispatch and the grouped FFN running at the same time on
 * two parts of the device (GC-MoE explainer, "GC-MoE's Core Idea": a small
 * partition of SMs dispatches while the rest computes; "Three-Node CUDA Graph
 * and token-ring Handshake": the two kernels are concurrent, and the GEMM
 * starts on the first filled tiles). On `stream`: route, then the counting
 * pass (per-expert pair counts, and the compact window layout), then the
 * grouped FFN on ffn_sms SMs, which takes its unit table from those counts
 * and starts each tile once dispatch has published its sentinel; on
 * dispatch_stream, between the fork and join events: dispatch; on `stream`
 * after the join: combine. The result equals moe_layer's bit for bit.
 *   arguments as moe_layer (ws of moe_layer_workspace_bytes, prepared by
 *   moe_workspace_init), plus `ov`
 * MOE_ERR_UNSUPPORTED for layers the tensor-core FFN does not run (fp32
 * expert rows, identity experts); MOE_ERR_INVALID_ARG for a missing stream or
 * event or SM counts out of range. A dispatch that never publishes a tile
 * the FFN waits for ends in MOE_ERR_TIMEOUT (bounded waits), not a hang.
 */
MOE_API moe_status moe_layer_overlap(const moe_shape* shape, const void* x, const float* logits,
                     const moe_weights* w, void* ws, void* out, moe_stream_t stream,
                     const moe_overlap* ov);

/*
 * moe_dispatch without a workspace argument, for callers that may not
 * allocate device memory where they dispatch (an engine that hands all device
 * memory to its own pool at start-up and forbids cudaMalloc while serving, or
 * a latency-bound decode loop that cannot afford the device synchronisation
 * an allocation brings). The pages have no counterpart of this call.
 *
 * Arguments and outputs are those of moe_dispatch (bufs: xq, xs, counts,
 * offsets, row_src, pos). The dispatch kernel's own state (counters, tile
 * sentinels and the tile ring) lives instead in a fixed 4 MiB array of device
 * memory inside the library, which every GPU that loads the library holds
 * until the process exits; a shape whose counters, sentinels and ring need
 * more than 4 MiB is rejected with MOE_ERR_INVALID_ARG (the scale atoms that
 * moe_dispatch also writes into its workspace are not made here, so they do
 * not count). The first call on each device looks up that array's device
 * address (with the device current), so make it before any stream capture.
 * Every call clears what the kernel needs zeroed, then dispatches; calls that
 * overlap on the GPU share the array and race. Device-detected errors are not
 * reported through a workspace: a pair that could not be placed has pos = -1.
 *
 * Its outputs may be read by the host or passed to moe_combine with identity
 * experts (identity_experts = 1, which reads xq/xs through pos). They must
 * not be passed to moe_grouped_ffn or moe_layer: those read the tile
 * sentinels, ring and scale atoms from their workspace, which this call does
 * not write, and a workspace that an earlier moe_dispatch used would hand them
 * stale ones.
 */
MOE_API moe_status moe_dispatch_noalloc(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                                        const moe_dispatch_bufs* bufs, moe_stream_t stream);

/*
 * Rearrange MX FP4 weight scales from row order into the scale-atom order
 * moe_weights wants for MOE_E2M1 weights (a byte permutation on the device,
 * no arithmetic; the GC-MoE explainer's "Two MMA Implementations" gives the
 * 32-element shared exponent, the atom order is the tensor cores' own).
 *   n     matrices (experts), >= 0
 *   rows  rows of each matrix (I for gate/up, H for down), a multiple of 128
 *   cols  elements per row (H for gate/up, I for down), a multiple of 128
 *   src   [n, rows, cols / 32] UE8M0 bytes, device, read only
 *   dst   [n, rows / 128, cols / 128, 512] bytes, device, written: inside the
 *         atom of a 128 x 128 block, row r's scale of block elements
 *         32 b .. 32 b + 31 is byte (r % 32) * 16 + (r / 32) * 4 + b
 * src and dst must not overlap. Enqueued on `stream`; MOE_ERR_INVALID_ARG
 * for bad sizes or NULL pointers (n * rows * cols == 0 enqueues nothing).
 */
MOE_API moe_status moe_pack_mx_scales(int64_t n, int64_t rows, int64_t cols, const void* src, void* dst,
                                      moe_stream_t stream);

/* ---- expert parallelism ------------------------------------------------------
 *
 * R ranks (one per GPU of one NVLink domain) each own E / R experts, rank d
 * experts [d E/R, (d + 1) E/R), and each dispatches its own tokens. The pages'
 * design (NVLinkOneSided abstract): every source rank pushes its tokens,
 * without exchanging metadata first, into rank-major buffers on the target
 * ranks, where the grouped GEMM reads them in place; Fence and Sentinel are
 * the two ways to synchronise, for throughput and for latency.
 *
 * Windows. Every rank receives into the windows of V = E virtual experts,
 * v = el * R + src for local expert el and source rank src: the rows one
 * source sends one expert form that source's own region, so it fills it with
 * its own counters and nobody else's.
 *   MOE_EP_SENTINEL  regions of round_up(t_max, 128) rows; a source publishes
 *                    each filled 128-row tile with a sentinel word and, when
 *                    done, its partial tiles and its per-region counts; the
 *                    receiver's grouped FFN starts once all R sources closed
 *   MOE_EP_FENCE     sources first write their per-expert pair counts to the
 *                    owners (moe_ep_count), each owner lays its regions out
 *                    back to back in whole tiles (moe_ep_layout), and sources
 *                    then place rows at exact offsets: smaller windows
 *                    (prefill), one more round of flags
 * Tokens, h and y keep the single-GPU formats (moe_dispatch_bufs).
 *
 * Addressing. Rank d's windows and workspace are reached at d * stride inside
 * rank-major address ranges that cover all ranks (moe_ep_windows): one
 * allocation when the ranks are emulated on one device, or, across GPUs, each
 * peer's allocation mapped into consecutive parts of one reserved virtual
 * range (CUDA virtual memory management with imported peer handles). Every
 * cross-rank write is a plain store or atomic to peer memory over NVLink,
 * released at system scope; no TMA multicast and no library kernel ever
 * reads a peer's memory, and the grouped FFN reads only its own rank's part.
 *
 * Per layer, every rank enqueues, in order: moe_route (with the global
 * shape), [Fence: moe_ep_count, then moe_ep_layout], moe_ep_dispatch,
 * moe_ep_grouped_ffn, moe_ep_combine. Cross-rank waits inside those calls are
 * bounded (MOE_ERR_TIMEOUT after 200 ms). Ranks emulated on one device must
 * enqueue each step for every rank before the next step of any rank (stream
 * order then satisfies every wait before it starts).
 */
enum { MOE_EP_SENTINEL = 0, MOE_EP_FENCE = 1 };

typedef struct moe_ep {
  int32_t ranks;      /* R, 1..64, dividing E */
  int32_t rank;       /* this rank, 0..R-1 */
  int32_t protocol;   /* MOE_EP_SENTINEL or MOE_EP_FENCE */
  int32_t reserved;   /* 0 */
  int64_t t_max;      /* most tokens any rank dispatches in one call (shape->T <= t_max) */
} moe_ep;

/* Rank-major address ranges: rank d's part starts at d * rows rows (or at
 * d * ws_bytes bytes for ws), rows and ws_bytes from moe_ep_sizes. */
typedef struct moe_ep_windows {
  void* xq;          /* [R * rows, H] xq_dtype: tokens pushed by the sources */
  float* xs;         /* [R * rows, H/128] fp32 scales (e4m3 tokens, else NULL) */
  int32_t* row_src;  /* [R * rows]: src * t_max * topk + (t * topk + j) of each placed row */
  void* hq;          /* [R * rows, I] h_dtype: written by each owner in its own part */
  float* hs;         /* [R * rows, I/128] (e4m3 h, else NULL) */
  void* y;           /* [R * rows, H] y_dtype: each owner's expert outputs */
  void* ws;          /* [R * ws_bytes]: each rank's workspace (moe_ep_workspace_init) */
} moe_ep_windows;

/* Rows of one rank's windows and bytes of one rank's workspace (host only).
 * `shape` is the global layer (E = all experts, T = this rank's tokens). */
MOE_API moe_status moe_ep_sizes(const moe_shape* shape, const moe_ep* ep, int64_t* rows, size_t* ws_bytes);

/* Prepare this rank's workspace (its part of all->ws): counters zeroed, epoch 1. */
MOE_API moe_status moe_ep_workspace_init(const moe_shape* shape, const moe_ep* ep,
                                         const moe_ep_windows* all, moe_stream_t stream);

/* Fence, first step: this rank's pair counts per expert, written to the
 * owners' workspaces (topk_idx [T, topk] from moe_route). */
MOE_API moe_status moe_ep_count(const moe_shape* shape, const moe_ep* ep, const int32_t* topk_idx,
                                const moe_ep_windows* all, moe_stream_t stream);

/* Fence, second step: once all R sources' counts are here, lay this rank's
 * regions out (whole tiles, back to back) and flag the layout ready. */
MOE_API moe_status moe_ep_layout(const moe_shape* shape, const moe_ep* ep, const moe_ep_windows* all,
                                 moe_stream_t stream);

/* Push this rank's tokens into their owners' windows (one-pass: atomic claim
 * in the source's own region, e4m3 per-128 quantisation as moe_dispatch,
 * sentinel per filled tile, partial tiles and counts at close).
 *   x   [T, H] act_dtype; topk_idx [T, topk] (global experts)
 *   pos [T * topk] int32 (out): d * rows + r for a pair placed in row r of
 *       rank d's windows, -1 if not placed (MOE_ERR_CAPACITY latched) */
MOE_API moe_status moe_ep_dispatch(const moe_shape* shape, const moe_ep* ep, const void* x,
                                   const int32_t* topk_idx, const moe_ep_windows* all, int32_t* pos,
                                   moe_stream_t stream);

/* This rank's grouped FFN over the rows all sources pushed into its windows
 * (waits, bounded, until all R sources have closed), then its y flagged ready.
 *   w  this rank's E/R experts' weights, laid out as moe_weights for E/R experts */
MOE_API moe_status moe_ep_grouped_ffn(const moe_shape* shape, const moe_ep* ep, const moe_weights* w,
                                      const moe_ep_windows* all, moe_stream_t stream);

/* Weighted combine of this rank's tokens, reading every pair's expert output
 * in place in its owner's window (the Ascend report's relay-free combine):
 * out[t] = sum_j topk_w[t, j] * y_all[pos[t * topk + j]], as moe_combine
 * (identity experts read the pushed tokens). Waits, bounded, until every
 * owner has flagged its y ready. */
MOE_API moe_status moe_ep_combine(const moe_shape* shape, const moe_ep* ep, const int32_t* pos,
                                  const float* topk_w, const moe_ep_windows* all, void* out,
                                  moe_stream_t stream);

/*
 * Synchronises `stream`, returns the first device error latched in `ws`
 * since the last poll (MOE_OK if none) and clears it.
 */
MOE_API moe_status moe_poll_status(void* ws, moe_stream_t stream);

/* Static description of a status code. */
MOE_API const char* moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */

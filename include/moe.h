/*
 * moe.h -- C ABI of libmoe: one capacity-limited, pooled-wave MoE block on one B200.
 *
 * The block (the Marin 535B-A23B MoE branch, "Marin начинает открытое обучение
 * MoE-модели с 535 млрд параметров", §2, and "Marin 535B-A23B：一场完全公开的前沿 MoE
 * 训练直播", §2.2 and §3.2):
 *
 *   z      = x W_lat_down^T                         latent down-projection
 *   logits = z W_router^T (+ logit_offset)          router, float32
 *   top-k of logits + bias                          bias: zero-mean, no gradient
 *   gates  = softmax of the chosen unbiased logits
 *   slots  : sender cap C_s per (destination, wave) pool, receiver cap C_r per
 *            expert, given in (token, rank) order; overflow is dropped and counted
 *   pools  : one fixed pool per (destination, wave), expert id packed in each row
 *   Y_e    = (silu(X_e w1_e^T) * (X_e w3_e^T)) w2_e^T  per expert, kept rows only
 *   r_t    = sum_j kept gate_tj Y(t, j)              combine in latent space
 *   y      = r W_lat_up^T + sum_s SwiGLU_s(x)        up-projection + shared experts
 *
 * with C_s = ceil(cap_send * T*k / (D*W)) and C_r = ceil(cap_recv * T*k / E), the
 * factors 1.10 and 1.15 given as integer ratios.  Expert e lives on destination
 * e / L, local index e % L, wave (e % L) / P, pool (e / L) * W + (e % L) / P, with
 * L = E / D and P = L / W.  One GPU is one source; the D destinations are pools
 * in this GPU's memory.
 *
 * Conventions for every call
 *   - Pointers named "device" are CUDA device pointers; others are host pointers.
 *     bf16 tensors are passed as uint16_t bit patterns.  All tensors are dense,
 *     row-major, with the shapes given; weights are [out][in].
 *   - Precision: operands and every tensor passed between two steps are bf16, all
 *     accumulation is float32; the block's outputs (y, dx, weight gradients) are
 *     returned in float32, unrounded.
 *   - The caller owns every buffer.  The library never allocates device memory.
 *     Scratch ("ws") and the forward context kept for the backward ("saved") are
 *     caller-allocated with the sizes moe_plan_info reports, 256-byte aligned.
 *   - Calls are asynchronous on the given stream (a cudaStream_t, or NULL for the
 *     legacy default stream) and never synchronise the host.
 *   - Every call validates its arguments before it launches anything and returns a
 *     status; nothing is thrown across the ABI.  moe_last_error() gives a message
 *     for the last failing call on this thread.  Drops are data, not errors.
 *   - Kernels that wait on a barrier give up after about a second and record
 *     MOE_ERR_TIMEOUT in the status word of the stats buffer instead of hanging.
 *   - Sizes: d_model, d_latent multiples of 64; hidden_routed, hidden_shared
 *     multiples of 128; E % D == 0, (E / D) % n_waves == 0, 1 <= top_k <= min(E, 32),
 *     E <= 1024.  T >= 0 (T == 0 is a no-op).  Needs an sm_100 device.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad ratio */
  MOE_ERR_UNSUPPORTED = 2,  /* shape outside the supported set, or no sm_100 device */
  MOE_ERR_WORKSPACE = 3,    /* ws / saved smaller than moe_plan_info reports */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime or driver call failed */
  MOE_ERR_TIMEOUT = 5       /* a kernel gave up waiting (recorded in the stats status word) */
} moe_status_t;

/* Block shape.  All sizes in elements. */
typedef struct {
  int32_t T;              /* tokens of this source */
  int32_t d_model;        /* model width (6144 at full width) */
  int32_t d_latent;       /* latent width of the routed path (3072) */
  int32_t n_experts;      /* routed experts E (384) */
  int32_t top_k;          /* experts per token k (8) */
  int32_t n_dest;         /* virtual destinations D (64) */
  int32_t n_waves;        /* waves W per destination (3) */
  int32_t hidden_routed;  /* hidden width of a routed expert (3072) */
  int32_t n_shared;       /* shared experts S (2) */
  int32_t hidden_shared;  /* hidden width of a shared expert (3072) */
  int32_t cap_send_num, cap_send_den;  /* sender factor, 110/100 */
  int32_t cap_recv_num, cap_recv_den;  /* receiver factor, 115/100 */
  /* cap_send_num = cap_recv_num = 0 selects the dropless variant ("Marin 535B-A23B"
   * page on ranhao.site, §3.3 token dropping and §7: the run later switched to a
   * dropless ragged all-to-all): no cap binds, every assignment is kept.  Pools are
   * then packed back to back in pool order (T*k rows in all) and the expert buffers
   * by expert, each expert's rows padded to a multiple of 128 (T*k + 127*E rows);
   * moe_plan_info reports cap_send = cap_recv = 0 and those sizes.  The dropless
   * variant runs through moe_forward / moe_backward; moe_dispatch, moe_expert_ffn,
   * moe_combine and moe_dispatch_noalloc return MOE_ERR_UNSUPPORTED for it. */
  int32_t n_sources;      /* virtual sources S (0 or 1: one).  T splits into S equal,
                           * contiguous token ranges, each sending its own D*W pools with
                           * its own sender cap C_s = ceil(1.10 * (T/S)*k / (D*W)), as each
                           * GPU does under expert parallelism ("Marin 535B-A23B" page on
                           * ranhao.site, §3.1 topology; lamjinlab.com §2 caps per pool).
                           * Pools are source-major; a destination's receiver reads its
                           * pools source by source.  T/S must be a multiple of 32. */
  /* Expert parallelism over ep_ranks GPUs (0 or 1: none), this GPU being rank ep_rank:
   * every rank is one source of T tokens and the receiver of destinations
   * [ep_rank * D/G, (ep_rank + 1) * D/G), i.e. of experts [ep_rank * E/G, ...), with
   * G = ep_ranks ("Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播", §3.1 topology and
   * §3.2: 64-way expert parallelism, six experts per GPU, one fixed-shape exchange per
   * wave).  Sender caps use this rank's T; receiver caps all ranks' tokens,
   * C_r = ceil(1.15 * G*T*k / E).  EP plans run through the moe_ep_* calls only. */
  int32_t ep_ranks;
  int32_t ep_rank;
} moe_config_t;

typedef struct moe_plan* moe_plan_t;

/* Derived sizes of a plan.  Byte counts are for caller allocations. */
typedef struct {
  int32_t local_experts;     /* L = E / D */
  int32_t experts_per_wave;  /* P = L / W */
  int32_t n_pools;           /* pools in the buffer: S * D * W (source-major) */
  int32_t cap_send;          /* C_s, rows of one pool (0: dropless) */
  int32_t cap_recv;          /* C_r, rows of one expert (0: dropless) */
  int32_t pool_row_elems;    /* bf16 elements per pool row: d_latent payload + 8 header */
  uint64_t pools_bytes;      /* [D*W][C_s][pool_row_elems] bf16 (dropless: [T*k][...]) */
  uint64_t expert_out_bytes; /* [E][C_r][d_latent] bf16 (dropless: [T*k + 127*E][...]) */
  uint64_t slot_bytes;       /* [T][k][2] int32 */
  uint64_t stats_bytes;      /* moe_stats_t + per-expert and per-pool counters */
  uint64_t saved_bytes;      /* forward context for moe_backward */
  uint64_t workspace_bytes;  /* scratch that suffices for every call */
} moe_plan_info_t;

/* Device-side counters, the head of the stats buffer.  It is followed in the same
 * buffer by int32 hist[E] (pre-drop selections), expert_kept[E],
 * expert_dropped_sender[E], expert_dropped_receiver[E] and pool_fill[D*W]. */
typedef struct {
  int32_t kept;              /* assignments that reached their expert */
  int32_t dropped_sender;    /* assignments past C_s of their pool */
  int32_t dropped_receiver;  /* sender-kept assignments past C_r of their expert */
  int32_t status;            /* 0, or a moe_status_t recorded by a kernel */
  int32_t max_pool_fill;
  int32_t max_expert_fill;
  int32_t assignments;       /* T * k */
  int32_t nan_logits;        /* router logits or bias that were NaN (input error) */
} moe_stats_t;

/* Block weights, all bf16 device pointers, [out][in]. */
typedef struct {
  const uint16_t* w_lat_down;  /* [d_latent][d_model] */
  const uint16_t* w_router;    /* [E][d_latent] */
  const uint16_t* w1;          /* [E][hidden_routed][d_latent]  routed gate */
  const uint16_t* w3;          /* [E][hidden_routed][d_latent]  routed value */
  const uint16_t* w2;          /* [E][d_latent][hidden_routed]  routed down */
  const uint16_t* w_lat_up;    /* [d_model][d_latent] */
  const uint16_t* ws1;         /* [S*hidden_shared][d_model]  shared gate, expert s on rows s*h_s.. */
  const uint16_t* ws3;         /* [S*hidden_shared][d_model]  shared value */
  const uint16_t* ws2;         /* [d_model][S*hidden_shared]  shared down, expert s on columns s*h_s.. */
} moe_weights_t;

/* Weight gradients, float32 device pointers, same shapes as moe_weights_t.  They
 * are the float32 accumulators of the wgrad GEMMs, not rounded to bf16 (the
 * precision of fp32 main-gradient buffers in mixed-precision training). */
typedef struct {
  float *w_lat_down, *w_router, *w1, *w3, *w2, *w_lat_up, *ws1, *ws3, *ws2;
} moe_grads_t;

/* The routed experts alone (for moe_expert_ffn). */
typedef struct {
  const uint16_t* w1;  /* [E][hidden_routed][d_latent] */
  const uint16_t* w3;  /* [E][hidden_routed][d_latent] */
  const uint16_t* w2;  /* [E][d_latent][hidden_routed] */
} moe_expert_weights_t;

/* Device pointers into a forward context ("saved"), for inspection. */
typedef struct {
  const uint16_t* z;          /* [T][d_latent] bf16 */
  const float* logits;        /* [T][E] float32 (logit_offset included) */
  const int32_t* topk_idx;    /* [T][k] */
  const float* topk_gate;     /* [T][k] */
  const int32_t* slot;        /* [T][k][2]: sender slot, receiver slot (-1 = dropped) */
  const int32_t* expert_rows; /* [E] rows each expert received (<= C_r) */
  const uint16_t* expert_in;  /* [E][C_r][d_latent] bf16, receiver-side rows */
  const uint16_t* expert_out; /* [E][C_r][d_latent] bf16 */
  const uint16_t* r;          /* [T][d_latent] bf16, combined routed output */
} moe_saved_view_t;

/* Create a plan for one block shape (host only: checks sizes, computes C_s, C_r
 * and the buffer layouts).  Returns MOE_ERR_UNSUPPORTED for shapes outside the
 * supported set, MOE_ERR_INVALID_ARG for nonsense.  The capacities are the expected
 * rows times the factors, rounded up: C_s = ceil(1.10 * (T/S)*k / (D*W)) per
 * (destination, wave) pool of a source, C_r = ceil(1.15 * T*k / E) per expert.
 * ("Marin начинает открытое обучение MoE-модели с 535 млрд параметров", §2: six
 * experts per GPU, three waves of identical shape, sender cap 1.10 per pool,
 * receiver cap 1.15 per local expert; "Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播",
 * §2.1 spec table: 384 routed experts, top-8, 64-way expert parallelism.) */
MOE_API moe_status_t moe_plan_create(const moe_config_t* cfg, moe_plan_t* out);
MOE_API moe_status_t moe_plan_destroy(moe_plan_t plan);
MOE_API moe_status_t moe_plan_info(moe_plan_t plan, moe_plan_info_t* out);

/* Router: top-k of float32 scores logits + bias (ties to the lower expert index),
 * softmax gates over the k chosen unbiased logits, histogram of selections.
 *   logits [T][E] float32 device, bias [E] float32 device,
 *   topk_idx [T][k] int32 device (selection order), topk_gate [T][k] float32 device,
 *   hist [E] int32 device (overwritten).
 * ("Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播", §2.2: top-8 routing with a
 * histogram-based router and a zero-mean bias.) */
MOE_API moe_status_t moe_route(moe_plan_t plan, const float* logits, const float* bias,
                       int32_t* topk_idx, float* topk_gate, int32_t* hist, void* stream);

/* Sender side of the dispatch: capacity-limited slot assignment in (token, rank)
 * order, then packing of z rows into the fixed pools.
 *   z [T][d_latent] bf16 device; topk_idx [T][k] int32 device;
 *   pools [D*W][C_s][d_latent + 8] bf16 device: row = payload, then a 16-byte header
 *     whose first int32 is the global expert id (-1 for an empty row);
 *   slot [T][k][2] int32 device: (sender slot | -1, receiver slot | -1);
 *   stats: stats buffer (device), counters overwritten (hist left as is);
 *   ws: scratch of ws_bytes >= workspace_bytes.
 * ("Marin начинает открытое обучение MoE-модели с 535 млрд параметров", §2: one
 * fixed pool per receiving GPU, three waves, expert ids in the payload, caps 1.10
 * and 1.15, overflow dropped and counted separately.) */
MOE_API moe_status_t moe_dispatch(moe_plan_t plan, const uint16_t* z, const int32_t* topk_idx,
                          uint16_t* pools, int32_t* slot, void* stats,
                          void* ws, size_t ws_bytes, void* stream);

/* moe_dispatch for callers that cannot allocate device memory.  Some callers have no
 * allocator of their own: a plugin inside a host program that owns the whole
 * device-memory budget, or code whose buffers are laid out before the block's sizes
 * are known.  This variant takes no workspace: the counters of its slot scan live in
 * a static array inside the library (2^21 int32 words, 8 MiB, held on every GPU that
 * loads the library until the process exits).  Inputs and outputs are those of
 * moe_dispatch, with the same results.
 *   - Plans whose scan needs more than 2^21 words (ceil(T/32) * (D*W + E) +
 *     n_sources * D*W) are rejected with MOE_ERR_UNSUPPORTED; use moe_dispatch for
 *     them.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any stream
 *     capture.  The address is kept for the life of the process, so do not use the
 *     library across a cudaDeviceReset of a device it has already run on.
 *   - Every call uses the same array.  Calls whose work overlaps on the GPU (other
 *     streams, other threads) race on it; order them on one stream.  Nothing in the
 *     array has to start at zero: each call writes every word it reads.
 * It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * The source pages have no counterpart of this entry point. */
MOE_API moe_status_t moe_dispatch_noalloc(moe_plan_t plan, const uint16_t* z, const int32_t* topk_idx,
                                          uint16_t* pools, int32_t* slot, void* stats, void* stream);

/* Receiver side and the routed experts: unpack each pool by the packed expert ids
 * (first C_r rows per expert in pool order), then the grouped SwiGLU GEMMs
 * Y_e = (silu(X_e w1_e^T) * (X_e w3_e^T)) w2_e^T.  ("Marin начинает открытое обучение
 * MoE-модели с 535 млрд параметров", §2: the receiver learns each row's expert from
 * the id in the payload, with no separate count or metadata exchange;
 * "Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播", §2.2: SwiGLU experts of width 3072.)
 *   pools as written by moe_dispatch; expert_out [E][C_r][d_latent] bf16 device
 *   (rows at and past the expert's row count are zero or unspecified);
 *   expert_rows [E] int32 device, rows each expert received (may be NULL). */
MOE_API moe_status_t moe_expert_ffn(moe_plan_t plan, const moe_expert_weights_t* w,
                            const uint16_t* pools, uint16_t* expert_out, int32_t* expert_rows,
                            void* ws, size_t ws_bytes, void* stream);

/* Combine: r_t = sum_j kept gate_tj * expert_out[e_tj][rslot_tj], in rank order,
 * float32 accumulation, bf16 result.  r [T][d_latent] bf16 device.  Dropped
 * assignments contribute nothing and the gates are not renormalised.
 * ("Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播", §2.2 diagram: the routed
 * outputs are weighted and summed in the latent space, then projected back to
 * d_model before they meet the shared path.) */
MOE_API moe_status_t moe_combine(moe_plan_t plan, const uint16_t* expert_out, const float* topk_gate,
                         const int32_t* topk_idx, const int32_t* slot, uint16_t* r,
                         void* stream);

/* Whole forward pass: y [T][d_model] float32 device from x [T][d_model] bf16 device.
 * bias [E] float32 device; logit_offset [E] float32 device or NULL.  stats: stats
 * buffer (device), fully overwritten.  saved: forward context for moe_backward
 * (saved_bytes) or NULL for inference.  Steps, in order: latent down-projection,
 * router, top-k, slot assignment, pack, unpack, grouped SwiGLU experts, combine,
 * shared experts, up-projection with the shared down-projection.
 * ("Marin начинает открытое обучение MoE-модели с 535 млрд параметров", §2, and
 * "Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播", §2.2: the 6144 -> 3072 latent
 * projection around the routed path, top-8 of 384 routed experts, two always-on
 * shared SwiGLU experts on every token; "Treinamento aberto do Marin 535B",
 * "A matemática do MoE": the shared experts at half width.) */
MOE_API moe_status_t moe_forward(moe_plan_t plan, const moe_weights_t* w, const uint16_t* x,
                         const float* bias, const float* logit_offset, float* y,
                         void* stats, void* saved, void* ws, size_t ws_bytes, void* stream);

/* Whole backward pass for the loss sum(y * dy): dy [T][d_model] bf16 device, dx
 * [T][d_model] float32 device and every weight gradient (overwritten, float32).
 * Dropped assignments get no gradient; the bias gets none, while the router weights
 * get theirs through the gates.  x must be the forward's input, saved its context.
 * ("Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播", §2.2: the balancing bias stays
 * outside backpropagation and does not change the router's gradients;
 * "Marin начинает открытое обучение MoE-модели с 535 млрд параметров", §2: dropped
 * rows are counted and contribute nothing.) */
MOE_API moe_status_t moe_backward(moe_plan_t plan, const moe_weights_t* w, const void* saved,
                          const uint16_t* x, const uint16_t* dy, float* dx,
                          const moe_grads_t* grads, void* ws, size_t ws_bytes, void* stream);

/* Bias step from a selection histogram: sgn_e = sign(T*k - E*hist_e) decided on
 * integers, b_e += step * (sgn_e - sum(sgn)/E) in float32, which keeps the bias
 * zero-mean.  hist [E] int32 device, bias [E] float32 device (updated in place).
 * ("Marin 535B-A23B：一场完全公开的前沿 MoE 训练直播", §2.2: next-step zero-mean bias
 * outside backpropagation.) */
MOE_API moe_status_t moe_bias_update(moe_plan_t plan, const int32_t* hist, float* bias, float step,
                             void* stream);

/* ---------------------------------------------------------------- expert parallelism
 *
 * A plan with ep_ranks = G >= 2 makes this GPU rank ep_rank of G: one source of T tokens
 * and the receiver of destinations [rank * D/G, (rank + 1) * D/G), i.e. of experts
 * [rank * E/G, (rank + 1) * E/G).  ("Marin начинает открытое обучение MoE-модели с 535 млрд
 * параметров", §2: one fixed pool per receiving GPU, three waves of identical shape, ids
 * in the payload, no count or metadata exchange; "Marin 535B-A23B：一场完全公开的前沿 MoE
 * 训练直播", §3.1 topology and §3.2 three-wave buffers.)  A training step is six calls
 * with an exchange of fixed-shape blocks between consecutive ones, which the caller makes
 * (capacity_limited_routed_b200/parallel.py uses NCCL send/recv):
 *
 *   moe_ep_forward_send      x -> send pools (router, top-k, sender slots, pack)
 *     exchange 1: pools      send_pools -> every rank's recv_pools
 *   moe_ep_forward_experts   recv pools -> this rank's experts -> y rows to send back
 *     exchange 2: y rows     y_send -> every source's y_recv
 *   moe_ep_forward_combine   y rows -> y (combine, up-projection, shared experts)
 *   moe_ep_backward_send     dy -> dY rows to send, dW_up, shared gradients
 *     exchange 3: dY rows    dy_send -> every rank's dy_recv
 *   moe_ep_backward_experts  dY rows -> this rank's expert gradients -> dX rows to send back
 *     exchange 4: dX rows    dx_send -> every source's dx_recv
 *   moe_ep_backward_finish   dX rows -> dx, dW_router, dW_lat_down
 *
 * Blocks.  Every exchange buffer holds D*W blocks of C_s rows (pools: d_latent + 8
 * elements per row, the others d_latent), block b = (a * D/G + d) * W + w for peer a,
 * local destination d < D/G and wave w.  In every exchange a rank sends block b of its
 * send buffer to peer a and receives block b of its receive buffer from peer a; wave w
 * may travel as soon as it is ready.  The receiving side sees its blocks source-major,
 * so its receiver walks sources in rank order (the virtual-sources layout, n_sources).
 * Receiver-dropped rows travel back as zeros.  A forward on G ranks gives the results of
 * a one-GPU forward with n_sources = G over all ranks' tokens in rank order.
 *
 * Buffers: saved and ws have the sizes moe_plan_info reports for the EP plan; the same
 * saved and ws go to all six calls of a step (the backward keeps state in ws from its
 * first call to its last).  Expert weights and gradients are this rank's E/G experts. */
typedef struct {
  int32_t ranks, rank, dest_per_rank, n_waves, cap_send;
  int32_t pool_row_elems;     /* d_latent + 8 */
  int32_t row_elems;          /* d_latent */
  uint16_t* send_pools;       /* [D*W*C_s][d_latent + 8] bf16 (ws) */
  uint16_t* recv_pools;       /* [D*W*C_s][d_latent + 8] bf16 (saved): blocks from every source */
  uint16_t* y_send;           /* [D*W*C_s][d_latent] (ws): expert outputs back to their sources */
  uint16_t* y_recv;           /* [D*W*C_s][d_latent] (saved): this source's rows back */
  uint16_t* dy_send;          /* [D*W*C_s][d_latent] (ws) */
  uint16_t* dy_recv;          /* [D*W*C_s][d_latent] (ws) */
  uint16_t* dx_send;          /* [D*W*C_s][d_latent] (ws) */
  uint16_t* dx_recv;          /* [D*W*C_s][d_latent] (ws) */
  int32_t* expert_rows;       /* [E/G] (saved): rows this rank's experts kept */
  int32_t* topk_idx;          /* [T][k] (saved): this source's choices */
  int32_t* slot;              /* [T][k][2] (saved): sender slot (receiver slots live at the receivers) */
} moe_ep_view_t;

MOE_API moe_status_t moe_ep_view(moe_plan_t plan, void* saved, void* ws, moe_ep_view_t* out);
MOE_API moe_status_t moe_ep_forward_send(moe_plan_t plan, const moe_weights_t* w, const uint16_t* x,
                                         const float* bias, const float* logit_offset, void* stats, void* saved,
                                         void* ws, size_t ws_bytes, void* stream);
MOE_API moe_status_t moe_ep_forward_experts(moe_plan_t plan, const moe_expert_weights_t* w, void* stats, void* saved,
                                            void* ws, size_t ws_bytes, void* stream);
MOE_API moe_status_t moe_ep_forward_combine(moe_plan_t plan, const moe_weights_t* w, float* y, void* saved, void* ws,
                                            size_t ws_bytes, void* stream);
MOE_API moe_status_t moe_ep_backward_send(moe_plan_t plan, const moe_weights_t* w, const void* saved,
                                          const uint16_t* x, const uint16_t* dy, const moe_grads_t* grads, void* ws,
                                          size_t ws_bytes, void* stream);
MOE_API moe_status_t moe_ep_backward_experts(moe_plan_t plan, const moe_expert_weights_t* w, const void* saved,
                                             const moe_grads_t* grads, void* ws, size_t ws_bytes, void* stream);
MOE_API moe_status_t moe_ep_backward_finish(moe_plan_t plan, const moe_weights_t* w, const void* saved,
                                            const uint16_t* x, float* dx, const moe_grads_t* grads, void* ws,
                                            size_t ws_bytes, void* stream);

/* Pointers into a forward context written by moe_forward (no device access). */
MOE_API moe_status_t moe_saved_view(moe_plan_t plan, const void* saved, moe_saved_view_t* out);

/* Tensor-core GEMM used by the block, exposed for testing:
 *   D[m][n] = sum_k A(m, k) * B(n, k), float32 accumulation.
 *   A: a_mn_major == 0 -> stored [M][K]; 1 -> stored [K][M].  bf16 device.
 *   B: b_mn_major == 0 -> stored [N][K]; 1 -> stored [K][N].  bf16 device.
 *   D: [M][N] float32 (d_f32 != 0) or bf16 device.
 *   M, N, K >= 1; the contiguous dimension of each operand a multiple of 8. */
MOE_API moe_status_t moe_gemm_bf16(int32_t M, int32_t N, int32_t K, const uint16_t* A, int32_t a_mn_major,
                           const uint16_t* B, int32_t b_mn_major, void* D, int32_t d_f32,
                           int32_t* status, void* stream);

/* Per-step timing.  Between moe_profile_start and moe_profile_stop every step of the
 * forward / backward calls (a GEMM, the slot scan, the pack, ...) is bracketed by a pair
 * of CUDA events on the call's stream.  moe_profile_stop waits for those events and
 * returns one record per step in launch order (at most cap; *count is the number
 * recorded).  launches counts the kernels the step launched. */
typedef struct {
  char name[40];
  float ms;
  int32_t launches;
} moe_profile_record_t;

MOE_API moe_status_t moe_profile_start(void);
MOE_API moe_status_t moe_profile_stop(moe_profile_record_t* out, int32_t cap, int32_t* count);

/* Kernels launched by this library since it was loaded. */
MOE_API int64_t moe_kernel_launches(void);

/* Streams of moe_forward / moe_backward.  side_stream = 1 (the default): the shared
 * experts, which do not depend on routing, run on a second stream of this library that
 * forks from the caller's stream by an event and joins back by another (forward: beside
 * the routing, slot scan, dispatch, unpack and first routed launches; backward: beside
 * un-dispatch and the router's backward).  side_stream = 0: every step of a call runs in
 * order on the caller's stream, so per-step event times (moe_profile_start) are each
 * step's own.  The results are the same either way.  Process-wide; takes effect for calls
 * made after it returns.  Any value other than 0 or 1 is rejected with
 * MOE_ERR_INVALID_ARG. */
MOE_API moe_status_t moe_set_side_stream(int32_t side_stream);

/* Message for the last failing call on this thread ("" if none). */
MOE_API const char* moe_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */

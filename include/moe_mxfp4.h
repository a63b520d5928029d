/*
 * moe_mxfp4.h -- C ABI of the routed MXFP4 Mixture-of-Experts FFN layer on
 * B200 (sm_100a).
 *
 * The layer (rabbit README, ferrumox/rabbit, model table row "MoE routing":
 * softmax routing to 10 of 512 experts plus a gated shared expert, routed
 * experts read as OCP MXFP4; the "expert matmul" phase of its decode-step
 * breakdown) computes, for
 * every token t of x [T, H]:
 *
 *   logits = Wr x_t                         router, fp32 accumulate
 *   idx, w = top-k of softmax(logits)       lowest index wins ties, w renormalised
 *   y_t    = sum_j w_j * FFN_{idx_j}(x_t)  routed SwiGLU experts on MXFP4 weights
 *          + sigmoid(w_sg . x_t) * FFN_shared(x_t)      gated bf16 shared expert
 *
 * with FFN_e(x) = Wd_e (silu(Wg_e x) * (Wu_e x)). The latent-width variant
 * ("Ran Moonshot's 2.8T-parameter Kimi K3 on a GPU-less mini-PC", architecture
 * paragraph: Stable LatentMoE, routed experts compute in a narrower latent
 * width) runs the routed experts on x_lat = bf16(W_ld x) [T, L] and maps their
 * weighted sum back with W_lu [H, L] before the shared expert is added.
 *
 * Conventions shared by every call
 * --------------------------------
 * - All pointers are DEVICE pointers on the current CUDA device unless a
 *   parameter says otherwise; the caller owns every buffer. No call allocates
 *   or frees device memory; scratch comes from the caller's workspace.
 * - bf16 tensors are passed as uint16_t bit patterns. Matrices are row-major;
 *   weight matrices are [out, in] with the input dimension contiguous.
 * - MXFP4 matrix [N, K] (OCP MX v1.0, section 5: E2M1 elements, E8M0 scale per
 *   32 elements): q [N, K/2] uint8, element 2j of a row is the LOW nibble of
 *   byte j and element 2j+1 the HIGH nibble; s [N, K/32] uint8, one E8M0 code
 *   per 32 consecutive elements of a row (value 2^(c-127); code 255 is NaN and
 *   poisons its block, IEEE propagation, not an error). Experts are stacked:
 *   Wg, Wu as q [E, I, W/2] + s [E, I, W/32]; Wd as q [E, W, I/2] + s [E, W, I/32],
 *   where W = L for latent layers, else H.
 * - `stream` is a cudaStream_t (NULL = legacy default stream). Every call only
 *   enqueues work on it and returns; nothing is synchronised.
 * - Synchronous validation: null or misaligned (16-byte) pointers, shapes this
 *   build does not support, or a workspace smaller than moe_workspace_size()
 *   return an error status and enqueue NOTHING. moe_last_error() then holds a
 *   one-line reason (thread-local).
 * - Data errors found on the device (an expert index outside [0, E) or repeated
 *   within a token) set a status word in the workspace; the affected call then
 *   produces empty routing (all counts 0) instead of touching memory out of
 *   range. Read it with moe_device_status().
 *
 * Supported shapes: 1 <= T <= 65536; H, I, I_shared and L (when non-zero)
 * multiples of 128 in [128, 65536]; 1 <= E <= 1024; 1 <= k <= min(E, 32);
 * T*k <= 2^24.
 */
#ifndef MOE_MXFP4_H
#define MOE_MXFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* null pointer, null dims, bad enum */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,  /* a dimension outside the supported set */
  MOE_ERR_ALIGNMENT = 3,          /* a pointer not 16-byte aligned */
  MOE_ERR_WORKSPACE_TOO_SMALL = 4,
  MOE_ERR_CUDA = 5,               /* a CUDA runtime call failed (launch, event) */
  MOE_ERR_DEVICE_STATUS = 6       /* returned by moe_device_status() when the
                                     device flagged a data error */
} moe_status;

/* How the routed experts receive their activations. */
typedef enum {
  /* bf16 activations. x is carried exactly (as f16 times one power-of-two
   * scale per token row); h = silu(g)*u enters the down projection as f16
   * times a power of two per group (32 elements on the single-token path, a
   * whole row on the multi-token TMA-ring path, 16 elements on the per-warp
   * path): relative rounding <= 2^-11 for every element within 2^-28 of its
   * group's largest magnitude. Decode path: grouped MXFP4 GEMVs. */
  MOE_ACT_BF16 = 0,
  /* MXFP4 activations: x rows and h are quantised to OCP MXFP4 (32-element
   * blocks, OCP MX v1.0 section 6.3 conversion) and the experts run as
   * block-scaled MXF4 tensor-core GEMMs (prefill path). */
  MOE_ACT_MXFP4 = 1
} moe_act_mode;

/* How the router scores experts (rabbit README, model table row "MoE
 * routing": a softmax over 512 experts keeping the best 10 for Qwen3.8-Max,
 * the router named noaux_tc sigmoid for GLM-5.2 and grouped routing for Kimi
 * Linear; the pages name the last two only, so their definitions here are
 * readings). */
typedef enum {
  /* softmax: experts ranked by logit; w = the softmax renormalised over the
   * selected experts (times route_scale). */
  MOE_SCORE_SOFTMAX = 0,
  /* sigmoid: s_e = sigmoid(logit_e); experts ranked by s_e + e_bias[e] (the
   * bias steers the selection only; NULL = 0); w_j = s_j / sum of the
   * selected s (times route_scale). */
  MOE_SCORE_SIGMOID = 1
} moe_score_fn;

typedef struct {
  int32_t T;         /* tokens */
  int32_t H;         /* hidden width */
  int32_t I;         /* routed-expert intermediate width */
  int32_t E;         /* routed experts */
  int32_t k;         /* experts per token */
  int32_t I_shared;  /* shared-expert intermediate width */
  int32_t L;         /* latent width of the routed experts; 0 = none (W = H) */
  int32_t act_mode;  /* moe_act_mode */
  /* router variant (all zero: the softmax router) */
  int32_t score_fn;     /* moe_score_fn */
  int32_t n_group;      /* 0 or 1: no groups. 2..64: group-limited selection: the
                           E experts form n_group groups of E / n_group
                           consecutive ids; a group scores the sum of its two
                           largest expert scores (the softmax probability, or
                           the biased sigmoid score); the topk_group best groups
                           are kept (ties: lower group); top-k among their
                           experts. Needs E % n_group == 0 and
                           topk_group * E / n_group >= k. */
  int32_t topk_group;   /* groups kept, 1..n_group (ignored without groups) */
  float route_scale;    /* multiplies the routing weights; 0 means 1 */
} moe_dims;

/* One-line description of a status code (static storage). */
const char* moe_status_string(moe_status s);

/* Reason for the last non-OK status returned on this host thread. */
const char* moe_last_error(void);

/* Bytes of device workspace every call below needs for `dims` (the same
 * buffer serves all calls; it must stay valid until the enqueued work has
 * run). Returns 0 for dims that fail validation. */
size_t moe_workspace_size(const moe_dims* dims);

/* Bytes of the activation operand buffer written by moe_permute and read by
 * moe_expert_ffn (x_op below). Returns 0 for invalid dims. */
size_t moe_x_op_size(const moe_dims* dims);

/* Clear the device status word in `ws` and the counters the one-token
 * routed launch hands work out with (enqueued on `stream`). Call once after
 * allocating a workspace, before its first use: those counters must start at
 * zero (every one-token call leaves them at zero again). Calls that share a
 * workspace must not overlap in time. */
moe_status moe_workspace_init(const moe_dims* dims, void* ws, size_t ws_bytes, void* stream);

/* Wait for `stream`, then copy the device status word into *host_status
 * (HOST pointer; 0 = no error). Returns MOE_ERR_DEVICE_STATUS when the word is
 * non-zero, MOE_OK otherwise. Bits (OR-ed by every call that sees them, kept
 * until moe_workspace_init clears them):
 *   1 (bit 0)  an expert index outside [0, E) (the dispatch is emptied);
 *   2 (bit 1)  an expert repeated within one token (the dispatch is emptied);
 *   4 (bit 2)  a bounded device wait gave up: a kernel waited for a shared-
 *              memory stage (a TMA or bulk copy, or another role of its CTA)
 *              for about five seconds without it arriving; that kernel
 *              stopped early, so the outputs of the call are incomplete. */
moe_status moe_device_status(const void* ws, int32_t* host_status, void* stream);

/* --- a1-a2: router ---------------------------------------------------------
 * (rabbit README, model table row "MoE routing": softmax routing to 10 of 512 experts; the
 * lowest-index tie-break and the renormalisation are readings of it.)
 * logits[t, e] = sum_h x[t, h] Wr[e, h] (bf16 products are exact, fp32
 * accumulation), p = softmax(logits[t]) in fp32, the k largest logits are
 * selected (equal logits: lower expert index first; slots ordered by
 * descending logit) and topk_w[t, j] = p[idx_j] / sum_j' p[idx_j'].
 *   x         [T, H] bf16           w_router [E, H] bf16
 *   topk_idx  [T, k] int32 (out)    topk_w   [T, k] fp32 (out)
 *   logits    [T, E] fp32 (out, may be NULL)
 */
moe_status moe_route(const moe_dims* dims, const uint16_t* x, const uint16_t* w_router,
                     int32_t* topk_idx, float* topk_w, float* logits,
                     void* ws, size_t ws_bytes, void* stream);

/* moe_route with the router's per-expert selection bias e_bias [E] fp32
 * (device; used by MOE_SCORE_SIGMOID, ignored by the softmax router; NULL =
 * no bias). The selection and weight rules are those of dims->score_fn,
 * n_group, topk_group and route_scale (see moe_dims). moe_route is this call
 * with e_bias = NULL. */
moe_status moe_route_biased(const moe_dims* dims, const uint16_t* x, const uint16_t* w_router,
                            const float* e_bias, int32_t* topk_idx, float* topk_w, float* logits,
                            void* ws, size_t ws_bytes, void* stream);

/* --- router without a workspace ---------------------------------------------
 * (No counterpart in the pages: an interface convenience of this library.)
 * The router step of moe_route (same inputs, outputs, selection and weight
 * rule) for callers that cannot supply device scratch memory: a plug-in given
 * only its input and output tensors, or a runtime whose memory plan allows no
 * extra buffer. Its split-K partial sums go to a 4 MiB device array built
 * into the library. It does not run moe_route's logit kernels: its logits
 * come from a split-K CUDA-core GEMV summed in another order, so they agree
 * with moe_route's to fp32 rounding; the selected experts are the same
 * except at near ties of two router logits (every call on the same inputs
 * gives the same bits). Shapes needing more than 4 MiB of partials (S * T * E
 * fp32 values, S = its K-split count, up to 16) return
 * MOE_ERR_UNSUPPORTED_SHAPE before anything is enqueued. The array is shared
 * by every call on a device: calls that overlap on the GPU race on it. The
 * first call on each device looks up the array's address; make it before
 * capturing a stream into a CUDA graph. Nothing is allocated.
 */
moe_status moe_route_noalloc(const moe_dims* dims, const uint16_t* x, const uint16_t* w_router,
                             int32_t* topk_idx, float* topk_w, float* logits, void* stream);

/* --- a3-a4: permutation ----------------------------------------------------
 * (The pages do not describe the dispatch; grouping the routed (token, slot)
 * pairs by expert is what running each expert once on its own tokens needs.)
 * Groups the T*k (token, slot) pairs by expert: counts[e] pairs per expert,
 * offsets = exclusive prefix sum (E+1 entries), permuted rows ordered by
 * expert and, inside an expert, by ascending token; expert_list[0] = number
 * of experts with at least one pair, expert_list[1..] = those experts in
 * ascending order (the work list of the expert kernels). row_token[r] / row_slot[r]
 * give the pair at permuted row r; slot_row[t, j] the row of pair (t, j).
 * It also writes the activation operand x_op from x_in ([T, W] bf16: x, or
 * x_lat for latent layers).
 *   x_op format, MOE_ACT_BF16: ONE ROW PER TOKEN (the grouped GEMVs gather
 *     rows through row_token): f16 values [T, W], then (at the next 256-byte
 *     boundary) fp32 row scales [T]: value = f16 * scale, the scale a power of
 *     two that maps the row's largest magnitude into [2^14, 2^15).
 *   x_op format, MOE_ACT_MXFP4: ONE ROW PER PERMUTED ROW, ready for the tensor
 *     cores (offsets of the parts from moe_mxf4_layout_of):
 *       codes [T*k, W/2] uint8 (low nibble = even element; OCP MX v1.0
 *         conversion of the token's bf16 row, ties to even), row r = token
 *         row_token[r];
 *       E8M0 scales in the TILED layout below, K = W;
 *       the tile list: tiles[t] = {expert, first permuted row, rows, 0} int32x4,
 *         each expert's rows cut into tiles of at most tile_rows consecutive
 *         rows, experts in expert_list order; tile_base[e] int32 = the first
 *         tile of active expert e; n_tiles int32 = number of tiles.
 *   TILED scale layout (what tcgen05 block-scaled MMAs read): for row n of
 *     tile t (0 <= n < 128) and K-block j (32 elements), the byte at
 *     (t * K/128 + j/4) * 512 + 16*(n % 32) + 4*(n / 32) + j % 4. For weight
 *     matrices the tiles are the 128-row blocks (t = row / 128, n = row % 128),
 *     see moe_tile_scales.
 *   topk_idx [T, k] int32; counts [E], offsets [E+1], expert_list [E+1],
 *   row_token [T*k], row_slot [T*k], slot_row [T, k] int32 (out);
 *   x_op moe_x_op_size() bytes (out)
 */
moe_status moe_permute(const moe_dims* dims, const int32_t* topk_idx, const uint16_t* x_in,
                       int32_t* counts, int32_t* offsets, int32_t* expert_list, int32_t* row_token,
                       int32_t* row_slot, int32_t* slot_row, void* x_op,
                       void* ws, size_t ws_bytes, void* stream);

/* --- a5-a7: routed experts (the "expert matmul") ----------------------------
 * (rabbit README: the "expert matmul" phase of its decode-step breakdown, on
 * routed experts read as OCP MXFP4, model table row "native quantization
 * read"; the SwiGLU activation is a reading.)
 * For every permuted row r of expert e (offsets[e] <= r < offsets[e+1]) and
 * its token t = row_token[r]:
 *   y_perm[r] = Wd_e ( silu(Wg_e x_t) * (Wu_e x_t) )      [W] fp32
 * Weights in the canonical MXFP4 layout above, decoded exactly (E2M1 value x
 * E8M0 scale); products accumulate in fp32. One token (T = 1, MOE_ACT_BF16):
 * both projections of its experts run in one launch whose CTAs take work
 * from counters in `ws` (see moe_workspace_init).
 * MOE_ACT_MXFP4 (tcgen05 block-scaled MMAs): x and h = silu(Wg x) * (Wu x)
 * enter their products as MXFP4 (h quantised per 32-element block along I);
 * wg_s, wu_s and wd_s must then be in the TILED layout (moe_tile_scales of the
 * canonical [E*N, K/32] arrays); the codes keep the canonical layout.
 *   x_op, offsets, expert_list, row_token as written by moe_permute;
 *   y_perm [T*k, W] fp32 (out)
 */
moe_status moe_expert_ffn(const moe_dims* dims, const void* x_op, const int32_t* offsets,
                          const int32_t* expert_list, const int32_t* row_token,
                          const uint8_t* wg_q, const uint8_t* wg_s,
                          const uint8_t* wu_q, const uint8_t* wu_s,
                          const uint8_t* wd_q, const uint8_t* wd_s,
                          float* y_perm, void* ws, size_t ws_bytes, void* stream);

/* --- routed experts streamed from host memory --------------------------------
 * (rabbit README: the routed experts do not stay resident but are fetched
 * when a token needs them, through an LRU cache per layer, and its per-expert
 * early drain starts an expert's matmul as soon as that expert's own bytes
 * have arrived.)
 * A cache of `slots` expert slots in device memory (caller-owned, sized by
 * moe_expert_cache_bytes, 256-byte aligned) in front of experts kept in host
 * memory. MOE_ACT_BF16 layers only.
 *
 * moe_expert_ffn_streamed computes what moe_expert_ffn computes (the same
 * kernels, bit for bit) for the experts listed in `active` (HOST array of
 * n_active distinct ids, e.g. expert_list[1..] of moe_permute read back;
 * n_active <= slots): experts already in a slot (hits) keep it; every other
 * one takes the least recently used slot that this call does not use and is
 * copied there from host_experts (HOST array of E*6 pointers: per expert its
 * wg_q, wg_s, wu_q, wu_s, wd_q, wd_s in the canonical layout, in page-locked
 * host memory for the copies to be asynchronous) on the cache's own copy
 * stream, after the last launch that read the slot. Each expert's gate/up and
 * down launches wait (on `stream`) only for their own expert's copy, in list
 * order; hits start at once. x_op, offsets, row_token, y_perm, ws as for
 * moe_expert_ffn. The cache is not capturable in a CUDA graph (its copies run
 * on a stream of its own). Calls on one cache are serialised by a lock.
 */
typedef struct moe_expert_cache moe_expert_cache;   /* opaque, host side */
size_t moe_expert_cache_bytes(const moe_dims* dims, int32_t slots);
moe_status moe_expert_cache_create(const moe_dims* dims, int32_t slots, void* dev_mem, size_t dev_bytes,
                                   moe_expert_cache** out);
/* Waits for the cache's copies, then frees its host-side state (not dev_mem). */
moe_status moe_expert_cache_destroy(moe_expert_cache* cache);
/* Running totals: experts found in a slot, experts copied, bytes copied. */
moe_status moe_expert_cache_stats(const moe_expert_cache* cache, int64_t* hits, int64_t* misses,
                                  int64_t* bytes_copied);
moe_status moe_expert_ffn_streamed(moe_expert_cache* cache, const moe_dims* dims, const int32_t* active,
                                   int32_t n_active, const void* x_op, const int32_t* offsets,
                                   const int32_t* row_token, const uint8_t* const* host_experts,
                                   float* y_perm, void* ws, size_t ws_bytes, void* stream);

/* --- MXFP4 tensor-core operands ----------------------------------------------
 * (No counterpart in the pages: data layout of this library.)
 * moe_tile_scales: canonical row-major E8M0 scales [rows, K/32] (src) -> the
 * TILED layout with 128-row tiles (dst, the same rows*K/32 bytes), as
 * moe_expert_ffn / moe_layer take them for MOE_ACT_MXFP4. rows and K
 * multiples of 128; enqueued on `stream`; src and dst device pointers.
 */
moe_status moe_tile_scales(const uint8_t* src, int64_t rows, int32_t K, uint8_t* dst, void* stream);

/* Byte offsets of the MOE_ACT_MXFP4 operands, for inspection and tests:
 * inside x_op: x_codes, x_scales (tiled), tiles, tile_base, n_tiles (see
 * moe_permute); inside the workspace, where moe_expert_ffn leaves h exactly as
 * the down projection consumed it: h_codes [T*k, I/2] uint8 and h_scales
 * (tiled, K = I, tiles of the tile list). Valid until the next call that uses
 * the buffer. MOE_ACT_BF16 returns MOE_ERR_UNSUPPORTED_SHAPE. */
typedef struct {
  size_t x_codes, x_scales, tiles, tile_base, n_tiles;   /* in x_op */
  size_t h_codes, h_scales;                              /* in the workspace */
  int32_t max_tiles, tile_rows;
} moe_mxf4_layout;
moe_status moe_mxf4_layout_of(const moe_dims* dims, moe_mxf4_layout* out);

/* --- a8-a9 (+a10 up): shared expert and combine ------------------------------
 * (rabbit README, model table row "MoE routing": a gated shared expert runs
 * beside the routed ones; the per-token sigmoid gate is a reading.)
 *   s_t = sigmoid(w_sgate . x_t) * Ws_down (silu(Ws_gate x_t) * (Ws_up x_t))
 *   y_t = [W_lu] (sum_j topk_w[t, j] * y_perm[slot_row[t, j]]) + s_t
 * W_lu is applied only for latent layers (w_lat_up non-NULL iff L > 0).
 *   x [T, H] bf16; w_sgate [H]; ws_gate, ws_up [I_shared, H]; ws_down
 *   [H, I_shared]; w_lat_up [H, L] bf16; y [T, H] fp32 (out)
 */
moe_status moe_combine(const moe_dims* dims, const float* y_perm, const int32_t* slot_row,
                       const float* topk_w, const uint16_t* x, const uint16_t* w_sgate,
                       const uint16_t* ws_gate, const uint16_t* ws_up, const uint16_t* ws_down,
                       const uint16_t* w_lat_up, float* y,
                       void* ws, size_t ws_bytes, void* stream);

/* --- a10: latent down-projection (latent layers only) ------------------------
 * ("Ran Moonshot's 2.8T-parameter Kimi K3 on a GPU-less mini-PC", architecture
 * paragraph: Stable LatentMoE, routed experts in a narrower latent width; the
 * dense bf16 projection and the bf16 rounding point are readings.)
 * x_lat[t] = bf16_rne( W_ld x_t ),  W_ld [L, H] bf16, x_lat [T, L] bf16 (out).
 */
moe_status moe_latent_down(const moe_dims* dims, const uint16_t* x, const uint16_t* w_lat_down,
                           uint16_t* x_lat, void* ws, size_t ws_bytes, void* stream);

/* --- diagnostics: the bounded device waits ----------------------------------
 * (No counterpart in the pages: a check of this library's failure handling.)
 * Every stage-ring kernel waits for its shared-memory stages with a bounded
 * wait; when a stage's bytes do not arrive in time it raises an abort flag,
 * every role of the CTA stops, and bit 2 (value 4) of the status word is set
 * (see moe_device_status). This call runs one CTA that uses the same waits
 * on one 512-byte stage, with `limit` tries (1..4096; about 20 us each at
 * most) instead of the multi-second default:
 *   deliver != 0: the stage is filled by a bulk copy from `src` (a 16-byte
 *     aligned DEVICE buffer of 512 bytes); the waits succeed and *status is
 *     left unchanged;
 *   deliver == 0: nothing delivers the stage's bytes; both waits give up, the
 *     kernel returns and ORs 4 into *status (a DEVICE int32).
 * No copy is in flight when a wait gives up, so the context stays usable.
 * Enqueued on `stream`; invalid arguments return an error and enqueue nothing.
 */
moe_status moe_selftest_bounded_wait(int32_t* status, const void* src, int deliver,
                                     uint32_t limit, void* stream);

/* --- the whole layer ---------------------------------------------------------
 * Every buffer of the calls above in one struct; moe_layer enqueues the same
 * arithmetic as route -> (latent_down) -> permute -> expert_ffn -> combine
 * (bit for bit: the latent down-projection rows ride in the router's pass over
 * x with the same splits as the stand-alone call; for one token in bf16 mode
 * without a latent projection the top-k launch also writes what moe_permute
 * writes), with the first half of the shared expert on a second stream forked
 * from and joined back into `stream` (capturable in a CUDA graph).
 */
typedef struct {
  const uint16_t* x;
  const uint16_t* w_router;
  const uint8_t *wg_q, *wg_s, *wu_q, *wu_s, *wd_q, *wd_s;
  const uint16_t* w_sgate;
  const uint16_t *ws_gate, *ws_up, *ws_down;
  const uint16_t *w_lat_down, *w_lat_up;   /* NULL unless L > 0 */
  /* outputs and intermediates (all caller-owned) */
  int32_t* topk_idx;   /* [T, k] */
  float* topk_w;       /* [T, k] */
  int32_t *counts, *offsets, *expert_list, *row_token, *row_slot, *slot_row;
  uint16_t* x_lat;     /* [T, L], NULL unless L > 0 */
  void* x_op;          /* moe_x_op_size() bytes */
  float* y_perm;       /* [T*k, W] */
  float* y;            /* [T, H] */
  const float* e_bias; /* [E] router selection bias (MOE_SCORE_SIGMOID), or NULL */
} moe_layer_args;

moe_status moe_layer(const moe_dims* dims, const moe_layer_args* args,
                     void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_MXFP4_H */

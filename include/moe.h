/*
 * moe.h — C ABI of the B200 (sm_100a) sparse Mixture-of-Experts FFN forward.
 *
 * The layer computes, for every token x_t (pages cited by title and listing):
 *
 *   z_t   = W_r x_t (+ b_r) (+ logit_bias)                      router
 *   S_t   = top-k experts of z_t (descending; ties -> lower index)
 *   g_t,s = gate of slot s (three modes, see MOE_GATE_*)
 *   y_t   = sum_{s kept} g_t,s * E_{S_t,s}(x_t) (+ sum_j Shared_j(x_t))
 *
 *   "MoE (Mixture of Experts) 아키텍처 완전 정복" (devtips.kr): MoELayer, DeepSeekMoE,
 *       the capacity snippet.
 *   "Mixture of Experts（MoE）架构深度解析" (youngju.dev, zh): GatingNetwork, MoELayer,
 *       SwitchRouter, load_balancing_loss, MixtralMoELayer, SwiGLUExpert,
 *       DeepSeekMoELayer.
 *   "Sparse Mixture of Experts（MoE）アーキテクチャ深層分析" (youngju.dev, ja): the gating
 *       equation y = sum_i G(x)_i E_i(x), SwiGLUExpert, TopKGating,
 *       compute_load_balancing_loss, router_z_loss.
 *   "Mixture of Experts" (study-site lecture 03): Token Routing, the SwiGLU table.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Ownership: the caller allocates and owns every buffer (device memory unless
 *   stated). The library never allocates, frees or keeps pointers after a call.
 * - Asynchrony: every call only enqueues kernels on `stream` and returns; none
 *   synchronises except moe_last_device_error(). The layer's kernels are launched
 *   with programmatic stream serialisation: each may begin its set-up while the
 *   kernel before it in the stream finishes, and waits for that kernel before it
 *   reads that kernel's output or writes anything. Before that wait the expert
 *   GEMMs only read the weights and the routing tables of this call, and request
 *   their first weight slices. The tables are complete by then: they come from an
 *   earlier kernel of the same call that the kernel ahead waited for, or (the
 *   tile table of moe_expert_ffn) from the kernel ahead itself, which does not let
 *   its successor begin before it has completed.
 * - Layout: row-major. Weights use the nn.Linear [out_features, in_features]
 *   layout, stacked over experts. Activations, weights, x_perm, y_perm and y are
 *   stored in cfg->dtype (fp32 or bf16); biases, logits, gates are fp32; index
 *   arrays are int32.
 * - Alignment: every pointer must be 16-byte aligned, the workspace 256-byte.
 * - Validation: arguments are checked on the host before anything is launched;
 *   a failed check returns an error status and enqueues nothing. No call aborts
 *   or throws.
 * - Device-side errors (an expert index out of range, offsets that are not a
 *   valid partition, a bounded wait that gave up) are recorded in a sticky error
 *   word at the start of the workspace; read and clear it with
 *   moe_last_device_error(). A kernel that detects one skips the offending
 *   access instead of faulting.
 * - Workspace: one buffer of moe_workspace_size() bytes serves every entry point
 *   of a configuration. Zero it once with moe_workspace_init() before first use.
 *   Calls that share a workspace must not overlap on the GPU.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (NULL = the legacy default stream). */
typedef struct CUstream_st *moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* a size, mode or pointer is out of range / NULL */
  MOE_ERR_UNSUPPORTED = 2,  /* valid, but outside what the kernels implement */
  MOE_ERR_MISALIGNED = 3,   /* a pointer breaks the 16-byte (256 for ws) rule */
  MOE_ERR_WORKSPACE = 4,    /* ws_bytes < moe_workspace_size() */
  MOE_ERR_CUDA = 5,         /* a CUDA runtime call failed (launch, attribute) */
  MOE_ERR_DEVICE = 6        /* moe_last_device_error() found a device-side error */
} moe_status_t;

/* Device error codes (the `code` of moe_last_device_error). */
enum {
  MOE_DEVERR_NONE = 0,
  MOE_DEVERR_EXPERT_INDEX = 1,  /* topk_idx outside [0, E); info = token*k + slot */
  MOE_DEVERR_OFFSETS = 2,       /* offsets not non-decreasing within [0, T*k]; info = expert */
  MOE_DEVERR_ROW_INDEX = 3,     /* inv outside [-1, T*k); info = token*k + slot */
  MOE_DEVERR_WAIT_TIMEOUT = 4   /* a pipeline wait exceeded its bound; info = site */
};

/* Expert FFN kinds. */
enum {
  MOE_ACT_RELU = 0,   /* Linear(d,F)+b1 -> ReLU -> Linear(F,d)+b2   (devtips.kr MoELayer)   */
  MOE_ACT_GELU = 1,   /* Linear(d,F)+b1 -> GELU(erf) -> Linear(F,d)+b2 (youngju zh MoELayer) */
  MOE_ACT_SWIGLU = 2  /* w_down(silu(w_gate x) * w_up x), no bias     (SwiGLUExpert)        */
};

/* Gate modes. Selection is always the top-k of the fp32 logits. */
enum {
  MOE_GATE_TOPK_SOFTMAX = 0,        /* softmax over the k selected logits (MoELayer, GatingNetwork) */
  MOE_GATE_SOFTMAX_TOPK_RENORM = 1, /* full softmax, selected probs / their sum (TopKGating)     */
  MOE_GATE_SOFTMAX_TOPK_RAW = 2     /* full softmax, selected probs as they are (SwitchRouter)   */
};

enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 };

/* Routing. Token choice: every token picks its top-k experts (all gate modes,
 * capacity drops). Expert choice (youngju.dev (zh) "ExpertChoiceRouter", youngju.dev
 * (ja) "ExpertChoiceGating"): every expert takes the C = floor(cf * T / E) tokens with
 * the highest score, score = its softmax over the tokens of the call; a token's
 * output is the score-weighted sum over the experts that took it (the dispatch mask
 * as the gate), 0 if none did. top_k and gate_mode are not used. */
enum { MOE_ROUTING_TOKEN_CHOICE = 0, MOE_ROUTING_EXPERT_CHOICE = 1 };

/* Layer configuration (MoEConfig of the ja page, plus routing and storage fields).
 * Limits: 1 <= E <= 256; 1 <= k <= min(E, 8); T >= 0 (T = 0 is a no-op);
 * d_model, d_ff, d_ff_shared multiples of 64 for bf16 (tensor-core path) and of
 * 4 for fp32; n_shared >= 0 (shared experts are SwiGLU). */
typedef struct {
  int32_t n_tokens;        /* T: tokens of the call (batch and sequence flattened) */
  int32_t d_model;         /* d */
  int32_t n_experts;       /* E routed experts */
  int32_t top_k;           /* k */
  int32_t d_ff;            /* F of each routed expert */
  int32_t act;             /* MOE_ACT_* */
  int32_t gate_mode;       /* MOE_GATE_* */
  int32_t dtype;           /* MOE_DTYPE_*: storage of x, weights, x_perm, y_perm, y */
  float capacity_factor;   /* > 0: capacity = floor(cf*T*k/E) rows per expert, overflow
                              dropped in token-major then slot order; <= 0: unlimited */
  float aux_alpha;         /* weight of the load-balancing loss (0.01 on the pages) */
  int32_t n_shared;        /* always-on SwiGLU experts, added unweighted (0 = none) */
  int32_t d_ff_shared;     /* F of each shared expert */
  int32_t routing;         /* MOE_ROUTING_*; expert choice: capacity_factor > 0 gives C,
                              1 <= C <= 8192, T <= 32768, n_shared = 0 */
} moe_cfg_t;

/* Device pointers to the parameters. Unused entries must be NULL. */
typedef struct {
  const void *w_router;     /* [E, d]              dtype */
  const float *b_router;    /* [E]  fp32 router bias, or NULL */
  const float *logit_bias;  /* [E]  fp32 added to the logits, or NULL */
  const void *w1;           /* [E, F, d]  dtype; SwiGLU: w_gate */
  const void *w3;           /* [E, F, d]  dtype; SwiGLU: w_up (NULL for MLP experts) */
  const void *w2;           /* [E, d, F]  dtype; w_down */
  const float *b1;          /* [E, F] fp32 or NULL (MLP experts only) */
  const float *b2;          /* [E, d] fp32 or NULL (MLP experts only) */
  const void *ws_gate;      /* [n_shared*F_sh, d] dtype: shared experts' w_gate, concatenated */
  const void *ws_up;        /* [n_shared*F_sh, d] dtype */
  const void *ws_down;      /* [d, n_shared*F_sh] dtype */
  const void *w_noise;      /* [E, d]  dtype: noise projection of noisy top-k gating
                               (moe_route_noisy / moe_forward_noisy), else NULL */
} moe_weights_t;

/* Optional device buffers that moe_forward fills with its intermediates
 * (any member may be NULL). Sizes as in moe_route / moe_permute. */
typedef struct {
  float *logits;       /* [T, E] */
  int32_t *topk_idx;   /* [T, k] */
  float *topk_gate;    /* [T, k] */
  int32_t *counts;     /* [E]   assignments per expert before capacity drops */
  int32_t *offsets;    /* [E+1] kept-row prefix: expert e owns rows [offsets[e], offsets[e+1]) */
  int32_t *perm;       /* [T*k] row -> token (rows >= offsets[E] are left unspecified) */
  int32_t *inv;        /* [T*k] (token, slot) -> row, -1 when dropped */
} moe_taps_t;

/* Bytes of workspace every entry point needs for `cfg`. */
moe_status_t moe_workspace_size(const moe_cfg_t *cfg, size_t *bytes);

/* Zero the workspace header (the sticky device error word, and the ticket word
 * that the permute step's scan CTAs share; every launch leaves it at zero again).
 * Call once after allocating a workspace. */
moe_status_t moe_workspace_init(void *ws, size_t ws_bytes, moe_stream_t stream);

/* Router + selection + gates ("GatingNetwork"/"TopKGating"/"SwitchRouter").
 * x [T, d] dtype, or NULL: then `logits` is an INPUT [T, E] and only selection
 * and gates run. Otherwise logits [T, E] fp32 is an output (may be NULL).
 * topk_idx [T, k] int32 and topk_gate [T, k] fp32 are outputs: slots in
 * descending logit order, equal logits -> lower expert index first. */
moe_status_t moe_route(const moe_cfg_t *cfg, const moe_weights_t *w, const void *x,
                       float *logits, int32_t *topk_idx, float *topk_gate,
                       void *ws, size_t ws_bytes, moe_stream_t stream);

/* Histogram, capacity, prefix sum and permutation ("SwitchRouter" drop rule).
 * In: x [T, d] dtype, topk_idx [T, k]. Out: counts [E] (before drops), offsets
 * [E+1] (kept-row prefix), perm [T*k] (row -> token), inv [T*k] ((t,s) -> row or
 * -1), x_perm [T*k, d] dtype (row r holds x[perm[r]]; rows of expert e are in
 * token order). Rows past offsets[E] are left unspecified. */
moe_status_t moe_permute(const moe_cfg_t *cfg, const void *x, const int32_t *topk_idx,
                         int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv,
                         void *x_perm, void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_permute for callers that cannot allocate device memory. (No counterpart on
 * the pages: it is a deployment variant of the permute step above.)
 * Some callers own no device memory beyond their inputs and outputs — a plugin
 * or operator inside a framework that manages every other byte through its own
 * arena, or a latency-critical loop where cudaMalloc (which may synchronise the
 * device) is not allowed — so they cannot pass the workspace moe_permute needs.
 * This variant takes the same inputs and outputs, with the same meaning, and
 * keeps its scratch (per-tile expert counts and their prefix sums) in a fixed
 * static device array of the library (about 0.5 MB, held on every GPU that uses
 * the library until the process exits). It allocates nothing.
 * Limit: n_experts * ceil(T / tile) <= 65536, with tile = 32 tokens for E <= 32,
 * 64 for E <= 128 and 32 above (E = 8: T <= 262144; E = 128: T <= 32768);
 * larger problems return MOE_ERR_WORKSPACE. d_model * element size must be a
 * multiple of 16 bytes.
 * All calls share the static array: calls that overlap on the GPU race, so the
 * caller must serialise them (one stream, or explicit ordering). The array's
 * address belongs to a CUDA context: the first call in each context (the device's
 * primary context, a context the caller created, or a primary context re-created
 * after a reset) looks it up with cudaGetSymbolAddress and caches it under the
 * context's ID; make that first call before any stream capture. Out-of-range expert indices are not
 * reported (there is no workspace for the error word); such a pair is treated as
 * dropped (inv = -1). */
moe_status_t moe_permute_noalloc(const moe_cfg_t *cfg, const void *x, const int32_t *topk_idx,
                                 int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv,
                                 void *x_perm, moe_stream_t stream);

/* Expert FFNs on expert-contiguous rows ("SwiGLUExpert", MLP experts).
 * Rows [offsets[e], offsets[e+1]) of x_perm [R, d] go through expert e and the
 * result is written to the same rows of y_perm [R, d] (dtype), R = T*k (token
 * choice) or E*C (expert choice). offsets is a device array [E+1]; it must be
 * non-decreasing from 0 to at most R (checked on the device: MOE_DEVERR_OFFSETS,
 * nothing computed). For the shared experts call
 * it with n_experts = 1, d_ff = n_shared*F_sh, w1/w3/w2 = ws_gate/ws_up/ws_down. */
moe_status_t moe_expert_ffn(const moe_cfg_t *cfg, const moe_weights_t *w, const void *x_perm,
                            const int32_t *offsets, void *y_perm, void *ws, size_t ws_bytes,
                            moe_stream_t stream);

/* Gate-weighted combine (the gating equation; "MoELayer" scatter-add).
 * y[t] = sum_{s: inv[t*k+s] >= 0} topk_gate[t*k+s] * y_perm[inv[t*k+s]]
 *        (+ shared_y[t] when shared_y != NULL, fp32 [T, d]); y [T, d] dtype.
 * Computed in fp32, rounded once. A token with every slot dropped gets 0 (+ shared). */
moe_status_t moe_combine(const moe_cfg_t *cfg, const void *y_perm, const int32_t *inv,
                         const float *topk_gate, const float *shared_y, void *y,
                         void *ws, size_t ws_bytes, moe_stream_t stream);

/* Load-balancing statistics ("load_balancing_loss", "compute_load_balancing_loss",
 * "router_z_loss", devtips.kr "load_balancing_loss").
 * out [3 + 2E] fp32 = { aux, z_loss, balance_sq, f[0..E), P[0..E) } with
 *   f_i = assignments to i (before drops) / (T*k), P_i = mean_t softmax(z_t)_i,
 *   aux = alpha*E*sum_i f_i P_i, z_loss = mean_t logsumexp(z_t)^2,
 *   balance_sq = sum_i (f_i - 1/E)^2. */
moe_status_t moe_aux_stats(const moe_cfg_t *cfg, const float *logits, const int32_t *topk_idx,
                           float *out, void *ws, size_t ws_bytes, moe_stream_t stream);

/* The whole layer: route, permute, expert FFNs, shared experts, combine.
 * x [T, d] and y [T, d] in dtype. aux_out (nullable) receives the moe_aux_stats
 * vector [3 + 2E]. taps (nullable) receives intermediates.
 * With cfg->routing == MOE_ROUTING_EXPERT_CHOICE: router, expert choice, gather of
 * each expert's C rows, expert FFNs, score-weighted combine; aux_out must be NULL
 * and of the taps only `logits` is filled. */
moe_status_t moe_forward(const moe_cfg_t *cfg, const moe_weights_t *w, const void *x, void *y,
                         float *aux_out, const moe_taps_t *taps, void *ws, size_t ws_bytes,
                         moe_stream_t stream);

/* A cudaEvent_t. */
typedef struct CUevent_st *moe_event_t;

/* Stages of one layer call, in launch order. Token choice: ROUTE = router GEMM,
 * softmax, top-k, gates and per-tile histogram (noisy gating: both projections and
 * the noise); SCAN = counts, capacity, offsets and the GEMM tile table; PERMUTE =
 * ranks, drops and the row gather; SHARED_FFN = the always-on experts; EXPERT_FFN =
 * the routed experts' GEMMs; COMBINE = the gate-weighted sum. Expert choice: ROUTE =
 * router and each expert's picks, SCAN = tile table, PERMUTE = row gather,
 * SHARED_FFN = nothing. */
enum {
  MOE_STAGE_ROUTE = 0,
  MOE_STAGE_SCAN = 1,
  MOE_STAGE_PERMUTE = 2,
  MOE_STAGE_SHARED_FFN = 3,
  MOE_STAGE_EXPERT_FFN = 4,
  MOE_STAGE_COMBINE = 5,
  MOE_STAGE_COUNT = 6
};

/* Events that moe_forward_staged records on `stream`: ev[i] before stage i and
 * ev[MOE_STAGE_COUNT] after the last one, so stage i's device time is the elapsed
 * time from ev[i] to ev[i + 1]. NULL entries are not recorded. The caller creates the
 * events (with timing enabled) and owns them. */
typedef struct {
  moe_event_t ev[MOE_STAGE_COUNT + 1];
} moe_stage_events_t;

/* The noise of noisy top-k gating for moe_forward_staged: the caller's draws eps
 * [T, E] fp32 (device), or, when eps is NULL, the counter-based draws for (seed,
 * offset) (see moe_noise_draws). */
typedef struct {
  const float *eps;
  uint64_t seed;
  uint64_t offset;
} moe_noise_t;

/* moe_forward (noise == NULL) or moe_forward_noisy / moe_forward_noisy_seeded (noise
 * given) that also records `events` (nullable) at its stage boundaries and marks
 * each stage with an NVTX range (named "moe_route", "moe_scan", ...). The kernels and
 * results are those of the plain entry points. The entry points launch each kernel
 * so that it may begin while the one before it finishes (programmatic dependent
 * launch); the kernel launched right after a recorded event starts after the event
 * instead, so that each timed stage is its own kernels' time. A failed event record
 * returns MOE_ERR_CUDA. */
moe_status_t moe_forward_staged(const moe_cfg_t *cfg, const moe_weights_t *w, const void *x,
                                const moe_noise_t *noise, void *y, float *aux_out,
                                const moe_taps_t *taps, const moe_stage_events_t *events,
                                void *ws, size_t ws_bytes, moe_stream_t stream);

/* Noisy top-k gating, the training mode of youngju.dev (ja) "TopKGating" (Noisy Top-K
 * Gating): the logits are z + softplus(x W_noise^T) * eps, z as in moe_route, softplus
 * the identity above 20 (as F.softplus), eps [T, E] fp32 standard normal draws made by
 * the caller (device memory); then selection and gates exactly as moe_route on those
 * logits (cfg->gate_mode; the page's mode is MOE_GATE_SOFTMAX_TOPK_RENORM). logits
 * [T, E] fp32 receives the noisy logits. Token-choice configurations only. bf16 layers
 * with at most 128 experts compute both projections in one tensor-core pass over x;
 * the others take two router passes and an elementwise step. */
moe_status_t moe_route_noisy(const moe_cfg_t *cfg, const moe_weights_t *w, const void *x,
                             const float *eps, float *logits, int32_t *topk_idx,
                             float *topk_gate, void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_forward with noisy top-k gating (see moe_route_noisy): the whole layer, routed
 * on the noisy logits; aux_out and the logits tap see the noisy logits. */
moe_status_t moe_forward_noisy(const moe_cfg_t *cfg, const moe_weights_t *w, const void *x,
                               const float *eps, void *y, float *aux_out, const moe_taps_t *taps,
                               void *ws, size_t ws_bytes, moe_stream_t stream);

/* The standard normal draws of the seeded noisy gate, for (seed, offset): eps [T, E]
 * fp32 (device) and, when raw != NULL, the generator's words raw [T, ceil(E/4), 4]
 * uint32 (device, 16-byte aligned). A pure function of (seed, offset, token, expert),
 * so calls may be repeated or split freely. Generator: Philox4x32-10 (J. K. Salmon,
 * M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel Random Numbers: As Easy as 1, 2,
 * 3", SC'11) with counter (t, e / 4, offset mod 2^32, offset >> 32) and key (seed mod
 * 2^32, seed >> 32); each output word r gives u = (2 (r >> 9) + 1) 2^-24 in (0, 1),
 * and the Box-Muller transform (rho = sqrt(-2 ln u0), rho cos 2 pi u1, rho sin 2 pi
 * u1) of words (0, 1) gives experts 4q, 4q + 1 and of words (2, 3) experts 4q + 2,
 * 4q + 3 (computed in fp32 with the device's logf, sqrtf and sincospif). A training
 * loop advances `offset` once per call: different offsets use disjoint counters. */
moe_status_t moe_noise_draws(int32_t n_tokens, int32_t n_experts, uint64_t seed,
                             uint64_t offset, float *eps, uint32_t *raw, moe_stream_t stream);

/* moe_route_noisy with the noise drawn inside the library for (seed, offset), the
 * draws of moe_noise_draws (kept in the workspace). */
moe_status_t moe_route_noisy_seeded(const moe_cfg_t *cfg, const moe_weights_t *w,
                                    const void *x, uint64_t seed, uint64_t offset,
                                    float *logits, int32_t *topk_idx, float *topk_gate,
                                    void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_forward_noisy with the noise drawn inside the library for (seed, offset). */
moe_status_t moe_forward_noisy_seeded(const moe_cfg_t *cfg, const moe_weights_t *w,
                                      const void *x, uint64_t seed, uint64_t offset, void *y,
                                      float *aux_out, const moe_taps_t *taps, void *ws,
                                      size_t ws_bytes, moe_stream_t stream);

/* Expert-Choice routing step (youngju.dev (zh) "ExpertChoiceRouter", youngju.dev (ja)
 * "ExpertChoiceGating"): logits as in moe_route, then for every expert e its C =
 * floor(cf * T / E) tokens of highest logit in descending order (equal logits: lower
 * token first; the per-expert softmax over tokens is monotone in the logit, so this
 * is the order of the scores), and their scores exp(z - m_e) / sum_t exp(z_t - m_e)
 * with m_e the expert's largest logit. A NaN logit counts as -inf.
 *   x         [T, d] dtype, or NULL: then `logits` [T, E] fp32 is the input
 *   logits    [T, E] fp32 output (input when x == NULL)
 *   ec_idx    [E, C] int32 output: token index of expert e's j-th pick
 *   ec_score  [E, C] fp32 output: its score
 * Requires cfg->routing == MOE_ROUTING_EXPERT_CHOICE (MOE_ERR_INVALID_ARG otherwise)
 * and the limits of moe_cfg_t (MOE_ERR_UNSUPPORTED beyond them). This is the pages'
 * router module (scores and indices per expert); moe_forward runs it as its first
 * step. */
moe_status_t moe_route_expert_choice(const moe_cfg_t *cfg, const moe_weights_t *w,
                                     const void *x, float *logits, int32_t *ec_idx,
                                     float *ec_score, void *ws, size_t ws_bytes,
                                     moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * Token-sharded batches. One batch of T_total tokens is split into n_shards
 * consecutive slices (shard 0 first), one per rank, with the weights replicated.
 * The pages define the layer on one batch; the entries below give each shard
 * exactly its slice of that single call's results. Tokens are independent given
 * the routing except in two places, and these entries carry both:
 *  - the capacity drop of youngju.dev (zh) "SwitchRouter" takes every expert's
 *    (token, slot) pairs in token-major order over the whole batch, with capacity
 *    floor(cf * T_total * k / E); shard r may keep max(0, cap - before_e) pairs for
 *    expert e, before_e = the pairs shards 0..r-1 routed to e before drops. So the
 *    shards first exchange their pre-drop counts [E] (an all-gather, the caller's
 *    collective) and pass them in as counts_all;
 *  - the statistics of moe_aux_stats are means over the batch: each shard emits
 *    fp64 sums, the caller adds them over the shards (a sum all-reduce), and
 *    moe_aux_finalize turns the sums into the statistics.
 * Sequence per rank: moe_route_shard -> all-gather counts, all-reduce aux_part ->
 * moe_forward_shard (or moe_permute_shard + moe_expert_ffn + moe_combine) and
 * moe_aux_finalize. Token-choice configurations only (MOE_ERR_INVALID_ARG with
 * MOE_ROUTING_EXPERT_CHOICE). cfg->n_tokens is the shard's token count. */
typedef struct {
  long long n_tokens_total;   /* tokens of the whole batch, >= cfg->n_tokens */
  int n_shards;               /* >= 1 */
  int shard;                  /* this shard's place, 0 <= shard < n_shards */
  const int32_t *counts_all;  /* device [n_shards, E] int32: every shard's pre-drop
                                 counts (moe_route_shard's `counts`), shard-major */
} moe_shard_t;

/* moe_route on this shard's tokens, plus its pre-drop counts per expert
 * (counts [E] int32, device) and, when aux_part != NULL, its fp64 sums for the
 * statistics: aux_part [1 + 2E] = { sum_t logsumexp(z_t)^2, count[0..E),
 * sum_t softmax(z_t)[0..E) } (device). x == NULL: logits is the input, as in
 * moe_route. An empty shard writes zero counts and sums. */
moe_status_t moe_route_shard(const moe_cfg_t *cfg, const moe_weights_t *w, const void *x,
                             float *logits, int32_t *topk_idx, float *topk_gate,
                             int32_t *counts, double *aux_part, void *ws, size_t ws_bytes,
                             moe_stream_t stream);

/* moe_permute for one shard: the same outputs, with the capacity of the whole batch
 * shared out as described above (counts are this shard's, before drops; offsets,
 * perm and inv index this shard's rows and tokens). */
moe_status_t moe_permute_shard(const moe_cfg_t *cfg, const moe_shard_t *shard, const void *x,
                               const int32_t *topk_idx, int32_t *counts, int32_t *offsets,
                               int32_t *perm, int32_t *inv, void *x_perm, void *ws,
                               size_t ws_bytes, moe_stream_t stream);

/* moe_forward for one shard that moe_route_shard has routed: taps->topk_idx and
 * taps->topk_gate are INPUTS (required); the other taps are outputs as in
 * moe_forward (taps->logits is not written). Permute with the shared-out capacity,
 * shared experts, expert FFNs and combine; y [n_tokens, d]. */
moe_status_t moe_forward_shard(const moe_cfg_t *cfg, const moe_shard_t *shard,
                               const moe_weights_t *w, const void *x, const moe_taps_t *taps,
                               void *y, void *ws, size_t ws_bytes, moe_stream_t stream);

/* The moe_aux_stats vector out [3 + 2E] fp32 (device) from aux_part [1 + 2E] fp64
 * summed over all shards (device), for a batch of n_tokens_total >= 1 tokens.
 * Needs no workspace. */
moe_status_t moe_aux_finalize(const moe_cfg_t *cfg, long long n_tokens_total,
                              const double *aux_part, float *out, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * Test hooks for failure detection (no counterpart on the pages). Every pipeline
 * wait inside the tensor-core kernels is bounded; a wait that runs out records
 * MOE_DEVERR_WAIT_TIMEOUT (info = the wait's site), lets the copies and MMAs the CTA
 * already issued finish, frees its tensor memory and returns, so the context stays
 * usable. These two calls make that happen on purpose, without a fault:
 * moe_test_set_wait_limit sets the bound (ns; 0 restores 2 s) of the single-CTA
 * expert GEMM's pipeline waits in launches that follow; moe_test_withhold_load makes
 * the next n_calls launches of that GEMM's up projection withhold each CTA's first
 * operand load, so its MMA issuer waits for data that never comes. Both are
 * process-wide host settings read at launch. */
moe_status_t moe_test_set_wait_limit(uint64_t ns);
moe_status_t moe_test_withhold_load(int32_t n_calls);

/* Synchronise `stream`, read and clear the sticky device error word.
 * Returns MOE_ERR_DEVICE when *code != 0, MOE_ERR_CUDA when the sync failed. */
moe_status_t moe_last_device_error(void *ws, int32_t *code, int32_t *info, moe_stream_t stream);

/* Human-readable name of a status. */
const char *moe_status_string(moe_status_t s);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */

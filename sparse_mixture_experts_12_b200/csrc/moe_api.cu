// C ABI of the MoE FFN forward: host-side validation, workspace layout and the
// launch sequence. Every step of the layer runs in this library's kernels.
#include <math.h>
#include <string.h>

#include <atomic>
#include <climits>

#include <nvtx3/nvToolsExt.h>

#include "shard.cuh"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace moe {

thread_local bool t_pdl_blocked = false;

namespace {

enum Buf {
  B_ERR, B_TILE_COUNTS, B_TILE_BASE, B_TILE_P, B_TILE_Z, B_COUNTS, B_OFFSETS, B_MPREFIX, B_SH_TBL,
  B_LOGITS, B_IDX, B_GATE, B_PERM, B_INV, B_XPERM, B_H, B_YPERM, B_SH_H, B_SH_Y, B_YPART,
  B_EC_ZT, B_EC_IDX, B_EC_SCORE, B_EC_SLOT, B_NOISE, B_CAP_E, B_EPS, B_NBUF
};

struct Layout {
  size_t off[B_NBUF];
  size_t total;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool expert_choice(const moe_cfg_t &c) { return c.routing == MOE_ROUTING_EXPERT_CHOICE; }
long long ec_picks(const moe_cfg_t &c);

// rows of the expert-contiguous buffers (x_perm, h, y_perm): T*k (token choice) or
// E*C (expert choice)
long long expert_rows(const moe_cfg_t &c) {
  return expert_choice(c) ? (long long)c.n_experts * ec_picks(c)
                          : (long long)c.n_tokens * c.top_k;
}

// tokens each expert takes under Expert-Choice routing: floor(cf * T / E)
long long ec_picks(const moe_cfg_t &c) {
  if (!(c.capacity_factor > 0.f)) return 0;
  const double v = floor((double)c.capacity_factor * (double)c.n_tokens / (double)c.n_experts);
  return v > 1e18 ? (long long)1e18 : (long long)v;
}

Layout layout_for(const moe_cfg_t &c) {
  const size_t T = (size_t)c.n_tokens, E = (size_t)c.n_experts, k = (size_t)c.top_k;
  const size_t d = (size_t)c.d_model, F = (size_t)c.d_ff;
  const size_t eb = c.dtype == MOE_DTYPE_F32 ? 4 : 2;
  const size_t NT = (size_t)ceil_div(c.n_tokens > 0 ? c.n_tokens : 1, router_bm(c.n_experts));
  const size_t Fs = (size_t)c.n_shared * (size_t)c.d_ff_shared;
  const bool ec = expert_choice(c);
  const size_t C = ec ? (size_t)ec_picks(c) : 0;
  // rows of the expert-contiguous buffers: T*k (token choice) or E*C (expert choice)
  const size_t R = ec ? E * C : T * k;
  size_t sz[B_NBUF];
  sz[B_ERR] = 4 * sizeof(int32_t);  // error code, its info, the scan's ticket, spare
  sz[B_TILE_COUNTS] = E * NT * 4;
  sz[B_TILE_BASE] = E * NT * 4;
  sz[B_TILE_P] = E * NT * 4;
  sz[B_TILE_Z] = NT * 4;
  sz[B_COUNTS] = E * 4;
  sz[B_OFFSETS] = (E + 1) * 4;
  sz[B_MPREFIX] = (E + 1) * 4;
  sz[B_SH_TBL] = 4 * 4;
  sz[B_LOGITS] = T * E * 4;
  sz[B_IDX] = T * k * 4;
  sz[B_GATE] = T * k * 4;
  sz[B_PERM] = T * k * 4;
  sz[B_INV] = T * k * 4;
  sz[B_XPERM] = R * d * eb;
  sz[B_H] = R * F * eb;
  sz[B_YPERM] = R * d * eb;
  sz[B_SH_H] = Fs ? T * Fs * eb : 0;
  sz[B_SH_Y] = Fs ? T * d * 4 : 0;
  // split-K partials of the small-batch expert GEMM (bf16, few tokens)
  sz[B_YPART] = (c.dtype == MOE_DTYPE_BF16 && T <= (size_t)kDecodeMaxRows)
                    ? ffn_decode_partial_bytes((int)(R > T ? R : T), (int)d)
                    : 0;
  sz[B_EC_ZT] = ec ? E * T * 4 : 0;
  sz[B_EC_IDX] = ec ? E * C * 4 : 0;
  sz[B_EC_SCORE] = ec ? E * C * 4 : 0;
  sz[B_EC_SLOT] = ec ? T * E * 4 : 0;
  sz[B_NOISE] = T * E * 4;  // x W_noise^T of noisy top-k gating
  sz[B_CAP_E] = E * 4;      // per-expert capacity left to one shard of a batch
  sz[B_EPS] = T * E * 4;    // the seeded noise draws of noisy top-k gating
  Layout L;
  size_t o = 0;
  for (int i = 0; i < B_NBUF; ++i) {
    L.off[i] = o;
    o += align256(sz[i]);
  }
  L.total = o;
  return L;
}

size_t layout_size(const Layout &L, Buf b) {
  return (b + 1 < B_NBUF ? L.off[b + 1] : L.total) - L.off[b];
}

template <typename P>
P *at(void *ws, const Layout &L, Buf b) {
  return reinterpret_cast<P *>(static_cast<char *>(ws) + L.off[b]);
}

// The scan's ticket word: the third word of the workspace header (after the sticky
// error code and its info), zeroed by moe_workspace_init.
unsigned *scan_ticket(void *ws, const Layout &L) {
  return reinterpret_cast<unsigned *>(at<int32_t>(ws, L, B_ERR) + 2);
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status_t check_cfg(const moe_cfg_t *c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  if (c->n_tokens < 0 || c->d_model <= 0 || c->d_ff <= 0) return MOE_ERR_INVALID_ARG;
  if (c->n_experts < 1 || c->n_experts > kMaxExperts) return MOE_ERR_INVALID_ARG;
  if (c->top_k < 1 || c->top_k > c->n_experts || c->top_k > kMaxTopK) return MOE_ERR_INVALID_ARG;
  if (c->act < MOE_ACT_RELU || c->act > MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (c->gate_mode < MOE_GATE_TOPK_SOFTMAX || c->gate_mode > MOE_GATE_SOFTMAX_TOPK_RAW)
    return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_DTYPE_F32 && c->dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
  if (!isfinite(c->capacity_factor) || !isfinite(c->aux_alpha)) return MOE_ERR_INVALID_ARG;
  if (c->n_shared < 0 || (c->n_shared > 0 && c->d_ff_shared <= 0)) return MOE_ERR_INVALID_ARG;
  if (c->routing != MOE_ROUTING_TOKEN_CHOICE && c->routing != MOE_ROUTING_EXPERT_CHOICE)
    return MOE_ERR_INVALID_ARG;
  if (expert_choice(*c)) {
    if (!(c->capacity_factor > 0.f)) return MOE_ERR_INVALID_ARG;
    const long long C = ec_picks(*c);
    if (c->n_tokens > 0 && C < 1) return MOE_ERR_INVALID_ARG;  // every expert takes a token
    if (C > c->n_tokens) return MOE_ERR_INVALID_ARG;           // cf > E: more picks than tokens
    if (c->n_tokens > kEcMaxTokens || C > kEcMaxPicks || c->n_shared > 0)
      return MOE_ERR_UNSUPPORTED;
  }
  const long long rows = expert_choice(*c) ? (long long)c->n_experts * ec_picks(*c)
                                           : (long long)c->n_tokens * c->top_k;
  if (rows > INT_MAX / 2) return MOE_ERR_UNSUPPORTED;
  const long long fs = (long long)c->n_shared * c->d_ff_shared;
  if (fs > INT_MAX / 2 || c->d_model > INT_MAX / 4 || c->d_ff > INT_MAX / 4)
    return MOE_ERR_UNSUPPORTED;
  if (c->dtype == MOE_DTYPE_BF16) {
    if (c->d_model % 64 || c->d_ff % 64 || fs % 64) return MOE_ERR_UNSUPPORTED;
    if ((long long)c->n_experts * c->d_ff > INT_MAX || (long long)c->n_experts * c->d_model > INT_MAX)
      return MOE_ERR_UNSUPPORTED;
  } else {
    if (c->d_model % 4) return MOE_ERR_UNSUPPORTED;
    // the fp32 path launches one CTA row per 128-row tile (grid.y limit)
    if (rows / kRowTile + c->n_experts + 1 > 65535 || c->n_tokens / kRowTile + 2 > 65535)
      return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

moe_status_t check_ws(const moe_cfg_t *c, const void *ws, size_t ws_bytes) {
  if (ws == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_MISALIGNED;
  if (ws_bytes < layout_for(*c).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// every pointer in the list: non-null required unless allowed, 16-byte aligned
moe_status_t check_ptrs(std::initializer_list<std::pair<const void *, bool>> ps) {
  for (auto &p : ps) {
    if (p.first == nullptr) {
      if (p.second) return MOE_ERR_INVALID_ARG;
      continue;
    }
    if (!aligned(p.first, 16)) return MOE_ERR_MISALIGNED;
  }
  return MOE_OK;
}

moe_status_t check_expert_weights(const moe_cfg_t *c, const moe_weights_t *w) {
  if (w == nullptr) return MOE_ERR_INVALID_ARG;
  const bool swiglu = c->act == MOE_ACT_SWIGLU;
  if (swiglu && (w->b1 || w->b2)) return MOE_ERR_INVALID_ARG;  // SwiGLU experts have no bias
  if (!swiglu && w->w3) return MOE_ERR_INVALID_ARG;
  return check_ptrs({{w->w1, true}, {w->w2, true}, {w->w3, swiglu}, {w->b1, false},
                     {w->b2, false}});
}

moe_status_t check_shared_weights(const moe_cfg_t *c, const moe_weights_t *w) {
  const bool need = c->n_shared > 0;
  if (!need) return MOE_OK;
  return check_ptrs({{w->ws_gate, true}, {w->ws_up, true}, {w->ws_down, true}});
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                        \
  do {                                       \
    moe_status_t s_ = (expr);                \
    if (s_ != MOE_OK) return s_;             \
  } while (0)
#define MOE_CUDA(expr) MOE_TRY(cuda_status(expr))

// Stage boundaries of one layer call: an event (when the caller gave one) and an
// NVTX range per stage. Stages are entered in increasing order; skipped stages
// still record their event, so every interval is defined.
class Stages {
 public:
  Stages(const moe_stage_events_t *ev, cudaStream_t st) : ev_(ev), st_(st) {}
  ~Stages() {
    if (open_) nvtxRangePop();
  }
  moe_status_t enter(int stage) {
    static const char *kNames[MOE_STAGE_COUNT] = {"moe_route", "moe_scan", "moe_permute",
                                                  "moe_shared_ffn", "moe_expert_ffn",
                                                  "moe_combine"};
    for (; next_ <= stage; ++next_) MOE_TRY(record(next_));
    if (open_) nvtxRangePop();
    nvtxRangePushA(kNames[stage]);
    open_ = true;
    return MOE_OK;
  }
  moe_status_t finish() {
    for (; next_ <= MOE_STAGE_COUNT; ++next_) MOE_TRY(record(next_));
    if (open_) nvtxRangePop();
    open_ = false;
    t_pdl_blocked = false;  // a flag left by the last event stays in this call
    return MOE_OK;
  }

 private:
  moe_status_t record(int i) {
    if (ev_ == nullptr || ev_->ev[i] == nullptr) return MOE_OK;
    t_pdl_blocked = true;  // the kernel after the event starts after it
    return cuda_status(cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev_->ev[i]), st_));
  }
  const moe_stage_events_t *ev_;
  cudaStream_t st_;
  int next_ = 0;
  bool open_ = false;
};

int capacity_of(const moe_cfg_t &c) {
  if (!(c.capacity_factor > 0.f)) return -1;
  const double cap = floor((double)c.capacity_factor * (double)c.n_tokens * (double)c.top_k /
                           (double)c.n_experts);
  return cap > (double)INT_MAX ? INT_MAX : (int)cap;
}

// capacity of a batch of n_tokens tokens: floor(cf * n_tokens * k / E), -1 = unlimited
int capacity_for_tokens(const moe_cfg_t &c, long long n_tokens) {
  if (!(c.capacity_factor > 0.f)) return -1;
  const double cap = floor((double)c.capacity_factor * (double)n_tokens * (double)c.top_k /
                           (double)c.n_experts);
  return cap > (double)INT_MAX ? INT_MAX : (int)cap;
}

// One shard of a token-sharded batch (see moe_shard_t).
moe_status_t check_shard(const moe_cfg_t &c, const moe_shard_t *sh) {
  if (sh == nullptr) return MOE_ERR_INVALID_ARG;
  if (sh->n_shards < 1 || sh->shard < 0 || sh->shard >= sh->n_shards) return MOE_ERR_INVALID_ARG;
  if (sh->n_tokens_total < c.n_tokens) return MOE_ERR_INVALID_ARG;
  if (sh->counts_all == nullptr) return MOE_ERR_INVALID_ARG;
  if (expert_choice(c)) return MOE_ERR_INVALID_ARG;  // picks are per expert over all tokens
  return MOE_OK;
}

int m_tiles_ub(long long rows, int groups) {
  long long ub = ceil_div((int)rows, kRowTile) + groups;
  if (ub > rows) ub = rows;
  return (int)ub;
}

// Process-wide test settings of the single-CTA tensor-core GEMM (see
// moe_test_set_wait_limit and moe_test_withhold_load).
std::atomic<uint64_t> g_wait_limit_ns{0};
std::atomic<int> g_withhold_loads{0};

cudaError_t run_ffn(const moe_cfg_t &c, GroupedFfnArgs a, cudaStream_t st) {
  if (c.dtype == MOE_DTYPE_F32) return launch_ffn_simt(a, st);
  a.wait_limit_ns = g_wait_limit_ns.load();
  // the test hook is taken by the next call that reaches the single-CTA kernel path
  if (a.max_group_rows > kDecodeMaxRows && g_withhold_loads.load() > 0) {
    int n = g_withhold_loads.load();
    while (n > 0 && !g_withhold_loads.compare_exchange_weak(n, n - 1)) {
    }
    a.withhold_load = n > 0 ? 1 : 0;
  }
  // few rows in any group: stream the weights with the tokens on the MMA's N side
  if (a.max_group_rows <= kDecodeMaxRows) return launch_ffn_tc_decode(a, st);
  return launch_ffn_tc(a, st);
}

GroupedFfnArgs routed_ffn_args(const moe_cfg_t &c, const moe_weights_t &w, const void *x_perm,
                               const int32_t *offsets, const int32_t *mprefix, void *h,
                               void *y_perm, int32_t *err, int max_group_rows, float *part) {
  GroupedFfnArgs a{};
  a.max_group_rows = max_group_rows;
  a.part = part;
  a.a = x_perm;
  a.a_rows = (int)expert_rows(c);
  a.offsets = offsets;
  a.mprefix = mprefix;
  a.G = c.n_experts;
  a.m_tiles_ub = m_tiles_ub(a.a_rows, c.n_experts);
  a.d = c.d_model;
  a.F = c.d_ff;
  a.act = c.act;
  a.w1 = w.w1;
  a.w3 = w.w3;
  a.w2 = w.w2;
  a.b1 = w.b1;
  a.b2 = w.b2;
  a.h = h;
  a.out = y_perm;
  a.out_f32 = 0;
  a.err = err;
  return a;
}

// Noisy top-k gating logits: z (router, biases) + softplus(x W_noise^T) * eps, into
// `logits`; the two router passes' own selections go to scratch.
moe_status_t noisy_logits(const moe_cfg_t &c, const moe_weights_t *w, const void *x,
                          const float *eps, float *logits, void *ws, const Layout &L,
                          cudaStream_t stream) {
  RouterArgs r{};
  r.x = x;
  r.w = w->w_router;
  r.b_router = w->b_router;
  r.logit_bias = w->logit_bias;
  r.logits_out = logits;
  r.topk_idx = at<int32_t>(ws, L, B_IDX);
  r.topk_gate = at<float>(ws, L, B_GATE);
  r.T = c.n_tokens;
  r.d = c.d_model;
  r.E = c.n_experts;
  r.k = c.top_k;
  r.gate_mode = c.gate_mode;
  r.err = at<int32_t>(ws, L, B_ERR);
  MOE_CUDA(launch_router(r, c.dtype, stream));
  float *zn = at<float>(ws, L, B_NOISE);
  r.w = w->w_noise;
  r.b_router = nullptr;
  r.logit_bias = nullptr;
  r.logits_out = zn;
  MOE_CUDA(launch_router(r, c.dtype, stream));
  MOE_CUDA(launch_noisy_logits(logits, zn, eps, (size_t)c.n_tokens * c.n_experts, stream));
  return MOE_OK;
}

// The noise of noisy top-k gating: the caller's draws, or the counter-based draws
// for (seed, offset).
struct NoiseSpec {
  const float *eps;  // [T, E] or nullptr: draw from (seed, offset)
  uint64_t seed, offset;
};

// Noisy routing: r carries the selection outputs (topk_idx, topk_gate, the per-tile
// partials, logits_out = the noisy-logits tap or nullptr). For bf16 layers with at
// most 128 experts one tensor-core pass computes both projections and the noisy
// logits and selects on them; otherwise the noisy logits go to logits_buf by two
// router passes and an elementwise kernel, and a second pass selects on them.
moe_status_t route_noisy(const moe_cfg_t &c, const moe_weights_t *w, const void *x,
                         const NoiseSpec &ns, RouterArgs r, float *logits_buf, void *ws,
                         const Layout &L, cudaStream_t stream) {
  const float *eps = ns.eps;
  if (eps == nullptr) {
    float *draws = at<float>(ws, L, B_EPS);
    MOE_CUDA(launch_noise_draws(c.n_tokens, c.n_experts, ns.seed, ns.offset, draws, nullptr,
                                stream));
    eps = draws;
  }
  RouterArgs f = r;
  f.x = x;
  f.w = w->w_router;
  f.b_router = w->b_router;
  f.logit_bias = w->logit_bias;
  f.logits_in = nullptr;
  f.w_noise = w->w_noise;
  f.eps = eps;
  if (c.dtype == MOE_DTYPE_BF16 && router_tc_supported(f)) {
    MOE_CUDA(launch_router(f, c.dtype, stream));
    return MOE_OK;
  }
  MOE_TRY(noisy_logits(c, w, x, eps, logits_buf, ws, L, stream));
  RouterArgs sel = r;
  sel.x = nullptr;
  sel.logits_in = logits_buf;
  sel.logits_out = nullptr;
  MOE_CUDA(launch_router(sel, c.dtype, stream));
  return MOE_OK;
}

// Expert-Choice routing: router logits (unless x is NULL: logits are the input),
// then every expert's picks. slot/offsets (nullable) feed the forward's later steps.
moe_status_t ec_route(const moe_cfg_t &c, const moe_weights_t *w, const void *x, float *logits,
                      int32_t *ec_idx, float *ec_score, int32_t *slot, int32_t *offsets,
                      void *ws, const Layout &L, cudaStream_t stream) {
  if (x != nullptr) {
    RouterArgs r{};
    r.x = x;
    r.w = w->w_router;
    r.b_router = w->b_router;
    r.logit_bias = w->logit_bias;
    r.logits_out = logits;
    r.topk_idx = at<int32_t>(ws, L, B_IDX);  // the router's own top-1, not used here
    r.topk_gate = at<float>(ws, L, B_GATE);
    r.T = c.n_tokens;
    r.d = c.d_model;
    r.E = c.n_experts;
    r.k = 1;
    r.gate_mode = MOE_GATE_TOPK_SOFTMAX;
    r.err = at<int32_t>(ws, L, B_ERR);
    MOE_CUDA(launch_router(r, c.dtype, stream));
  }
  if (slot != nullptr)
    MOE_CUDA(cudaMemsetAsync(slot, 0xFF, (size_t)c.n_tokens * c.n_experts * sizeof(int32_t),
                             stream));
  EcArgs a{};
  a.logits = logits;
  a.zt = at<float>(ws, L, B_EC_ZT);
  a.ec_idx = ec_idx;
  a.ec_score = ec_score;
  a.slot = slot;
  a.offsets = offsets;
  a.T = c.n_tokens;
  a.E = c.n_experts;
  a.C = (int)ec_picks(c);
  a.err = at<int32_t>(ws, L, B_ERR);
  MOE_CUDA(launch_ec_route(a, stream));
  return MOE_OK;
}

// Expert-Choice forward: route, gather each expert's C rows, expert FFNs, combine.
moe_status_t ec_forward(const moe_cfg_t &c, const moe_weights_t *w, const void *x, void *y,
                        float *logits, void *ws, const Layout &L, cudaStream_t stream,
                        Stages &sg) {
  const int T = c.n_tokens, E = c.n_experts, C = (int)ec_picks(c);
  int32_t *err = at<int32_t>(ws, L, B_ERR);
  int32_t *ec_idx = at<int32_t>(ws, L, B_EC_IDX);
  float *ec_score = at<float>(ws, L, B_EC_SCORE);
  int32_t *slot = at<int32_t>(ws, L, B_EC_SLOT);
  int32_t *offsets = at<int32_t>(ws, L, B_OFFSETS);
  int32_t *mprefix = at<int32_t>(ws, L, B_MPREFIX);
  MOE_TRY(sg.enter(MOE_STAGE_ROUTE));
  MOE_TRY(ec_route(c, w, x, logits, ec_idx, ec_score, slot, offsets, ws, L, stream));
  const int eb = c.dtype == MOE_DTYPE_F32 ? 4 : 2;
  void *x_perm = at<void>(ws, L, B_XPERM);
  void *y_perm = at<void>(ws, L, B_YPERM);
  MOE_TRY(sg.enter(MOE_STAGE_SCAN));
  MOE_CUDA(launch_tile_table(offsets, E, E * C, mprefix, err, stream));
  MOE_TRY(sg.enter(MOE_STAGE_PERMUTE));
  MOE_CUDA(launch_ec_gather(x, T, ec_idx, E * C, c.d_model * eb, x_perm, stream));
  float *part = layout_size(L, B_YPART) > 0 ? at<float>(ws, L, B_YPART) : nullptr;
  GroupedFfnArgs a = routed_ffn_args(c, *w, x_perm, offsets, mprefix, at<void>(ws, L, B_H),
                                     y_perm, err, C, part);  // E*C rows, C per expert
  MOE_TRY(sg.enter(MOE_STAGE_EXPERT_FFN));
  MOE_CUDA(run_ffn(c, a, stream));
  MOE_TRY(sg.enter(MOE_STAGE_COMBINE));
  MOE_CUDA(launch_ec_combine(y_perm, slot, ec_score, T, E, C, c.d_model, c.dtype, y, stream));
  return sg.finish();
}

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API moe_status_t moe_workspace_size(const moe_cfg_t *cfg, size_t *bytes) {
  MOE_TRY(check_cfg(cfg));
  if (bytes == nullptr) return MOE_ERR_INVALID_ARG;
  *bytes = layout_for(*cfg).total;
  return MOE_OK;
}

MOE_API moe_status_t moe_workspace_init(void *ws, size_t ws_bytes, moe_stream_t stream) {
  if (ws == nullptr || ws_bytes < 256) return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_MISALIGNED;
  MOE_CUDA(cudaMemsetAsync(ws, 0, 256, stream));
  return MOE_OK;
}

MOE_API moe_status_t moe_route(const moe_cfg_t *cfg, const moe_weights_t *w, const void *x,
                               float *logits, int32_t *topk_idx, float *topk_gate, void *ws,
                               size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  if (cfg->n_tokens == 0) return MOE_OK;
  if (w == nullptr) return MOE_ERR_INVALID_ARG;
  if (x != nullptr) {
    MOE_TRY(check_ptrs({{x, true}, {w->w_router, true}, {logits, false}}));
  } else {
    MOE_TRY(check_ptrs({{logits, true}}));
  }
  MOE_TRY(check_ptrs({{topk_idx, true}, {topk_gate, true}, {w->b_router, false},
                      {w->logit_bias, false}}));
  const moe_cfg_t &c = *cfg;
  const Layout L = layout_for(c);
  RouterArgs r{};
  r.x = x;
  r.w = w->w_router;
  r.b_router = w->b_router;
  r.logit_bias = w->logit_bias;
  r.logits_in = x ? nullptr : logits;
  r.logits_out = x ? logits : nullptr;
  r.topk_idx = topk_idx;
  r.topk_gate = topk_gate;
  r.tile_counts = at<int32_t>(ws, L, B_TILE_COUNTS);
  r.T = c.n_tokens;
  r.d = c.d_model;
  r.E = c.n_experts;
  r.k = c.top_k;
  r.gate_mode = c.gate_mode;
  r.err = at<int32_t>(ws, L, B_ERR);
  MOE_CUDA(launch_router(r, c.dtype, stream));
  return MOE_OK;
}

namespace moe {
namespace {
moe_status_t route_noisy_entry(const moe_cfg_t *cfg, const moe_weights_t *w, const void *x,
                               const NoiseSpec &ns, float *logits, int32_t *topk_idx,
                               float *topk_gate, void *ws, size_t ws_bytes, cudaStream_t stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  if (expert_choice(*cfg)) return MOE_ERR_INVALID_ARG;
  if (cfg->n_tokens == 0) return MOE_OK;
  if (w == nullptr) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ptrs({{x, true}, {logits, true}, {topk_idx, true}, {topk_gate, true},
                      {w->w_router, true}, {w->w_noise, true}, {w->b_router, false},
                      {w->logit_bias, false}}));
  const moe_cfg_t &c = *cfg;
  const Layout L = layout_for(c);
  RouterArgs r{};
  r.logits_out = logits;
  r.topk_idx = topk_idx;
  r.topk_gate = topk_gate;
  r.tile_counts = at<int32_t>(ws, L, B_TILE_COUNTS);
  r.T = c.n_tokens;
  r.d = c.d_model;
  r.E = c.n_experts;
  r.k = c.top_k;
  r.gate_mode = c.gate_mode;
  r.err = at<int32_t>(ws, L, B_ERR);
  return route_noisy(c, w, x, ns, r, logits, ws, L, stream);
}
}  // namespace
}  // namespace moe

MOE_API moe_status_t moe_route_noisy(const moe_cfg_t *cfg, const moe_weights_t *w,
                                     const void *x, const float *eps, float *logits,
                                     int32_t *topk_idx, float *topk_gate, void *ws,
                                     size_t ws_bytes, moe_stream_t stream) {
  if (eps == nullptr) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ptrs({{eps, true}}));
  return route_noisy_entry(cfg, w, x, NoiseSpec{eps, 0, 0}, logits, topk_idx, topk_gate, ws,
                           ws_bytes, stream);
}

MOE_API moe_status_t moe_route_noisy_seeded(const moe_cfg_t *cfg, const moe_weights_t *w,
                                            const void *x, uint64_t seed, uint64_t offset,
                                            float *logits, int32_t *topk_idx, float *topk_gate,
                                            void *ws, size_t ws_bytes, moe_stream_t stream) {
  return route_noisy_entry(cfg, w, x, NoiseSpec{nullptr, seed, offset}, logits, topk_idx,
                           topk_gate, ws, ws_bytes, stream);
}

MOE_API moe_status_t moe_noise_draws(int32_t n_tokens, int32_t n_experts, uint64_t seed,
                                     uint64_t offset, float *eps, uint32_t *raw,
                                     moe_stream_t stream) {
  if (n_tokens < 0 || n_experts < 1 || n_experts > kMaxExperts) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ptrs({{eps, true}, {raw, false}}));
  MOE_CUDA(launch_noise_draws(n_tokens, n_experts, seed, offset, eps, raw, stream));
  return MOE_OK;
}

MOE_API moe_status_t moe_route_expert_choice(const moe_cfg_t *cfg, const moe_weights_t *w,
                                             const void *x, float *logits, int32_t *ec_idx,
                                             float *ec_score, void *ws, size_t ws_bytes,
                                             moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  if (!expert_choice(*cfg)) return MOE_ERR_INVALID_ARG;
  if (cfg->n_tokens == 0) return MOE_OK;
  if (x != nullptr) {
    if (w == nullptr) return MOE_ERR_INVALID_ARG;
    MOE_TRY(check_ptrs({{x, true}, {w->w_router, true}, {w->b_router, false},
                        {w->logit_bias, false}}));
  }
  MOE_TRY(check_ptrs({{logits, true}, {ec_idx, true}, {ec_score, true}}));
  const Layout L = layout_for(*cfg);
  return ec_route(*cfg, w, x, logits, ec_idx, ec_score, nullptr, nullptr, ws, L, stream);
}

MOE_API moe_status_t moe_permute(const moe_cfg_t *cfg, const void *x, const int32_t *topk_idx,
                                 int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv,
                                 void *x_perm, void *ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_TRY(check_ptrs({{x, true}, {topk_idx, true}, {counts, true}, {offsets, true}, {perm, true},
                      {inv, true}, {x_perm, true}}));
  const moe_cfg_t &c = *cfg;
  if (c.n_tokens == 0) {
    MOE_CUDA(cudaMemsetAsync(counts, 0, sizeof(int32_t) * c.n_experts, stream));
    MOE_CUDA(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (c.n_experts + 1), stream));
    return MOE_OK;
  }
  const Layout L = layout_for(c);
  int32_t *err = at<int32_t>(ws, L, B_ERR);
  int32_t *tile_counts = at<int32_t>(ws, L, B_TILE_COUNTS);
  MOE_CUDA(launch_tile_counts(topk_idx, c.n_tokens, c.top_k, c.n_experts, tile_counts, err, stream));
  ScanArgs s{};
  s.ticket = scan_ticket(ws, L);
  s.tile_counts = tile_counts;
  s.tile_base = at<int32_t>(ws, L, B_TILE_BASE);
  s.counts = counts;
  s.offsets = offsets;
  s.mprefix = at<int32_t>(ws, L, B_MPREFIX);
  s.E = c.n_experts;
  s.NT = ceil_div(c.n_tokens, router_bm(c.n_experts));
  s.cap = capacity_of(c);
  s.T = c.n_tokens;
  s.k = c.top_k;
  MOE_CUDA(launch_scan(s, stream));
  ScatterArgs p{};
  p.x = x;
  p.topk_idx = topk_idx;
  p.tile_base = s.tile_base;
  p.offsets = offsets;
  p.perm = perm;
  p.inv = inv;
  p.x_perm = x_perm;
  p.T = c.n_tokens;
  p.d = c.d_model;
  p.E = c.n_experts;
  p.k = c.top_k;
  p.cap = s.cap;
  p.elem_bytes = c.dtype == MOE_DTYPE_F32 ? 4 : 2;
  p.err = err;
  MOE_CUDA(launch_scatter(p, stream));
  return MOE_OK;
}

MOE_API moe_status_t moe_expert_ffn(const moe_cfg_t *cfg, const moe_weights_t *w,
                                    const void *x_perm, const int32_t *offsets, void *y_perm,
                                    void *ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  if (cfg->n_tokens == 0) return MOE_OK;
  MOE_TRY(check_expert_weights(cfg, w));
  MOE_TRY(check_ptrs({{x_perm, true}, {offsets, true}, {y_perm, true}}));
  const moe_cfg_t &c = *cfg;
  const Layout L = layout_for(c);
  int32_t *err = at<int32_t>(ws, L, B_ERR);
  int32_t *mprefix = at<int32_t>(ws, L, B_MPREFIX);
  const int rows = (int)expert_rows(c);
  MOE_CUDA(launch_tile_table(offsets, c.n_experts, rows, mprefix, err, stream));
  GroupedFfnArgs a = routed_ffn_args(c, *w, x_perm, offsets, mprefix, at<void>(ws, L, B_H),
                                     y_perm, err, rows,
                                     layout_size(L, B_YPART) > 0 ? at<float>(ws, L, B_YPART) : nullptr);
  MOE_CUDA(run_ffn(c, a, stream));
  return MOE_OK;
}

MOE_API moe_status_t moe_combine(const moe_cfg_t *cfg, const void *y_perm, const int32_t *inv,
                                 const float *topk_gate, const float *shared_y, void *y,
                                 void *ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  if (cfg->n_tokens == 0) return MOE_OK;
  MOE_TRY(check_ptrs({{y_perm, true}, {inv, true}, {topk_gate, true}, {shared_y, false},
                      {y, true}}));
  const moe_cfg_t &c = *cfg;
  const Layout L = layout_for(c);
  CombineArgs a{};
  a.y_perm = y_perm;
  a.inv = inv;
  a.gate = topk_gate;
  a.shared_y = shared_y;
  a.y = y;
  a.T = c.n_tokens;
  a.d = c.d_model;
  a.k = c.top_k;
  a.R = c.n_tokens * c.top_k;
  a.err = at<int32_t>(ws, L, B_ERR);
  MOE_CUDA(launch_combine(a, c.dtype, stream));
  return MOE_OK;
}

MOE_API moe_status_t moe_aux_stats(const moe_cfg_t *cfg, const float *logits,
                                   const int32_t *topk_idx, float *out, void *ws, size_t ws_bytes,
                                   moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_TRY(check_ptrs({{logits, true}, {topk_idx, true}, {out, true}}));
  const moe_cfg_t &c = *cfg;
  if (c.n_tokens == 0) return MOE_ERR_INVALID_ARG;  // the statistics are means over tokens
  const Layout L = layout_for(c);
  int32_t *err = at<int32_t>(ws, L, B_ERR);
  // softmax partial sums from the given logits (selection outputs go to scratch)
  RouterArgs r{};
  r.logits_in = logits;
  r.topk_idx = at<int32_t>(ws, L, B_IDX);
  r.topk_gate = at<float>(ws, L, B_GATE);
  r.tile_p = at<float>(ws, L, B_TILE_P);
  r.tile_z = at<float>(ws, L, B_TILE_Z);
  r.T = c.n_tokens;
  r.d = c.d_model;
  r.E = c.n_experts;
  r.k = c.top_k;
  r.gate_mode = c.gate_mode;
  r.err = err;
  MOE_CUDA(launch_router(r, c.dtype, stream));
  int32_t *tile_counts = at<int32_t>(ws, L, B_TILE_COUNTS);
  MOE_CUDA(launch_tile_counts(topk_idx, c.n_tokens, c.top_k, c.n_experts, tile_counts, err, stream));
  ScanArgs s{};
  s.ticket = scan_ticket(ws, L);
  s.tile_counts = tile_counts;
  s.tile_base = at<int32_t>(ws, L, B_TILE_BASE);
  s.counts = at<int32_t>(ws, L, B_COUNTS);
  s.offsets = at<int32_t>(ws, L, B_OFFSETS);
  s.mprefix = at<int32_t>(ws, L, B_MPREFIX);
  s.E = c.n_experts;
  s.NT = ceil_div(c.n_tokens, router_bm(c.n_experts));
  s.cap = -1;
  s.tile_p = r.tile_p;
  s.tile_z = r.tile_z;
  s.aux_out = out;
  s.T = c.n_tokens;
  s.k = c.top_k;
  s.alpha = c.aux_alpha;
  MOE_CUDA(launch_scan(s, stream));
  return MOE_OK;
}

namespace moe {
namespace {
// the whole layer; noise != NULL: noisy top-k gating (token choice only)
// sh != NULL: one shard of a token-sharded batch, routed already (topk_idx and
// topk_gate in taps, the capacity of the whole batch shared out per expert)
moe_status_t forward_impl(const moe_cfg_t *cfg, const moe_weights_t *w, const void *x,
                          const NoiseSpec *noise, void *y, float *aux_out, const moe_taps_t *taps,
                          void *ws, size_t ws_bytes, moe_stream_t stream,
                          const moe_shard_t *sh = nullptr,
                          const moe_stage_events_t *events = nullptr) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  if (sh != nullptr) {
    MOE_TRY(check_shard(*cfg, sh));
    if (aux_out != nullptr || noise != nullptr) return MOE_ERR_INVALID_ARG;
    if (cfg->n_tokens > 0 &&
        (taps == nullptr || taps->topk_idx == nullptr || taps->topk_gate == nullptr))
      return MOE_ERR_INVALID_ARG;
  }
  Stages sg(events, stream);
  if (cfg->n_tokens == 0) return sg.finish();  // nothing is read or written
  if (w == nullptr) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ptrs({{x, true}, {y, true}, {aux_out, false}, {w->w_router, sh == nullptr},
                      {w->b_router, false}, {w->logit_bias, false}}));
  MOE_TRY(check_expert_weights(cfg, w));
  MOE_TRY(check_shared_weights(cfg, w));
  moe_taps_t tp{};
  if (taps) {
    tp = *taps;
    MOE_TRY(check_ptrs({{tp.logits, false}, {tp.topk_idx, false}, {tp.topk_gate, false},
                        {tp.counts, false}, {tp.offsets, false}, {tp.perm, false},
                        {tp.inv, false}}));
  }
  const moe_cfg_t &c = *cfg;
  const Layout L = layout_for(c);
  int32_t *err = at<int32_t>(ws, L, B_ERR);
  float *logits = tp.logits ? tp.logits : at<float>(ws, L, B_LOGITS);
  if (expert_choice(c)) {
    if (aux_out != nullptr || noise != nullptr) return MOE_ERR_INVALID_ARG;
    return ec_forward(c, w, x, y, logits, ws, L, stream, sg);
  }
  if (noise != nullptr) MOE_TRY(check_ptrs({{noise->eps, false}, {w->w_noise, true}}));
  int32_t *idx = tp.topk_idx ? tp.topk_idx : at<int32_t>(ws, L, B_IDX);
  float *gate = tp.topk_gate ? tp.topk_gate : at<float>(ws, L, B_GATE);
  int32_t *counts = tp.counts ? tp.counts : at<int32_t>(ws, L, B_COUNTS);
  int32_t *offsets = tp.offsets ? tp.offsets : at<int32_t>(ws, L, B_OFFSETS);
  int32_t *perm = tp.perm ? tp.perm : at<int32_t>(ws, L, B_PERM);
  int32_t *inv = tp.inv ? tp.inv : at<int32_t>(ws, L, B_INV);
  int32_t *mprefix = at<int32_t>(ws, L, B_MPREFIX);
  int32_t *sh_tbl = at<int32_t>(ws, L, B_SH_TBL);
  const bool want_aux = aux_out != nullptr;

  // 1. router GEMM + softmax + top-k + gates + per-tile histogram (noisy gating:
  //    on z + softplus(x W_noise^T) * eps)
  MOE_TRY(sg.enter(MOE_STAGE_ROUTE));
  RouterArgs r{};
  if (noise == nullptr) {
    r.x = x;
    r.w = w->w_router;
    r.b_router = w->b_router;
    r.logit_bias = w->logit_bias;
  }
  r.logits_out = tp.logits;  // the statistics come from the router's own partial sums
  r.topk_idx = idx;
  r.topk_gate = gate;
  r.tile_counts = at<int32_t>(ws, L, B_TILE_COUNTS);
  r.tile_p = want_aux ? at<float>(ws, L, B_TILE_P) : nullptr;
  r.tile_z = want_aux ? at<float>(ws, L, B_TILE_Z) : nullptr;
  r.T = c.n_tokens;
  r.d = c.d_model;
  r.E = c.n_experts;
  r.k = c.top_k;
  r.gate_mode = c.gate_mode;
  r.err = err;
  // decode-sized batches: the router also lays out the experts (no scan kernel)
  const bool small = noise == nullptr && sh == nullptr && c.dtype == MOE_DTYPE_BF16 &&
                     small_route_supported(r);
  if (small) {
    SmallRouteArgs sr{};
    sr.r = r;
    sr.cap = capacity_of(c);
    sr.counts = counts;
    sr.offsets = offsets;
    sr.mprefix = mprefix;
    sr.tile_base = at<int32_t>(ws, L, B_TILE_BASE);
    sr.sh_tbl = c.n_shared > 0 ? sh_tbl : nullptr;
    MOE_CUDA(launch_route_small(sr, stream));
  } else if (noise != nullptr) {
    MOE_TRY(route_noisy(c, w, x, *noise, r, logits, ws, L, stream));
  } else if (sh == nullptr) {
    MOE_CUDA(launch_router(r, c.dtype, stream));
  } else {  // routed by the caller: only the per-tile histogram
    MOE_CUDA(launch_tile_counts(idx, c.n_tokens, c.top_k, c.n_experts, r.tile_counts, err,
                                stream));
  }
  // 2. scan: counts, capacity, offsets, GEMM tile table (+ aux statistics)
  MOE_TRY(sg.enter(MOE_STAGE_SCAN));
  ScanArgs s{};
  s.ticket = scan_ticket(ws, L);
  s.tile_counts = r.tile_counts;
  s.tile_base = at<int32_t>(ws, L, B_TILE_BASE);
  s.counts = counts;
  s.offsets = offsets;
  s.mprefix = mprefix;
  s.E = c.n_experts;
  s.NT = ceil_div(c.n_tokens, router_bm(c.n_experts));
  s.cap = capacity_of(c);
  s.tile_p = r.tile_p;
  s.tile_z = r.tile_z;
  s.aux_out = aux_out;
  s.T = c.n_tokens;
  s.k = c.top_k;
  s.alpha = c.aux_alpha;
  s.sh_tbl = c.n_shared > 0 ? sh_tbl : nullptr;
  ShardCaps sc{};
  if (small) {
    // laid out by the router
  } else if (sh == nullptr) {
    MOE_CUDA(launch_scan(s, stream));
  } else {
    s.cap = capacity_for_tokens(c, sh->n_tokens_total);
    sc = ShardCaps{sh->counts_all, at<int32_t>(ws, L, B_CAP_E), sh->n_shards, sh->shard};
    MOE_CUDA(launch_scan_shard(s, sc, stream));
  }
  // 3. stable permutation with capacity drops + row gather
  MOE_TRY(sg.enter(MOE_STAGE_PERMUTE));
  ScatterArgs p{};
  p.x = x;
  p.topk_idx = idx;
  p.tile_base = s.tile_base;
  p.offsets = offsets;
  p.perm = perm;
  p.inv = inv;
  p.x_perm = at<void>(ws, L, B_XPERM);
  p.T = c.n_tokens;
  p.d = c.d_model;
  p.E = c.n_experts;
  p.k = c.top_k;
  p.cap = s.cap;
  p.elem_bytes = c.dtype == MOE_DTYPE_F32 ? 4 : 2;
  p.err = err;
  if (sh == nullptr) MOE_CUDA(launch_scatter(p, stream));
  else MOE_CUDA(launch_scatter_shard(p, sc.cap_e, stream));
  // 4. always-on shared experts: one SwiGLU over all tokens, experts concatenated along F
  float *sh_y = nullptr;
  float *part = layout_size(L, B_YPART) > 0 ? at<float>(ws, L, B_YPART) : nullptr;
  MOE_TRY(sg.enter(MOE_STAGE_SHARED_FFN));
  if (c.n_shared > 0) {
    GroupedFfnArgs a{};
    a.a = x;
    a.a_rows = c.n_tokens;
    a.offsets = sh_tbl;
    a.mprefix = sh_tbl + 2;
    a.G = 1;
    a.m_tiles_ub = ceil_div(c.n_tokens, kRowTile);
    a.d = c.d_model;
    a.F = c.n_shared * c.d_ff_shared;
    a.act = MOE_ACT_SWIGLU;
    a.w1 = w->ws_gate;
    a.w3 = w->ws_up;
    a.w2 = w->ws_down;
    a.h = at<void>(ws, L, B_SH_H);
    sh_y = at<float>(ws, L, B_SH_Y);
    a.out = sh_y;
    a.out_f32 = 1;
    a.max_group_rows = c.n_tokens;
    a.part = part;
    a.err = err;
    MOE_CUDA(run_ffn(c, a, stream));
  }
  // 5. routed experts on the expert-contiguous rows (a token adds at most one row to
  //    any expert, so no group holds more than T rows)
  GroupedFfnArgs a = routed_ffn_args(c, *w, p.x_perm, offsets, mprefix, at<void>(ws, L, B_H),
                                     at<void>(ws, L, B_YPERM), err, c.n_tokens, part);
  MOE_TRY(sg.enter(MOE_STAGE_EXPERT_FFN));
  MOE_CUDA(run_ffn(c, a, stream));
  // 6. gate-weighted combine (+ shared output)
  MOE_TRY(sg.enter(MOE_STAGE_COMBINE));
  CombineArgs cb{};
  cb.y_perm = a.out;
  cb.inv = inv;
  cb.gate = gate;
  cb.shared_y = sh_y;
  cb.y = y;
  cb.T = c.n_tokens;
  cb.d = c.d_model;
  cb.k = c.top_k;
  cb.R = c.n_tokens * c.top_k;
  cb.err = err;
  MOE_CUDA(launch_combine(cb, c.dtype, stream));
  return sg.finish();
}
}  // namespace
}  // namespace moe

MOE_API moe_status_t moe_forward(const moe_cfg_t *cfg, const moe_weights_t *w, const void *x,
                                 void *y, float *aux_out, const moe_taps_t *taps, void *ws,
                                 size_t ws_bytes, moe_stream_t stream) {
  return forward_impl(cfg, w, x, nullptr, y, aux_out, taps, ws, ws_bytes, stream);
}

MOE_API moe_status_t moe_forward_noisy(const moe_cfg_t *cfg, const moe_weights_t *w,
                                       const void *x, const float *eps, void *y,
                                       float *aux_out, const moe_taps_t *taps, void *ws,
                                       size_t ws_bytes, moe_stream_t stream) {
  if (eps == nullptr) return MOE_ERR_INVALID_ARG;
  const NoiseSpec ns{eps, 0, 0};
  return forward_impl(cfg, w, x, &ns, y, aux_out, taps, ws, ws_bytes, stream);
}

MOE_API moe_status_t moe_forward_noisy_seeded(const moe_cfg_t *cfg, const moe_weights_t *w,
                                              const void *x, uint64_t seed, uint64_t offset,
                                              void *y, float *aux_out, const moe_taps_t *taps,
                                              void *ws, size_t ws_bytes, moe_stream_t stream) {
  const NoiseSpec ns{nullptr, seed, offset};
  return forward_impl(cfg, w, x, &ns, y, aux_out, taps, ws, ws_bytes, stream);
}

MOE_API moe_status_t moe_forward_staged(const moe_cfg_t *cfg, const moe_weights_t *w,
                                        const void *x, const moe_noise_t *noise, void *y,
                                        float *aux_out, const moe_taps_t *taps,
                                        const moe_stage_events_t *events, void *ws,
                                        size_t ws_bytes, moe_stream_t stream) {
  if (noise == nullptr)
    return forward_impl(cfg, w, x, nullptr, y, aux_out, taps, ws, ws_bytes, stream, nullptr,
                        events);
  const NoiseSpec ns{noise->eps, noise->seed, noise->offset};
  return forward_impl(cfg, w, x, &ns, y, aux_out, taps, ws, ws_bytes, stream, nullptr, events);
}

// ----------------------------------------------------- token-sharded batches
MOE_API moe_status_t moe_route_shard(const moe_cfg_t *cfg, const moe_weights_t *w,
                                     const void *x, float *logits, int32_t *topk_idx,
                                     float *topk_gate, int32_t *counts, double *aux_part,
                                     void *ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  if (expert_choice(*cfg)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ptrs({{counts, true}, {aux_part, false}}));
  const moe_cfg_t &c = *cfg;
  if (c.n_tokens == 0) {  // an empty shard: no assignments, zero sums
    MOE_CUDA(cudaMemsetAsync(counts, 0, sizeof(int32_t) * c.n_experts, stream));
    if (aux_part != nullptr)
      MOE_CUDA(cudaMemsetAsync(aux_part, 0, sizeof(double) * (1 + 2 * c.n_experts), stream));
    return MOE_OK;
  }
  if (w == nullptr) return MOE_ERR_INVALID_ARG;
  if (x != nullptr) {
    MOE_TRY(check_ptrs({{x, true}, {w->w_router, true}, {logits, false}}));
  } else {
    MOE_TRY(check_ptrs({{logits, true}}));
  }
  MOE_TRY(check_ptrs({{topk_idx, true}, {topk_gate, true}, {w->b_router, false},
                      {w->logit_bias, false}}));
  const Layout L = layout_for(c);
  int32_t *err = at<int32_t>(ws, L, B_ERR);
  RouterArgs r{};
  r.x = x;
  r.w = w->w_router;
  r.b_router = w->b_router;
  r.logit_bias = w->logit_bias;
  r.logits_in = x ? nullptr : logits;
  r.logits_out = x ? logits : nullptr;
  r.topk_idx = topk_idx;
  r.topk_gate = topk_gate;
  r.tile_counts = at<int32_t>(ws, L, B_TILE_COUNTS);
  r.tile_p = aux_part ? at<float>(ws, L, B_TILE_P) : nullptr;
  r.tile_z = aux_part ? at<float>(ws, L, B_TILE_Z) : nullptr;
  r.T = c.n_tokens;
  r.d = c.d_model;
  r.E = c.n_experts;
  r.k = c.top_k;
  r.gate_mode = c.gate_mode;
  r.err = err;
  MOE_CUDA(launch_router(r, c.dtype, stream));
  // the shard's assignments per expert before any drop (offsets etc. to scratch)
  const int NT = ceil_div(c.n_tokens, router_bm(c.n_experts));
  ScanArgs s{};
  s.ticket = scan_ticket(ws, L);
  s.tile_counts = r.tile_counts;
  s.tile_base = at<int32_t>(ws, L, B_TILE_BASE);
  s.counts = counts;
  s.offsets = at<int32_t>(ws, L, B_OFFSETS);
  s.mprefix = at<int32_t>(ws, L, B_MPREFIX);
  s.E = c.n_experts;
  s.NT = NT;
  s.cap = -1;
  s.T = c.n_tokens;
  s.k = c.top_k;
  MOE_CUDA(launch_scan(s, stream));
  if (aux_part != nullptr)
    MOE_CUDA(launch_aux_partials(r.tile_counts, r.tile_p, r.tile_z, c.n_experts, NT, aux_part,
                                 stream));
  return MOE_OK;
}

MOE_API moe_status_t moe_permute_shard(const moe_cfg_t *cfg, const moe_shard_t *shard,
                                       const void *x, const int32_t *topk_idx, int32_t *counts,
                                       int32_t *offsets, int32_t *perm, int32_t *inv,
                                       void *x_perm, void *ws, size_t ws_bytes,
                                       moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  MOE_TRY(check_shard(*cfg, shard));
  MOE_TRY(check_ptrs({{x, true}, {topk_idx, true}, {counts, true}, {offsets, true}, {perm, true},
                      {inv, true}, {x_perm, true}, {shard->counts_all, true}}));
  const moe_cfg_t &c = *cfg;
  if (c.n_tokens == 0) {
    MOE_CUDA(cudaMemsetAsync(counts, 0, sizeof(int32_t) * c.n_experts, stream));
    MOE_CUDA(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (c.n_experts + 1), stream));
    return MOE_OK;
  }
  const Layout L = layout_for(c);
  int32_t *err = at<int32_t>(ws, L, B_ERR);
  int32_t *tile_counts = at<int32_t>(ws, L, B_TILE_COUNTS);
  MOE_CUDA(launch_tile_counts(topk_idx, c.n_tokens, c.top_k, c.n_experts, tile_counts, err, stream));
  ScanArgs s{};
  s.ticket = scan_ticket(ws, L);
  s.tile_counts = tile_counts;
  s.tile_base = at<int32_t>(ws, L, B_TILE_BASE);
  s.counts = counts;
  s.offsets = offsets;
  s.mprefix = at<int32_t>(ws, L, B_MPREFIX);
  s.E = c.n_experts;
  s.NT = ceil_div(c.n_tokens, router_bm(c.n_experts));
  s.cap = capacity_for_tokens(c, shard->n_tokens_total);
  s.T = c.n_tokens;
  s.k = c.top_k;
  const ShardCaps sc{shard->counts_all, at<int32_t>(ws, L, B_CAP_E), shard->n_shards,
                     shard->shard};
  MOE_CUDA(launch_scan_shard(s, sc, stream));
  ScatterArgs p{};
  p.x = x;
  p.topk_idx = topk_idx;
  p.tile_base = s.tile_base;
  p.offsets = offsets;
  p.perm = perm;
  p.inv = inv;
  p.x_perm = x_perm;
  p.T = c.n_tokens;
  p.d = c.d_model;
  p.E = c.n_experts;
  p.k = c.top_k;
  p.cap = s.cap;
  p.elem_bytes = c.dtype == MOE_DTYPE_F32 ? 4 : 2;
  p.err = err;
  MOE_CUDA(launch_scatter_shard(p, sc.cap_e, stream));
  return MOE_OK;
}

MOE_API moe_status_t moe_forward_shard(const moe_cfg_t *cfg, const moe_shard_t *shard,
                                       const moe_weights_t *w, const void *x,
                                       const moe_taps_t *taps, void *y, void *ws,
                                       size_t ws_bytes, moe_stream_t stream) {
  if (shard == nullptr) return MOE_ERR_INVALID_ARG;
  return forward_impl(cfg, w, x, nullptr, y, nullptr, taps, ws, ws_bytes, stream, shard);
}

MOE_API moe_status_t moe_aux_finalize(const moe_cfg_t *cfg, long long n_tokens_total,
                                      const double *aux_part, float *out, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  if (n_tokens_total < 1) return MOE_ERR_INVALID_ARG;  // the statistics are means over tokens
  MOE_TRY(check_ptrs({{aux_part, true}, {out, true}}));
  MOE_CUDA(launch_aux_finalize(aux_part, cfg->n_experts, n_tokens_total, cfg->top_k,
                               cfg->aux_alpha, out, stream));
  return MOE_OK;
}

MOE_API moe_status_t moe_last_device_error(void *ws, int32_t *code, int32_t *info,
                                           moe_stream_t stream) {
  if (ws == nullptr || code == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_MISALIGNED;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t h[2] = {0, 0};
  if (cudaMemcpy(h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(ws, 0, sizeof(h)) != cudaSuccess) return MOE_ERR_CUDA;
  *code = h[0];
  if (info) *info = h[1];
  return h[0] != 0 ? MOE_ERR_DEVICE : MOE_OK;
}

MOE_API moe_status_t moe_test_set_wait_limit(uint64_t ns) {
  g_wait_limit_ns.store(ns);
  return MOE_OK;
}

MOE_API moe_status_t moe_test_withhold_load(int32_t n_calls) {
  if (n_calls < 0) return MOE_ERR_INVALID_ARG;
  g_withhold_loads.store(n_calls);
  return MOE_OK;
}

MOE_API const char *moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_MISALIGNED: return "misaligned pointer";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_DEVICE: return "device-side error";
  }
  return "unknown status";
}

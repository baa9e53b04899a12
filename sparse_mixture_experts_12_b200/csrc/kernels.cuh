// Internal launch interface between the C-ABI layer and the kernel files.
#pragma once

#include "common.cuh"

namespace moe {

struct RouterArgs {
  const void *x;            // [T, d] dtype, or nullptr when logits_in is given
  const void *w;            // [E, d] dtype
  const float *b_router;    // [E] or nullptr
  const float *logit_bias;  // [E] or nullptr
  const float *logits_in;   // [T, E] when x == nullptr
  float *logits_out;        // [T, E] or nullptr
  int32_t *topk_idx;        // [T, k]
  float *topk_gate;         // [T, k]
  int32_t *tile_counts;     // [E, NT] or nullptr
  float *tile_p;            // [E, NT] or nullptr: per-tile sums of softmax probabilities
  float *tile_z;            // [NT] or nullptr: per-tile sums of logsumexp^2
  int T, d, E, k, gate_mode;
  int32_t *err;             // device error word (pipeline timeouts) or nullptr
  // noisy top-k gating (tensor-core router only): when w_noise != nullptr the logits
  // are z + softplus(x W_noise^T) * eps before the selection
  const void *w_noise;      // [E, d] dtype
  const float *eps;         // [T, E] standard normal draws
};

struct ScanArgs {
  const int32_t *tile_counts;  // [E, NT]
  int32_t *tile_base;          // [E, NT] exclusive prefix over tiles, per expert
  int32_t *counts;             // [E]
  int32_t *offsets;            // [E+1]
  int32_t *mprefix;            // [E+1] prefix of ceil(kept_e / kRowTile)
  int E, NT, cap;              // cap < 0: unlimited
  // optional aux statistics
  const float *tile_p;         // [E, NT]
  const float *tile_z;         // [NT]
  float *aux_out;              // [3 + 2E] or nullptr
  int T, k;
  float alpha;
  int32_t *sh_tbl;             // [4] or nullptr: {0, T, 0, ceil(T/kRowTile)} for the shared experts
  unsigned *ticket;            // zero-initialised word shared by the scan's CTAs (it returns to
                               // zero after every launch), or nullptr: one CTA does the scan
};

struct ScatterArgs {
  const void *x;               // [T, d] dtype
  const int32_t *topk_idx;     // [T, k]
  const int32_t *tile_base;    // [E, NT]
  const int32_t *offsets;      // [E+1]
  int32_t *perm;               // [T*k]
  int32_t *inv;                // [T*k]
  void *x_perm;                // [T*k, d]
  int T, d, E, k, cap, elem_bytes;
  int32_t *err;
};

struct CombineArgs {
  const void *y_perm;          // [R, d] dtype
  const int32_t *inv;          // [T*k]
  const float *gate;           // [T*k]
  const float *shared_y;       // [T, d] fp32 or nullptr
  void *y;                     // [T, d] dtype
  int T, d, k, R;
  int32_t *err;
};

// Grouped GEMM over expert-contiguous rows. Group g owns rows
// [offsets[g], offsets[g+1]) of A and the weight rows of expert g.
struct GroupedFfnArgs {
  const void *a;          // [rows, d] dtype (x_perm, or x for the shared experts)
  int a_rows;             // rows allocated in a/h/out (for the TMA bounds)
  const int32_t *offsets; // [G+1]
  const int32_t *mprefix; // [G+1]
  int G;                  // groups (experts)
  int m_tiles_ub;         // host upper bound on sum_g ceil(rows_g / kRowTile)
  int d, F, act;
  const void *w1, *w3, *w2;  // [G, F, d], [G, F, d] (SwiGLU), [G, d, F]
  const float *b1, *b2;      // [G, F], [G, d] or nullptr
  void *h;                // [a_rows, F] dtype (intermediate)
  void *out;              // [a_rows, d]
  int out_f32;            // 1: out is fp32 (shared experts), else dtype
  int max_group_rows;     // host bound on the rows of any one group
  float *part;            // fp32 split-K partials of the small-batch path, or nullptr
  int32_t *err;
  uint64_t wait_limit_ns; // bound on the pipeline waits of the single-CTA GEMM (0: default)
  int withhold_load;      // test hook: the single-CTA up-projection GEMM withholds one
                          // operand load per CTA (its bounded waits run out)
};

// Expert-Choice routing (see expert_choice.cu)
constexpr int kEcMaxTokens = 32768;  // one CTA holds an expert's whole column of logits
constexpr int kEcMaxPicks = 8192;    // C: the sort buffer of the picks
struct EcArgs {
  const float *logits;  // [T, E]
  float *zt;            // [E, T] scratch: transposed logits, NaN -> -inf
  int32_t *ec_idx;      // [E, C]
  float *ec_score;      // [E, C]
  int32_t *slot;        // [T, E] or nullptr: pick slot j of token t in expert e, -1 if none
                        // (the caller sets it to -1 first)
  int32_t *offsets;     // [E+1] or nullptr: e * C
  int T, E, C;
  int32_t *err;         // device error word or nullptr
};
cudaError_t launch_ec_route(const EcArgs &a, cudaStream_t st);
cudaError_t launch_ec_gather(const void *x, int T, const int32_t *ec_idx, int rows,
                             int row_bytes, void *x_perm, cudaStream_t st);
cudaError_t launch_ec_combine(const void *y_perm, const int32_t *slot, const float *score,
                              int T, int E, int C, int d, int dtype, void *y, cudaStream_t st);

cudaError_t launch_router(const RouterArgs &a, int dtype, cudaStream_t st);
// Decode-sized batches (bf16, at most 8 tokens and 32 experts, no noise and no
// statistics): the router and the scan's layout in one launch (route_small.cu). The
// router arguments' tile_counts are not written: the layout comes with the routing.
// Up to 8 tokens the one CTA beats the tensor-core router and the scan (measured:
// decode T = 1 -5 %, T = 8 -1 % per layer call); at 32 tokens it is slower (+2.4 %).
constexpr int kSmallRouteMaxT = 8;
constexpr int kSmallRouteMaxE = 32;
struct SmallRouteArgs {
  RouterArgs r;
  int cap;              // rows per expert kept, < 0: unlimited
  int32_t *counts;      // [E]
  int32_t *offsets;     // [E+1] prefix of the kept rows
  int32_t *mprefix;     // [E+1] prefix of ceil(kept_e / kRowTile)
  int32_t *tile_base;   // [E] the permute step's per-tile bases (one token tile: zero)
  int32_t *sh_tbl;      // [4] or nullptr: {0, T, 0, ceil(T/kRowTile)} for the shared experts
};
bool small_route_supported(const RouterArgs &a);
cudaError_t launch_route_small(const SmallRouteArgs &a, cudaStream_t st);
// noisy top-k gating: z[i] += softplus(zn[i]) * eps[i] over n logits
cudaError_t launch_noisy_logits(float *z, const float *zn, const float *eps, size_t n,
                                cudaStream_t st);
// bf16 router on the tensor cores (x given, d a multiple of 64, T > 0; with
// w_noise, at most 128 experts)
bool router_tc_supported(const RouterArgs &a);
// the seeded noise draws eps [T, E] (and the raw Philox words [T, ceil(E/4), 4])
cudaError_t launch_noise_draws(int T, int E, uint64_t seed, uint64_t offset, float *eps,
                               uint32_t *raw, cudaStream_t st);
cudaError_t launch_router_tc(const RouterArgs &a, cudaStream_t st);
cudaError_t launch_tile_counts(const int32_t *topk_idx, int T, int k, int E, int32_t *tile_counts,
                               int32_t *err, cudaStream_t st);
cudaError_t launch_scan(const ScanArgs &a, cudaStream_t st);
cudaError_t launch_scatter(const ScatterArgs &a, cudaStream_t st);
cudaError_t launch_combine(const CombineArgs &a, int dtype, cudaStream_t st);
// mprefix (and offset validation) from a caller-supplied offsets array
cudaError_t launch_tile_table(const int32_t *offsets, int G, int max_rows, int32_t *mprefix,
                              int32_t *err, cudaStream_t st);
// fp32 SIMT path (any sizes)
cudaError_t launch_ffn_simt(const GroupedFfnArgs &a, cudaStream_t st);
// bf16 tcgen05 path
cudaError_t launch_ffn_tc(const GroupedFfnArgs &a, cudaStream_t st);
// bf16 tcgen05 path for small groups (weights on the M side, tokens in 32-row
// chunks); used when no group can hold more than kDecodeMaxRows rows
constexpr int kDecodeMaxRows = 64;
cudaError_t launch_ffn_tc_decode(const GroupedFfnArgs &a, cudaStream_t st);
size_t ffn_decode_partial_bytes(int max_rows, int d);

}  // namespace moe

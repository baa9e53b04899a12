// Router on the 5th-generation tensor cores for every bf16 layer: logits =
// x W_r^T (+ router bias, + per-expert logit bias) by tcgen05.mma with an fp32
// TMEM accumulator, fused with the softmax, the top-k selection, the gate values
// and the per-tile statistics that the permute step (capacity ranks) and the
// auxiliary losses consume.
//
// Gating network: youngju.dev (zh) "GatingNetwork" / "SwitchRouter" and the
// devtips.kr "MoELayer" gate (a Linear over d_model, with or without bias);
// gate modes: top-k then softmax (GatingNetwork, MixtralMoELayer), softmax then
// top-k renormalised (youngju.dev ja "TopKGating"), softmax then top-1 raw
// (SwitchRouter).
//
// The router streams x (T x d) once and is bound by HBM. One cluster of S CTAs
// (S = 1, 2 or 4) covers 128 tokens; CTA r of the cluster reduces its own share
// of the d columns (a split of K), so that small batches still spread over the
// SMs. Per CTA, 576 threads:
//   warp 0       TMA producer: 128 x 64 slices of x and EPAD x 64 slices of W_r
//                (rows >= E read as zeros), 128-byte swizzle, a ring of stages.
//   warp 1       TMEM owner and MMA issuer (M = 128, N = EPAD, K = 16 per MMA).
//   warps 2..17  epilogue.
// The epilogue parks each CTA's fp32 partial logits in its shared memory; after a
// cluster barrier, CTA r takes tokens [r * 128/S, (r+1) * 128/S) and sums the S
// partials of each in rank order (distributed shared memory), so the result does
// not depend on timing. G threads share a token (consecutive lanes, expert columns
// e = g, g + G, ...): the max and the k argmax rounds (value, then lower expert
// index) and the exp sum run over shared memory with fixed shuffle trees across
// the G lanes. The permute tiles (router_bm(E) tokens) lie inside one CTA's token
// share, so their histograms and sums need no exchange.
//
// Noisy top-k gating (youngju.dev (ja) "TopKGating", training mode): W_r and W_noise
// are stacked on the MMA's N side (EX columns each), so one pass over x gives both
// x W_r^T and x W_noise^T; the epilogue forms z + softplus(x W_noise^T) * eps, with
// softplus the identity above 20 (as F.softplus), before the selection.
#include <mutex>

#include "tc_ptx.cuh"

namespace moe {

namespace {

using namespace tc;

constexpr int kRtM = 128;           // tokens per cluster (the MMA's M)
constexpr int kRtEpiWarps = 16;
constexpr int kRtEpiThreads = 32 * kRtEpiWarps;
constexpr int kRtThreads = 64 + kRtEpiThreads;
constexpr int kRtABytes = kRtM * kBlockK * 2;
constexpr int kRtMaxStages = 8;
constexpr int kRtRingBudget = 144 * 1024;  // shared memory for the operand ring
constexpr int kRtMaxSubs = 4;              // permute tiles in one CTA's token share

struct RtCtl {
  uint64_t full[kRtMaxStages];
  uint64_t empty[kRtMaxStages];
  uint64_t tfull;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int epi_ok;
  float br[kMaxExperts];  // router bias (0 when absent)
  float lb[kMaxExperts];  // per-expert logit bias (0 when absent)
  int cnt[kRtMaxSubs][kMaxExperts];
  float lse[kRtM];      // per token of the CTA's share: logsumexp of the logits
  float inv_s[kRtM];    // 1 / sum exp(z - max)
  float sel_v[kRtM][kMaxTopK];  // the top-k picks, value and expert
  int sel_i[kRtM][kMaxTopK];
};

template <int EPAD, int S, bool NOISY> struct RtCfg {
  static_assert(EPAD == 16 || EPAD == 32 || EPAD == 64 || EPAD == 128 || EPAD == 256, "EPAD");
  static_assert(S == 1 || S == 2 || S == 4, "S");
  // expert columns the selection runs over: all of N, or its first half when the
  // noise projection fills the second
  static constexpr int kEx = NOISY ? EPAD / 2 : EPAD;
  static constexpr int kBBytes = EPAD * kBlockK * 2;
  static constexpr int kStageBytes = kRtABytes + kBBytes;  // a multiple of 1024
  static constexpr int kStages = kRtRingBudget / kStageBytes < kRtMaxStages
                                     ? kRtRingBudget / kStageBytes : kRtMaxStages;
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kTok = kRtM / S;             // tokens of one CTA's epilogue
  static constexpr int kGmax = kRtEpiThreads / kTok;
  static constexpr int kG = kGmax < kEx ? kGmax : kEx;  // threads per token
  // Row stride (floats) of the logit tiles: at least EPAD and congruent to G modulo
  // 32, so that the 32 / G tokens x G lanes of a warp, reading column g + j G of
  // their token, hit 32 different banks. A multiple of 4 (G >= 4): 16-byte rows.
  static constexpr int kLdp = EPAD + ((kG - EPAD) % 32 + 32) % 32;
  static constexpr int kPartBytes = kRtM * kLdp * 4;
  // the share's logits (zb): in place of the partial tile when S = 1, after it when
  // the cluster's other CTAs still read the partials
  static constexpr int kZBytes = S == 1 ? 0 : (kRtM / S) * kLdp * 4;
  static constexpr int kBody =
      kRing > kPartBytes + kZBytes ? kRing : kPartBytes + kZBytes;
  static constexpr size_t kSmem = (size_t)kBody + sizeof(RtCtl) + 1024;
  static constexpr uint32_t kTmemCols = EPAD < 32 ? 32 : EPAD;
  static_assert(kG >= 4 && kG <= 32 && kEx % kG == 0, "token groups");
  static_assert(kLdp % 4 == 0, "16-byte rows");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ bool rt_wait(uint64_t *bar, uint32_t parity, RtCtl *ctl, int32_t *err,
                                        int site, bool honour_abort = true) {
  return wait_mbar(bar, parity, &ctl->abort_flag, 0u, err, site, honour_abort, kWaitLimitNs);
}

// (v, i) ranks above (bv, bi): larger value, ties to the lower expert index
__device__ __forceinline__ bool rt_better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

__device__ __forceinline__ void rt_epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kRtEpiThreads) : "memory");
}

// every thread of the cluster (S > 1) or of the CTA (S = 1)
template <int S>
__device__ __forceinline__ void rt_sync_all() {
  if constexpr (S == 1) {
    __syncthreads();
  } else {
    __syncwarp();
    cluster_sync_all();
  }
}

// TMEM -> this CTA's partial tile [128][EPAD] (row stride kLdp). Warp w reads TMEM
// lanes [32 (w % 4), +32) (its lane quarter); the four warps of a quarter take
// every fourth 32-column chunk. 16-byte stores.
template <int EPAD, int S, bool NOISY>
__device__ __forceinline__ void stage_partial(float *part, uint32_t tmem, int warp, int lane) {
  using C = RtCfg<EPAD, S, NOISY>;
  const int q = warp & 3;
  const int h = (warp - 2) >> 2;
  const int r = q * 32 + lane;
  float4 *row = reinterpret_cast<float4 *>(part + r * C::kLdp);
  const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16);
  if constexpr (EPAD == 16) {
    if (h == 0) {
      uint32_t v[16];
      tmem_ld16(tb, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 4; ++j)
        row[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                             __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
    }
  } else {
#pragma unroll 1
    for (int c = h; c < EPAD / 32; c += 4) {
      uint32_t v[32];
      tmem_ld32(tb + c * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 8; ++j)
        row[c * 8 + j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                     __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
    }
  }
}

// Group reductions over the G consecutive lanes that share a token (fixed trees).
template <int G>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o, G));
  return v;
}
template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, G);
  return v;
}
template <int G>
__device__ __forceinline__ void group_argmax(float &v, int &i) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o, G);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o, G);
    if (rt_better(ov, oi, v, i)) { v = ov; i = oi; }
  }
}

// The epilogue of CTA `rank`: tokens [rank * kTok, +kTok) of the cluster's 128. The
// logits live in shared memory and every pass is a compact loop: the router's
// epilogue runs once per call, after the expert GEMMs have flushed its code from
// L2, so code size (instruction fetch) costs more here than a few shared loads.
// G threads per token (consecutive lanes), thread g on expert columns g, g + G, ...
//  1. one pass over the thread's columns, kB at a time: the S partials summed in
//     rank order, the biases, the noise term, the logits written out, z (NaN and
//     padding -> -inf) kept in zb, and the best (value, then lower index) entry,
//     which after a fixed shuffle tree across the G lanes is both the maximum and
//     the first pick;
//  2. the other k - 1 argmax rounds (each the best entry ranked below the previous
//     pick), then sum exp(z - max) with exp(z - max) kept in zb; one thread per
//     token forms the gates and writes the token's outputs;
//  3. per permute tile: counts, and (statistics) the probability sums, each column
//     summed over the tile's tokens in token order, and the sum of lse^2.
template <int EPAD, int S, bool NOISY>
__device__ __forceinline__ void epilogue_tokens(const RouterArgs &a, RtCtl *ctl, float *part,
                                                float *zb, int tile, int rank, int NT, int BM,
                                                int et) {
  using C = RtCfg<EPAD, S, NOISY>;
  constexpr int EX = C::kEx, G = C::kG, TOK = C::kTok, LD = C::kLdp;
  const int E = a.E, T = a.T, k = a.k;
  const int t_base = tile * kRtM + rank * TOK;  // token of this CTA's first row

  if (et < TOK * G) {  // whole warps
    const int m = et / G, g = et % G;
    const int t = t_base + m;
    const bool valid = t < T;
    const int row = rank * TOK + m;  // the token's row in every rank's partial tile
    float *zr = zb + m * LD;
    constexpr int kEpl = EX / G;  // expert columns of this thread
    constexpr int kB = kEpl < 4 ? kEpl : 4;

    // ---- 1. logits, the maximum and the first pick. All kB columns' loads (the S
    // ranks' partials) are issued before any is used or any zb store is made, since
    // a store between two loads of the same array keeps them apart.
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    {
      const uint32_t part_s = smem_u32(part);
#pragma unroll 1
      for (int j0 = 0; j0 < kEpl; j0 += kB) {
        float acc[kB], accn[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int e = g + (j0 + u) * G;
          accn[u] = 0.f;
          if constexpr (S == 1) {
            acc[u] = part[row * LD + e];
            if constexpr (NOISY) accn[u] = part[row * LD + EX + e];
          } else {
            const uint32_t off = 4u * (uint32_t)(row * LD + e);
            float v[S], vn[S];
#pragma unroll
            for (int r = 0; r < S; ++r) {
              const uint32_t rb = mapa_rank(part_s, (uint32_t)r) + off;
              v[r] = ld_cluster_f32(rb);
              if constexpr (NOISY) vn[r] = ld_cluster_f32(rb + 4u * EX);
            }
            acc[u] = v[0];  // the ranks' partials in rank order
#pragma unroll
            for (int r = 1; r < S; ++r) acc[u] += v[r];
            if constexpr (NOISY) {
              accn[u] = vn[0];
#pragma unroll
              for (int r = 1; r < S; ++r) accn[u] += vn[r];
            }
          }
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int e = g + (j0 + u) * G;
          const bool live = valid && e < E;
          float v = acc[u];
          if (a.b_router) v += ctl->br[e];
          if (a.logit_bias) v += ctl->lb[e];
          if constexpr (NOISY) {
            if (live) {
              const float sp = accn[u] > 20.f ? accn[u] : log1pf(expf(accn[u]));
              v = v + sp * a.eps[(size_t)t * E + e];
            }
          }
          if (a.logits_out != nullptr && live) a.logits_out[(size_t)t * E + e] = v;
          const float z = (e >= E || v != v) ? -INFINITY : v;  // padding, NaN never win
          zr[e] = z;
          if (rt_better(z, e, bv, bi)) { bv = z; bi = e; }
        }
      }
    }
    group_argmax<G>(bv, bi);
    const float mx = bv;
    if (g == 0) {
      ctl->sel_v[m][0] = bv;
      ctl->sel_i[m][0] = bi;
    }

    // ---- 2. the other picks, the exp sum, the gates
    float pv = bv;
    int pi = bi;
#pragma unroll 1
    for (int s = 1; s < k; ++s) {
      bv = -INFINITY;
      bi = 0x7fffffff;
#pragma unroll 4
      for (int e = g; e < EX; e += G) {
        const float z = zr[e];
        const bool below = z < pv || (z == pv && e > pi);
        if (below && rt_better(z, e, bv, bi)) { bv = z; bi = e; }
      }
      group_argmax<G>(bv, bi);
      pv = bv;
      pi = bi;
      if (g == 0) {
        ctl->sel_v[m][s] = bv;
        ctl->sel_i[m][s] = bi;
      }
    }
    float ssum = 0.f;
#pragma unroll 1
    for (int j0 = 0; j0 < kEpl; j0 += kB) {  // kB loads before the kB stores
      float ex[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) ex[u] = zr[g + (j0 + u) * G];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        ex[u] = expf(ex[u] - mx);
        ssum += ex[u];
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) zr[g + (j0 + u) * G] = ex[u];  // for the probability sums
    }
    ssum = group_sum<G>(ssum);
    const float inv_s = 1.f / ssum;
    __syncwarp();  // the group's sel_v / sel_i are written
    if (g == 0) {
      ctl->lse[m] = valid ? mx + logf(ssum) : 0.f;
      ctl->inv_s[m] = valid ? inv_s : 0.f;
      const float *tv = ctl->sel_v[m];
      const int *ti = ctl->sel_i[m];
      float gv[kMaxTopK];
      float gs = 0.f;
      if (a.gate_mode == MOE_GATE_TOPK_SOFTMAX) {
#pragma unroll
        for (int s = 0; s < kMaxTopK; ++s)
          if (s < k) { gv[s] = expf(tv[s] - tv[0]); gs += gv[s]; }
        const float inv = 1.f / gs;
#pragma unroll
        for (int s = 0; s < kMaxTopK; ++s) if (s < k) gv[s] *= inv;
      } else {
#pragma unroll
        for (int s = 0; s < kMaxTopK; ++s)
          if (s < k) { gv[s] = expf(tv[s] - mx) * inv_s; gs += gv[s]; }
        if (a.gate_mode == MOE_GATE_SOFTMAX_TOPK_RENORM) {
#pragma unroll
          for (int s = 0; s < kMaxTopK; ++s) if (s < k) gv[s] = gv[s] / gs;
        }
      }
      if (valid) {
#pragma unroll
        for (int s = 0; s < kMaxTopK; ++s) {
          if (s < k) {
            a.topk_idx[(size_t)t * k + s] = ti[s];
            a.topk_gate[(size_t)t * k + s] = gv[s];
            // integer counts: the result does not depend on the order of the adds
            if (ti[s] < E) atomicAdd(&ctl->cnt[m / BM][ti[s]], 1);
          }
        }
      }
    }
  }
  rt_epi_sync();

  // ---- 3. per permute tile (BM tokens, whole tiles inside this CTA's share)
  const int subs = TOK / BM;
  const int tile0 = t_base / BM;
  for (int i = et; i < subs * E; i += kRtEpiThreads) {
    const int sub = i / E, e = i - sub * E;
    const int pt = tile0 + sub;
    if (pt >= NT) continue;
    if (a.tile_counts) a.tile_counts[(size_t)e * NT + pt] = ctl->cnt[sub][e];
    if (a.tile_p != nullptr) {
      const int rows = min(BM, T - pt * BM);
      const float *col = zb + sub * BM * LD + e;
      const float *is = ctl->inv_s + sub * BM;
      float s = 0.f;
      for (int mm = 0; mm < rows; ++mm) s += col[mm * LD] * is[mm];
      a.tile_p[(size_t)e * NT + pt] = s;
    }
  }
  if (a.tile_z && et < subs) {
    const int pt = tile0 + et;
    if (pt < NT) {
      const int rows = min(BM, T - pt * BM);
      float s = 0.f;
      for (int mm = 0; mm < rows; ++mm) {
        const float l = ctl->lse[et * BM + mm];
        s += l * l;
      }
      a.tile_z[pt] = s;
    }
  }
}

template <int EPAD, int S, bool NOISY>
__global__ void __launch_bounds__(kRtThreads, 1)
k_router_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
            const __grid_constant__ CUtensorMap tmN, RouterArgs a, int NT, int BM) {
  using C = RtCfg<EPAD, S, NOISY>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  RtCtl *ctl = reinterpret_cast<RtCtl *>(smem + C::kBody);
  float *part = reinterpret_cast<float *>(smem);  // [128][EPAD+1], reuses the ring
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E;
  const int rank = S == 1 ? 0 : (int)cluster_ctarank();
  const int tile = blockIdx.x / S;
  const int t0 = tile * kRtM;
  const int nkb = ceil_div(a.d, kBlockK);
  const int kb0 = rank * nkb / S, kb1 = (rank + 1) * nkb / S;  // this CTA's K share

  for (int e = tid; e < kMaxExperts; e += kRtThreads) {
    ctl->br[e] = (a.b_router && e < E) ? a.b_router[e] : 0.f;
    ctl->lb[e] = (a.logit_bias && e < E) ? a.logit_bias[e] : 0.f;
  }
  for (int i = tid; i < kRtMaxSubs * kMaxExperts; i += kRtThreads) (&ctl->cnt[0][0])[i] = 0;
  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->tfull, 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    ctl->epi_ok = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  // the set-up above overlaps the previous kernel; x, the weights and every output
  // are touched only after it has completed
  pdl_wait();
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    prefetch_map(&tmX);
    prefetch_map(&tmW);
    if (NOISY) prefetch_map(&tmN);
    int stage = 0;
    uint32_t phase = 0, issued = 0, last_phase = 0;
    bool ok = true;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!rt_wait(&ctl->empty[stage], phase ^ 1u, ctl, a.err, 11)) { ok = false; break; }
      uint8_t *sa = smem + (size_t)stage * C::kStageBytes;
      mbar_expect_tx(&ctl->full[stage], C::kStageBytes);
      tma_load_2d(&tmX, &ctl->full[stage], sa, kb * kBlockK, t0);
      tma_load_2d(&tmW, &ctl->full[stage], sa + kRtABytes, kb * kBlockK, 0);
      if (NOISY)  // the noise projection's rows follow W_r's (whole 1024-byte atoms)
        tma_load_2d(&tmN, &ctl->full[stage], sa + kRtABytes + C::kEx * kBlockK * 2,
                    kb * kBlockK, 0);
      issued |= 1u << stage;
      last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
      if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
    }
    // every copy issued has landed before the ring is reused, whichever role gave up
    // (a no-op wait on a normal run: the MMAs consumed them all)
    for (int s = 0; s < C::kStages; ++s)
      if (issued & (1u << s)) rt_wait(&ctl->full[s], (last_phase >> s) & 1u, ctl, nullptr, 0, false);
    (void)ok;
  } else if (warp == 1 && lane == 0) {
    // --------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = make_idesc(kRtM, EPAD);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true, any = false;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!rt_wait(&ctl->full[stage], phase, ctl, a.err, 12)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + (size_t)stage * C::kStageBytes);
      const uint64_t da = sw128_desc(sa);
      const uint64_t db = sw128_desc(sa + kRtABytes);
#pragma unroll
      for (int kk = 0; kk < kBlockK / 16; ++kk)
        umma_bf16(tmem, da + 2 * kk, db + 2 * kk, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
      any = true;
      umma_commit(&ctl->empty[stage]);
      if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
    }
    if (ok) {
      umma_commit(&ctl->tfull);
    } else if (any) {  // retire the MMAs in flight before TMEM is released
      umma_commit(&ctl->drain);
      rt_wait(&ctl->drain, 0, ctl, nullptr, 0, false);
    }
  } else if (warp >= 2) {
    // ------------------------------------------ epilogue, 1: TMEM -> partial tile
    const int et = tid - 64;
    // one thread waits; the named barrier is reached by all epilogue threads
    if (et == 0) ctl->epi_ok = rt_wait(&ctl->tfull, 0, ctl, a.err, 13) ? 1 : 0;
    rt_epi_sync();
    if (ctl->epi_ok) {
      tc_fence_after();
      stage_partial<EPAD, S, NOISY>(part, tmem, warp, lane);
    }
  }
  // the partial tiles of the whole cluster are complete
  tc_fence_before();
  rt_sync_all<S>();
  tc_fence_after();
  if (warp >= 2 && ctl->epi_ok)
    epilogue_tokens<EPAD, S, NOISY>(a, ctl, part, S == 1 ? part : part + kRtM * C::kLdp, tile,
                                    rank, NT, BM, tid - 64);
  // no CTA leaves (its shared memory) while another may still read its partials
  rt_sync_all<S>();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

std::mutex g_rt_mu;

template <int EPAD, int S, bool NOISY>
cudaError_t launch_rt(const RouterArgs &a, cudaStream_t st) {
  using C = RtCfg<EPAD, S, NOISY>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(g_rt_mu);
    if (!attr_set[dev & 63]) {
      e = cudaFuncSetAttribute(k_router_tc<EPAD, S, NOISY>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
      if (e != cudaSuccess) return e;
      attr_set[dev & 63] = true;
    }
  }
  CUtensorMap mx, mw, mn;
  if (!make_map(&mx, a.x, (uint64_t)a.T, (uint64_t)a.d, kRtM)) return cudaErrorInvalidValue;
  if (!make_map(&mw, a.w, (uint64_t)a.E, (uint64_t)a.d, C::kEx)) return cudaErrorInvalidValue;
  if (NOISY) {
    if (!make_map(&mn, a.w_noise, (uint64_t)a.E, (uint64_t)a.d, C::kEx))
      return cudaErrorInvalidValue;
  } else {
    mn = mw;
  }
  const int BM = router_bm(a.E);
  const int NT = ceil_div(a.T, BM);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(ceil_div(a.T, kRtM) * S));
  cfg.blockDim = dim3(kRtThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = take_pdl() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k_router_tc<EPAD, S, NOISY>, mx, mw, mn, a, NT, BM);
}

// K splits: at most four, each CTA's token share (128 / S) a whole number of permute
// tiles, at least two 64-column blocks of K per split, and only while the grid
// stays under one CTA per SM.
int router_splits(int T, int d, int E, int ex) {
  const int BM = router_bm(E);
  const int tiles = ceil_div(T, kRtM);
  const int nkb = d / kBlockK;
  const int sms = sm_count();
  int S = 1;
  while (S < 4 && kRtM / (2 * S) >= BM && 2 * S <= nkb && tiles * 2 * S <= sms) S *= 2;
  (void)ex;
  return S;
}

template <int EPAD, bool NOISY>
cudaError_t launch_rt_e(const RouterArgs &a, cudaStream_t st) {
  constexpr int kEx = NOISY ? EPAD / 2 : EPAD;  // the expert columns of the selection
  const int S = router_splits(a.T, a.d, a.E, kEx);
  if (S == 4) return launch_rt<EPAD, 4, NOISY>(a, st);
  if (S == 2) return launch_rt<EPAD, 2, NOISY>(a, st);
  return launch_rt<EPAD, 1, NOISY>(a, st);
}

}  // namespace

bool router_tc_supported(const RouterArgs &a) {
  if (a.x == nullptr || a.E < 1 || a.E > kMaxExperts || a.d % kBlockK != 0 || a.T <= 0)
    return false;
  if (a.w_noise != nullptr) return a.E <= 128 && a.eps != nullptr;
  return true;
}

cudaError_t launch_router_tc(const RouterArgs &a, cudaStream_t st) {
  if (!router_tc_supported(a)) return cudaErrorInvalidValue;
  if (a.w_noise != nullptr) {  // N = 2 x (E rounded up to 8 .. 128)
    if (a.E <= 8) return launch_rt_e<16, true>(a, st);
    if (a.E <= 16) return launch_rt_e<32, true>(a, st);
    if (a.E <= 32) return launch_rt_e<64, true>(a, st);
    if (a.E <= 64) return launch_rt_e<128, true>(a, st);
    return launch_rt_e<256, true>(a, st);
  }
  if (a.E <= 16) return launch_rt_e<16, false>(a, st);
  if (a.E <= 32) return launch_rt_e<32, false>(a, st);
  if (a.E <= 64) return launch_rt_e<64, false>(a, st);
  if (a.E <= 128) return launch_rt_e<128, false>(a, st);
  return launch_rt_e<256, false>(a, st);
}

}  // namespace moe

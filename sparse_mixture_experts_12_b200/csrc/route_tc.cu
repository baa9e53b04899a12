// Router on the 5th-generation tensor cores for bf16 layers with 16..256
// experts: logits = x W_r^T (+ router bias, + per-expert logit bias) by
// tcgen05.mma with an fp32 TMEM accumulator, fused with the softmax, the top-k
// selection, the gate values and the per-tile statistics that the permute step
// (capacity ranks) and the auxiliary losses consume.
//
// Gating network: youngju.dev (zh) "GatingNetwork" / "SwitchRouter" and the
// devtips.kr "MoELayer" gate (a Linear over d_model, with or without bias);
// gate modes: top-k then softmax (GatingNetwork, MixtralMoELayer), softmax then
// top-k renormalised (youngju.dev ja "TopKGating"), softmax then top-1 raw
// (SwitchRouter).
//
// One CTA per 128 tokens, 320 threads:
//   warp 0      TMA producer: 128 x 64 slices of x and EPAD x 64 slices of W_r
//               (rows >= E read as zeros), 128-byte swizzle, 4..9-stage ring.
//   warp 1      TMEM owner and MMA issuer (M = 128, N = EPAD, K = 16 per MMA).
//   warps 2..9  epilogue, two threads per token.
// Same results as the SIMT router up to the fp32 summation order of the dot
// products: same bias order, NaN -> -inf before selection, ties to the lower
// expert index, same gate formulas, same fixed-order per-tile sums.
#include <mutex>

#include "tc_ptx.cuh"

namespace moe {

namespace {

using namespace tc;

constexpr int kRtMaxStages = 10;
constexpr int kRtRingBudget = 192 * 1024;  // shared memory for the operand ring
constexpr int kRtM = 128;  // tokens per CTA
constexpr int kRtEpiThreads = 256;  // two threads per token
constexpr int kRtThreads = 64 + kRtEpiThreads;
constexpr int kRtABytes = kRtM * kBlockK * 2;
constexpr int kRtMaxSubs = 4;  // permute tiles per CTA: 128 / router_bm(E)

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
  float lse[kRtM];
  int cnt[kRtMaxSubs][kMaxExperts];
  // the two threads of a token meet here: max, top-k candidates (double-buffered
  // by round parity), exp sums
  float hmax[2][kRtM];
  float cand_v[2][2][kRtM];
  int cand_i[2][2][kRtM];
  float hsum[2][kRtM];
};

template <int EPAD> struct RtCfg {
  static_assert(EPAD == 32 || EPAD == 64 || EPAD == 128 || EPAD == 256, "EPAD");
  static constexpr int kBBytes = EPAD * kBlockK * 2;
  static constexpr int kStageBytes = kRtABytes + kBBytes;  // a multiple of 1024
  // as many stages as the budget holds: one CTA per SM streams x, so the bytes in
  // flight per SM set the achievable bandwidth
  static constexpr int kStages = kRtRingBudget / kStageBytes < kRtMaxStages
                                     ? kRtRingBudget / kStageBytes : kRtMaxStages;
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kLdl = EPAD + 1;  // probability tile row stride (floats)
  static constexpr int kProbBytes = kRtM * kLdl * 4;
  static constexpr int kBody = kRing > kProbBytes ? kRing : kProbBytes;
  static constexpr size_t kSmem = (size_t)kBody + sizeof(RtCtl) + 1024;
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

// Two threads per token. Pass 1: the two warps that may read a TMEM lane quarter
// take alternate 32-column chunks of their 32 tokens: logits (+ biases in the
// CUDA-core router's order) are written out and z (NaN -> -inf) parked in the
// token's row of the shared-memory tile. Then thread (token r, half h) owns row r,
// columns [h*E0, min(E, (h+1)*E0)): the max, k argmax rounds (each the best entry
// ranked below the previous pick: value, then lower index) and sum exp(z - max) are
// taken over each half and merged through shared memory in a fixed order.
template <int EPAD>
__device__ __forceinline__ void epilogue_rows(const RouterArgs &a, RtCtl *ctl, float *prob,
                                              uint32_t tmem, int t0, int NT, int BM, int warp,
                                              int lane) {
  constexpr int LDL = RtCfg<EPAD>::kLdl;
  const int E = a.E, T = a.T, k = a.k;
  const int et = (warp - 2) * 32 + lane;  // 0..255 over the epilogue threads
  // one thread waits; the named barrier is reached by all epilogue threads
  if (et == 0) ctl->epi_ok = rt_wait(&ctl->tfull, 0, ctl, a.err, 13) ? 1 : 0;
  rt_epi_sync();
  if (!ctl->epi_ok) return;
  tc_fence_after();

  {  // ---- pass 1: TMEM -> logits out, z into the row
    const int ew = warp & 3;                // TMEM lanes [32 ew, 32 ew + 32) (warp % 4)
    const int c_first = (warp - 2) >> 2;    // this warp's chunks: c_first, c_first + 2, ...
    const int r = ew * 32 + lane;
    const int t = t0 + r;
    const bool valid = t < T;
    float *row = prob + r * LDL;
    const uint32_t tb = tmem + ((uint32_t)(ew * 32) << 16);
    const bool vec_out = valid && a.logits_out != nullptr && (E & 3) == 0;
#pragma unroll 1
    for (int c = c_first; c < EPAD / 32; c += 2) {
      uint32_t v[32];
      tmem_ld32(tb + c * 32, v);
      tmem_ld_wait();
      float lo[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int e = c * 32 + j;
        float val = __uint_as_float(v[j]);
        if (a.b_router) val += ctl->br[e];
        if (a.logit_bias) val += ctl->lb[e];
        lo[j] = val;
        if (e < E) row[e] = (val != val) ? -INFINITY : val;  // a NaN logit never wins a slot
      }
      const int n_out = min(32, E - c * 32);
      if (vec_out && n_out == 32) {
        float4 *dst = reinterpret_cast<float4 *>(a.logits_out + (size_t)t * E + c * 32);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_float4(lo[4 * q], lo[4 * q + 1], lo[4 * q + 2], lo[4 * q + 3]);
      } else if (valid && a.logits_out != nullptr) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < n_out) a.logits_out[(size_t)t * E + c * 32 + j] = lo[j];
      }
    }
  }
  rt_epi_sync();

  // ---- the rest: thread (token r, half h); a warp holds 32 consecutive tokens
  const int r = et & (kRtM - 1), h = et / kRtM;
  const int t = t0 + r;
  const bool valid = t < T;
  float *row = prob + r * LDL;
  const int E0 = (E + 1) >> 1;
  const int e_lo = h * E0, e_hi = min(E, e_lo + E0);

  float mx = -INFINITY;
  for (int e = e_lo; e < e_hi; ++e) mx = fmaxf(mx, row[e]);
  ctl->hmax[h][r] = mx;
  rt_epi_sync();
  mx = fmaxf(ctl->hmax[0][r], ctl->hmax[1][r]);

  float tv[kMaxTopK];
  int ti[kMaxTopK];
  float pv = INFINITY;
  int pi = -1;
#pragma unroll
  for (int s = 0; s < kMaxTopK; ++s) {
    tv[s] = -INFINITY;
    ti[s] = 0x7fffffff;
    if (s < k) {
      float bv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      int bi[4] = {0x7fffffff, 0x7fffffff, 0x7fffffff, 0x7fffffff};
      int e = e_lo;
#pragma unroll 2
      for (; e + 4 <= e_hi; e += 4) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float z = row[e + q];
          const bool below = z < pv || (z == pv && e + q > pi);
          if (below && rt_better(z, e + q, bv[q], bi[q])) { bv[q] = z; bi[q] = e + q; }
        }
      }
      for (; e < e_hi; ++e) {
        const float z = row[e];
        const bool below = z < pv || (z == pv && e > pi);
        if (below && rt_better(z, e, bv[0], bi[0])) { bv[0] = z; bi[0] = e; }
      }
#pragma unroll
      for (int q = 1; q < 4; ++q)
        if (rt_better(bv[q], bi[q], bv[0], bi[0])) { bv[0] = bv[q]; bi[0] = bi[q]; }
      ctl->cand_v[s & 1][h][r] = bv[0];
      ctl->cand_i[s & 1][h][r] = bi[0];
      rt_epi_sync();
      float b0 = ctl->cand_v[s & 1][0][r], b1 = ctl->cand_v[s & 1][1][r];
      int i0 = ctl->cand_i[s & 1][0][r], i1 = ctl->cand_i[s & 1][1][r];
      if (rt_better(b1, i1, b0, i0)) { b0 = b1; i0 = i1; }
      tv[s] = pv = b0;
      ti[s] = pi = i0;
    }
  }

  float ssum = 0.f;
#pragma unroll 4
  for (int e = e_lo; e < e_hi; ++e) {
    const float ex = expf(row[e] - mx);
    ssum += ex;
    row[e] = ex;
  }
  ctl->hsum[h][r] = ssum;
  rt_epi_sync();
  ssum = ctl->hsum[0][r] + ctl->hsum[1][r];
  const float inv_s = 1.f / ssum;
  if (a.tile_p != nullptr)
    for (int e = e_lo; e < e_hi; ++e) row[e] *= inv_s;

  if (h == 0) {
    ctl->lse[r] = mx + logf(ssum);
    float g[kMaxTopK];
    float gs = 0.f;
    if (a.gate_mode == MOE_GATE_TOPK_SOFTMAX) {
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s)
        if (s < k) { g[s] = expf(tv[s] - tv[0]); gs += g[s]; }
      const float inv = 1.f / gs;
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s) if (s < k) g[s] *= inv;
    } else {
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s)
        if (s < k) { g[s] = expf(tv[s] - mx) * inv_s; gs += g[s]; }
      if (a.gate_mode == MOE_GATE_SOFTMAX_TOPK_RENORM) {
#pragma unroll
        for (int s = 0; s < kMaxTopK; ++s) if (s < k) g[s] = g[s] / gs;
      }
    }
    if (valid) {
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s) {
        if (s < k) {
          a.topk_idx[(size_t)t * k + s] = ti[s];
          a.topk_gate[(size_t)t * k + s] = g[s];
          if (ti[s] < E) atomicAdd(&ctl->cnt[r / BM][ti[s]], 1);
        }
      }
    }
  }
  rt_epi_sync();

  // per permute tile (BM tokens): histogram, probability sums, sum of lse^2,
  // each in token order
  const int subs = kRtM / BM;
  for (int i = et; i < subs * E; i += kRtEpiThreads) {
    const int sub = i / E, e = i - sub * E;
    const int tile = blockIdx.x * subs + sub;
    if (tile >= NT) continue;
    if (a.tile_counts) a.tile_counts[(size_t)e * NT + tile] = ctl->cnt[sub][e];
    if (a.tile_p != nullptr) {
      const int rows = min(BM, T - tile * BM);
      float s = 0.f;
      for (int m = 0; m < rows; ++m) s += prob[(sub * BM + m) * LDL + e];
      a.tile_p[(size_t)e * NT + tile] = s;
    }
  }
  if (a.tile_z && et < subs) {
    const int tile = blockIdx.x * subs + et;
    if (tile < NT) {
      const int rows = min(BM, T - tile * BM);
      float s = 0.f;
      for (int m = 0; m < rows; ++m) {
        const float l = ctl->lse[et * BM + m];
        s += l * l;
      }
      a.tile_z[tile] = s;
    }
  }
}

template <int EPAD>
__global__ void __launch_bounds__(kRtThreads, 1)
k_router_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
            RouterArgs a, int NT, int BM) {
  using C = RtCfg<EPAD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  RtCtl *ctl = reinterpret_cast<RtCtl *>(smem + C::kBody);
  float *prob = reinterpret_cast<float *>(smem);  // [128][EPAD+1], reuses the ring
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E;
  const int t0 = blockIdx.x * kRtM;
  const int nkb = ceil_div(a.d, kBlockK);

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
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, EPAD);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    prefetch_map(&tmX);
    prefetch_map(&tmW);
    int stage = 0;
    uint32_t phase = 0, issued = 0, last_phase = 0;
    bool ok = true;
    for (int kb = 0; kb < nkb; ++kb) {
      if (!rt_wait(&ctl->empty[stage], phase ^ 1u, ctl, a.err, 11)) { ok = false; break; }
      uint8_t *sa = smem + (size_t)stage * C::kStageBytes;
      mbar_expect_tx(&ctl->full[stage], C::kStageBytes);
      tma_load_2d(&tmX, &ctl->full[stage], sa, kb * kBlockK, t0);
      tma_load_2d(&tmW, &ctl->full[stage], sa + kRtABytes, kb * kBlockK, 0);
      issued |= 1u << stage;
      last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
      if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
    }
    if (!ok) {  // let the copies already in flight land before the CTA exits
      for (int s = 0; s < C::kStages; ++s)
        if (issued & (1u << s)) rt_wait(&ctl->full[s], (last_phase >> s) & 1u, ctl, nullptr, 0, false);
    }
  } else if (warp == 1 && lane == 0) {
    // --------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = make_idesc(kRtM, EPAD);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true, any = false;
    for (int kb = 0; kb < nkb; ++kb) {
      if (!rt_wait(&ctl->full[stage], phase, ctl, a.err, 12)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + (size_t)stage * C::kStageBytes);
      const uint64_t da = sw128_desc(sa);
      const uint64_t db = sw128_desc(sa + kRtABytes);
#pragma unroll
      for (int kk = 0; kk < kBlockK / 16; ++kk)
        umma_bf16(tmem, da + 2 * kk, db + 2 * kk, idesc, (kb | kk) != 0);
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
    epilogue_rows<EPAD>(a, ctl, prob, tmem, t0, NT, BM, warp, lane);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, EPAD);
  }
}

std::mutex g_rt_mu;

template <int EPAD>
cudaError_t launch_rt(const RouterArgs &a, cudaStream_t st) {
  using C = RtCfg<EPAD>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(g_rt_mu);
    if (!attr_set[dev & 63]) {
      e = cudaFuncSetAttribute(k_router_tc<EPAD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)C::kSmem);
      if (e != cudaSuccess) return e;
      attr_set[dev & 63] = true;
    }
  }
  CUtensorMap mx, mw;
  if (!make_map(&mx, a.x, (uint64_t)a.T, (uint64_t)a.d, kRtM)) return cudaErrorInvalidValue;
  if (!make_map(&mw, a.w, (uint64_t)a.E, (uint64_t)a.d, EPAD)) return cudaErrorInvalidValue;
  const int BM = router_bm(a.E);
  const int NT = ceil_div(a.T, BM);
  k_router_tc<EPAD><<<ceil_div(a.T, kRtM), kRtThreads, C::kSmem, st>>>(mx, mw, a, NT, BM);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_tc(const RouterArgs &a, cudaStream_t st) {
  if (a.x == nullptr || a.E < 1 || a.E > kMaxExperts || a.d % kBlockK != 0)
    return cudaErrorInvalidValue;
  if (a.E <= 32) return launch_rt<32>(a, st);
  if (a.E <= 64) return launch_rt<64>(a, st);
  if (a.E <= 128) return launch_rt<128>(a, st);
  return launch_rt<256>(a, st);
}

}  // namespace moe

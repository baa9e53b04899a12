// Router GEMM (CUDA cores, fp32 accumulate) fused with softmax, top-k, gates,
// per-tile expert histogram and per-tile softmax/logsumexp partial sums.
//
// Gating network: youngju.dev (zh) "GatingNetwork" / "SwitchRouter" and the
// devtips.kr "MoELayer" gate (a Linear over d_model, with or without bias);
// gate modes: top-k then softmax (GatingNetwork, MixtralMoELayer), softmax then
// top-k renormalised (youngju.dev ja "TopKGating"), softmax then top-1 raw
// (SwitchRouter). Top-k is taken on the fp32 logits in every mode; equal logits
// go to the lower expert index first.
#include <atomic>

#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kRouterThreads = 256;
constexpr int kBK = 32;  // K elements per slice per iteration
constexpr int kRouterStages = 3;  // cp.async ring depth

template <int EPAD> struct RouterShape;
template <> struct RouterShape<8>   { static constexpr int BM = 32, TM = 1, TN = 8, KS = 8; };
template <> struct RouterShape<16>  { static constexpr int BM = 32, TM = 1, TN = 8, KS = 4; };
template <> struct RouterShape<32>  { static constexpr int BM = 32, TM = 2, TN = 8, KS = 4; };
template <> struct RouterShape<64>  { static constexpr int BM = 64, TM = 4, TN = 8, KS = 2; };
template <> struct RouterShape<128> { static constexpr int BM = 64, TM = 4, TN = 8, KS = 1; };
template <> struct RouterShape<256> { static constexpr int BM = 32, TM = 4, TN = 8, KS = 1; };

template <int EPAD> struct RouterSmem {
  using S = RouterShape<EPAD>;
  static constexpr int XS = kBK + 4;                          // padded fp32 row (x and W)
  static constexpr int SLICE = (S::BM + EPAD) * XS;           // fp32 floats per K slice
  static constexpr int TILE_FLOATS = S::KS * SLICE;
  static constexpr int LG_FLOATS = S::BM * (EPAD + 1);
  static constexpr int FLOATS = TILE_FLOATS > LG_FLOATS ? TILE_FLOATS : LG_FLOATS;
  // raw (storage dtype) copy of one iteration: KS slices x (BM x rows + EPAD w rows) x kBK
  static constexpr int raw_bytes(int eb) { return S::KS * (S::BM + EPAD) * kBK * eb; }
  static constexpr int bytes(int eb) { return FLOATS * 4 + kRouterStages * raw_bytes(eb); }
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename ET, int EPAD>
__global__ void __launch_bounds__(kRouterThreads)
k_router(RouterArgs a) {
  using S = RouterShape<EPAD>;
  using L = RouterSmem<EPAD>;
  constexpr int BM = S::BM, TM = S::TM, TN = S::TN, KS = S::KS;
  static_assert(BM == router_bm(EPAD), "router tile must match the permute tiles");
  static_assert((BM / TM) * (EPAD / TN) * KS == kRouterThreads, "thread layout");
  constexpr int VE = Elem<ET>::kPerVec;
  constexpr int EB = sizeof(ET);
  constexpr int XS = L::XS;
  constexpr int SLICE = L::SLICE;
  extern __shared__ __align__(16) float smem[];  // fp32 tile, then the raw ring
  uint8_t *raw = reinterpret_cast<uint8_t *>(smem + L::FLOATS);
  constexpr int RAW = L::raw_bytes(EB);
  __shared__ int cnt[EPAD];
  __shared__ float lse_s[BM];

  const int tid = threadIdx.x;
  const int E = a.E, d = a.d, T = a.T, k = a.k;
  const int t0 = blockIdx.x * BM;
  const int tile = blockIdx.x;
  float *lg = smem;  // [BM][EPAD+1] after the GEMM
  constexpr int LDL = EPAD + 1;

  for (int i = tid; i < EPAD; i += kRouterThreads) cnt[i] = 0;

  if (a.x != nullptr) {
    // -------------------------------------------------------------- GEMM part
    constexpr int TPS = kRouterThreads / KS;  // threads per K slice
    const int ks = tid / TPS;
    const int r = tid % TPS;
    const int tn = r % (EPAD / TN);
    const int tm = r / (EPAD / TN);
    float acc[TM][TN];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
      for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;

    // Each thread owns the same 16-byte vectors of every iteration: it copies them
    // into the raw ring (cp.async, zero-filled out of range) and later converts
    // exactly those vectors to fp32, so only its own copies must have landed.
    constexpr int VPR = kBK / VE;              // vectors per row of a slice
    constexpr int XV = KS * BM * VPR;          // x vectors per iteration
    constexpr int WV = KS * EPAD * VPR;        // W vectors per iteration
    constexpr int NV = XV + WV;
    constexpr int VPT = (NV + kRouterThreads - 1) / kRouterThreads;
    const ET *x = static_cast<const ET *>(a.x);
    const ET *w = static_cast<const ET *>(a.w);
    const int kstep = KS * kBK;
    const int n_iter = ceil_div(d, kstep);
    const uint32_t raw_base = static_cast<uint32_t>(__cvta_generic_to_shared(raw));

    auto issue = [&](int it) {
      if (it < n_iter) {
        const int kb = it * kstep;
        const uint32_t stage = raw_base + (uint32_t)((it % kRouterStages) * RAW);
#pragma unroll
        for (int q = 0; q < VPT; ++q) {
          const int v = tid + q * kRouterThreads;
          if (v < NV) {
            // slice-major: a warp covers consecutive 16-byte chunks of one slice
            const bool isx = v < XV;
            const int u = isx ? v : v - XV;
            const int rows = isx ? BM : EPAD;
            const int sl = u / (rows * VPR);
            const int row = (u % (rows * VPR)) / VPR;       // token (x) or expert (W)
            const int c = (u % VPR) * VE;                   // column inside the slice
            const int col = kb + sl * kBK + c;
            bool ok;
            const ET *src;
            if (isx) {
              ok = (t0 + row < T) && (col < d);
              src = x + (size_t)(ok ? t0 + row : 0) * d + (ok ? col : 0);
            } else {
              ok = (row < E) && (col < d);
              src = w + (size_t)(ok ? row : 0) * d + (ok ? col : 0);
            }
            const int prow = isx ? row : BM + row;
            const uint32_t dst = stage + (uint32_t)(((sl * (BM + EPAD) + prow) * kBK + c) * EB);
            cp_async16(dst, src, ok);
          }
        }
      }
      cp_async_commit();  // an empty group past the end keeps the wait counts uniform
    };
    auto convert = [&](int it) {
      const uint8_t *stage = raw + (size_t)(it % kRouterStages) * RAW;
#pragma unroll
      for (int q = 0; q < VPT; ++q) {
        const int v = tid + q * kRouterThreads;
        if (v < NV) {
          const bool isx = v < XV;
          const int u = isx ? v : v - XV;
          const int rows = isx ? BM : EPAD;
          const int sl = u / (rows * VPR);
          const int row = (u % (rows * VPR)) / VPR;
          const int c = (u % VPR) * VE;
          const int prow = isx ? row : BM + row;
          const uint4 val =
              *reinterpret_cast<const uint4 *>(stage + ((sl * (BM + EPAD) + prow) * kBK + c) * EB);
          float f[VE];
          unpack16(val, f);
          // x rows then W rows, both row-major with a padded stride: the 16-byte
          // stores of a warp spread over all banks
          float *dst = smem + sl * SLICE + prow * XS + c;
#pragma unroll
          for (int e = 0; e < VE; e += 4)
            *reinterpret_cast<float4 *>(dst + e) = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
        }
      }
    };

#pragma unroll
    for (int s = 0; s < kRouterStages - 1; ++s) issue(s);
    for (int it = 0; it < n_iter; ++it) {
      cp_async_wait<kRouterStages - 2>();  // this thread's copies of iteration `it` landed
      __syncthreads();                      // everyone is done computing on the fp32 tile
      convert(it);
      issue(it + kRouterStages - 1);        // refills the raw stage converted last iteration
      __syncthreads();
      const float *xs = smem + ks * SLICE;
      const float *wsm = xs + BM * XS;
#pragma unroll 2
      for (int kk = 0; kk < kBK; kk += 4) {
        float xv[TM][4];
#pragma unroll
        for (int i = 0; i < TM; ++i) {
          const float4 q = *reinterpret_cast<const float4 *>(xs + (tm * TM + i) * XS + kk);
          xv[i][0] = q.x; xv[i][1] = q.y; xv[i][2] = q.z; xv[i][3] = q.w;
        }
        // this thread's experts are tn + (EPAD/TN)*j: the float4 reads of W rows by
        // the lanes of a warp fall in distinct banks
#pragma unroll
        for (int j = 0; j < TN; ++j) {
          const float4 q = *reinterpret_cast<const float4 *>(wsm + (tn + (EPAD / TN) * j) * XS + kk);
#pragma unroll
          for (int i = 0; i < TM; ++i) {
            acc[i][j] = fmaf(xv[i][0], q.x, acc[i][j]);
            acc[i][j] = fmaf(xv[i][1], q.y, acc[i][j]);
            acc[i][j] = fmaf(xv[i][2], q.z, acc[i][j]);
            acc[i][j] = fmaf(xv[i][3], q.w, acc[i][j]);
          }
        }
      }
    }
    cp_async_wait<0>();
    __syncthreads();
    // reduce the K slices in a fixed order into lg
    for (int s = 0; s < KS; ++s) {
      if (ks == s) {
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
          for (int j = 0; j < TN; ++j) {
            float *p = lg + (tm * TM + i) * LDL + tn + (EPAD / TN) * j;
            *p = (s == 0) ? acc[i][j] : *p + acc[i][j];
          }
      }
      __syncthreads();
    }
    // biases, then write the logits out
    for (int i = tid; i < BM * EPAD; i += kRouterThreads) {
      const int m = i / EPAD, e = i % EPAD;
      if (e < E) {
        float v = lg[m * LDL + e];
        if (a.b_router) v += a.b_router[e];
        if (a.logit_bias) v += a.logit_bias[e];
        lg[m * LDL + e] = v;
        if (a.logits_out && t0 + m < T) a.logits_out[(size_t)(t0 + m) * E + e] = v;
      }
    }
  } else {
    // logits are an input
    for (int i = tid; i < BM * EPAD; i += kRouterThreads) {
      const int m = i / EPAD, e = i % EPAD;
      if (e < E) lg[m * LDL + e] = (t0 + m < T) ? a.logits_in[(size_t)(t0 + m) * E + e] : 0.f;
    }
  }
  __syncthreads();

  // ------------------------------------------------ softmax + top-k, warp per token
  const int warp = tid >> 5, lane = tid & 31;
  constexpr int EPL = (EPAD + 31) / 32;  // experts per lane
  for (int m = warp; m < BM; m += kRouterThreads / 32) {
    const int t = t0 + m;
    if (t >= T) break;
    float z[EPL];
    bool taken[EPL];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      const float v = (e < E) ? lg[m * LDL + e] : -INFINITY;
      z[j] = (v != v) ? -INFINITY : v;  // a NaN logit never wins a slot
      taken[j] = false;
      mx = fmaxf(mx, z[j]);
    }
    mx = warp_max(mx);
    float ex[EPL], ssum = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      ex[j] = (lane + 32 * j < E) ? expf(z[j] - mx) : 0.f;
      ssum += ex[j];
    }
    ssum = warp_sum(ssum);
    const float inv_s = 1.f / ssum;
    // probabilities back into the tile (for the P_i partial sums)
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = lane + 32 * j;
      if (e < E) lg[m * LDL + e] = ex[j] * inv_s;
    }
    if (lane == 0) lse_s[m] = mx + logf(ssum);
    // k rounds of warp argmax
    float sel_v[kMaxTopK];
    int sel_i[kMaxTopK];
#pragma unroll
    for (int s = 0; s < kMaxTopK; ++s) {
      if (s < k) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
          const int e = lane + 32 * j;
          if (e < E && !taken[j] && (z[j] > bv || (z[j] == bv && e < bi))) { bv = z[j]; bi = e; }
        }
        warp_argmax(bv, bi);
        sel_v[s] = bv;
        sel_i[s] = bi;
#pragma unroll
        for (int j = 0; j < EPL; ++j)
          if (lane + 32 * j == bi) taken[j] = true;
      }
    }
    if (lane == 0) {
      float g[kMaxTopK];
      float gs = 0.f;
      if (a.gate_mode == MOE_GATE_TOPK_SOFTMAX) {
#pragma unroll
        for (int s = 0; s < kMaxTopK; ++s)
          if (s < k) { g[s] = expf(sel_v[s] - sel_v[0]); gs += g[s]; }
        const float inv = 1.f / gs;
#pragma unroll
        for (int s = 0; s < kMaxTopK; ++s) if (s < k) g[s] *= inv;
      } else {
#pragma unroll
        for (int s = 0; s < kMaxTopK; ++s)
          if (s < k) { g[s] = expf(sel_v[s] - mx) * inv_s; gs += g[s]; }
        if (a.gate_mode == MOE_GATE_SOFTMAX_TOPK_RENORM) {
#pragma unroll
          for (int s = 0; s < kMaxTopK; ++s) if (s < k) g[s] = g[s] / gs;
        }
      }
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s) {
        if (s < k) {
          a.topk_idx[(size_t)t * k + s] = sel_i[s];
          a.topk_gate[(size_t)t * k + s] = g[s];
          if (sel_i[s] < E) atomicAdd(&cnt[sel_i[s]], 1);
        }
      }
    }
  }
  __syncthreads();

  // -------------------------------------------- per-tile histogram and partial sums
  const int NT = gridDim.x;
  const int rows = min(BM, T - t0);
  for (int e = tid; e < E; e += kRouterThreads) {
    if (a.tile_counts) a.tile_counts[(size_t)e * NT + tile] = cnt[e];
    if (a.tile_p) {
      float s = 0.f;
      for (int m = 0; m < rows; ++m) s += lg[m * LDL + e];
      a.tile_p[(size_t)e * NT + tile] = s;
    }
  }
  if (tid == 0 && a.tile_z) {
    float s = 0.f;
    for (int m = 0; m < rows; ++m) s += lse_s[m] * lse_s[m];
    a.tile_z[tile] = s;
  }
}

template <typename ET, int EPAD>
cudaError_t launch_router_t(const RouterArgs &a, cudaStream_t st) {
  const int smem = RouterSmem<EPAD>::bytes(sizeof(ET));
  static std::atomic<bool> attr_done[64];  // idempotent: a racing second call sets the same value
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!attr_done[dev & 63].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(k_router<ET, EPAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_done[dev & 63].store(true, std::memory_order_release);
  }
  const int NT = ceil_div(a.T, RouterShape<EPAD>::BM);
  k_router<ET, EPAD><<<NT, kRouterThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int EPAD>
cudaError_t launch_router_e(const RouterArgs &a, int dtype, cudaStream_t st) {
  return dtype == MOE_DTYPE_F32 ? launch_router_t<float, EPAD>(a, st)
                                : launch_router_t<__nv_bfloat16, EPAD>(a, st);
}

// --------------------------------------------------------- GEMV router, E <= 8
// A skinny GEMM (N <= 8) over a long K: W_r [E, d] is staged once in shared memory,
// each warp streams the rows of 4 tokens with many 16-byte loads in flight (lane l
// reads columns [8l, 8l+8) of every 256-column step for bf16), keeps 4 x 8 partial
// sums and folds them with a reduce-scatter shuffle tree (fixed order) so that lane
// l ends with the logit of token l/8, expert l%8. Softmax, top-k and the gates then
// run in groups of 8 lanes. Same token tiles, outputs and per-tile partials as the
// tiled router.
constexpr int kGemvTokensPerWarp = 4;
constexpr int kGemvUnroll = 4;

__device__ __forceinline__ float group8_max(float v) {
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o, 8));
  return v;
}
__device__ __forceinline__ float group8_sum(float v) {
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, 8);
  return v;
}

template <typename ET>
__global__ void __launch_bounds__(kRouterThreads)
k_router_gemv(RouterArgs a) {
  constexpr int BM = 32;  // router_bm(E) for E <= 32
  static_assert(BM == router_bm(8), "router tile must match the permute tiles");
  static_assert(BM == (kRouterThreads / 32) * kGemvTokensPerWarp, "one token quad per warp");
  constexpr int VE = Elem<ET>::kPerVec;
  extern __shared__ __align__(16) uint8_t wsm_raw[];
  const ET *wsm = reinterpret_cast<const ET *>(wsm_raw);  // [8][d]
  __shared__ int cnt[8];
  __shared__ float prob_s[BM][9];
  __shared__ float lse_s[BM];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E, d = a.d, T = a.T, k = a.k;
  const int t0 = blockIdx.x * BM;
  const int tile = blockIdx.x;
  if (tid < 8) cnt[tid] = 0;
  {  // stage W_r (rows >= E are zero)
    const int nv = 8 * d / VE;
    const uint4 *src = static_cast<const uint4 *>(a.w);
    uint4 *dst = reinterpret_cast<uint4 *>(wsm_raw);
    for (int v = tid; v < nv; v += kRouterThreads)
      dst[v] = (v < E * d / VE) ? __ldg(src + v) : make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();

  const ET *x = static_cast<const ET *>(a.x);
  float acc[kGemvTokensPerWarp][8];
#pragma unroll
  for (int i = 0; i < kGemvTokensPerWarp; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
  const ET *xrow[kGemvTokensPerWarp];
  bool tok_ok[kGemvTokensPerWarp];
#pragma unroll
  for (int i = 0; i < kGemvTokensPerWarp; ++i) {
    const int t = t0 + warp * kGemvTokensPerWarp + i;
    tok_ok[i] = t < T;
    xrow[i] = x + (size_t)(tok_ok[i] ? t : 0) * d;
  }
  constexpr int STEP = 32 * VE;
  for (int c0 = 0; c0 < d; c0 += STEP * kGemvUnroll) {
    uint4 xv[kGemvUnroll][kGemvTokensPerWarp];
#pragma unroll
    for (int u = 0; u < kGemvUnroll; ++u) {
      const int c = c0 + u * STEP + lane * VE;
#pragma unroll
      for (int i = 0; i < kGemvTokensPerWarp; ++i)
        xv[u][i] = (tok_ok[i] && c < d) ? __ldg(reinterpret_cast<const uint4 *>(xrow[i] + c))
                                        : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kGemvUnroll; ++u) {
      const int c = c0 + u * STEP + lane * VE;
      if (c >= d) break;
      float xf[kGemvTokensPerWarp][VE];
#pragma unroll
      for (int i = 0; i < kGemvTokensPerWarp; ++i) unpack16(xv[u][i], xf[i]);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float wf[VE];
        unpack16(*reinterpret_cast<const uint4 *>(wsm + (size_t)e * d + c), wf);
#pragma unroll
        for (int i = 0; i < kGemvTokensPerWarp; ++i)
#pragma unroll
          for (int j = 0; j < VE; ++j) acc[i][e] = fmaf(xf[i][j], wf[j], acc[i][e]);
      }
    }
  }
  // reduce-scatter over the warp: 32 partial sums -> lane l holds q = l = 8*i + e
  float v[32];
#pragma unroll
  for (int i = 0; i < kGemvTokensPerWarp; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) v[i * 8 + e] = acc[i][e];
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int q = 0; q < o; ++q) {
      const float send = upper ? v[q] : v[q + o];
      const float keep = upper ? v[q + o] : v[q];
      v[q] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  const int iq = lane >> 3, e = lane & 7;
  const int m = warp * kGemvTokensPerWarp + iq;  // token inside the tile
  const int t = t0 + m;
  const bool valid_e = e < E;
  float z = v[0];
  if (a.b_router && valid_e) z += a.b_router[e];
  if (a.logit_bias && valid_e) z += a.logit_bias[e];
  if (a.logits_out && valid_e && t < T) a.logits_out[(size_t)t * E + e] = z;
  z = (!valid_e || z != z) ? -INFINITY : z;  // padding experts and NaN never win a slot
  const float mx = group8_max(z);
  const float ex = valid_e ? expf(z - mx) : 0.f;
  const float ssum = group8_sum(ex);
  const float p = ex / ssum;
  prob_s[m][e] = valid_e ? p : 0.f;
  if (e == 0) lse_s[m] = mx + logf(ssum);
  // k rounds of argmax inside the 8-lane group (value desc, index asc)
  bool taken = false;
  int my_slot = -1;
  float top0 = 0.f;
  for (int s = 0; s < k; ++s) {
    float bv = taken ? -INFINITY : z;
    int bi = taken ? 0x7fffffff : e;
    if (taken) bv = -INFINITY;
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o, 8);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o, 8);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (s == 0) top0 = bv;
    if (bi == e && !taken) { taken = true; my_slot = s; }
  }
  float g;
  if (a.gate_mode == MOE_GATE_TOPK_SOFTMAX) {
    const float es = taken ? expf(z - top0) : 0.f;
    g = es / group8_sum(es);
  } else {
    const float ps = taken ? ex / ssum : 0.f;
    g = (a.gate_mode == MOE_GATE_SOFTMAX_TOPK_RENORM) ? ps / group8_sum(ps) : ps;
  }
  if (taken && t < T) {
    a.topk_idx[(size_t)t * k + my_slot] = e;
    a.topk_gate[(size_t)t * k + my_slot] = g;
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  const int NT = gridDim.x;
  const int rows = min(BM, T - t0);
  if (tid < E) {
    if (a.tile_counts) a.tile_counts[(size_t)tid * NT + tile] = cnt[tid];
    if (a.tile_p) {
      float sp = 0.f;
      for (int r = 0; r < rows; ++r) sp += prob_s[r][tid];
      a.tile_p[(size_t)tid * NT + tile] = sp;
    }
  }
  if (tid == 0 && a.tile_z) {
    float sz = 0.f;
    for (int r = 0; r < rows; ++r) sz += lse_s[r] * lse_s[r];
    a.tile_z[tile] = sz;
  }
}

template <typename ET>
cudaError_t launch_router_gemv(const RouterArgs &a, cudaStream_t st) {
  const int smem = 8 * a.d * (int)sizeof(ET);
  static int attr_bytes[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (smem > 48 * 1024 && attr_bytes[dev & 63] < smem) {
    e = cudaFuncSetAttribute(k_router_gemv<ET>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_bytes[dev & 63] = smem;
  }
  k_router_gemv<ET><<<ceil_div(a.T, 32), kRouterThreads, smem, st>>>(a);
  return cudaGetLastError();
}

// Histogram of a given topk_idx per token tile (the standalone permute path).
__global__ void __launch_bounds__(256) k_tile_counts(const int32_t *__restrict__ topk_idx, int T,
                                                     int k, int E, int bm,
                                                     int32_t *__restrict__ tile_counts,
                                                     int32_t *err) {
  __shared__ int cnt[kMaxExperts];
  const int tile = blockIdx.x, NT = gridDim.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int p0 = tile * bm * k;
  const int p1 = min(T, (tile + 1) * bm) * k;
  for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
    const int e = topk_idx[p];
    if (e >= 0 && e < E)
      atomicAdd(&cnt[e], 1);
    else
      report_error(err, MOE_DEVERR_EXPERT_INDEX, p);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) tile_counts[(size_t)e * NT + tile] = cnt[e];
}

}  // namespace

cudaError_t launch_router(const RouterArgs &a, int dtype, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int E = a.E;
  // the fused noisy gate exists on the tensor-core router only
  if (a.w_noise != nullptr && !(dtype == MOE_DTYPE_BF16 && router_tc_supported(a)))
    return cudaErrorInvalidValue;
  // bf16: the tensor-core router (x W_r^T is a contraction; on the CUDA cores it is
  // bound by the FMA rate rather than by reading x)
  if (dtype == MOE_DTYPE_BF16 && router_tc_supported(a)) return launch_router_tc(a, st);
  // fp32, small expert counts with W_r fitting in shared memory: the GEMV-shaped router
  if (E <= 8 && a.x != nullptr &&
      8LL * a.d * (dtype == MOE_DTYPE_F32 ? 4 : 2) <= 96LL * 1024)
    return dtype == MOE_DTYPE_F32 ? launch_router_gemv<float>(a, st)
                                  : launch_router_gemv<__nv_bfloat16>(a, st);
  if (E <= 8) return launch_router_e<8>(a, dtype, st);
  if (E <= 16) return launch_router_e<16>(a, dtype, st);
  if (E <= 32) return launch_router_e<32>(a, dtype, st);
  if (E <= 64) return launch_router_e<64>(a, dtype, st);
  if (E <= 128) return launch_router_e<128>(a, dtype, st);
  return launch_router_e<256>(a, dtype, st);
}

// Noisy Top-K Gating (youngju.dev (ja) "TopKGating", training mode): the router
// logits plus softplus(x W_noise^T) times the caller's standard normal draws.
// softplus switches to the identity above 20, as F.softplus does.
__global__ void __launch_bounds__(256) k_noisy_logits(float *__restrict__ z,
                                                      const float *__restrict__ zn,
                                                      const float *__restrict__ eps, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const float v = zn[i];
    const float sp = v > 20.f ? v : log1pf(expf(v));
    z[i] = z[i] + sp * eps[i];
  }
}

cudaError_t launch_noisy_logits(float *z, const float *zn, const float *eps, size_t n,
                                cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const size_t blocks = std::min<size_t>((n + 255) / 256, 148 * 16);
  k_noisy_logits<<<(unsigned)blocks, 256, 0, st>>>(z, zn, eps, n);
  return cudaGetLastError();
}

cudaError_t launch_tile_counts(const int32_t *topk_idx, int T, int k, int E, int32_t *tile_counts,
                               int32_t *err, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int bm = router_bm(E);
  k_tile_counts<<<ceil_div(T, bm), 256, 0, st>>>(topk_idx, T, k, E, bm, tile_counts, err);
  return cudaGetLastError();
}

}  // namespace moe

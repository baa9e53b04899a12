// Router GEMM (CUDA cores, fp32 accumulate) fused with softmax, top-k, gates,
// per-tile expert histogram and per-tile softmax/logsumexp partial sums.
//
// Gating network: youngju.dev (zh) "GatingNetwork" / "SwitchRouter" and the
// devtips.kr "MoELayer" gate (a Linear over d_model, with or without bias);
// gate modes: top-k then softmax (GatingNetwork, MixtralMoELayer), softmax then
// top-k renormalised (youngju.dev ja "TopKGating"), softmax then top-1 raw
// (SwitchRouter). Top-k is taken on the fp32 logits in every mode; equal logits
// go to the lower expert index first.
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kRouterThreads = 256;
constexpr int kBK = 32;  // K elements per slice per iteration

template <int EPAD> struct RouterShape;
template <> struct RouterShape<8>   { static constexpr int BM = 32, TM = 1, TN = 8, KS = 8; };
template <> struct RouterShape<16>  { static constexpr int BM = 32, TM = 1, TN = 8, KS = 4; };
template <> struct RouterShape<32>  { static constexpr int BM = 32, TM = 2, TN = 8, KS = 4; };
template <> struct RouterShape<64>  { static constexpr int BM = 64, TM = 4, TN = 8, KS = 2; };
template <> struct RouterShape<128> { static constexpr int BM = 64, TM = 4, TN = 8, KS = 1; };
template <> struct RouterShape<256> { static constexpr int BM = 32, TM = 4, TN = 8, KS = 1; };

template <typename ET, int EPAD>
__global__ void __launch_bounds__(kRouterThreads)
k_router(RouterArgs a) {
  using S = RouterShape<EPAD>;
  constexpr int BM = S::BM, TM = S::TM, TN = S::TN, KS = S::KS;
  static_assert(BM == router_bm(EPAD), "router tile must match the permute tiles");
  static_assert((BM / TM) * (EPAD / TN) * KS == kRouterThreads, "thread layout");
  constexpr int VE = Elem<ET>::kPerVec;
  constexpr int XS = kBK + 4;                      // padded x row (floats)
  constexpr int SLICE = BM * XS + kBK * EPAD;      // floats per K slice
  constexpr int TILE_FLOATS = KS * SLICE;
  constexpr int LG_FLOATS = BM * (EPAD + 1);
  constexpr int SMEM_FLOATS = TILE_FLOATS > LG_FLOATS ? TILE_FLOATS : LG_FLOATS;
  __shared__ __align__(16) float smem[SMEM_FLOATS];
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

    // global -> register staging of one iteration (KS slices x kBK columns)
    constexpr int XV = BM * KS * kBK / VE;      // x vectors per iteration
    constexpr int WV = EPAD * KS * kBK / VE;    // W vectors per iteration
    constexpr int XPT = (XV + kRouterThreads - 1) / kRouterThreads;
    constexpr int WPT = (WV + kRouterThreads - 1) / kRouterThreads;
    uint4 xr[XPT], wr[WPT];
    const ET *x = static_cast<const ET *>(a.x);
    const ET *w = static_cast<const ET *>(a.w);
    const int kstep = KS * kBK;
    const int n_iter = ceil_div(d, kstep);

    auto load_iter = [&](int it) {
      const int kb = it * kstep;
#pragma unroll
      for (int q = 0; q < XPT; ++q) {
        const int v = tid + q * kRouterThreads;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (v < XV) {
          const int row = v / (KS * kBK / VE);
          const int col = (v % (KS * kBK / VE)) * VE + kb;
          if (t0 + row < T && col < d)
            u = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)(t0 + row) * d + col));
        }
        xr[q] = u;
      }
#pragma unroll
      for (int q = 0; q < WPT; ++q) {
        const int v = tid + q * kRouterThreads;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (v < WV) {
          const int e = v / (KS * kBK / VE);
          const int col = (v % (KS * kBK / VE)) * VE + kb;
          if (e < E && col < d)
            u = __ldg(reinterpret_cast<const uint4 *>(w + (size_t)e * d + col));
        }
        wr[q] = u;
      }
    };
    auto store_iter = [&]() {
#pragma unroll
      for (int q = 0; q < XPT; ++q) {
        const int v = tid + q * kRouterThreads;
        if (v < XV) {
          const int row = v / (KS * kBK / VE);
          const int cc = (v % (KS * kBK / VE)) * VE;  // column inside the iteration
          const int sl = cc / kBK, c = cc % kBK;
          float f[VE];
          unpack16(xr[q], f);
          float *dst = smem + sl * SLICE + row * XS + c;
#pragma unroll
          for (int u = 0; u < VE; u += 4)
            *reinterpret_cast<float4 *>(dst + u) = make_float4(f[u], f[u + 1], f[u + 2], f[u + 3]);
        }
      }
#pragma unroll
      for (int q = 0; q < WPT; ++q) {
        const int v = tid + q * kRouterThreads;
        if (v < WV) {
          const int e = v / (KS * kBK / VE);
          const int cc = (v % (KS * kBK / VE)) * VE;
          const int sl = cc / kBK, c = cc % kBK;
          float f[VE];
          unpack16(wr[q], f);
          float *dst = smem + sl * SLICE + BM * XS;
#pragma unroll
          for (int u = 0; u < VE; ++u) dst[(c + u) * EPAD + e] = f[u];
        }
      }
    };

    load_iter(0);
    for (int it = 0; it < n_iter; ++it) {
      __syncthreads();  // previous compute finished with the tiles
      store_iter();
      __syncthreads();
      if (it + 1 < n_iter) load_iter(it + 1);
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
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float wv[TN];
#pragma unroll
          for (int j = 0; j < TN; j += 4) {
            const float4 q = *reinterpret_cast<const float4 *>(wsm + (kk + u) * EPAD + tn * TN + j);
            wv[j] = q.x; wv[j + 1] = q.y; wv[j + 2] = q.z; wv[j + 3] = q.w;
          }
#pragma unroll
          for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(xv[i][u], wv[j], acc[i][j]);
        }
      }
    }
    __syncthreads();
    // reduce the K slices in a fixed order into lg
    for (int s = 0; s < KS; ++s) {
      if (ks == s) {
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
          for (int j = 0; j < TN; ++j) {
            float *p = lg + (tm * TM + i) * LDL + tn * TN + j;
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

template <int EPAD>
cudaError_t launch_router_e(const RouterArgs &a, int dtype, cudaStream_t st) {
  const int NT = ceil_div(a.T, RouterShape<EPAD>::BM);
  if (dtype == MOE_DTYPE_F32)
    k_router<float, EPAD><<<NT, kRouterThreads, 0, st>>>(a);
  else
    k_router<__nv_bfloat16, EPAD><<<NT, kRouterThreads, 0, st>>>(a);
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
  if (E <= 8) return launch_router_e<8>(a, dtype, st);
  if (E <= 16) return launch_router_e<16>(a, dtype, st);
  if (E <= 32) return launch_router_e<32>(a, dtype, st);
  if (E <= 64) return launch_router_e<64>(a, dtype, st);
  if (E <= 128) return launch_router_e<128>(a, dtype, st);
  return launch_router_e<256>(a, dtype, st);
}

cudaError_t launch_tile_counts(const int32_t *topk_idx, int T, int k, int E, int32_t *tile_counts,
                               int32_t *err, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int bm = router_bm(E);
  k_tile_counts<<<ceil_div(T, bm), 256, 0, st>>>(topk_idx, T, k, E, bm, tile_counts, err);
  return cudaGetLastError();
}

}  // namespace moe

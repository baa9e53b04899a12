// fp32 expert FFNs on CUDA cores (FFMA), for fp32 layers.
//
// Tensor cores have no fp32 MMA kind (tf32 rounds the operands to 10-bit
// mantissas), so an fp32 layer runs its two grouped GEMMs here, exactly in fp32:
//   h = act(x W1^T + b1)  or  silu(x Wg^T) * (x Wu^T)   (SwiGLUExpert)
//   o = h W2^T + b2
// Experts: devtips.kr "MoELayer" (ReLU MLP with bias), youngju.dev (zh)
// "MoELayer" (GELU MLP), youngju.dev "SwiGLUExpert".
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int BM = kRowTile, BN = 64, BK = 32;
constexpr int kAPer = BM * BK / 256, kBPer = BN * BK / 256;  // slice elements per thread
constexpr int TM = 8, TN = 4;  // per-thread micro tile; (BM/TM)*(BN/TN) = 256 threads

struct SimtGemm {
  const float *a;        // [rows, K]
  const int32_t *offsets, *mprefix;
  int G, K, N;
  const float *b, *b3;   // [G, N, K] (b3: SwiGLU up projection) or nullptr
  const float *bias;     // [G, N] or nullptr
  float *out;            // [rows, N]
  int act;               // MOE_ACT_* for the up projection; -1: plain (down projection)
};

__device__ __forceinline__ float apply_act(int act, float v) {
  if (act == MOE_ACT_RELU) return fmaxf(v, 0.f);
  if (act == MOE_ACT_GELU) return 0.5f * v * (1.f + erff(v * 0.70710678118654752f));
  return v;
}

template <bool kSwiGLU>
__global__ void __launch_bounds__(256) k_simt_gemm(SimtGemm s) {
  __shared__ __align__(16) float As[BK][BM + 4];
  __shared__ __align__(16) float Bs[BK][BN + 4];
  __shared__ __align__(16) float B3s[kSwiGLU ? BK : 1][BN + 4];
  __shared__ int grp_s, row0_s, nrows_s;
  const int tid = threadIdx.x;
  const int mt = blockIdx.y;
  if (tid == 0) {
    int g = -1;
    if (mt < s.mprefix[s.G]) {
      int lo = 0, hi = s.G - 1;  // last g with mprefix[g] <= mt
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.mprefix[mid] <= mt) lo = mid; else hi = mid - 1;
      }
      g = lo;
    }
    grp_s = g;
    if (g >= 0) {
      row0_s = s.offsets[g] + (mt - s.mprefix[g]) * BM;
      nrows_s = min(BM, s.offsets[g + 1] - row0_s);
    }
  }
  __syncthreads();
  const int g = grp_s;
  if (g < 0) return;
  const int row0 = row0_s, nrows = nrows_s;
  const int n0 = blockIdx.x * BN;
  const int tx = tid % (BN / TN), ty = tid / (BN / TN);
  const float *bw = s.b + (size_t)g * s.N * s.K;
  const float *bw3 = kSwiGLU ? s.b3 + (size_t)g * s.N * s.K : nullptr;
  float acc[TM][TN], acc3[kSwiGLU ? TM : 1][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      acc[i][j] = 0.f;
      if (kSwiGLU) acc3[i][j] = 0.f;
    }
  // the next K slice is read from global memory into registers while this one is
  // multiplied out of shared memory (rows of 32 consecutive K values per 32 threads)
  float ra[kAPer], rb[kBPer], rb3[kSwiGLU ? kBPer : 1];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int j = 0; j < kAPer; ++j) {
      const int i = tid + 256 * j, m = i / BK, kk = i % BK;
      ra[j] = (m < nrows && k0 + kk < s.K) ? s.a[(size_t)(row0 + m) * s.K + k0 + kk] : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kBPer; ++j) {
      const int i = tid + 256 * j, n = i / BK, kk = i % BK;
      const bool ok = n0 + n < s.N && k0 + kk < s.K;
      rb[j] = ok ? bw[(size_t)(n0 + n) * s.K + k0 + kk] : 0.f;
      if (kSwiGLU) rb3[j] = ok ? bw3[(size_t)(n0 + n) * s.K + k0 + kk] : 0.f;
    }
  };
  fetch(0);
  for (int k0 = 0; k0 < s.K; k0 += BK) {
#pragma unroll
    for (int j = 0; j < kAPer; ++j) {
      const int i = tid + 256 * j;
      As[i % BK][i / BK] = ra[j];
    }
#pragma unroll
    for (int j = 0; j < kBPer; ++j) {
      const int i = tid + 256 * j;
      Bs[i % BK][i / BK] = rb[j];
      if (kSwiGLU) B3s[i % BK][i / BK] = rb3[j];
    }
    __syncthreads();
    if (k0 + BK < s.K) fetch(k0 + BK);
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float av[TM], bv[TN], bv3[TN];
#pragma unroll
      for (int i = 0; i < TM; i += 4) {
        const float4 q = *reinterpret_cast<const float4 *>(&As[kk][ty * TM + i]);
        av[i] = q.x; av[i + 1] = q.y; av[i + 2] = q.z; av[i + 3] = q.w;
      }
      const float4 qb = *reinterpret_cast<const float4 *>(&Bs[kk][tx * TN]);
      bv[0] = qb.x; bv[1] = qb.y; bv[2] = qb.z; bv[3] = qb.w;
      if (kSwiGLU) {
        const float4 q3 = *reinterpret_cast<const float4 *>(&B3s[kk][tx * TN]);
        bv3[0] = q3.x; bv3[1] = q3.y; bv3[2] = q3.z; bv3[3] = q3.w;
      }
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) {
          acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
          if (kSwiGLU) acc3[i][j] = fmaf(av[i], bv3[j], acc3[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int m = ty * TM + i;
    if (m >= nrows) continue;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const int n = n0 + tx * TN + j;
      if (n >= s.N) continue;
      float v;
      if (kSwiGLU) {
        const float gt = acc[i][j];
        v = (gt / (1.f + expf(-gt))) * acc3[i][j];
      } else {
        v = acc[i][j];
        if (s.bias) v += s.bias[(size_t)g * s.N + n];
        v = apply_act(s.act, v);
      }
      s.out[(size_t)(row0 + m) * s.N + n] = v;
    }
  }
}

}  // namespace

cudaError_t launch_ffn_simt(const GroupedFfnArgs &a, cudaStream_t st) {
  if (a.m_tiles_ub <= 0) return cudaSuccess;
  SimtGemm up{static_cast<const float *>(a.a), a.offsets, a.mprefix, a.G, a.d, a.F,
              static_cast<const float *>(a.w1), static_cast<const float *>(a.w3), a.b1,
              static_cast<float *>(a.h), a.act};
  dim3 g1(ceil_div(a.F, BN), a.m_tiles_ub);
  if (a.act == MOE_ACT_SWIGLU)
    k_simt_gemm<true><<<g1, 256, 0, st>>>(up);
  else
    k_simt_gemm<false><<<g1, 256, 0, st>>>(up);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  SimtGemm down{static_cast<const float *>(a.h), a.offsets, a.mprefix, a.G, a.F, a.d,
                static_cast<const float *>(a.w2), nullptr, a.b2,
                static_cast<float *>(a.out), -1};
  dim3 g2(ceil_div(a.d, BN), a.m_tiles_ub);
  k_simt_gemm<false><<<g2, 256, 0, st>>>(down);
  return cudaGetLastError();
}

}  // namespace moe

// Routing of decode-sized batches in one CTA: at most 8 tokens over at most 32
// experts. The router logits on the CUDA cores, softmax, top-k and gates, and the
// expert layout that the permute step and the grouped GEMM read (counts, capacity,
// offsets, the 128-row tile prefix), in one launch instead of a router kernel
// followed by the scan.
//
// Gating network: youngju.dev (zh) "GatingNetwork" / "SwitchRouter" and the
// devtips.kr "MoELayer" gate (a Linear over d_model, with or without bias); gate
// modes as in the other routers: top-k then softmax (GatingNetwork,
// MixtralMoELayer), softmax then top-k renormalised (youngju.dev ja "TopKGating"),
// softmax then top-1 raw (SwitchRouter). Capacity floor(cf T k / E) as in
// "SwitchRouter" and the devtips.kr capacity snippet.
//
// The logits: thread j of the CTA takes the columns 4 j + 2048 i of x and
// W_r (8-byte loads, coalesced over the warp) for blocks of 4 tokens x 8 experts;
// each warp reduces its 32 partial sums to one per lane (a fixed shuffle pattern),
// and the warps' partials are added in warp order. Then a warp per token takes the
// selection, a lane per expert: the maximum and the k argmax rounds
// (value, then lower expert index) and the exp sum over fixed shuffle trees. No
// value depends on timing.
#include <cuda_bf16.h>

#include <atomic>

#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kSrThreads = 512;
constexpr int kSrWarps = kSrThreads / 32;
constexpr int kSrTok = 4;  // tokens per accumulator block
constexpr int kSrExp = 8;  // experts per accumulator block

__device__ __forceinline__ bool sr_better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// the best (value, then lower index) over the warp's lanes (a fixed xor tree)
__device__ __forceinline__ void sr_argmax(float &v, int &i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (sr_better(ov, oi, v, i)) { v = ov; i = oi; }
  }
}

__device__ __forceinline__ void bf16x4(uint2 u, float (&f)[4]) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}

__global__ void __launch_bounds__(kSrThreads, 1) k_route_small(SmallRouteArgs a) {
  extern __shared__ float red[];  // [blocks][kSrWarps][32]
  __shared__ float lg[kSmallRouteMaxT][kSmallRouteMaxE + 1];
  __shared__ int sel[kSmallRouteMaxT * kMaxTopK];
  const RouterArgs &r = a.r;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = r.T, E = r.E, k = r.k, d = r.d;
  const int ntg = ceil_div(T, kSrTok), neg = ceil_div(E, kSrExp);
  // every output below is read by the kernels before this one's successors
  pdl_wait();
  pdl_trigger();
  const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(r.x);
  const __nv_bfloat16 *w = static_cast<const __nv_bfloat16 *>(r.w);

  // ---- 1. partial dot products, one (token block, expert block) at a time
  for (int eg = 0; eg < neg; ++eg) {
    for (int tg = 0; tg < ntg; ++tg) {
      float acc[kSrTok][kSrExp];
#pragma unroll
      for (int i = 0; i < kSrTok; ++i)
#pragma unroll
        for (int e = 0; e < kSrExp; ++e) acc[i][e] = 0.f;
      for (int c = 4 * tid; c < d; c += 4 * kSrThreads) {
        float xf[kSrTok][4];
#pragma unroll
        for (int i = 0; i < kSrTok; ++i) {
          const int t = tg * kSrTok + i;
          const uint2 u = t < T ? __ldg(reinterpret_cast<const uint2 *>(x + (size_t)t * d + c))
                                : make_uint2(0u, 0u);
          bf16x4(u, xf[i]);
        }
#pragma unroll
        for (int e = 0; e < kSrExp; ++e) {
          const int ee = eg * kSrExp + e;
          float wf[4];
          const uint2 u = ee < E ? __ldg(reinterpret_cast<const uint2 *>(w + (size_t)ee * d + c))
                                 : make_uint2(0u, 0u);
          bf16x4(u, wf);
#pragma unroll
          for (int i = 0; i < kSrTok; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][e] = fmaf(xf[i][j], wf[j], acc[i][e]);
        }
      }
      // reduce over the warp: value q = 8 i + e ends, summed, in lane q
      float v[32];
#pragma unroll
      for (int i = 0; i < kSrTok; ++i)
#pragma unroll
        for (int e = 0; e < kSrExp; ++e) v[i * kSrExp + e] = acc[i][e];
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
      red[((size_t)(eg * ntg + tg) * kSrWarps + warp) * 32 + lane] = v[0];
    }
  }
  __syncthreads();

  // ---- 2. logits: the warps' partials added in warp order
  for (int i = tid; i < neg * ntg * 32; i += kSrThreads) {
    const int blk = i >> 5, q = i & 31;
    const int eg = blk / ntg, tg = blk - eg * ntg;
    const int t = tg * kSrTok + (q >> 3), e = eg * kSrExp + (q & 7);
    if (t < T && e < E) {
      const float *p = red + (size_t)blk * kSrWarps * 32 + q;
      float s = p[0];
#pragma unroll
      for (int ww = 1; ww < kSrWarps; ++ww) s += p[ww * 32];
      lg[t][e] = s;
    }
  }
  __syncthreads();

  // ---- 3. selection, gates and outputs: a warp per token, a lane per expert
  for (int t = warp; t < T; t += kSrWarps) {
    const int e = lane;
    float v = 0.f;
    if (e < E) {
      v = lg[t][e];
      if (r.b_router) v += r.b_router[e];
      if (r.logit_bias) v += r.logit_bias[e];
      if (r.logits_out) r.logits_out[(size_t)t * E + e] = v;
    }
    const float z = (e >= E || v != v) ? -INFINITY : v;  // padding, NaN never win
    float bv = z;
    int bi = e;
    sr_argmax(bv, bi);
    const float mx = bv;
    float tv[kMaxTopK];
    int ti[kMaxTopK];
    tv[0] = bv;
    ti[0] = bi;
#pragma unroll
    for (int s = 1; s < kMaxTopK; ++s) {
      if (s < k) {
        const bool below = z < tv[s - 1] || (z == tv[s - 1] && e > ti[s - 1]);
        float cv = below ? z : -INFINITY;
        int ci = below ? e : 0x7fffffff;
        sr_argmax(cv, ci);
        tv[s] = cv;
        ti[s] = ci;
      }
    }
    float ex = expf(z - mx);  // 0 for padding
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ex += __shfl_xor_sync(0xffffffffu, ex, o);
    const float ssum = ex;
    if (lane == 0) {
      const float inv_s = 1.f / ssum;
      float gv[kMaxTopK];
      float gs = 0.f;
      if (r.gate_mode == MOE_GATE_TOPK_SOFTMAX) {
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
        if (r.gate_mode == MOE_GATE_SOFTMAX_TOPK_RENORM) {
#pragma unroll
          for (int s = 0; s < kMaxTopK; ++s) if (s < k) gv[s] = gv[s] / gs;
        }
      }
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s) {
        if (s < k) {
          r.topk_idx[(size_t)t * k + s] = ti[s];
          r.topk_gate[(size_t)t * k + s] = gv[s];
          sel[t * k + s] = ti[s];
        }
      }
    }
  }
  __syncthreads();

  // ---- 4. counts, capacity, offsets, the 128-row tile prefix; the permute step's
  // per-tile bases are all zero (one token tile)
  if (warp == 0) {
    int c = 0;
    if (lane < E)
      for (int p = 0; p < T * k; ++p) c += sel[p] == lane;
    const int kept = (a.cap < 0) ? c : min(c, a.cap);
    const int mt = ceil_div(kept, kRowTile);
    int ik = kept, im = mt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vk = __shfl_up_sync(0xffffffffu, ik, o);
      const int vm = __shfl_up_sync(0xffffffffu, im, o);
      if (lane >= o) { ik += vk; im += vm; }
    }
    if (lane < E) {
      a.counts[lane] = c;
      a.offsets[lane] = ik - kept;
      a.mprefix[lane] = im - mt;
      a.tile_base[lane] = 0;
    }
    if (lane == 31) {
      a.offsets[E] = ik;
      a.mprefix[E] = im;
    }
    if (lane == 0 && a.sh_tbl) {
      a.sh_tbl[0] = 0;
      a.sh_tbl[1] = T;
      a.sh_tbl[2] = 0;
      a.sh_tbl[3] = ceil_div(T, kRowTile);
    }
  }
}

}  // namespace

bool small_route_supported(const RouterArgs &a) {
  return a.x != nullptr && a.w_noise == nullptr && a.T >= 1 && a.T <= kSmallRouteMaxT &&
         a.E >= 1 && a.E <= kSmallRouteMaxE && a.k >= 1 && a.k <= a.E && a.k <= kMaxTopK &&
         a.d % 4 == 0 && a.tile_p == nullptr && a.tile_z == nullptr;
}

cudaError_t launch_route_small(const SmallRouteArgs &a, cudaStream_t st) {
  if (!small_route_supported(a.r)) return cudaErrorInvalidValue;
  const int blocks = ceil_div(a.r.T, kSrTok) * ceil_div(a.r.E, kSrExp);
  const size_t smem = (size_t)blocks * kSrWarps * 32 * sizeof(float);
  static std::atomic<bool> attr_done[64];  // idempotent: a racing second call sets the same value
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!attr_done[dev & 63].load(std::memory_order_acquire)) {
    constexpr int kMaxSmem = (kSmallRouteMaxT / kSrTok) * (kSmallRouteMaxE / kSrExp) * kSrWarps * 32 *
                             (int)sizeof(float);
    e = cudaFuncSetAttribute(k_route_small, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e != cudaSuccess) return e;
    attr_done[dev & 63].store(true, std::memory_order_release);
  }
  return launch_pdl(k_route_small, dim3(1), dim3(kSrThreads), smem, st, a);
}

}  // namespace moe

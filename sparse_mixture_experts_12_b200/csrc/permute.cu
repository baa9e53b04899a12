// Histogram -> scan -> stable permutation with capacity drops, and the
// gate-weighted combine.
//
// Dispatch follows youngju.dev (zh) "SwitchRouter": per expert, the (token, slot)
// pairs routed to it are taken in token-major order and those whose position is
// >= capacity are dropped; capacity = floor(cf*T*k/E) (devtips.kr capacity
// snippet, with k). The kept pairs are laid out expert-contiguously, in token
// order inside each expert, which is what the grouped expert GEMM consumes.
// Combine is the gating equation y = sum_i G(x)_i E_i(x) of youngju.dev (ja),
// i.e. the masked scatter-add of the "MoELayer" listings, done as a gather.
//
// Everything is atomic-free in global memory and deterministic: ranks come from
// per-tile counts, an exclusive scan over (expert, tile), and in-tile warp matching.
#include "kernels.cuh"

namespace moe {

namespace {

// ----------------------------------------------------------------- block scan
template <int NTHREADS>
__device__ int block_inclusive_scan(int v, int *warp_buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_buf[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < NTHREADS / 32) ? warp_buf[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < NTHREADS / 32) warp_buf[lane] = w;
  }
  __syncthreads();
  if (warp > 0) v += warp_buf[warp - 1];
  return v;
}

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) k_scan(ScanArgs a) {
  __shared__ int warp_buf[32];
  __shared__ int seg_start[kMaxExperts + 1];
  __shared__ int kept_s[kMaxExperts];
  __shared__ float red[kScanThreads];
  const int E = a.E, NT = a.NT;
  const int N = E * NT;
  const int tid = threadIdx.x;
  const int chunk = ceil_div(N, kScanThreads);
  const int i0 = min(N, tid * chunk), i1 = min(N, i0 + chunk);

  int s = 0;
  for (int i = i0; i < i1; ++i) s += a.tile_counts[i];
  const int incl = block_inclusive_scan<kScanThreads>(s, warp_buf);
  int run = incl - s;
  for (int i = i0; i < i1; ++i) {
    if (i % NT == 0) seg_start[i / NT] = run;
    run += a.tile_counts[i];
  }
  if (tid == kScanThreads - 1) seg_start[E] = incl;
  __syncthreads();
  run = incl - s;
  for (int i = i0; i < i1; ++i) {
    a.tile_base[i] = run - seg_start[i / NT];
    run += a.tile_counts[i];
  }
  if (tid < E) {
    const int c = seg_start[tid + 1] - seg_start[tid];
    a.counts[tid] = c;
    kept_s[tid] = (a.cap < 0) ? c : min(c, a.cap);
  }
  __syncthreads();
  if (tid == 0) {
    int off = 0, mp = 0;
    for (int e = 0; e < E; ++e) {
      a.offsets[e] = off;
      a.mprefix[e] = mp;
      off += kept_s[e];
      mp += ceil_div(kept_s[e], kRowTile);
    }
    a.offsets[E] = off;
    a.mprefix[E] = mp;
    if (a.sh_tbl) {
      a.sh_tbl[0] = 0;
      a.sh_tbl[1] = a.T;
      a.sh_tbl[2] = 0;
      a.sh_tbl[3] = ceil_div(a.T, kRowTile);
    }
  }
  if (a.aux_out == nullptr) return;

  // ---- load-balancing statistics (fixed-order reductions, deterministic)
  int epow = 1;
  while (epow < E) epow <<= 1;
  const int G = kScanThreads / epow;  // threads per expert (>= 4)
  {
    const int e = tid / G, g = tid % G;
    float p = 0.f;
    if (e < E)
      for (int tl = g; tl < NT; tl += G) p += a.tile_p[(size_t)e * NT + tl];
    red[tid] = p;
    __syncthreads();
    for (int h = G / 2; h > 0; h >>= 1) {
      if (g < h) red[tid] += red[tid + h];
      __syncthreads();
    }
  }
  __shared__ float P_s[kMaxExperts];
  if (tid < E) P_s[tid] = red[tid * G] / (float)a.T;
  __syncthreads();
  float z = 0.f;
  for (int tl = tid; tl < NT; tl += kScanThreads) z += a.tile_z[tl];
  red[tid] = z;
  __syncthreads();
  for (int h = kScanThreads / 2; h > 0; h >>= 1) {
    if (tid < h) red[tid] += red[tid + h];
    __syncthreads();
  }
  if (tid == 0) {
    const double inv_tk = 1.0 / ((double)a.T * (double)a.k);
    double fp = 0.0, bsq = 0.0;
    for (int e = 0; e < E; ++e) {
      const double f = (double)(seg_start[e + 1] - seg_start[e]) * inv_tk;
      fp += f * (double)P_s[e];
      bsq += (f - 1.0 / E) * (f - 1.0 / E);
      a.aux_out[3 + e] = (float)f;
      a.aux_out[3 + E + e] = P_s[e];
    }
    a.aux_out[0] = (float)((double)a.alpha * E * fp);
    a.aux_out[1] = red[0] / (float)a.T;
    a.aux_out[2] = (float)bsq;
  }
}

// ------------------------------------------------------------------- scatter
constexpr int kScatterThreads = 256;

__global__ void __launch_bounds__(kScatterThreads) k_scatter(ScatterArgs a) {
  extern __shared__ int32_t sh[];
  const int E = a.E, k = a.k, T = a.T;
  const int bm = router_bm(E);
  const int tile = blockIdx.x, NT = gridDim.x;
  const int t0 = tile * bm;
  const int rows = min(bm, T - t0);
  const int P = rows * k;
  const int NC = ceil_div(bm * k, 32);
  int32_t *hist = sh;               // [NC][E]
  int32_t *prow = hist + NC * E;    // [bm*k]: in-chunk rank, then the destination row
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t *idx = a.topk_idx + (size_t)t0 * k;

  for (int i = tid; i < NC * E; i += kScatterThreads) hist[i] = 0;
  __syncthreads();
  for (int c = warp; c < NC; c += kScatterThreads / 32) {
    const int p = c * 32 + lane;
    int e = (p < P) ? idx[p] : -1;
    if (e < 0 || e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int within = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && within == 0) hist[c * E + e] = __popc(peers);
    if (p < P) prow[p] = within;
  }
  __syncthreads();
  for (int e = tid; e < E; e += kScatterThreads) {
    int run = 0;
    for (int c = 0; c < NC; ++c) {
      const int v = hist[c * E + e];
      hist[c * E + e] = run;
      run += v;
    }
  }
  __syncthreads();
  for (int p = tid; p < P; p += kScatterThreads) {
    const int e = idx[p];
    const int t = t0 + p / k;
    int row = -1;
    if (e < 0 || e >= E) {
      report_error(a.err, MOE_DEVERR_EXPERT_INDEX, t0 * k + p);
    } else {
      const int rank = a.tile_base[(size_t)e * NT + tile] + hist[(p / 32) * E + e] + prow[p];
      if (a.cap < 0 || rank < a.cap) {
        row = a.offsets[e] + rank;
        a.perm[row] = t;
      }
    }
    a.inv[(size_t)t0 * k + p] = row;
    prow[p] = row;
  }
  __syncthreads();
  // gather: warp per token, the source row is read once and written to each kept slot
  const int nvec = a.d * a.elem_bytes / 16;
  const size_t row_bytes = (size_t)a.d * a.elem_bytes;
  const char *xb = static_cast<const char *>(a.x);
  char *xp = static_cast<char *>(a.x_perm);
  for (int m = warp; m < rows; m += kScatterThreads / 32) {
    int dst[kMaxTopK];
#pragma unroll
    for (int s = 0; s < kMaxTopK; ++s) dst[s] = (s < k) ? prow[m * k + s] : -1;
    const uint4 *src = reinterpret_cast<const uint4 *>(xb + (size_t)(t0 + m) * row_bytes);
    for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
      uint4 u[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int v = v0 + 32 * q;
        if (v < nvec) u[q] = __ldg(src + v);
      }
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s) {
        if (dst[s] < 0) continue;
        uint4 *o = reinterpret_cast<uint4 *>(xp + (size_t)dst[s] * row_bytes);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int v = v0 + 32 * q;
          if (v < nvec) o[v] = u[q];
        }
      }
    }
  }
}

// ------------------------------------------------------------------- combine
template <typename T>
__global__ void __launch_bounds__(256) k_combine(CombineArgs a) {
  constexpr int VE = Elem<T>::kPerVec;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= a.T) return;
  const int k = a.k;
  int row[kMaxTopK];
  float g[kMaxTopK];
#pragma unroll
  for (int s = 0; s < kMaxTopK; ++s) {
    row[s] = -1;
    g[s] = 0.f;
    if (s < k) {
      int r = a.inv[(size_t)t * k + s];
      if (r < -1 || r >= a.R) {
        if (lane == 0) report_error(a.err, MOE_DEVERR_ROW_INDEX, t * k + s);
        r = -1;
      }
      row[s] = r;
      g[s] = a.gate[(size_t)t * k + s];
    }
  }
  const T *yp = static_cast<const T *>(a.y_perm);
  T *y = static_cast<T *>(a.y);
  const int nvec = a.d / VE;
  for (int v = lane; v < nvec; v += 32) {
    float acc[VE];
#pragma unroll
    for (int i = 0; i < VE; ++i) acc[i] = 0.f;
#pragma unroll
    for (int s = 0; s < kMaxTopK; ++s) {
      if (row[s] < 0) continue;
      float f[VE];
      unpack16(__ldg(reinterpret_cast<const uint4 *>(yp + (size_t)row[s] * a.d) + v), f);
#pragma unroll
      for (int i = 0; i < VE; ++i) acc[i] = fmaf(g[s], f[i], acc[i]);
    }
    if (a.shared_y) {
      const float4 *sp = reinterpret_cast<const float4 *>(a.shared_y + (size_t)t * a.d + v * VE);
#pragma unroll
      for (int i = 0; i < VE; i += 4) {
        const float4 q = __ldg(sp + i / 4);
        acc[i] += q.x; acc[i + 1] += q.y; acc[i + 2] += q.z; acc[i + 3] += q.w;
      }
    }
    reinterpret_cast<uint4 *>(y + (size_t)t * a.d)[v] = pack16(acc);
  }
}

// ---------------------------------------------------------------- tile table
__global__ void k_tile_table(const int32_t *offsets, int G, int max_rows, int32_t *mprefix,
                             int32_t *err) {
  if (threadIdx.x != 0) return;
  bool ok = offsets[0] >= 0;
  int bad = 0;
  for (int g = 0; g < G && ok; ++g) {
    if (offsets[g + 1] < offsets[g] || offsets[g + 1] > max_rows) { ok = false; bad = g; }
  }
  int mp = 0;
  for (int g = 0; g < G; ++g) {
    mprefix[g] = mp;
    if (ok) mp += ceil_div(offsets[g + 1] - offsets[g], kRowTile);
  }
  mprefix[G] = mp;
  if (!ok) report_error(err, MOE_DEVERR_OFFSETS, bad);
}

}  // namespace

cudaError_t launch_scan(const ScanArgs &a, cudaStream_t st) {
  k_scan<<<1, kScanThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_scatter(const ScatterArgs &a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int bm = router_bm(a.E);
  const int NT = ceil_div(a.T, bm);
  const int NC = ceil_div(bm * a.k, 32);
  const size_t smem = (size_t)(NC * a.E + bm * a.k) * sizeof(int32_t);
  k_scatter<<<NT, kScatterThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs &a, int dtype, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int grid = ceil_div(a.T, 8);
  if (dtype == MOE_DTYPE_F32)
    k_combine<float><<<grid, 256, 0, st>>>(a);
  else
    k_combine<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_tile_table(const int32_t *offsets, int G, int max_rows, int32_t *mprefix,
                              int32_t *err, cudaStream_t st) {
  k_tile_table<<<1, 32, 0, st>>>(offsets, G, max_rows, mprefix, err);
  return cudaGetLastError();
}

}  // namespace moe

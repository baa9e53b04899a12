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
#include "shard.cuh"

namespace moe {

namespace {

// ----------------------------------------------------------------- warp scan
__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kScanVPL = 8;  // tiles per lane per batch (loads issued together)

// Warp per expert, eight experts per CTA and E / 8 CTAs (one CTA looping over all
// experts when there is no ticket word): the exclusive prefix of the expert's
// per-tile counts over the token tiles (tile_counts is [E][NT], so a warp reads
// consecutive tiles), its pre-drop count and (statistics) its probability sum.
// The last CTA to finish (an atomic ticket that wraps back to zero, so nothing
// waits) then does counts, capacity, kept-row offsets and the 128-row tile prefix
// over the experts, and the load-balancing statistics (fixed-order sums).
// SHARD: the tokens are one shard of a larger batch; expert e keeps at most
// max(0, cap - pairs routed to e by the earlier shards), written to sc.cap_e.
template <bool SHARD>
__global__ void __launch_bounds__(kScanThreads) k_scan(ScanArgs a, ShardCaps sc) {
  __shared__ float red[kScanWarps];
  __shared__ int last_s;
  pdl_wait();
  pdl_trigger();
  const int E = a.E, NT = a.NT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool want_p = a.aux_out != nullptr;
  for (int e = blockIdx.x * kScanWarps + warp; e < E; e += gridDim.x * kScanWarps) {
    const int32_t *tc = a.tile_counts + (size_t)e * NT;
    int32_t *tb = a.tile_base + (size_t)e * NT;
    const float *tp = want_p ? a.tile_p + (size_t)e * NT : nullptr;
    int run = 0;
    float p = 0.f;  // this lane's tiles t = lane, lane + 32, ... in order
    for (int b0 = 0; b0 < NT; b0 += 32 * kScanVPL) {
      // the counts and the probability sums of this block, all requested at once
      int v[kScanVPL];
      float pv[kScanVPL];
#pragma unroll
      for (int j = 0; j < kScanVPL; ++j) {
        const int t = b0 + j * 32 + lane;
        v[j] = t < NT ? tc[t] : 0;
        pv[j] = (tp != nullptr && t < NT) ? tp[t] : 0.f;
      }
#pragma unroll
      for (int j = 0; j < kScanVPL; ++j) {
        const int incl = warp_incl_scan(v[j]);
        const int t = b0 + j * 32 + lane;
        if (t < NT) tb[t] = run + incl - v[j];
        run += __shfl_sync(0xffffffffu, incl, 31);
        p += pv[j];
      }
    }
    if (want_p) p = warp_sum(p);
    if (lane == 0) {
      a.counts[e] = run;
      if (want_p) a.aux_out[3 + E + e] = p / (float)a.T;
    }
  }
  if (gridDim.x > 1) {  // only the last CTA goes on, after every CTA's writes
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      last_s = atomicInc(a.ticket, gridDim.x - 1) == gridDim.x - 1;
    }
    __syncthreads();
    if (!last_s) return;
    __threadfence();
  } else {
    __syncthreads();
  }
  if (warp == 0) {
    // E <= 256: eight experts per lane
    int cnt[8], kept[8], mt[8];
    int sk = 0, sm = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      const int c = e < E ? __ldcg(a.counts + e) : 0;
      cnt[j] = c;
      int cap = a.cap;
      if constexpr (SHARD) {
        if (cap >= 0 && e < E) {
          long long before = 0;
          for (int r = 0; r < sc.rank; ++r) before += sc.counts_all[(size_t)r * E + e];
          cap = (int)max(0LL, (long long)a.cap - before);
          sc.cap_e[e] = cap;
        }
      }
      kept[j] = (a.cap < 0) ? c : min(c, cap);
      mt[j] = ceil_div(kept[j], kRowTile);
      sk += kept[j];
      sm += mt[j];
    }
    const int ik = warp_incl_scan(sk), im = warp_incl_scan(sm);
    int ok = ik - sk, om = im - sm;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      if (e < E) {
        a.counts[e] = cnt[j];
        a.offsets[e] = ok;
        a.mprefix[e] = om;
      }
      ok += kept[j];
      om += mt[j];
    }
    if (lane == 31) {
      a.offsets[E] = ik;
      a.mprefix[E] = im;
    }
    if (lane == 0 && a.sh_tbl) {
      a.sh_tbl[0] = 0;
      a.sh_tbl[1] = a.T;
      a.sh_tbl[2] = 0;
      a.sh_tbl[3] = ceil_div(a.T, kRowTile);
    }
  }
  if (a.aux_out == nullptr) return;

  // ---- load-balancing statistics
  float z = 0.f;
  for (int t = threadIdx.x; t < NT; t += kScanThreads) z += a.tile_z[t];
  z = warp_sum(z);
  if (lane == 0) red[warp] = z;
  __syncthreads();
  if (warp == 0) {
    // fp64 sums over the experts: lane l takes experts l, l + 32, ..., then a
    // fixed shuffle tree
    const double inv_tk = 1.0 / ((double)a.T * (double)a.k);
    double fp = 0.0, bsq = 0.0;
    // E <= 256: the lane's (up to) eight experts' counts and probability sums are all
    // requested before any f is stored into aux_out (a store there would keep the
    // next loads of the same array behind it)
    int cnt[8];
    float pe[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      cnt[j] = e < E ? __ldcg(a.counts + e) : 0;
      pe[j] = e < E ? __ldcg(a.aux_out + 3 + E + e) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (e < E) {
        const double f = (double)cnt[j] * inv_tk;
        fp += f * (double)pe[j];
        bsq += (f - 1.0 / E) * (f - 1.0 / E);
        a.aux_out[3 + e] = (float)f;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      fp += __shfl_xor_sync(0xffffffffu, fp, o);
      bsq += __shfl_xor_sync(0xffffffffu, bsq, o);
    }
    if (lane == 0) {
      float zs = 0.f;
      for (int w = 0; w < kScanWarps; ++w) zs += red[w];
      a.aux_out[0] = (float)((double)a.alpha * E * fp);
      a.aux_out[1] = zs / (float)a.T;
      a.aux_out[2] = (float)bsq;
    }
  }
}

// ------------------------------------------------------------------- scatter
constexpr int kScatterThreads = 256;

template <bool SHARD>
__global__ void __launch_bounds__(kScatterThreads) k_scatter(ScatterArgs a, const int32_t *cap_e) {
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
  int32_t *base = prow + bm * k;    // [E]: this tile's base rank in each expert
  int32_t *first = base + E;        // [E]: the expert's first row (offsets)
  int32_t *capv = first + E;        // [E]: the pairs the expert may keep
  int32_t *eidx = capv + E;         // [bm*k]: the routing indices of the tile
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kScatterThreads / 32;
  const int32_t *idx = a.topk_idx + (size_t)t0 * k;
  pdl_wait();
  pdl_trigger();

  // the tile's routing indices (at most two 32-pair chunks per warp: bm * k <= 512)
  // and the per-expert values of phase 3 are all requested before the first barrier
  int ev[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int p = (warp + u * kWarps) * 32 + lane;
    ev[u] = (p < P) ? idx[p] : -1;
  }
  for (int e = tid; e < E; e += kScatterThreads) {
    base[e] = a.tile_base[(size_t)e * NT + tile];
    first[e] = a.offsets[e];
    capv[e] = a.cap < 0 ? INT_MAX : (SHARD ? cap_e[e] : a.cap);
  }
  for (int i = tid; i < NC * E; i += kScatterThreads) hist[i] = 0;
  __syncthreads();
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int c = warp + u * kWarps;
    if (c >= NC) break;
    const int p = c * 32 + lane;
    if (p < P) eidx[p] = ev[u];
    const int e = (ev[u] < 0 || ev[u] >= E) ? -1 : ev[u];
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
    const int e = eidx[p];
    const int t = t0 + p / k;
    int row = -1;
    if (e < 0 || e >= E) {
      report_error(a.err, MOE_DEVERR_EXPERT_INDEX, t0 * k + p);
    } else {
      const int rank = base[e] + hist[(p / 32) * E + e] + prow[p];
      if (rank < capv[e]) {
        row = first[e] + rank;
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
    bool any = false;
#pragma unroll
    for (int s = 0; s < kMaxTopK; ++s) {
      dst[s] = (s < k) ? prow[m * k + s] : -1;
      any |= dst[s] >= 0;
    }
    if (!any) continue;  // every slot dropped: the row is not read at all
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
// A warp per token. Each lane takes NB 16-byte vectors of the row per batch and
// requests every kept slot's vectors (and, SHARED, the shared-expert row) before
// using any, so a warp keeps NB x k loads in flight; KMAX bounds k (register
// budget). A token whose every slot was dropped (and that has no shared-expert
// row) is written as zeros without loading or converting anything: in a layer
// with tight capacity (Switch keeps 1721 of 16384 tokens) that is most of them.
template <typename T, int KMAX, int NB, bool SHARED>
__global__ void __launch_bounds__(256, SHARED ? 2 : (KMAX <= 2 ? 4 : 3)) k_combine(CombineArgs a) {
  constexpr int VE = Elem<T>::kPerVec;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  pdl_wait();
  pdl_trigger();
  if (t >= a.T) return;
  const int k = a.k;
  int row[KMAX];
  float g[KMAX];
#pragma unroll
  for (int s = 0; s < KMAX; ++s) {
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
  if (!SHARED) {
    bool any = false;
#pragma unroll
    for (int s = 0; s < KMAX; ++s) any |= row[s] >= 0;
    if (!any) {
      uint4 *dst = reinterpret_cast<uint4 *>(y + (size_t)t * a.d);
      for (int v = lane; v < nvec; v += 32) dst[v] = make_uint4(0u, 0u, 0u, 0u);
      return;
    }
  }
  for (int v0 = lane; v0 < nvec; v0 += 32 * NB) {
    // a dropped slot reads nothing and contributes zero
    uint4 u[KMAX][NB];
#pragma unroll
    for (int s = 0; s < KMAX; ++s)
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int v = v0 + 32 * b;
        u[s][b] = (row[s] >= 0 && v < nvec)
                      ? __ldg(reinterpret_cast<const uint4 *>(yp + (size_t)row[s] * a.d) + v)
                      : make_uint4(0u, 0u, 0u, 0u);
      }
    float4 sh[SHARED ? NB : 1][VE / 4];
    if (SHARED) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int v = v0 + 32 * b;
        const float4 *sp = reinterpret_cast<const float4 *>(a.shared_y + (size_t)t * a.d + v * VE);
#pragma unroll
        for (int i = 0; i < VE / 4; ++i)
          sh[b][i] = (v < nvec) ? __ldg(sp + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int v = v0 + 32 * b;
      if (v >= nvec) break;
      float acc[VE];
#pragma unroll
      for (int i = 0; i < VE; ++i) acc[i] = 0.f;
#pragma unroll
      for (int s = 0; s < KMAX; ++s) {
        if (s >= k) break;
        float f[VE];
        unpack16(u[s][b], f);
#pragma unroll
        for (int i = 0; i < VE; ++i) acc[i] = fmaf(g[s], f[i], acc[i]);
      }
      if (SHARED) {
#pragma unroll
        for (int i = 0; i < VE; i += 4) {
          const float4 q = sh[SHARED ? b : 0][i / 4];
          acc[i] += q.x; acc[i + 1] += q.y; acc[i + 2] += q.z; acc[i + 3] += q.w;
        }
      }
      reinterpret_cast<uint4 *>(y + (size_t)t * a.d)[v] = pack16(acc);
    }
  }
}

// ---------------------------------------------------------------- tile table
// One warp: validate a caller-supplied offsets array and build the 128-row tile
// prefix from it (all zero, so nothing is computed, when the offsets are invalid).
__global__ void k_tile_table(const int32_t *offsets, int G, int max_rows, int32_t *mprefix,
                             int32_t *err) {
  // waits for the kernel before it, and never lets the one after it begin early: the
  // GEMMs read mprefix before their own wait
  pdl_wait();
  const int lane = threadIdx.x;
  int bad = G;
  for (int g = lane; g < G; g += 32) {
    const int a0 = offsets[g], a1 = offsets[g + 1];
    if (a0 < 0 || a1 < a0 || a1 > max_rows) bad = min(bad, g);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bad = min(bad, __shfl_xor_sync(0xffffffffu, bad, o));
  const bool ok = bad == G;
  int mt[8], sm = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int g = lane * 8 + j;
    mt[j] = (ok && g < G) ? ceil_div(offsets[g + 1] - offsets[g], kRowTile) : 0;
    sm += mt[j];
  }
  const int incl = warp_incl_scan(sm);
  int run = incl - sm;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int g = lane * 8 + j;
    if (g < G) mprefix[g] = run;
    run += mt[j];
  }
  if (lane == 31) mprefix[G] = incl;
  if (!ok && lane == 0) report_error(err, MOE_DEVERR_OFFSETS, bad);
}

}  // namespace

// E / 8 CTAs with a ticket word, else one CTA over all experts
unsigned scan_grid(const ScanArgs &a) {
  return a.ticket != nullptr ? (unsigned)ceil_div(a.E, kScanWarps) : 1u;
}

cudaError_t launch_scan(const ScanArgs &a, cudaStream_t st) {
  return launch_pdl(k_scan<false>, dim3(scan_grid(a)), dim3(kScanThreads), 0, st, a,
                    ShardCaps{});
}

cudaError_t launch_scan_shard(const ScanArgs &a, const ShardCaps &sc, cudaStream_t st) {
  k_scan<true><<<scan_grid(a), kScanThreads, 0, st>>>(a, sc);
  return cudaGetLastError();
}

namespace {
template <bool SHARD>
cudaError_t scatter(const ScatterArgs &a, const int32_t *cap_e, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int bm = router_bm(a.E);
  const int NT = ceil_div(a.T, bm);
  const int NC = ceil_div(bm * a.k, 32);
  if (bm * a.k > 2 * kScatterThreads) return cudaErrorInvalidValue;  // two chunks per warp
  const size_t smem = (size_t)(NC * a.E + 2 * bm * a.k + 3 * a.E) * sizeof(int32_t);
  return launch_pdl(k_scatter<SHARD>, dim3(NT), dim3(kScatterThreads), smem, st, a, cap_e);
}
}  // namespace

cudaError_t launch_scatter(const ScatterArgs &a, cudaStream_t st) {
  return scatter<false>(a, nullptr, st);
}

cudaError_t launch_scatter_shard(const ScatterArgs &a, const int32_t *cap_e, cudaStream_t st) {
  return scatter<true>(a, cap_e, st);
}

cudaError_t launch_combine(const CombineArgs &a, int dtype, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int grid = ceil_div(a.T, 8);
  const bool f32 = dtype == MOE_DTYPE_F32;
  const dim3 g(grid), b(256);
  const bool sh = a.shared_y != nullptr;
  if (a.k <= 2) {
    if (f32)
      return sh ? launch_pdl(k_combine<float, 2, 4, true>, g, b, 0, st, a)
                : launch_pdl(k_combine<float, 2, 4, false>, g, b, 0, st, a);
    return sh ? launch_pdl(k_combine<__nv_bfloat16, 2, 4, true>, g, b, 0, st, a)
              : launch_pdl(k_combine<__nv_bfloat16, 2, 4, false>, g, b, 0, st, a);
  }
  if (f32)
    return sh ? launch_pdl(k_combine<float, kMaxTopK, 1, true>, g, b, 0, st, a)
              : launch_pdl(k_combine<float, kMaxTopK, 1, false>, g, b, 0, st, a);
  return sh ? launch_pdl(k_combine<__nv_bfloat16, kMaxTopK, 1, true>, g, b, 0, st, a)
            : launch_pdl(k_combine<__nv_bfloat16, kMaxTopK, 1, false>, g, b, 0, st, a);
}

cudaError_t launch_tile_table(const int32_t *offsets, int G, int max_rows, int32_t *mprefix,
                              int32_t *err, cudaStream_t st) {
  return launch_pdl(k_tile_table, dim3(1), dim3(32), 0, st, offsets, G, max_rows, mprefix, err);
}

}  // namespace moe

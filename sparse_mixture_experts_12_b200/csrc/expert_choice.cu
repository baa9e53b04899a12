// Expert-Choice routing (youngju.dev (zh) "ExpertChoiceRouter", youngju.dev (ja)
// "ExpertChoiceGating"): every expert takes the C tokens of highest score, score =
// the expert's softmax over the tokens; the layer output of a token is the
// score-weighted sum of the outputs of the experts that took it (the dispatch mask
// of "ExpertChoiceGating" used as the gate).
//
// The router logits come from the router kernels. Then:
//   k_ec_transpose  logits [T, E] -> zt [E, T] (NaN -> -inf), through 32 x 32 tiles
//   k_ec_select     one CTA per expert: max and sum exp over its T logits (fixed-order
//                   reductions), radix select of the C-th largest logit (4 passes of 8
//                   bits over order-preserving integer keys), the picks in token order,
//                   then a bitonic sort by (logit descending, token ascending) ->
//                   ec_idx, ec_score, the token -> pick slot map and the row offsets
//   k_ec_gather     x_perm[e*C + j] = x[ec_idx[e, j]]
//   k_ec_combine    y[t] = sum over experts e that took t, in expert order, of
//                   score * y_perm[e*C + j], in fp32, one rounding
// The grouped expert GEMMs in between are the token-choice ones (offsets e*C).
#include <mutex>

#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kSelThreads = 1024;

// order-preserving key of a logit: larger logit -> larger key; -0 counts as +0
// (they compare equal as floats, so they must tie), NaN as -inf
__device__ __forceinline__ uint32_t ec_key(float z) {
  if (z != z) z = -INFINITY;
  z = z + 0.f;
  const uint32_t u = __float_as_uint(z);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(1024) k_ec_transpose(const float *__restrict__ logits, int T,
                                                       int E, float *__restrict__ zt) {
  __shared__ float tile[32][33];
  pdl_wait();
  pdl_trigger();
  const int t0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int t = t0 + ty, e = e0 + tx;
  if (t < T && e < E) {
    const float v = logits[(size_t)t * E + e];
    tile[ty][tx] = (v != v) ? -INFINITY : v;
  }
  __syncthreads();
  const int e2 = e0 + ty, t2 = t0 + tx;
  if (e2 < E && t2 < T) zt[(size_t)e2 * T + t2] = tile[tx][ty];
}

// block-wide exclusive scan of one int per thread (1024 threads); returns the
// exclusive prefix and the total
__device__ __forceinline__ int block_excl_scan(int v, int *sh_warp, int &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) sh_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = sh_warp[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    sh_warp[lane] = wi - w;  // exclusive prefix of the warps
    if (lane == 31) sh_warp[32] = wi;
  }
  __syncthreads();
  const int r = sh_warp[warp] + incl - v;
  total = sh_warp[32];
  __syncthreads();  // sh_warp is reused by the next scan
  return r;
}

// fixed-order block reductions (every thread gets the result)
__device__ __forceinline__ float block_max(float v, float *sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  float r = sh[0];
  for (int w = 1; w < kSelThreads / 32; ++w) r = fmaxf(r, sh[w]);
  __syncthreads();
  return r;
}
__device__ __forceinline__ float block_sum(float v, float *sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < kSelThreads / 32; ++w) r += sh[w];
  __syncthreads();
  return r;
}

// One CTA per expert. Dynamic shared memory: keys [T] u32, then the sort buffer
// [P] u64 (P = C rounded up to a power of two).
__global__ void __launch_bounds__(kSelThreads, 1) k_ec_select(EcArgs a, int P) {
  extern __shared__ __align__(16) uint8_t ec_smem[];
  pdl_wait();
  pdl_trigger();
  const int T = a.T, C = a.C, E = a.E;
  const int e = blockIdx.x;
  uint32_t *key = reinterpret_cast<uint32_t *>(ec_smem);
  uint64_t *sbuf = reinterpret_cast<uint64_t *>(ec_smem + (((size_t)T * 4 + 15) & ~(size_t)15));
  __shared__ int hist[256];
  __shared__ int sh_warp[33];
  __shared__ float sh_red[32];
  __shared__ uint32_t sh_sel[2];  // bucket chosen in this pass, count still to take
  const int tid = threadIdx.x;
  const float *z = a.zt + (size_t)e * T;
  for (int i = tid; i < P; i += kSelThreads) sbuf[i] = ~0ull;  // (ordered by the scans' syncs)

  float m = -INFINITY;
  for (int t = tid; t < T; t += kSelThreads) {
    const float v = z[t];
    key[t] = ec_key(v);
    m = fmaxf(m, v);
  }
  m = block_max(m, sh_red);
  float s = 0.f;
  for (int t = tid; t < T; t += kSelThreads) s += expf(z[t] - m);
  s = block_sum(s, sh_red);

  // ---- radix select of the C-th largest key, most significant byte first
  uint32_t prefix = 0, mask = 0;
  int remaining = C;
  const int lane = tid & 31;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    // warp-aggregated counts: most keys share their leading bytes, so one add per
    // distinct bin and warp instead of one per key (integer adds: the counts do not
    // depend on their order)
    for (int t0 = 0; t0 < T; t0 += kSelThreads) {
      const int t = t0 + tid;
      const uint32_t k = t < T ? key[t] : 0u;
      const int bin = (t < T && (k & mask) == prefix) ? (int)((k >> shift) & 0xFF) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
    __syncthreads();
    if (tid < 32) {
      // the highest bin b whose keys, with those of the bins above it, reach
      // `remaining`: lane l holds bins 8l .. 8l + 7; suffix sums over the lanes
      int c[8], lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[8 * lane + j];
        lsum += c[j];
      }
      int suf = lsum;  // keys in this lane's bins and every bin above them
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += v;
      }
      int above = suf - lsum;
      if (above < remaining && remaining <= suf) {
        int b = 8 * lane + 7;
#pragma unroll
        for (int j = 7; j > 0; --j) {
          if (above + c[j] >= remaining) break;
          above += c[j];
          --b;
        }
        sh_sel[0] = (uint32_t)b;
        sh_sel[1] = (uint32_t)(remaining - above);
      }
    }
    __syncthreads();
    prefix |= sh_sel[0] << shift;
    mask |= 0xFFu << shift;
    remaining = (int)sh_sel[1];
    __syncthreads();
  }
  const uint32_t kstar = prefix;  // the C-th largest key; `remaining` of its ties are taken

  // ---- the picks in token order: every key above kstar, and the first
  // `remaining` tokens whose key equals kstar
  const int per = (T + kSelThreads - 1) / kSelThreads;
  const int t_lo = min(T, tid * per), t_hi = min(T, t_lo + per);
  int n_eq = 0;
  for (int t = t_lo; t < t_hi; ++t) n_eq += key[t] == kstar;
  int tot;
  int eq_before = block_excl_scan(n_eq, sh_warp, tot);
  int n_sel = 0;
  {
    int r = eq_before;
    for (int t = t_lo; t < t_hi; ++t) {
      const uint32_t k = key[t];
      if (k > kstar) ++n_sel;
      else if (k == kstar && r++ < remaining) ++n_sel;
    }
  }
  int pos = block_excl_scan(n_sel, sh_warp, tot);
  {
    int r = eq_before;
    for (int t = t_lo; t < t_hi; ++t) {
      const uint32_t k = key[t];
      bool take = k > kstar;
      if (k == kstar) take = r++ < remaining;
      if (take && pos < P) sbuf[pos++] = ((uint64_t)(~k) << 32) | (uint32_t)t;
    }
  }
  __syncthreads();

  // ---- bitonic sort, ascending: logit descending, then token ascending
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < P / 2; i += kSelThreads) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t x = sbuf[lo], y = sbuf[hi];
        if ((x > y) == up) {
          sbuf[lo] = y;
          sbuf[hi] = x;
        }
      }
      __syncthreads();
    }
  }

  const float inv_s = 1.f / s;
  for (int j = tid; j < C; j += kSelThreads) {
    const uint32_t tu = (uint32_t)(sbuf[j] & 0xffffffffu);
    if (tu >= (uint32_t)T) {  // a slot the selection did not fill: never expected
      report_error(a.err, MOE_DEVERR_ROW_INDEX, e);
      a.ec_idx[(size_t)e * C + j] = 0;
      a.ec_score[(size_t)e * C + j] = 0.f;
      continue;
    }
    const int t = (int)tu;
    a.ec_idx[(size_t)e * C + j] = t;
    a.ec_score[(size_t)e * C + j] = expf(z[t] - m) * inv_s;
    if (a.slot) a.slot[(size_t)t * E + e] = j;
  }
  if (a.offsets && tid == 0) {
    a.offsets[e] = e * C;
    if (e == E - 1) a.offsets[E] = E * C;
  }
}

__global__ void __launch_bounds__(256) k_ec_gather(const uint8_t *__restrict__ x, int T,
                                                   const int32_t *__restrict__ idx, int rows,
                                                   int row_bytes, uint8_t *__restrict__ x_perm) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;
  if (r >= rows) return;
  const int t = idx[r];
  if ((unsigned)t >= (unsigned)T) return;  // reported by the selection
  const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * row_bytes);
  uint4 *dst = reinterpret_cast<uint4 *>(x_perm + (size_t)r * row_bytes);
  const int nvec = row_bytes / 16;
  for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
    uint4 u[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (v0 + 32 * q < nvec) u[q] = __ldg(src + v0 + 32 * q);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (v0 + 32 * q < nvec) dst[v0 + 32 * q] = u[q];
  }
}

// A warp per token: the (row, score) list of the experts that took the token, in
// expert order, in shared memory; then each lane sums its 16-byte vectors over the
// list in that order.
template <typename ET>
__global__ void __launch_bounds__(256) k_ec_combine(const ET *__restrict__ y_perm,
                                                    const int32_t *__restrict__ slot,
                                                    const float *__restrict__ score, int T,
                                                    int E, int C, int d, ET *__restrict__ y) {
  constexpr int VE = Elem<ET>::kPerVec;
  __shared__ int l_row[8][kMaxExperts];
  __shared__ float l_g[8][kMaxExperts];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  pdl_wait();
  pdl_trigger();
  if (t >= T) return;
  int n = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    int j = e < E ? slot[(size_t)t * E + e] : -1;
    if (j >= C) j = -1;  // never expected: the selection writes slots below C
    const unsigned took = __ballot_sync(0xffffffffu, j >= 0);
    if (j >= 0) {
      const int p = n + __popc(took & ((1u << lane) - 1u));
      l_row[warp][p] = e * C + j;
      l_g[warp][p] = score[(size_t)e * C + j];
    }
    n += __popc(took);
  }
  __syncwarp();
  const int nvec = d / VE;
  constexpr int NB = 4;  // 16-byte vectors of a row per lane and batch
  for (int v0 = lane; v0 < nvec; v0 += 32 * NB) {
    float acc[NB][VE];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int i = 0; i < VE; ++i) acc[b][i] = 0.f;
    // two experts' rows requested together (eight 16-byte loads in flight per lane),
    // then added in expert order
    for (int i = 0; i < n; i += 2) {
      const bool two = i + 1 < n;
      uint4 u[2][NB];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = l_row[warp][two || h == 0 ? i + h : i];
        const uint4 *src = reinterpret_cast<const uint4 *>(y_perm + (size_t)row * d);
#pragma unroll
        for (int b = 0; b < NB; ++b)
          u[h][b] = ((h == 0 || two) && v0 + 32 * b < nvec) ? __ldg(src + v0 + 32 * b)
                                                             : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (h == 1 && !two) break;
        const float g = l_g[warp][i + h];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float f[VE];
          unpack16(u[h][b], f);
#pragma unroll
          for (int q = 0; q < VE; ++q) acc[b][q] = fmaf(g, f[q], acc[b][q]);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b)
      if (v0 + 32 * b < nvec)
        reinterpret_cast<uint4 *>(y + (size_t)t * d)[v0 + 32 * b] = pack16(acc[b]);
  }
}

std::mutex g_ec_mu;

}  // namespace

size_t ec_select_smem_bytes(int T, int C) {
  int P = 1;
  while (P < C) P <<= 1;
  return (((size_t)T * 4 + 15) & ~(size_t)15) + (size_t)P * 8;
}

cudaError_t launch_ec_route(const EcArgs &a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  dim3 tg(ceil_div(a.T, 32), ceil_div(a.E, 32));
  // programmatic dependent launches: each kernel waits for the one before it before
  // it touches global memory
  cudaError_t e = launch_pdl(k_ec_transpose, tg, dim3(1024), 0, st, a.logits, a.T, a.E, a.zt);
  if (e != cudaSuccess) return e;
  int P = 1;
  while (P < a.C) P <<= 1;
  const size_t smem = ec_select_smem_bytes(a.T, a.C);
  {
    static bool attr_set[64] = {};
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_ec_mu);
    if (!attr_set[dev & 63]) {
      e = cudaFuncSetAttribute(k_ec_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)ec_select_smem_bytes(kEcMaxTokens, kEcMaxPicks));
      if (e != cudaSuccess) return e;
      attr_set[dev & 63] = true;
    }
  }
  return launch_pdl(k_ec_select, dim3(a.E), dim3(kSelThreads), smem, st, a, P);
}

cudaError_t launch_ec_gather(const void *x, int T, const int32_t *ec_idx, int rows,
                             int row_bytes, void *x_perm, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  return launch_pdl(k_ec_gather, dim3(ceil_div(rows, 8)), dim3(256), 0, st,
                    static_cast<const uint8_t *>(x), T, ec_idx, rows, row_bytes,
                    static_cast<uint8_t *>(x_perm));
}

cudaError_t launch_ec_combine(const void *y_perm, const int32_t *slot, const float *score,
                              int T, int E, int C, int d, int dtype, void *y, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  // programmatic dependent launch: it waits for the down projection before it reads
  if (dtype == MOE_DTYPE_F32)
    return launch_pdl(k_ec_combine<float>, dim3(ceil_div(T, 8)), dim3(256), 0, st,
                      static_cast<const float *>(y_perm), slot, score, T, E, C, d,
                      static_cast<float *>(y));
  return launch_pdl(k_ec_combine<__nv_bfloat16>, dim3(ceil_div(T, 8)), dim3(256), 0, st,
                    static_cast<const __nv_bfloat16 *>(y_perm), slot, score, T, E, C, d,
                    static_cast<__nv_bfloat16 *>(y));
}

}  // namespace moe

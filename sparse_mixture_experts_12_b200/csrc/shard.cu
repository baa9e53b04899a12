// Load-balancing statistics of a token-sharded batch: per-shard fp64 sums, and the
// statistics from the summed parts (the sum itself is a collective of the caller).
// The statistics are those of "load_balancing_loss" / "compute_load_balancing_loss"
// (f_i counted before drops, over T*k; P_i the mean full softmax), "router_z_loss"
// (mean squared logsumexp) and the squared-deviation balance loss of the Shazeer-style
// "load_balancing_loss" (sum_i (f_i - 1/E)^2).
#include "shard.cuh"

namespace moe {
namespace {

constexpr int kPartThreads = 1024;

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One CTA: warp per expert over the tiles (lane-strided, then a fixed shuffle tree).
__global__ void __launch_bounds__(kPartThreads)
k_aux_partials(const int32_t *tile_counts, const float *tile_p, const float *tile_z, int E,
               int NT, double *part) {
  __shared__ double red[kPartThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int nw = kPartThreads / 32;
  for (int e = warp; e < E; e += nw) {
    long long c = 0;
    double p = 0.0;
    for (int t = lane; t < NT; t += 32) {
      c += tile_counts[(size_t)e * NT + t];
      p += (double)tile_p[(size_t)e * NT + t];
    }
    const double cs = warp_sum_f64((double)c);  // exact: counts are far below 2^53
    p = warp_sum_f64(p);
    if (lane == 0) {
      part[1 + e] = cs;
      part[1 + E + e] = p;
    }
  }
  double z = 0.0;
  for (int t = threadIdx.x; t < NT; t += kPartThreads) z += (double)tile_z[t];
  z = warp_sum_f64(z);
  if (lane == 0) red[warp] = z;
  __syncthreads();
  if (threadIdx.x == 0) {
    double zs = 0.0;
    for (int w = 0; w < nw; ++w) zs += red[w];
    part[0] = zs;
  }
}

// One warp.
__global__ void k_aux_finalize(const double *part, int E, long long T, int k, float alpha,
                               float *out) {
  const int lane = threadIdx.x;
  const double inv_t = 1.0 / (double)T;
  const double inv_tk = 1.0 / ((double)T * (double)k);
  double fp = 0.0, bsq = 0.0;
  for (int e = lane; e < E; e += 32) {
    const double f = part[1 + e] * inv_tk;
    const double P = part[1 + E + e] * inv_t;
    fp += f * P;
    bsq += (f - 1.0 / E) * (f - 1.0 / E);
    out[3 + e] = (float)f;
    out[3 + E + e] = (float)P;
  }
  fp = warp_sum_f64(fp);
  bsq = warp_sum_f64(bsq);
  if (lane == 0) {
    out[0] = (float)((double)alpha * E * fp);
    out[1] = (float)(part[0] * inv_t);
    out[2] = (float)bsq;
  }
}

}  // namespace

cudaError_t launch_aux_partials(const int32_t *tile_counts, const float *tile_p,
                                const float *tile_z, int E, int NT, double *part,
                                cudaStream_t st) {
  k_aux_partials<<<1, kPartThreads, 0, st>>>(tile_counts, tile_p, tile_z, E, NT, part);
  return cudaGetLastError();
}

cudaError_t launch_aux_finalize(const double *part, int E, long long T, int k, float alpha,
                                float *out, cudaStream_t st) {
  k_aux_finalize<<<1, 32, 0, st>>>(part, E, T, k, alpha, out);
  return cudaGetLastError();
}

}  // namespace moe

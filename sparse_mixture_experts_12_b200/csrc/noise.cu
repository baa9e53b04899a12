// Counter-based standard normal draws for the seeded noisy gate.
//
// youngju.dev (ja) "TopKGating" (Noisy Top-K Gating) adds softplus(x W_noise^T)
// times standard normal noise to the router logits in training. Drawn from a seed
// and an offset, the noise is a pure function of (seed, offset, token, expert): a
// counter-based generator, so that every CUDA thread computes its own draws
// without state and an independent CPU restatement reproduces them.
//
// Generator: Philox4x32-10 of J. K. Salmon, M. A. Moraes, R. O. Dror and D. E.
// Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11), written from that
// definition. Token t and expert group q = e / 4 use counter (t, q, offset lo,
// offset hi) and key (seed lo, seed hi). Each of the four output words r becomes a
// uniform u = (2 (r >> 9) + 1) 2^-24 in (0, 1), exact in fp32; the transform of
// Box and Muller (Ann. Math. Statist. 29, 1958) turns (u0, u1) into the draws of
// experts 4q, 4q + 1 (rho cos, rho sin of 2 pi u1, rho = sqrt(-2 ln u0)) and
// (u2, u3) into those of experts 4q + 2, 4q + 3.
#include <algorithm>

#include "kernels.cuh"

namespace moe {

namespace {

constexpr uint32_t kPhiloxM0 = 0xD2511F53u, kPhiloxM1 = 0xCD9E8D57u;  // round multipliers
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u, kPhiloxW1 = 0xBB67AE85u;  // key increments

// One Philox4x32-10 block: ten rounds of
// (c0, c1, c2, c3) -> (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)),
// the key advanced by (W0, W1) before every round but the first.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += kPhiloxW0;
      k1 += kPhiloxW1;
    }
    const uint32_t hi0 = __umulhi(kPhiloxM0, c.x), lo0 = kPhiloxM0 * c.x;
    const uint32_t hi1 = __umulhi(kPhiloxM1, c.z), lo1 = kPhiloxM1 * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

__device__ __forceinline__ float uniform_open(uint32_t r) {
  return __uint2float_rn(((r >> 9) << 1) | 1u) * 0x1p-24f;  // < 2^24: exact
}

__device__ __forceinline__ void box_muller(float ua, float ub, float &z0, float &z1) {
  const float rho = sqrtf(-2.f * logf(ua));
  float s, c;
  sincospif(2.f * ub, &s, &c);  // 2 ub is exact
  z0 = rho * c;
  z1 = rho * s;
}

// eps [T, E] fp32 and, when raw != NULL, the Philox words raw [T, ceil(E/4), 4].
__global__ void __launch_bounds__(256) k_noise_draws(int T, int E, uint32_t k0, uint32_t k1,
                                                     uint32_t o0, uint32_t o1,
                                                     float *__restrict__ eps,
                                                     uint4 *__restrict__ raw) {
  const int Q = (E + 3) >> 2;
  const long long n = (long long)T * Q;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i / Q), q = (int)(i - (long long)t * Q);
    const uint4 r = philox4x32_10(make_uint4((uint32_t)t, (uint32_t)q, o0, o1), k0, k1);
    if (raw != nullptr) raw[i] = r;
    float z[4];
    box_muller(uniform_open(r.x), uniform_open(r.y), z[0], z[1]);
    box_muller(uniform_open(r.z), uniform_open(r.w), z[2], z[3]);
    float *row = eps + (size_t)t * E;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (4 * q + j < E) row[4 * q + j] = z[j];
  }
}

}  // namespace

cudaError_t launch_noise_draws(int T, int E, uint64_t seed, uint64_t offset, float *eps,
                               uint32_t *raw, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const long long n = (long long)T * ((E + 3) / 4);
  const long long blocks = std::min<long long>((n + 255) / 256, 148LL * 8);
  k_noise_draws<<<(unsigned)blocks, 256, 0, st>>>(
      T, E, (uint32_t)seed, (uint32_t)(seed >> 32), (uint32_t)offset, (uint32_t)(offset >> 32),
      eps, reinterpret_cast<uint4 *>(raw));
  return cudaGetLastError();
}

}  // namespace moe

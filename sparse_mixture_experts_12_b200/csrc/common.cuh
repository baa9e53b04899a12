// Shared device/host helpers of the MoE kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

#define MOE_HIDDEN __attribute__((visibility("hidden")))

namespace moe {

constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;
constexpr int kRowTile = 128;  // rows of one grouped-GEMM M tile (and of the tile table)

// ---------------------------------------------------------------- element types
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
  static constexpr int kPerVec = 4;  // elements per 16-byte vector
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
  static constexpr int kPerVec = 8;
};

// 16-byte vector <-> float[kPerVec]
__device__ __forceinline__ void unpack16(const uint4 &u, float (&f)[4]) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void unpack16(const uint4 &u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ uint4 pack16(const float (&f)[4]) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                    __float_as_uint(f[3]));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint4 pack16(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

// ---------------------------------------------------------------- device errors
// err[0] = code (first error wins), err[1] = info.
__device__ __forceinline__ void report_error(int32_t *err, int32_t code, int32_t info) {
  if (err == nullptr) return;
  if (atomicCAS(err, 0, code) == 0) atomicExch(err + 1, info);
}

// ------------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialisation may begin while the
// kernel before it in the stream is still running. pdl_wait() blocks until that
// kernel has completed and its writes are visible: it comes before the first
// access to anything an earlier kernel writes, or reads while this one writes it.
// pdl_trigger() lets the next kernel in the stream begin its launch; a kernel
// calls it only after its own pdl_wait(), so every kernel that passes its wait
// knows that all earlier kernels have completed. Both are no-ops in a kernel
// launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- warp helpers
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// (value, index) argmax with ties to the lower index.
__device__ __forceinline__ void warp_argmax(float &v, int &i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
  }
}

// ---------------------------------------------------------------- router tiling
// Tokens per router CTA; the permute kernels use the same token tiles.
__host__ __device__ constexpr int router_bm(int E) {
  return E <= 32 ? 32 : (E <= 128 ? 64 : 32);
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Set when a layer call has just recorded a stage event on this host thread: the
// next launch is a plain one (it starts after the event, so that the stage's time is
// its kernels' own) and clears the flag; every other launch uses programmatic
// dependent launch.
extern thread_local bool t_pdl_blocked;

// Whether the next launch may use programmatic dependent launch (consumes the flag).
inline bool take_pdl() {
  const bool ok = !t_pdl_blocked;
  t_pdl_blocked = false;
  return ok;
}

// Launch `kernel` with programmatic stream serialisation (see pdl_wait), or as a
// plain launch right after a stage event.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = take_pdl() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace moe

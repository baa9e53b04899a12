// Grouped expert FFN on the 5th-generation tensor cores (tcgen05 + TMEM), bf16
// operands, fp32 accumulation.
//
// Experts: youngju.dev "SwiGLUExpert" (w_down(silu(w_gate x) * w_up x)), the
// "SiLU · SwiGLU · MoE" table of the study-site lecture, devtips.kr "MoELayer"
// (ReLU MLP) and youngju.dev (zh) "MoELayer" (GELU MLP). Only the rows routed to
// an expert are multiplied by its weights ("Token Routing": unselected experts
// are not computed at all).
//
// Design (one persistent CTA per SM, 256 threads, warp-specialised):
//   warp 0      TMA producer: A tile [128 rows x 64 k] of the expert-contiguous
//               activations and the B tile [256 rows x 64 k] of the expert's
//               weights into a 4-stage shared-memory ring (128-byte swizzle).
//               For SwiGLU the B tile is w_gate rows [n, n+128) stacked on w_up
//               rows [n, n+128), so one N=256 MMA yields both halves.
//   warp 1      MMA issuer: tcgen05.mma M=128 N=256 K=16, accumulator in TMEM,
//               two 256-column accumulators so the epilogue of tile i overlaps
//               the main loop of tile i+1.
//   warp 2      TMEM allocator.
//   warps 4..7  epilogue: tcgen05.ld, fused silu(g)*u / bias+ReLU / bias+GELU,
//               bf16 (or fp32) stores masked to the expert's rows.
// The tile list is built on the device (per-expert M-tile prefix), so no host
// synchronisation sits between routing and the expert GEMMs. Every wait is
// bounded; on a timeout the CTA records MOE_DEVERR_WAIT_TIMEOUT, drains its
// in-flight copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kStages = 4;
constexpr int kBlockK = 64;  // 64 bf16 = one 128-byte swizzle row
constexpr int kTileM = kRowTile;
constexpr int kMmaN = 256;
constexpr int kABytes = kTileM * kBlockK * 2;
constexpr int kBBytes = kMmaN * kBlockK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 2 * kMmaN;
constexpr int kThreads = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

enum { EPI_SWIGLU = 0, EPI_ACT = 1, EPI_DOWN = 2 };

struct TcArgs {
  const int32_t *offsets;
  const int32_t *mprefix;
  int G, N, K;
  int n_tiles;    // N tiles per group
  int b_rows;     // weight rows per group in the B map(s)
  void *out;      // [rows, N]
  int out_f32;
  const float *bias;  // [G, N] or nullptr
  int act;
  int32_t *err;
};

struct SmemCtl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int tbl[2 * (kMaxExperts + 1)];  // mprefix[G+1], offsets[G+1]
};

constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + sizeof(SmemCtl) + 1024;

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `parity` to complete. Gives up when another role has
// aborted (honour_abort) or after kWaitLimitNs, recording the site.
__device__ __noinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, SmemCtl *ctl,
                                          int32_t *err, int site, bool honour_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  volatile int *abort_flag = &ctl->abort_flag;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honour_abort && *abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      report_error(err, MOE_DEVERR_WAIT_TIMEOUT, site);
      return false;
    }
  }
}
__device__ __forceinline__ void tma_load_2d(const CUtensorMap *map, uint64_t *bar, void *dst,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void prefetch_map(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes grouped in 8-row (1024-byte) swizzle atoms.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);  // start address
  d |= (uint64_t)1 << 16;                    // leading-dim byte offset (unused here)
  d |= (uint64_t)(1024 >> 4) << 32;          // stride-dim byte offset: 8 rows x 128 B
  d |= (uint64_t)1 << 46;                    // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                    // SWIZZLE_128B
  return d;
}
// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void decode_tile(int tile, const int *mpre, int G, int n_tiles,
                                            int &g, int &n, int &m) {
  int lo = 0, hi = G - 1;  // last g with mpre[g] * n_tiles <= tile (never an empty group)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (mpre[mid] * n_tiles <= tile) lo = mid; else hi = mid - 1;
  }
  g = lo;
  const int mt = mpre[g + 1] - mpre[g];
  const int local = tile - mpre[g] * n_tiles;
  n = local / mt;
  m = local % mt;
}

__device__ __forceinline__ float gelu_erf(float v) {
  return 0.5f * v * (1.f + erff(v * 0.70710678118654752f));
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
k_ffn_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
         const __grid_constant__ CUtensorMap tmB3, TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  SmemCtl *ctl = reinterpret_cast<SmemCtl *>(smem + (size_t)kStages * kStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G;
  int *mpre = ctl->tbl;
  int *offs = ctl->tbl + (G + 1);
  for (int i = tid; i <= G; i += kThreads) {
    mpre[i] = a.mprefix[i];
    offs[i] = a.offsets[i];
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->tfull[s], 1);
      mbar_init(&ctl->tempty[s], 4 * 32);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const int total = mpre[G] * a.n_tiles;
  const int nkb = ceil_div(a.K, kBlockK);
  constexpr int kBStep = (EPI == EPI_SWIGLU) ? kMmaN / 2 : kMmaN;  // weight rows per N tile

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    prefetch_map(&tmA);
    prefetch_map(&tmB);
    if (EPI == EPI_SWIGLU) prefetch_map(&tmB3);
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, last_phase = 0;  // per-stage bit sets, for the abort drain
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      int g, n, m;
      decode_tile(tile, mpre, G, a.n_tiles, g, n, m);
      const int arow = offs[g] + m * kTileM;
      const int brow = g * a.b_rows + n * kBStep;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!wait_bounded(&ctl->empty[stage], phase ^ 1u, ctl, a.err, 1)) { ok = false; break; }
        uint8_t *sa = smem + (size_t)stage * kStageBytes;
        uint8_t *sb = sa + kABytes;
        mbar_expect_tx(&ctl->full[stage], kStageBytes);
        tma_load_2d(&tmA, &ctl->full[stage], sa, kb * kBlockK, arow);
        if (EPI == EPI_SWIGLU) {
          tma_load_2d(&tmB, &ctl->full[stage], sb, kb * kBlockK, brow);
          tma_load_2d(&tmB3, &ctl->full[stage], sb + kBBytes / 2, kb * kBlockK, brow);
        } else {
          tma_load_2d(&tmB, &ctl->full[stage], sb, kb * kBlockK, brow);
        }
        issued |= 1u << stage;
        last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok) {  // let the copies already in flight land before the CTA exits
      for (int s = 0; s < kStages; ++s)
        if (issued & (1u << s))
          wait_bounded(&ctl->full[s], (last_phase >> s) & 1u, ctl, nullptr, 0, false);
    }
  } else if (warp == 1 && lane == 0) {
    // --------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = make_idesc(kTileM, kMmaN);
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true, any = false;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      if (!wait_bounded(&ctl->tempty[acc], acc_phase ^ 1u, ctl, a.err, 2)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem + (uint32_t)(acc * kMmaN);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!wait_bounded(&ctl->full[stage], phase, ctl, a.err, 3)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + (size_t)stage * kStageBytes);
        const uint64_t da = sw128_desc(sa);
        const uint64_t db = sw128_desc(sa + kABytes);
#pragma unroll
        for (int kk = 0; kk < kBlockK / 16; ++kk)  // +32 bytes per K=16 step
          umma_bf16(d_tmem, da + 2 * kk, db + 2 * kk, idesc, (kb | kk) != 0);
        any = true;
        umma_commit(&ctl->empty[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      umma_commit(&ctl->tfull[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (!ok && any) {  // retire the MMAs in flight before TMEM is released
      umma_commit(&ctl->drain);
      wait_bounded(&ctl->drain, 0, ctl, nullptr, 0, false);
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------------- epilogue
    const int ew = warp - 4;  // TMEM lanes [32*ew, 32*ew + 32)
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int g, n, m;
      decode_tile(tile, mpre, G, a.n_tiles, g, n, m);
      bool ok = wait_bounded(&ctl->tfull[acc], acc_phase, ctl, a.err, 4);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int grow = m * kTileM + ew * 32 + lane;
      const bool valid = grow < offs[g + 1] - offs[g];
      const size_t orow = (size_t)offs[g] + grow;
      const uint32_t tbase = tmem + ((uint32_t)(ew * 32) << 16) + (uint32_t)(acc * kMmaN);
      if (EPI == EPI_SWIGLU) {
        __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(a.out);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t gv[32], uv[32];
          tmem_ld32(tbase + c * 32, gv);
          tmem_ld32(tbase + kMmaN / 2 + c * 32, uv);
          tmem_ld_wait();
          const int col0 = n * (kMmaN / 2) + c * 32;
          if (valid && col0 < a.N) {
            uint4 *dst = reinterpret_cast<uint4 *>(out + orow * a.N + col0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float h[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float gt = __uint_as_float(gv[q * 8 + j]);
                const float up = __uint_as_float(uv[q * 8 + j]);
                h[j] = gt / (1.f + __expf(-gt)) * up;
              }
              dst[q] = pack16(h);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < kMmaN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tbase + c * 32, v);
          tmem_ld_wait();
          const int col0 = n * kMmaN + c * 32;
          if (valid && col0 < a.N) {
            float f[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              float x = __uint_as_float(v[j]);
              if (a.bias) x += __ldg(a.bias + (size_t)g * a.N + col0 + j);
              if (EPI == EPI_ACT) x = (a.act == MOE_ACT_RELU) ? fmaxf(x, 0.f) : gelu_erf(x);
              f[j] = x;
            }
            if (a.out_f32) {
              float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + orow * a.N + col0);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
            } else {
              uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) +
                                                     orow * a.N + col0);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                float h[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) h[j] = f[q * 8 + j];
                dst[q] = pack16(h);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl->tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 map over a row-major [rows, cols] matrix; box = [box_rows, 64 cols].
bool make_map(CUtensorMap *map, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBlockK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct DeviceInfo {
  int sms = 0;
  bool attr_set[3] = {false, false, false};
};

DeviceInfo &device_info(int dev) {
  static DeviceInfo infos[64];
  return infos[dev & 63];
}

template <int EPI>
cudaError_t launch_one(const CUtensorMap &ma, const CUtensorMap &mb, const CUtensorMap &mb3,
                       const TcArgs &t, int grid, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  DeviceInfo &info = device_info(dev);
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!info.attr_set[EPI]) {
      e = cudaFuncSetAttribute(k_ffn_tc<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSmemBytes);
      if (e != cudaSuccess) return e;
      info.attr_set[EPI] = true;
    }
  }
  k_ffn_tc<EPI><<<grid, kThreads, kSmemBytes, st>>>(ma, mb, mb3, t);
  return cudaGetLastError();
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  DeviceInfo &info = device_info(dev);
  if (info.sms == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    info.sms = n;
  }
  return info.sms;
}

}  // namespace

cudaError_t launch_ffn_tc(const GroupedFfnArgs &a, cudaStream_t st) {
  if (a.m_tiles_ub <= 0) return cudaSuccess;
  const int sms = sm_count();
  const bool swiglu = a.act == MOE_ACT_SWIGLU;
  CUtensorMap ma, mb, mb3;
  // up projection: [rows, d] x [G*F, d]^T -> h [rows, F]
  if (!make_map(&ma, a.a, (uint64_t)a.a_rows, (uint64_t)a.d, kTileM)) return cudaErrorInvalidValue;
  if (!make_map(&mb, a.w1, (uint64_t)a.G * a.F, (uint64_t)a.d, swiglu ? kMmaN / 2 : kMmaN))
    return cudaErrorInvalidValue;
  if (swiglu) {
    if (!make_map(&mb3, a.w3, (uint64_t)a.G * a.F, (uint64_t)a.d, kMmaN / 2))
      return cudaErrorInvalidValue;
  } else {
    mb3 = mb;
  }
  TcArgs t{};
  t.offsets = a.offsets;
  t.mprefix = a.mprefix;
  t.G = a.G;
  t.N = a.F;
  t.K = a.d;
  t.n_tiles = ceil_div(a.F, swiglu ? kMmaN / 2 : kMmaN);
  t.b_rows = a.F;
  t.out = a.h;
  t.out_f32 = 0;
  t.bias = a.b1;
  t.act = a.act;
  t.err = a.err;
  int grid = (int)std::min<long long>((long long)a.m_tiles_ub * t.n_tiles, sms);
  cudaError_t e = swiglu ? launch_one<EPI_SWIGLU>(ma, mb, mb3, t, grid, st)
                         : launch_one<EPI_ACT>(ma, mb, mb3, t, grid, st);
  if (e != cudaSuccess) return e;
  // down projection: h [rows, F] x [G*d, F]^T -> out [rows, d]
  if (!make_map(&ma, a.h, (uint64_t)a.a_rows, (uint64_t)a.F, kTileM)) return cudaErrorInvalidValue;
  if (!make_map(&mb, a.w2, (uint64_t)a.G * a.d, (uint64_t)a.F, kMmaN)) return cudaErrorInvalidValue;
  t.N = a.d;
  t.K = a.F;
  t.n_tiles = ceil_div(a.d, kMmaN);
  t.b_rows = a.d;
  t.out = a.out;
  t.out_f32 = a.out_f32;
  t.bias = a.b2;
  t.act = -1;
  grid = (int)std::min<long long>((long long)a.m_tiles_ub * t.n_tiles, sms);
  return launch_one<EPI_DOWN>(ma, mb, mb, t, grid, st);
}

}  // namespace moe

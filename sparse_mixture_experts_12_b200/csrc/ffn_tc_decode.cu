// Expert FFN for small batches (decode-sized T: a few rows per expert).
//
// Same arithmetic as ffn_tc.cu (youngju.dev "SwiGLUExpert"; devtips.kr /
// youngju.dev (zh) "MoELayer" MLP experts), arranged for weight streaming: the
// expert's weight rows sit on the MMA's M side (128 per tile) and up to 32 of its
// token rows on its N side (more rows are handled as further 32-row chunks), so a
// tile costs 4 small MMAs per 64-wide K slice and the kernel is bound by reading
// the weights. The down projection splits
// K across CTAs, as many splits (up to 16) as it takes to even out the tiles of
// the persistent grid's CTAs when there are few (expert, 128-row) tiles; the
// splits write fp32 partial sums that a reduction kernel adds in a fixed order.
//
// Tile = (expert g, 32-row chunk c of its rows, 128 weight rows n, K split s). Warp 0: TMA producer
// (weight rows of W_gate [and W_up] + the expert's 32 activation rows per stage),
// warp 1: MMA issuer (tcgen05.mma M=128 N=32 K=16), warp 2: TMEM allocator,
// warps 4..7: epilogue (TMEM lane = weight row, columns = tokens), writing
// h[token][row] (coalesced across the warp's lanes) or the fp32 partials.
#include <algorithm>
#include <atomic>

#include "tc_ptx.cuh"

namespace moe {

namespace {

using namespace tc;

constexpr int kSwapN = 32;                       // token columns per tile
constexpr int kSwapM = 128;                      // weight rows per tile
constexpr int kSwapStages = 6;
constexpr int kWBytes = kSwapM * kBlockK * 2;    // one weight tile slice (16 KB)
constexpr int kXBytes = kSwapN * kBlockK * 2;    // the token slice (4 KB)
constexpr int kSwapStageBytes = 2 * kWBytes + kXBytes;
constexpr int kSwapThreads = 256;
constexpr int kSwapTmemCols = 128;               // 2 buffers x (gate 32 | up 32)
constexpr int kMaxSplit = 16;

enum { SW_SWIGLU = 0, SW_ACT = 1, SW_DOWN = 2 };
enum { OUT_BF16 = 0, OUT_F32 = 1, OUT_PARTIAL = 2 };

struct SwapArgs {
  const int32_t *offsets;
  const int32_t *mprefix;  // 128-row tile prefix (zero for empty experts / invalid offsets)
  int G;
  int n_blocks;            // 128-row weight blocks per expert
  int splits;              // K splits
  int kb_per_split;        // 64-wide K slices per split
  int K;
  int w_rows;              // weight rows per expert in the weight map (= N)
  int N;                   // output columns (F for the up projection, d for the down)
  void *out;               // h / y_perm / fp32 partials [splits][rows][N]
  size_t part_stride;      // elements between two splits' partials
  int out_mode;
  const float *bias;       // [G, N] or nullptr
  int act;
  int32_t *err;
};

struct SwapCtl {
  uint64_t full[kSwapStages];
  uint64_t empty[kSwapStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int tbl[2 * (kMaxExperts + 1)];  // 32-row chunk prefix [G+1], offsets [G+1]
};

constexpr size_t kSwapSmemBytes = (size_t)kSwapStages * kSwapStageBytes + sizeof(SwapCtl) + 1024;

__device__ __forceinline__ bool wait_swap(uint64_t *bar, uint32_t parity, SwapCtl *ctl,
                                          int32_t *err, int site, bool honour_abort = true) {
  return wait_mbar(bar, parity, &ctl->abort_flag, 0u, err, site, honour_abort, kWaitLimitNs);
}

template <int EPI>
__global__ void __launch_bounds__(kSwapThreads, 1)
k_ffn_swap(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmW3,
           const __grid_constant__ CUtensorMap tmX, SwapArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  SwapCtl *ctl = reinterpret_cast<SwapCtl *>(smem + (size_t)kSwapStages * kSwapStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G;
  int *cpre = ctl->tbl;  // prefix of 32-row chunks per expert
  int *offs = ctl->tbl + (G + 1);
  for (int i = tid; i <= G; i += kSwapThreads) offs[i] = a.offsets[i];
  if (warp == 3) {
    // chunks per expert = ceil(rows / 32), zero where the 128-row prefix says the
    // expert is empty (or the offsets failed validation); warp scan over experts
    const int per = ceil_div(G, 32);
    const int j0 = min(G, lane * per), j1 = min(G, j0 + per);
    auto chunks = [&](int j) {
      return (a.mprefix[j + 1] > a.mprefix[j]) ? ceil_div(a.offsets[j + 1] - a.offsets[j], kSwapN)
                                               : 0;
    };
    int sum = 0;
    for (int j = j0; j < j1; ++j) sum += chunks(j);
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - sum;
    for (int j = j0; j < j1; ++j) {
      cpre[j] = run;
      run += chunks(j);
    }
    if (lane == 31) cpre[G] = incl;
  }
  if (tid == 0) {
    for (int s = 0; s < kSwapStages; ++s) {
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
    tmem_alloc(&ctl->tmem_base, kSwapTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the kernel after this one may be placed as soon as SMs free up; it waits for
  // this grid before it reads anything this grid writes
  pdl_trigger();
  const uint32_t tmem = ctl->tmem_base;
  const int per_expert = a.n_blocks * a.splits;
  const int total = cpre[G] * per_expert;
  const int nkb = ceil_div(a.K, kBlockK);
  constexpr bool kTwo = (EPI == SW_SWIGLU);
  constexpr uint32_t kTxBytes = (kTwo ? 2 : 1) * kWBytes + kXBytes;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    prefetch_map(&tmW);
    prefetch_map(&tmX);
    if (kTwo) prefetch_map(&tmW3);
    int stage = 0;
    uint32_t phase = 0, issued = 0, last_phase = 0;
    bool ok = true;
    // The weights and the tile tables (from the routing, which has completed before
    // the kernel ahead of this one passed its own wait) do not depend on the kernel
    // ahead: the first stages' weight slices are requested before waiting for it.
    // The activation rows (its output) only after the wait.
    int early = 0;
    for (int tile = blockIdx.x; early < kSwapStages && tile < total; tile += gridDim.x) {
      int g, nn, ch;
      decode_tile(tile, cpre, G, per_expert, g, nn, ch);
      const int nb = nn / a.splits, sp = nn % a.splits;
      const int kb0 = sp * a.kb_per_split, kb1 = min(nkb, kb0 + a.kb_per_split);
      const int wrow = g * a.w_rows + nb * kSwapM;
      for (int kb = kb0; kb < kb1 && early < kSwapStages; ++kb, ++early) {
        uint8_t *sw = smem + (size_t)early * kSwapStageBytes;
        mbar_expect_tx(&ctl->full[early], kTxBytes);
        tma_load_2d(&tmW, &ctl->full[early], sw, kb * kBlockK, wrow);
        if (kTwo) tma_load_2d(&tmW3, &ctl->full[early], sw + kWBytes, kb * kBlockK, wrow);
      }
    }
    pdl_wait();
    int step = 0;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      int g, nn, ch;
      decode_tile(tile, cpre, G, per_expert, g, nn, ch);
      const int nb = nn / a.splits, sp = nn % a.splits;
      const int kb0 = sp * a.kb_per_split, kb1 = min(nkb, kb0 + a.kb_per_split);
      const int wrow = g * a.w_rows + nb * kSwapM;
      const int xrow = offs[g] + ch * kSwapN;
      for (int kb = kb0; kb < kb1; ++kb, ++step) {
        // the first `early` stages are free (first use) and already carry their weight
        // copies: they get their activation copies whatever happens, so that every
        // copy issued completes its stage's barrier
        if (step >= early &&
            !wait_swap(&ctl->empty[stage], phase ^ 1u, ctl, a.err, 11)) {
          ok = false;
          break;
        }
        uint8_t *sw = smem + (size_t)stage * kSwapStageBytes;
        if (step >= early) {
          mbar_expect_tx(&ctl->full[stage], kTxBytes);
          tma_load_2d(&tmW, &ctl->full[stage], sw, kb * kBlockK, wrow);
          if (kTwo) tma_load_2d(&tmW3, &ctl->full[stage], sw + kWBytes, kb * kBlockK, wrow);
        }
        tma_load_2d(&tmX, &ctl->full[stage], sw + 2 * kWBytes, kb * kBlockK, xrow);
        issued |= 1u << stage;
        last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == kSwapStages) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok) {
      for (int s = 0; s < kSwapStages; ++s)
        if (issued & (1u << s))
          wait_swap(&ctl->full[s], (last_phase >> s) & 1u, ctl, nullptr, 0, false);
    }
  } else if (warp == 1 && lane == 0) {
    // --------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = make_idesc(kSwapM, kSwapN);
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true, any = false;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      int g, nn, ch;
      decode_tile(tile, cpre, G, per_expert, g, nn, ch);
      const int sp = nn % a.splits;
      const int kb0 = sp * a.kb_per_split, kb1 = min(nkb, kb0 + a.kb_per_split);
      if (!wait_swap(&ctl->tempty[acc], acc_phase ^ 1u, ctl, a.err, 12)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d1 = tmem + (uint32_t)(acc * 2 * kSwapN);
      const uint32_t d3 = d1 + kSwapN;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_swap(&ctl->full[stage], phase, ctl, a.err, 13)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sw = smem_u32(smem + (size_t)stage * kSwapStageBytes);
        const uint64_t dw = sw128_desc(sw);
        const uint64_t dw3 = sw128_desc(sw + kWBytes);
        const uint64_t dx = sw128_desc(sw + 2 * kWBytes);
#pragma unroll
        for (int kk = 0; kk < kBlockK / 16; ++kk) {
          const uint32_t accum = (kb != kb0 || kk != 0) ? 1u : 0u;
          umma_bf16(d1, dw + 2 * kk, dx + 2 * kk, idesc, accum);
          if (kTwo) umma_bf16(d3, dw3 + 2 * kk, dx + 2 * kk, idesc, accum);
        }
        any = true;
        umma_commit(&ctl->empty[stage]);
        if (++stage == kSwapStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      umma_commit(&ctl->tfull[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (!ok && any) {
      umma_commit(&ctl->drain);
      wait_swap(&ctl->drain, 0, ctl, nullptr, 0, false);
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------------- epilogue
    const int ew = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int g, nn, ch;
      decode_tile(tile, cpre, G, per_expert, g, nn, ch);
      const int nb = nn / a.splits, sp = nn % a.splits;
      bool ok = wait_swap(&ctl->tfull[acc], acc_phase, ctl, a.err, 14);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int n = nb * kSwapM + ew * 32 + lane;  // output column of this lane
      const int row0 = offs[g] + ch * kSwapN;
      const int rows = min(kSwapN, offs[g + 1] - row0);
      const uint32_t tb = tmem + ((uint32_t)(ew * 32) << 16) + (uint32_t)(acc * 2 * kSwapN);
      uint32_t v1[32], v3[32];
      tmem_ld32(tb, v1);
      if (kTwo) tmem_ld32(tb + kSwapN, v3);
      tmem_ld_wait();
      if (n < a.N) {
        const float b = (a.bias && sp == 0) ? __ldg(a.bias + (size_t)g * a.N + n) : 0.f;
#pragma unroll
        for (int t = 0; t < kSwapN; ++t) {  // fully unrolled: v1/v3 stay in registers
          if (t >= rows) break;
          const size_t o = (size_t)(row0 + t) * a.N + n;
          float v = __uint_as_float(v1[t]);
          if (EPI == SW_SWIGLU) {
            v = __fdividef(v, 1.f + __expf(-v)) * __uint_as_float(v3[t]);
          } else if (EPI == SW_ACT) {
            v += b;
            v = (a.act == MOE_ACT_RELU) ? fmaxf(v, 0.f) : gelu_erf(v);
          } else {
            v += b;
          }
          if (a.out_mode == OUT_PARTIAL)
            static_cast<float *>(a.out)[(size_t)sp * a.part_stride + o] = v;
          else if (a.out_mode == OUT_F32)
            static_cast<float *>(a.out)[o] = v;
          else
            static_cast<__nv_bfloat16 *>(a.out)[o] = __float2bfloat16_rn(v);
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
    tmem_dealloc(tmem, kSwapTmemCols);
  }
}

// Sum the K-split partials in split order and store rows [0, offsets[G]).
__global__ void __launch_bounds__(256) k_splitk_reduce(const float *__restrict__ part, int splits,
                                                       size_t part_stride,
                                                       const int32_t *__restrict__ offsets, int G,
                                                       int N, void *out, int out_f32) {
  pdl_wait();
  pdl_trigger();
  const size_t n = (size_t)offsets[G] * N;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    float s = part[i];
    for (int sp = 1; sp < splits; ++sp) s += part[(size_t)sp * part_stride + i];
    if (out_f32)
      static_cast<float *>(out)[i] = s;
    else
      static_cast<__nv_bfloat16 *>(out)[i] = __float2bfloat16_rn(s);
  }
}

template <int EPI>
cudaError_t launch_swap(const CUtensorMap &mw, const CUtensorMap &mw3, const CUtensorMap &mx,
                        const SwapArgs &s, long long tiles_ub, cudaStream_t st) {
  static std::atomic<bool> attr_done[64];  // idempotent: a racing second call sets the same value
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!attr_done[dev & 63].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(k_ffn_swap<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSwapSmemBytes);
    if (e != cudaSuccess) return e;
    attr_done[dev & 63].store(true, std::memory_order_release);
  }
  const int grid = (int)std::max<long long>(1, std::min<long long>(tiles_ub, sm_count()));
  return launch_pdl(k_ffn_swap<EPI>, dim3(grid), dim3(kSwapThreads), kSwapSmemBytes, st, mw, mw3,
                    mx, s);
}

}  // namespace

size_t ffn_decode_partial_bytes(int max_rows, int d) {
  return (size_t)kMaxSplit * (size_t)max_rows * (size_t)d * sizeof(float);
}

cudaError_t launch_ffn_tc_decode(const GroupedFfnArgs &a, cudaStream_t st) {
  if (a.m_tiles_ub <= 0) return cudaSuccess;
  const bool swiglu = a.act == MOE_ACT_SWIGLU;
  // upper bound on the 32-row chunks over all experts
  const long long touched_ub = std::min<long long>(a.G, a.a_rows) + a.a_rows / kSwapN;
  CUtensorMap mw, mw3, mx;
  // up projection: h[t][f] = act(x_t . W1[f]) for the expert's rows
  if (!make_map(&mw, a.w1, (uint64_t)a.G * a.F, (uint64_t)a.d, kSwapM)) return cudaErrorInvalidValue;
  if (swiglu) {
    if (!make_map(&mw3, a.w3, (uint64_t)a.G * a.F, (uint64_t)a.d, kSwapM))
      return cudaErrorInvalidValue;
  } else {
    mw3 = mw;
  }
  if (!make_map(&mx, a.a, (uint64_t)a.a_rows, (uint64_t)a.d, kSwapN)) return cudaErrorInvalidValue;
  SwapArgs s{};
  s.offsets = a.offsets;
  s.mprefix = a.mprefix;
  s.G = a.G;
  s.n_blocks = ceil_div(a.F, kSwapM);
  s.splits = 1;
  s.K = a.d;
  s.kb_per_split = ceil_div(a.d, kBlockK);
  s.w_rows = a.F;
  s.N = a.F;
  s.out = a.h;
  s.out_mode = OUT_BF16;
  s.bias = a.b1;
  s.act = a.act;
  s.err = a.err;
  cudaError_t e = swiglu ? launch_swap<SW_SWIGLU>(mw, mw3, mx, s, touched_ub * s.n_blocks, st)
                         : launch_swap<SW_ACT>(mw, mw3, mx, s, touched_ub * s.n_blocks, st);
  if (e != cudaSuccess) return e;
  // down projection: y[t][c] = h_t . W2[c], K split so that enough CTAs stream weights
  if (!make_map(&mw, a.w2, (uint64_t)a.G * a.d, (uint64_t)a.F, kSwapM)) return cudaErrorInvalidValue;
  if (!make_map(&mx, a.h, (uint64_t)a.a_rows, (uint64_t)a.F, kSwapN)) return cudaErrorInvalidValue;
  const int nkb = ceil_div(a.F, kBlockK);
  const long long units = touched_ub * ceil_div(a.d, kSwapM);
  // K splits: the fewest that bring the K slices of the busiest CTA (whole tiles
  // over the persistent grid) to within 3 % of the best count up to kMaxSplit, so
  // that a last, partly filled wave of tiles does not leave a few CTAs streaming
  // alone (Mixtral T = 1: 64 weight blocks, 9 splits -> 576 tiles, 4 per CTA)
  const long long sms = sm_count();
  auto busiest = [&](int sp) {
    const int kb = ceil_div(nkb, sp);
    return (double)((units * sp + sms - 1) / sms) * kb;
  };
  double best = 1e300;
  for (int sp = 1; sp <= std::min(kMaxSplit, nkb); ++sp) best = std::min(best, busiest(sp));
  int splits = 1;
  while (splits < std::min(kMaxSplit, nkb) && busiest(splits) > 1.03 * best) ++splits;
  const int kbps = ceil_div(nkb, splits);
  splits = ceil_div(nkb, kbps);  // every split gets at least one K slice
  const bool partial = splits > 1 && a.part != nullptr;
  if (!partial) splits = 1;
  s.n_blocks = ceil_div(a.d, kSwapM);
  s.splits = splits;
  s.kb_per_split = partial ? kbps : nkb;
  s.K = a.F;
  s.w_rows = a.d;
  s.N = a.d;
  s.bias = a.b2;
  s.act = -1;
  s.part_stride = (size_t)a.a_rows * a.d;
  s.out = partial ? static_cast<void *>(a.part) : a.out;
  s.out_mode = partial ? OUT_PARTIAL : (a.out_f32 ? OUT_F32 : OUT_BF16);
  e = launch_swap<SW_DOWN>(mw, mw, mx, s, touched_ub * s.n_blocks * splits, st);
  if (e != cudaSuccess || !partial) return e;
  return launch_pdl(k_splitk_reduce, dim3(std::min(ceil_div(a.a_rows * a.d, 256), 4 * sm_count())),
                    dim3(256), 0, st, (const float *)a.part, splits, s.part_stride, a.offsets, a.G,
                    a.d, a.out, a.out_f32);
}

}  // namespace moe

// Grouped expert FFN on the 5th-generation tensor cores (tcgen05 + TMEM), bf16
// operands, fp32 accumulation.
//
// Experts: youngju.dev "SwiGLUExpert" (w_down(silu(w_gate x) * w_up x)), the
// "SiLU · SwiGLU · MoE" table of the study-site lecture, devtips.kr "MoELayer"
// (ReLU MLP) and youngju.dev (zh) "MoELayer" (GELU MLP). Only the rows routed to
// an expert are multiplied by its weights ("Token Routing": unselected experts
// are not computed at all).
//
// Design (persistent, warp-specialised):
//   warp 0      TMA producer: A rows of the expert-contiguous activations and the
//               expert's weight rows, 64-element K slices with 128-byte swizzle,
//               into a shared-memory ring.
//   warp 1      MMA issuer: tcgen05.mma (kind::f16, fp32 accumulate in TMEM).
//   warp 2      TMEM allocator.
//   warps 4..   epilogue (the warps of a TMEM lane quarter split the columns:
//               two per quarter in the CTA-pair kernel, four in the single-CTA
//               kernel): tcgen05.ld, fused silu(g)*u / bias+ReLU / bias+GELU,
//               bf16 (or fp32) stores masked to the expert's rows.
// Tile shapes, chosen per projection by its reduction length K:
//   K >= 2048  a CTA pair (cluster of 2, tcgen05.mma.cta_group::2): 256 rows x 512
//              columns, two M256 N256 MMAs per K step into one 512-column
//              accumulator, 4 x 48 KB stages per CTA;
//   K <  2048  a single CTA: 128 rows x 256 columns, two 256-column accumulators
//              (the epilogue overlaps the next tile), 4 x 48 KB stages.
// A 256 x 256 pair tile (6 x 32 KB stages) is built with -DMOE_TC_PAIR.
// For SwiGLU each 256 MMA columns are w_gate rows next to the same w_up rows, so
// one MMA yields both halves of silu(g) * u.
// The tile list is built on the device (per-expert M-tile prefix), so no host
// synchronisation sits between routing and the expert GEMMs. Every wait is
// bounded; on a timeout the CTA records MOE_DEVERR_WAIT_TIMEOUT, drains its
// in-flight copies and MMAs, frees TMEM and returns.
#include <algorithm>
#include <mutex>

#include "tc_ptx.cuh"

namespace moe {

namespace {

using namespace tc;

constexpr int kStages = 4;
constexpr int kTileM = kRowTile;
constexpr int kMmaN = 256;
constexpr int kABytes = kTileM * kBlockK * 2;
constexpr int kBBytes = kMmaN * kBlockK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 2 * kMmaN;
constexpr int kThreads = 384;  // warps 0-3: producer, MMA, TMEM, spare; 4-11: epilogue
constexpr int kEpiWarps = 8;
// single-CTA kernel: sixteen epilogue warps (four per TMEM lane quarter, a quarter
// of the columns each). Its tiles are short (K < 2048), so the fused activation of
// one tile must keep up with the next tile's main loop; the erf-GELU epilogue of
// eight warps did not (latency-bound, about a third of an instruction per cycle).
constexpr int kEpiWarps1 = 16;
constexpr int kThreads1 = 128 + 32 * kEpiWarps1;

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
  int tile_mode;  // TILES_ALL, or the pair / tail halves of a split launch
  int tma_store;  // pair kernel, bf16 output: full 32-row groups leave through TMA stores
  int pdl_mode;            // PDL_NONE, PDL_WAIT (wait before the first dependent access)
                           // or PDL_TAIL (the tail-tile launch: wait only before exit)
  uint64_t wait_limit_ns;  // single-CTA kernel: bound on its pipeline waits
  int withhold_load;       // single-CTA kernel, test hook: the first operand load of each
                           // CTA is never issued, so the waits on it run out
};

// The output path of one epilogue warp for one tile. With a map, a chunk whose 32
// rows are all the expert's is staged in the warp's 2 KB shared-memory buffer (64-
// byte swizzle) and written by one TMA store; other chunks use masked direct stores.
struct EpiStore {
  const CUtensorMap *map;  // 32 x 32 bf16 output boxes, or nullptr
  uint8_t *stage;          // this warp's staging buffer
  bool rows_full;          // all 32 rows of the warp belong to the expert
  int row0;                // output row of lane 0
};
constexpr int kStageOutBytes = kStoreBox * kStoreBox * 2;  // 2 KB per epilogue warp

// one 32-row x 32-column bf16 chunk (pk = this lane's row) to global memory
__device__ __forceinline__ void emit_chunk(const EpiStore &st, const uint4 (&pk)[4],
                                           __nv_bfloat16 *dst_row, int col0) {
  if (st.map != nullptr && st.rows_full) {
    const int lane = threadIdx.x & 31;
    if (lane == 0) bulk_wait_read_all();  // the previous store has read the buffer
    __syncwarp();
    uint4 *row = reinterpret_cast<uint4 *>(st.stage + lane * 64);
    const int sw = (lane >> 1) & 3;
#pragma unroll
    for (int q = 0; q < 4; ++q) row[q ^ sw] = pk[q];
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(st.map, st.stage, col0, st.row0);
      bulk_commit();
    }
  } else {
    uint4 *dst = reinterpret_cast<uint4 *>(dst_row + col0);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = pk[q];
  }
}

// Row tiles of an expert with c rows: mt = ceil(c / 128). A split launch gives the
// CTA-pair kernel the floor(mt / 2) full pair tiles and, when mt is odd (the last
// 128-row tile holds at most 128 rows), hands that tile to the single-CTA kernel
// instead of a 256-row pair tile that would be at least half empty.
enum { TILES_ALL = 0, TILES_PAIRS_NO_TAIL = 1, TILES_TAIL_ONLY = 2 };

// Programmatic dependent launch of a GEMM (see pdl_wait). PDL_TAIL: the tail-tile
// launch reads nothing the pair grid before it writes, so it starts at once; it
// waits for that grid only before it exits, so that its completion tells the
// kernels after it that the pair grid has completed too.
enum { PDL_NONE = 0, PDL_WAIT = 1, PDL_TAIL = 2 };

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


__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, SmemCtl *ctl,
                                             int32_t *err, int site, bool honour_abort = true,
                                             uint64_t limit_ns = kWaitLimitNs) {
  return wait_mbar(bar, parity, &ctl->abort_flag, 0u, err, site, honour_abort, limit_ns);
}

// ------------------------------------------------------------ shared epilogue
// One accumulator tile (this thread's TMEM lane = one output row) -> global.
// SwiGLU: columns [0,128) hold x.w_gate, [128,256) x.w_up; h = silu(g) * u.
// ACT: bias + ReLU / GELU. DOWN: + bias. Stores are masked to the valid row and
// to the N extent.
// Columns go in 32-wide chunks c in [c0, c1). SwiGLU: the gate value of chunk c
// sits at accumulator column acc_off + 32c and the up value 128 columns further;
// other tiles: accumulator column acc_off + 32c. Output column = out_base + 32c.
template <int EPI>
__device__ __forceinline__ void epilogue_tile(const TcArgs &a, uint32_t tbase, int g, int acc_off,
                                              int out_base, int c0, int c1, bool valid,
                                              size_t orow, const EpiStore &st) {
  if (EPI == EPI_SWIGLU) {
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(a.out);
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      uint32_t gv[32], uv[32];
      tmem_ld32(tbase + acc_off + c * 32, gv);
      tmem_ld32(tbase + acc_off + kMmaN / 2 + c * 32, uv);
      tmem_ld_wait();
      const int col0 = out_base + c * 32;
      if (valid && col0 < a.N) {  // rows_full implies valid on every lane
        uint4 pk[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float h[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float gt = __uint_as_float(gv[q * 8 + j]);
            const float up = __uint_as_float(uv[q * 8 + j]);
            h[j] = __fdividef(gt, 1.f + __expf(-gt)) * up;
          }
          pk[q] = pack16(h);
        }
        emit_chunk(st, pk, out + orow * a.N, col0);
      }
    }
  } else {
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      uint32_t v[32];
      tmem_ld32(tbase + acc_off + c * 32, v);
      tmem_ld_wait();
      const int col0 = out_base + c * 32;
      if (valid && col0 < a.N) {
        float f[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
        if (a.bias) {  // the same 32 values for every lane: broadcast 16-byte loads
          const float4 *b4 = reinterpret_cast<const float4 *>(a.bias + (size_t)g * a.N + col0);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 b = __ldg(b4 + q);
            f[4 * q] += b.x; f[4 * q + 1] += b.y; f[4 * q + 2] += b.z; f[4 * q + 3] += b.w;
          }
        }
        if (EPI == EPI_ACT) {
          if (a.act == MOE_ACT_RELU) {
#pragma unroll
            for (int j = 0; j < 32; ++j) f[j] = fmaxf(f[j], 0.f);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) f[j] = gelu_erf(f[j]);
          }
        }
        if (a.out_f32) {
          float4 *dst =
              reinterpret_cast<float4 *>(static_cast<float *>(a.out) + orow * a.N + col0);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
        } else {
          uint4 pk[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float h[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) h[j] = f[q * 8 + j];
            pk[q] = pack16(h);
          }
          emit_chunk(st, pk, static_cast<__nv_bfloat16 *>(a.out) + orow * a.N, col0);
        }
      }
    }
  }
}

// =========================================================== single-CTA kernel
template <int EPI>
__global__ void __launch_bounds__(kThreads1, 1)
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
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->tfull[s], 1);
      mbar_init(&ctl->tempty[s], kEpiWarps1 * 32);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // The set-up above overlaps the previous kernel. So do the tile tables: they come
  // from the routing, which completed before the kernel ahead of this one passed its
  // own wait (or, in a standalone call, from the table kernel, which does not let
  // this grid start early), and the first stages' weight slices. The producer waits
  // for the kernel ahead before it requests the activation rows (its output).
  for (int i = tid; i <= G; i += kThreads1) {
    if (a.tile_mode != TILES_TAIL_ONLY) mpre[i] = a.mprefix[i];
    offs[i] = a.offsets[i];
  }
  if (a.tile_mode == TILES_TAIL_ONLY && warp == 3) {
    // one tile per expert with an odd row-tile count: its last 128-row tile
    const int per = ceil_div(G, 32);
    const int j0 = min(G, lane * per), j1 = min(G, j0 + per);
    int sum = 0;
    for (int j = j0; j < j1; ++j) sum += (a.mprefix[j + 1] - a.mprefix[j]) & 1;
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - sum;
    for (int j = j0; j < j1; ++j) {
      mpre[j] = run;
      run += (a.mprefix[j + 1] - a.mprefix[j]) & 1;
    }
    if (lane == 31) mpre[G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (a.pdl_mode == PDL_WAIT) pdl_trigger();
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
    uint32_t issued = 0, last_phase = 0;  // per-stage bit sets, for the end-of-role drain
    bool ok = true;
    auto load_b = [&](int st, int kb, int brow) {
      uint8_t *sb = smem + (size_t)st * kStageBytes + kABytes;
      tma_load_2d(&tmB, &ctl->full[st], sb, kb * kBlockK, brow);
      if (EPI == EPI_SWIGLU)
        tma_load_2d(&tmB3, &ctl->full[st], sb + kBBytes / 2, kb * kBlockK, brow);
    };
    // test hook: the CTA's first stage is never loaded, so the MMA issuer's wait on it
    // (and then the producer's wait for that stage to drain) runs out
    auto withheld = [&](int tile, int kb) {
      return a.withhold_load && tile == (int)blockIdx.x && kb == 0;
    };
    // the first stages' weight slices, before the wait for the kernel ahead
    int early = 0;
    for (int tile = blockIdx.x; early < kStages && tile < total; tile += gridDim.x) {
      int g, n, m;
      decode_tile(tile, mpre, G, a.n_tiles, g, n, m);
      const int brow = g * a.b_rows + n * kBStep;
      for (int kb = 0; kb < nkb && early < kStages; ++kb, ++early) {
        if (withheld(tile, kb)) continue;
        mbar_expect_tx(&ctl->full[early], kStageBytes);
        load_b(early, kb, brow);
      }
    }
    if (a.pdl_mode == PDL_WAIT) pdl_wait();
    int step = 0;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      int g, n, m;
      decode_tile(tile, mpre, G, a.n_tiles, g, n, m);
      if (a.tile_mode == TILES_TAIL_ONLY) m = ceil_div(offs[g + 1] - offs[g], kTileM) - 1;
      const int arow = offs[g] + m * kTileM;
      const int brow = g * a.b_rows + n * kBStep;
      for (int kb = 0; kb < nkb; ++kb, ++step) {
        // the first `early` stages are free (first use) and already carry their weight
        // copies: they get their activation copies whatever happens, so that every
        // copy issued completes its stage's barrier
        if (step >= early && !wait_bounded(&ctl->empty[stage], phase ^ 1u, ctl, a.err, 1,
                                           true, a.wait_limit_ns)) {
          ok = false;
          break;
        }
        if (!withheld(tile, kb)) {
          uint8_t *sa = smem + (size_t)stage * kStageBytes;
          if (step >= early) {
            mbar_expect_tx(&ctl->full[stage], kStageBytes);
            load_b(stage, kb, brow);
          }
          tma_load_2d(&tmA, &ctl->full[stage], sa, kb * kBlockK, arow);
          issued |= 1u << stage;
          last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        }
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
    // every copy this CTA issued has landed before it can exit, whichever role gave
    // up (a no-op wait on a normal run: the MMAs consumed them all)
    for (int s = 0; s < kStages; ++s)
      if (issued & (1u << s))
        wait_bounded(&ctl->full[s], (last_phase >> s) & 1u, ctl, nullptr, 0, false);
  } else if (warp == 1 && lane == 0) {
    // --------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = make_idesc(kTileM, kMmaN);
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true, any = false;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      if (!wait_bounded(&ctl->tempty[acc], acc_phase ^ 1u, ctl, a.err, 2, true,
                        a.wait_limit_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem + (uint32_t)(acc * kMmaN);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!wait_bounded(&ctl->full[stage], phase, ctl, a.err, 3, true, a.wait_limit_ns)) {
          ok = false;
          break;
        }
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
    const int ew = warp & 3;          // TMEM lanes [32*ew, 32*ew + 32) (warp % 4)
    const int quarter = (warp - 4) >> 2;  // which quarter of the tile's columns
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int g, n, m;
      decode_tile(tile, mpre, G, a.n_tiles, g, n, m);
      if (a.tile_mode == TILES_TAIL_ONLY) m = ceil_div(offs[g + 1] - offs[g], kTileM) - 1;
      bool ok = wait_bounded(&ctl->tfull[acc], acc_phase, ctl, a.err, 4, true, a.wait_limit_ns);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int grow = m * kTileM + ew * 32 + lane;
      const bool valid = grow < offs[g + 1] - offs[g];
      const size_t orow = (size_t)offs[g] + grow;
      const uint32_t tbase = tmem + ((uint32_t)(ew * 32) << 16) + (uint32_t)(acc * kMmaN);
      // the four warps sharing a TMEM lane quarter take a quarter of the columns each
      const EpiStore st{nullptr, nullptr, false, 0};
      if (EPI == EPI_SWIGLU)
        epilogue_tile<EPI>(a, tbase, g, 0, n * (kMmaN / 2), quarter, quarter + 1, valid, orow,
                           st);
      else
        epilogue_tile<EPI>(a, tbase, g, 0, n * kMmaN, 2 * quarter, 2 * quarter + 2, valid, orow,
                           st);
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
  if (a.pdl_mode == PDL_TAIL) pdl_wait();
}

// ============================================================= CTA-pair kernel
// Two CTAs of a cluster share one 256-row tile: CTA r holds A rows [128r, 128r+128)
// and B rows [128r, 128r+128) of the 256-row B tile (for SwiGLU: CTA 0 the w_gate
// rows, CTA 1 the w_up rows). The leader (rank 0) issues tcgen05.mma.cta_group::2
// M=256 N=256 K=16, which reads both CTAs' shared memory and writes both CTAs'
// TMEM (rows 128r.. in CTA r). Each CTA's own TMA loads (no multicast) count on the
// leader's `full` barrier; the MMA commits release `empty` and `tfull` in both
// CTAs; both epilogues release the leader's `tempty`. Per CTA a stage is 32 KB
// (vs 48 KB for the single-CTA tile), so six stages fit.
constexpr int kStages2 = 6;  // ring depth of the 256-column pair tile
constexpr int kPairM = 2 * kTileM;
constexpr int kAHalf = kTileM * kBlockK * 2;
constexpr int kBHalf = (kMmaN / 2) * kBlockK * 2;
// NH = N halves per pair tile. NH = 1: 256 MMA columns, six 32 KB stages, two
// TMEM accumulators. NH = 2: 512 columns (two MMAs per K step), four 48 KB
// stages, one 512-column accumulator: twice the MMA work per stage and 25% fewer
// operand bytes per flop, but the epilogue no longer overlaps the next tile's
// main loop, so it pays off for long K.
template <int NH> struct PairCfg {
  static constexpr int kStages = NH == 1 ? kStages2 : 4;
  static constexpr int kStageBytes = kAHalf + NH * kBHalf;
  static constexpr int kAccBufs = NH == 1 ? 2 : 1;
  static constexpr size_t kRing = (size_t)kStages * kStageBytes;
};
constexpr uint64_t kDrainNs = 50000000ull;  // 50 ms bound on end-of-kernel drains

struct SmemCtl2 {
  uint64_t full[kStages2];   // leader: both CTAs' copies of the stage landed
  uint64_t empty[kStages2];  // each CTA: the pair's MMAs are done with the stage
  uint64_t tfull[2];         // each CTA: accumulator ready for the epilogue
  uint64_t tempty[2];        // leader: both epilogues have drained the accumulator
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int tbl[2 * (kMaxExperts + 1)];  // pair-tile prefix [G+1], offsets [G+1]
};

template <int NH>
constexpr size_t pair_smem_bytes() {
  return PairCfg<NH>::kRing + (size_t)kEpiWarps * kStageOutBytes + sizeof(SmemCtl2) + 1024;
}

// Work items of the persistent pair kernel. With NH = 2, when the last round of
// tiles would leave at least half of the CTA pairs idle (r = total % pairs tiles,
// 0 < 2r <= pairs), those r tiles are issued as 2r half tiles of one N half each,
// so the last round takes half as long. Item -> (tile, sel): sel = -1 for a whole
// tile, else the single N half it covers.
struct PairItems {
  int full, items;
  __device__ PairItems(int total, int pairs, int nh) : full(total), items(total) {
    const int r = total % pairs;
    if (nh == 2 && r > 0 && 2 * r <= pairs) {
      full = total - r;
      items = total + r;
    }
  }
  __device__ int tile(int it, int &sel) const {
    if (it < full) {
      sel = -1;
      return it;
    }
    sel = (it - full) & 1;
    return full + ((it - full) >> 1);
  }
};

// Bounded wait that, on its own timeout, also raises the peer CTA's abort flag.
__device__ __forceinline__ bool wait_pair(uint64_t *bar, uint32_t parity, SmemCtl2 *ctl,
                                          uint32_t peer_abort, int32_t *err, int site,
                                          bool honour_abort = true,
                                          uint64_t limit_ns = kWaitLimitNs) {
  return wait_mbar(bar, parity, &ctl->abort_flag, peer_abort, err, site, honour_abort, limit_ns);
}

template <int EPI, int NH>
__global__ void __launch_bounds__(kThreads, 1)
k_ffn_tc2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
          const __grid_constant__ CUtensorMap tmB3, const __grid_constant__ CUtensorMap tmO,
          TcArgs a) {
  using PC = PairCfg<NH>;
  constexpr int kS = PC::kStages;
  constexpr int kSB = PC::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // ring | 8 x 2 KB output staging (TMA stores) | control block
  SmemCtl2 *ctl = reinterpret_cast<SmemCtl2 *>(smem + PC::kRing + kEpiWarps * kStageOutBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int G = a.G;
  int *ppre = ctl->tbl;
  int *offs = ctl->tbl + (G + 1);
  if (tid == 0) {
    for (int s = 0; s < kS; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {  // NH = 1: two accumulators; NH = 2: two N halves
      mbar_init(&ctl->tfull[s], 1);
      mbar_init(&ctl->tempty[s], 2 * kEpiWarps * 32);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(&ctl->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  // the set-up above overlaps the previous kernel; the tile tables, the operands
  // and the outputs are touched only after it has completed
  if (a.pdl_mode == PDL_WAIT) pdl_wait();
  for (int i = tid; i <= G; i += kThreads) offs[i] = a.offsets[i];
  if (warp == 1) {
    // pair tiles per group = ceil(ceil(rows / 128) / 2) from the 128-row tile prefix
    // (all zero when the offsets failed validation); warp scan over the groups
    const int per = ceil_div(G, 32);
    const int j0 = min(G, lane * per), j1 = min(G, j0 + per);
    const int round_up = a.tile_mode == TILES_PAIRS_NO_TAIL ? 0 : 1;  // an odd last tile
    int sum = 0;
    for (int j = j0; j < j1; ++j) sum += (a.mprefix[j + 1] - a.mprefix[j] + round_up) >> 1;
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - sum;
    for (int j = j0; j < j1; ++j) {
      ppre[j] = run;
      run += (a.mprefix[j + 1] - a.mprefix[j] + round_up) >> 1;
    }
    if (lane == 31) ppre[G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers and TMEM exist before any cross-CTA use
  // a tail-tile launch queued behind this grid (it reads nothing this grid
  // writes) may start on the SMs that this grid's CTAs leave
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const int nkb = ceil_div(a.K, kBlockK);
  const uint32_t peer_abort = mapa_rank(smem_u32(&ctl->abort_flag), rank ^ 1u);
  const int c0 = (int)cluster_index(), cstep = (int)cluster_count();
  const PairItems work(ppre[G] * a.n_tiles, cstep, NH);

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    prefetch_map(&tmA);
    prefetch_map(&tmB);
    if (EPI == EPI_SWIGLU) prefetch_map(&tmB3);
    const uint32_t full0 = mapa_rank(smem_u32(&ctl->full[0]), 0);  // the leader's barriers
    const CUtensorMap *bmap = (EPI == EPI_SWIGLU && rank == 1) ? &tmB3 : &tmB;
    int stage = 0;
    uint32_t phase = 0, issued = 0, last_phase = 0;
    bool ok = true;
    for (int it = c0; ok && it < work.items; it += cstep) {
      int sel, g, n, m;
      decode_tile(work.tile(it, sel), ppre, G, a.n_tiles, g, n, m);
      const int h0 = sel < 0 ? 0 : sel, h1 = sel < 0 ? NH : sel + 1;
      const int arow = offs[g] + m * kPairM + (int)rank * kTileM;
      // this CTA's weight rows of N half h (SwiGLU: CTA 0 w_gate rows, CTA 1 w_up rows)
      constexpr int kHStep = (EPI == EPI_SWIGLU) ? kMmaN / 2 : kMmaN;
      const int brow0 = (EPI == EPI_SWIGLU)
                            ? g * a.b_rows + n * NH * (kMmaN / 2)
                            : g * a.b_rows + n * NH * kMmaN + (int)rank * (kMmaN / 2);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!wait_pair(&ctl->empty[stage], phase ^ 1u, ctl, peer_abort, a.err, 1)) {
          ok = false;
          break;
        }
        if (leader) mbar_expect_tx(&ctl->full[stage], 2 * (kAHalf + (h1 - h0) * kBHalf));
        uint8_t *sa = smem + (size_t)stage * kSB;
        const uint32_t fb = full0 + (uint32_t)(stage * sizeof(uint64_t));
        tma_load_2d_pair(&tmA, fb, sa, kb * kBlockK, arow);
#pragma unroll
        for (int h = 0; h < NH; ++h)
          if (h >= h0 && h < h1)
            tma_load_2d_pair(bmap, fb, sa + kAHalf + h * kBHalf, kb * kBlockK, brow0 + h * kHStep);
        issued |= 1u << stage;
        last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == kS) { stage = 0; phase ^= 1u; }
      }
    }
    // wait until the pair's MMAs have released every stage this CTA filled: the
    // last reads of our shared memory and the commit arrivals on our barriers are done
    for (int s = 0; s < kS; ++s)
      if (issued & (1u << s))
        wait_pair(&ctl->empty[s], (last_phase >> s) & 1u, ctl, peer_abort, nullptr, 0, false,
                  ok ? kWaitLimitNs : kDrainNs);
  } else if (warp == 1 && lane == 0 && leader) {
    // --------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = make_idesc(kPairM, kMmaN);
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true, any = false;
    // the MMAs of one K step (one ring stage) for N half h
    auto issue_half = [&](int st, int kb, int h) {
      const uint32_t sa = smem_u32(smem + (size_t)st * kSB);
      const uint64_t da = sw128_desc(sa), db = sw128_desc(sa + kAHalf + h * kBHalf);
#pragma unroll
      for (int kk = 0; kk < kBlockK / 16; ++kk)
        umma_bf16_pair(tmem + (uint32_t)(h * kMmaN), da + 2 * kk, db + 2 * kk, idesc,
                       (kb | kk) != 0);
    };
    // wait for the next stage to fill; returns its index and advances the ring
    auto next_full = [&](int &st) -> bool {
      if (!wait_pair(&ctl->full[stage], phase, ctl, peer_abort, a.err, 3)) return false;
      tc_fence_after();
      st = stage;
      if (++stage == kS) { stage = 0; phase ^= 1u; }
      return true;
    };
    if constexpr (NH == 2) {
      // The accumulator's two N halves are handed over one at a time. At the end of
      // a tile, half 0 of the last kS K steps is issued before half 1, so the
      // epilogue drains half 0 while half 1 finishes; at the start of the next tile,
      // half 0 of its first kS K steps runs as soon as half 0 is drained, while the
      // epilogue drains half 1. Tiles of one N half (sel >= 0) run in plain order.
      const bool split = nkb >= 2 * kS;
      for (int it = c0; ok && it < work.items; it += cstep) {
        int sel;
        work.tile(it, sel);
        if (!wait_pair(&ctl->tempty[0], acc_phase ^ 1u, ctl, peer_abort, a.err, 2)) {
          ok = false;
          break;
        }
        if (sel >= 0 || !split) {
          if (!wait_pair(&ctl->tempty[1], acc_phase ^ 1u, ctl, peer_abort, a.err, 2)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kb = 0; kb < nkb; ++kb) {
            int st;
            if (!(ok = next_full(st))) break;
            if (sel != 1) issue_half(st, kb, 0);
            if (sel != 0) issue_half(st, kb, 1);
            any = true;
            umma_commit_pair_both(&ctl->empty[st]);
          }
          if (!ok) break;
        } else {
          tc_fence_after();
          const int s0 = stage;
          for (int kb = 0; kb < kS; ++kb) {  // head: half 0 only
            int st;
            if (!(ok = next_full(st))) break;
            issue_half(st, kb, 0);
            any = true;
          }
          if (!ok) break;
          if (!wait_pair(&ctl->tempty[1], acc_phase ^ 1u, ctl, peer_abort, a.err, 2)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kb = 0; kb < kS; ++kb) {  // head: half 1, releasing the stages
            const int st = (s0 + kb) % kS;
            issue_half(st, kb, 1);
            umma_commit_pair_both(&ctl->empty[st]);
          }
          for (int kb = kS; kb < nkb - kS; ++kb) {  // body: both halves per stage
            int st;
            if (!(ok = next_full(st))) break;
            issue_half(st, kb, 0);
            issue_half(st, kb, 1);
            umma_commit_pair_both(&ctl->empty[st]);
          }
          if (!ok) break;
          const int s1 = stage;
          for (int kb = nkb - kS; kb < nkb; ++kb) {  // tail: half 0 first ...
            int st;
            if (!(ok = next_full(st))) break;
            issue_half(st, kb, 0);
          }
          if (!ok) break;
          umma_commit_pair_both(&ctl->tfull[0]);  // ... handed to the epilogue
          for (int kb = nkb - kS; kb < nkb; ++kb) {
            const int st = (s1 + kb - (nkb - kS)) % kS;
            issue_half(st, kb, 1);
            umma_commit_pair_both(&ctl->empty[st]);
          }
          umma_commit_pair_both(&ctl->tfull[1]);
          acc_phase ^= 1u;
          continue;
        }
        umma_commit_pair_both(&ctl->tfull[0]);
        umma_commit_pair_both(&ctl->tfull[1]);
        acc_phase ^= 1u;
      }
    } else {
      for (int it = c0; ok && it < work.items; it += cstep) {
        if (!wait_pair(&ctl->tempty[acc], acc_phase ^ 1u, ctl, peer_abort, a.err, 2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * kMmaN);
        for (int kb = 0; kb < nkb; ++kb) {
          int st;
          if (!(ok = next_full(st))) break;
          const uint32_t sa = smem_u32(smem + (size_t)st * kSB);
          const uint64_t da = sw128_desc(sa), db = sw128_desc(sa + kAHalf);
#pragma unroll
          for (int kk = 0; kk < kBlockK / 16; ++kk)
            umma_bf16_pair(d_tmem, da + 2 * kk, db + 2 * kk, idesc, (kb | kk) != 0);
          any = true;
          umma_commit_pair_both(&ctl->empty[st]);
        }
        if (!ok) break;
        umma_commit_pair_both(&ctl->tfull[acc]);
        if (++acc == PC::kAccBufs) { acc = 0; acc_phase ^= 1u; }
      }
    }
    if (!ok && any) {  // retire the MMAs in flight before TMEM is released
      umma_commit_pair_own(&ctl->drain);
      wait_pair(&ctl->drain, 0, ctl, peer_abort, nullptr, 0, false, kDrainNs);
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------------- epilogue
    const int ew = warp & 3;
    const int half = (warp - 4) >> 2;
    const uint32_t tempty0 = mapa_rank(smem_u32(&ctl->tempty[0]), 0);
    uint8_t *stage_out = smem + PC::kRing + (warp - 4) * kStageOutBytes;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int it = c0; ok && it < work.items; it += cstep) {
      int sel, g, n, m;
      decode_tile(work.tile(it, sel), ppre, G, a.n_tiles, g, n, m);
      const int grow = m * kPairM + (int)rank * kTileM + ew * 32 + lane;
      const bool valid = grow < offs[g + 1] - offs[g];
      const size_t orow = (size_t)offs[g] + grow;
      const bool rows_full = __all_sync(0xffffffffu, valid);
      const EpiStore st{a.tma_store ? &tmO : nullptr, stage_out, rows_full,
                        (int)(orow - (size_t)lane)};
      if constexpr (NH == 2) {
        // N half 0, then N half 1, each drained by all eight warps (the two warps of
        // a lane quarter take half of its columns each) and released on its own
        const uint32_t tbase = tmem + ((uint32_t)(ew * 32) << 16);
        for (int h = 0; h < 2; ++h) {
          ok = wait_pair(&ctl->tfull[h], acc_phase, ctl, peer_abort, a.err, 4);
          __syncwarp();
          if (!(ok = __all_sync(0xffffffffu, ok))) break;
          tc_fence_after();
          if (sel < 0 || sel == h) {
            if (EPI == EPI_SWIGLU)
              epilogue_tile<EPI>(a, tbase, g, h * kMmaN, n * kMmaN + h * (kMmaN / 2), 2 * half,
                                 2 * half + 2, valid, orow, st);
            else
              epilogue_tile<EPI>(a, tbase, g, h * kMmaN, (2 * n + h) * kMmaN, 4 * half,
                                 4 * half + 4, valid, orow, st);
          }
          tc_fence_before();
          mbar_arrive_cluster(tempty0 + (uint32_t)(h * sizeof(uint64_t)));
        }
        acc_phase ^= 1u;
      } else {
        ok = wait_pair(&ctl->tfull[acc], acc_phase, ctl, peer_abort, a.err, 4);
        __syncwarp();
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
        const uint32_t tbase = tmem + ((uint32_t)(ew * 32) << 16) + (uint32_t)(acc * kMmaN);
        // the two warps sharing a lane quarter take half the columns each
        if (EPI == EPI_SWIGLU)
          epilogue_tile<EPI>(a, tbase, g, 0, n * (kMmaN / 2), 2 * half, 2 * half + 2, valid, orow,
                             st);
        else
          epilogue_tile<EPI>(a, tbase, g, 0, n * kMmaN, 4 * half, 4 * half + 4, valid, orow, st);
        tc_fence_before();
        mbar_arrive_cluster(tempty0 + (uint32_t)(acc * sizeof(uint64_t)));
        if (++acc == PC::kAccBufs) { acc = 0; acc_phase ^= 1u; }
      }
    }
    if (a.tma_store && lane == 0) bulk_wait_all();  // this warp's output stores are done
    __syncwarp();
  }
  if (*(volatile int *)&ctl->abort_flag) settle_ns(100000);  // copies in flight land
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's remote arrivals are done before either CTA exits
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
struct DeviceInfo {
  bool attr_set[9] = {};  // [EPI]: single-CTA kernel; [3 + slot]: pair kernel
  int max_pairs[6] = {};  // [slot], slot = 3 * (NH - 1) + EPI
};

DeviceInfo &device_info(int dev) {
  static DeviceInfo infos[64];
  return infos[dev & 63];
}

std::mutex g_attr_mu;

// overlap = launch with programmatic stream serialisation: the grid may start
// while the preceding grid (which signals launch_dependents) is still running.
// Only for a grid that neither reads nor writes anything the preceding grid writes.
template <int EPI>
cudaError_t launch_single(const CUtensorMap &ma, const CUtensorMap &mb, const CUtensorMap &mb3,
                          TcArgs t, long long tiles_ub, bool overlap, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  DeviceInfo &info = device_info(dev);
  {
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (!info.attr_set[EPI]) {
      e = cudaFuncSetAttribute(k_ffn_tc<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSmemBytes);
      if (e != cudaSuccess) return e;
      info.attr_set[EPI] = true;
    }
  }
  const int grid = (int)std::max<long long>(1, std::min<long long>(tiles_ub, sm_count()));
  if (overlap) {
    t.pdl_mode = PDL_TAIL;
  } else if (t.pdl_mode == PDL_NONE) {
    k_ffn_tc<EPI><<<grid, kThreads1, kSmemBytes, st>>>(ma, mb, mb3, t);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k_ffn_tc<EPI>, ma, mb, mb3, t);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int EPI, int NH>
cudaError_t launch_pair(const CUtensorMap &ma, const CUtensorMap &mb, const CUtensorMap &mb3,
                        const CUtensorMap &mo, const TcArgs &t, long long tiles_ub,
                        cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  DeviceInfo &info = device_info(dev);
  constexpr int slot = 3 * (NH - 1) + EPI;
  constexpr size_t smem = pair_smem_bytes<NH>();
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  {
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (!info.attr_set[3 + slot]) {
      e = cudaFuncSetAttribute(k_ffn_tc2<EPI, NH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e != cudaSuccess) return e;
      cfg.gridDim = dim3(2 * (sm_count() / 2));
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, k_ffn_tc2<EPI, NH>, &cfg) != cudaSuccess || n <= 0)
        n = sm_count() / 2;
      info.max_pairs[slot] = n;
      info.attr_set[3 + slot] = true;
    }
  }
  const long long pairs = std::min<long long>(tiles_ub, info.max_pairs[slot]);
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cudaLaunchAttribute attr2[2] = {attr[0], attr[0]};
  if (t.pdl_mode == PDL_WAIT) {  // the cluster shape and programmatic serialisation
    attr2[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr2[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr2;
    cfg.numAttrs = 2;
  }
  e = cudaLaunchKernelEx(&cfg, k_ffn_tc2<EPI, NH>, ma, mb, mb3, mo, t);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Tile choice. A reduction of K >= kWideMinK over experts that average at least
// one 256-row pair tile takes the wide 256 x 512 CTA-pair tile: twice the MMA
// work per pipeline stage hides the operand-load latency that bounds the
// 128 x 256 single-CTA tile on long K. Short reductions keep the single-CTA tile,
// whose double-buffered accumulator hides the epilogue (a large share of a short
// tile), and so do experts with few rows (capacity-limited layers), where
// 128-row tiles waste less and give every SM a tile of its own. Building with
// MOE_TC_PAIR uses the 256 x 256 pair tile everywhere instead. All three compute
// the same result.
constexpr int kWideMinK = 2048;

#ifdef MOE_TC_PAIR
constexpr bool kUsePairs = true;
#else
constexpr bool kUsePairs = false;
#endif

inline bool use_wide(int K, long long rows, int groups) {
  return !kUsePairs && K >= kWideMinK && rows >= (long long)kPairM * groups;
}
inline bool uses_pairs(bool wide) { return kUsePairs || wide; }

// mb1 / mb31: the weight maps of the single-CTA kernel when they differ from the
// pair kernel's (non-SwiGLU tiles load 256 weight rows per copy there).
// split: with the wide tile, hand the odd last row tiles to the single-CTA kernel.
// Measured on routed loads: +5.5 % for DeepSeek (768 rows per expert on average,
// tails in half the experts), -2.5 % for Mixtral (1024 rows on average: its few
// small tails fill less than one extra round of the single-CTA kernel's tiles), so
// it is used below 1024 rows per expert on average.
inline bool split_tails(long long rows, int groups) { return rows < 4LL * kPairM * groups; }

// mo: the output map for the pair kernel's TMA stores (used when t.tma_store).
template <int EPI>
cudaError_t launch_gemm(const CUtensorMap &ma, const CUtensorMap &mb, const CUtensorMap &mb3,
                        const CUtensorMap &mb1, const CUtensorMap &mb31, const CUtensorMap &mo,
                        TcArgs t, int m_tiles_ub, int groups, int n_cols, bool wide, bool split,
                        cudaStream_t st) {
  // output columns per 256 accumulator columns
  const int per_n = (EPI == EPI_SWIGLU) ? kMmaN / 2 : kMmaN;
  const long long pair_m_ub = (long long)(m_tiles_ub + groups + 1) / 2;
  if (kUsePairs) {
    t.n_tiles = ceil_div(n_cols, per_n);
    t.tile_mode = TILES_ALL;
    return launch_pair<EPI, 1>(ma, mb, mb3, mo, t,
                               std::max<long long>(pair_m_ub * t.n_tiles, 1), st);
  }
  if (wide) {
    // full pair tiles on the wide kernel; with split, the odd last 128-row tiles
    // on the single-CTA kernel, which fills the SMs the pair grid's last round leaves
    t.n_tiles = ceil_div(n_cols, 2 * per_n);
    t.tile_mode = split ? TILES_PAIRS_NO_TAIL : TILES_ALL;
    cudaError_t e = launch_pair<EPI, 2>(ma, mb, mb3, mo, t,
                                        std::max<long long>(pair_m_ub * t.n_tiles, 1), st);
    if (e != cudaSuccess || !split) return e;
    t.n_tiles = ceil_div(n_cols, per_n);
    t.tile_mode = TILES_TAIL_ONLY;
    return launch_single<EPI>(ma, mb1, mb31, t, (long long)groups * t.n_tiles, true, st);
  }
  t.n_tiles = ceil_div(n_cols, per_n);
  t.tile_mode = TILES_ALL;
  return launch_single<EPI>(ma, mb1, mb31, t, (long long)m_tiles_ub * t.n_tiles, false, st);
}

}  // namespace

cudaError_t launch_ffn_tc(const GroupedFfnArgs &a, cudaStream_t st) {
  if (a.m_tiles_ub <= 0) return cudaSuccess;
  const bool swiglu = a.act == MOE_ACT_SWIGLU;
  const bool wide_up = use_wide(a.d, a.a_rows, a.G), wide_down = use_wide(a.F, a.a_rows, a.G);
  const bool split = split_tails(a.a_rows, a.G);
  // Weight-map boxes: pair tiles load 128 weight rows per CTA and N half; single-CTA
  // tiles 256 rows per copy, or two 128-row copies (W_gate, W_up) for SwiGLU.
  const uint32_t box_single = swiglu ? kMmaN / 2 : kMmaN;
  const uint32_t box_pair = kMmaN / 2;
  CUtensorMap ma, mb, mb3, mbs, mb3s;
  // up projection: [rows, d] x [G*F, d]^T -> h [rows, F]
  if (!make_map(&ma, a.a, (uint64_t)a.a_rows, (uint64_t)a.d, kTileM)) return cudaErrorInvalidValue;
  const bool pairs_up = uses_pairs(wide_up);
  if (!make_map(&mbs, a.w1, (uint64_t)a.G * a.F, (uint64_t)a.d, box_single))
    return cudaErrorInvalidValue;
  if (swiglu) {
    if (!make_map(&mb3s, a.w3, (uint64_t)a.G * a.F, (uint64_t)a.d, box_single))
      return cudaErrorInvalidValue;
  } else {
    mb3s = mbs;
  }
  if (pairs_up && box_pair != box_single) {
    if (!make_map(&mb, a.w1, (uint64_t)a.G * a.F, (uint64_t)a.d, box_pair))
      return cudaErrorInvalidValue;
    mb3 = mb;
  } else {
    mb = mbs;
    mb3 = mb3s;
  }
  TcArgs t{};
  t.offsets = a.offsets;
  t.mprefix = a.mprefix;
  t.G = a.G;
  t.N = a.F;
  t.K = a.d;
  t.b_rows = a.F;
  t.out = a.h;
  t.out_f32 = 0;
  t.bias = a.b1;
  t.act = a.act;
  t.err = a.err;
  t.wait_limit_ns = a.wait_limit_ns ? a.wait_limit_ns : kWaitLimitNs;
  t.withhold_load = a.withhold_load;  // the up projection only
  // both projections start while the kernel before them finishes (a tail-tile
  // launch of the up projection waits for its pair grid before it exits, so the
  // down projection's wait covers both)
  t.pdl_mode = take_pdl() ? PDL_WAIT : PDL_NONE;
  // pair tiles write bf16 outputs through TMA stores of 32 x 32 boxes
  CUtensorMap mo;
  if (!make_store_map(&mo, a.h, (uint64_t)a.a_rows, (uint64_t)a.F)) return cudaErrorInvalidValue;
  t.tma_store = 1;
  cudaError_t e =
      swiglu ? launch_gemm<EPI_SWIGLU>(ma, mb, mb3, mbs, mb3s, mo, t, a.m_tiles_ub, a.G, a.F,
                                       wide_up, split, st)
             : launch_gemm<EPI_ACT>(ma, mb, mb3, mbs, mb3s, mo, t, a.m_tiles_ub, a.G, a.F,
                                    wide_up, split, st);
  if (e != cudaSuccess) return e;
  // down projection: h [rows, F] x [G*d, F]^T -> out [rows, d]
  if (!make_map(&ma, a.h, (uint64_t)a.a_rows, (uint64_t)a.F, kTileM)) return cudaErrorInvalidValue;
  if (!make_map(&mbs, a.w2, (uint64_t)a.G * a.d, (uint64_t)a.F, kMmaN))
    return cudaErrorInvalidValue;
  if (uses_pairs(wide_down)) {
    if (!make_map(&mb, a.w2, (uint64_t)a.G * a.d, (uint64_t)a.F, box_pair))
      return cudaErrorInvalidValue;
  } else {
    mb = mbs;
  }
  t.N = a.d;
  t.K = a.F;
  t.b_rows = a.d;
  t.out = a.out;
  t.out_f32 = a.out_f32;
  t.bias = a.b2;
  t.act = -1;
  t.withhold_load = 0;
  t.pdl_mode = PDL_WAIT;  // follows the up projection's kernels directly
  t.tma_store = a.out_f32 ? 0 : 1;
  if (!a.out_f32 && !make_store_map(&mo, a.out, (uint64_t)a.a_rows, (uint64_t)a.d))
    return cudaErrorInvalidValue;
  return launch_gemm<EPI_DOWN>(ma, mb, mb, mbs, mbs, mo, t, a.m_tiles_ub, a.G, a.d, wide_down,
                               split, st);
}

}  // namespace moe

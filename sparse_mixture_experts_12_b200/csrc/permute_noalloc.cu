// moe_permute_noalloc: the histogram -> scan -> permute step for callers that
// cannot allocate device memory.
//
// Some callers of this library do not own device memory: a plugin or operator
// inside a host framework that hands it only its input and output buffers and
// manages every other byte through its own arena, or a latency-critical loop in
// which a cudaMalloc (which may synchronise the device) is not acceptable. Such a
// caller cannot provide the workspace moe_permute needs. This entry point keeps
// that scratch (the per-tile expert counts and their prefix sums) in a fixed
// file-scope device array instead, so the caller passes only inputs and outputs.
//
// The array is part of the library image: every GPU on which the library is used
// holds it (about 0.5 MB) until the process exits. All calls share it, so calls
// that overlap on the GPU (different streams, or different host threads on one
// device) race and must be serialised by the caller. Every entry the kernels
// read is written earlier in the same call, so nothing needs clearing between
// calls. Index errors are not recorded anywhere: a pair whose expert index is out
// of range is treated as dropped (inv = -1).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <climits>
#include <mutex>

#include "kernels.cuh"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace moe {
namespace {

// Largest (experts x token tiles) table the static scratch holds. A token tile
// is router_bm(E) tokens (32 for E <= 32, 64 for E <= 128, 32 above), so e.g.
// E = 8 allows T <= 262144 and E = 128 allows T <= 32768.
constexpr int kNoAllocMaxTileEntries = 65536;
// [tile_counts | tile_base] of kNoAllocMaxTileEntries each, then mprefix [E+1].
constexpr size_t kNoAllocInts = 2 * (size_t)kNoAllocMaxTileEntries + kMaxExperts + 1;

static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocInts];

// The device address of g_permute_scratch belongs to a CUDA context: each context
// that loads the library has its own copy of the array. So the address is cached per
// context, keyed on the driver's context ID, which is unique for the life of the
// process (a context created after a reset, or a non-primary context, gets a new
// ID even where its handle repeats an old one). Where the ID cannot be read, the
// address is looked up on every call (cudaGetSymbolAddress allocates nothing).
struct ScratchEntry {
  unsigned long long ctx_id;
  int32_t *addr;
};
constexpr int kScratchCache = 64;
ScratchEntry g_scratch_cache[kScratchCache];
int g_scratch_used = 0;
int g_scratch_next = 0;
std::mutex g_scratch_mu;

struct CtxQuery {
  PFN_cuCtxGetCurrent_v4000 current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};

const CtxQuery &ctx_query() {
  static CtxQuery q;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      q.current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      q.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  return q;
}

// ID of the context current on this thread; false when there is none (the runtime
// has not made the device's primary context current yet) or it cannot be read.
bool current_context_id(unsigned long long *id) {
  const CtxQuery &q = ctx_query();
  if (q.current == nullptr || q.get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (q.current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return q.get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_permute_scratch in the current context (in host code the
// symbol itself is only a host-side stand-in).
moe_status_t scratch_in_current_context(int32_t **out) {
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (have_id) {
    for (int i = 0; i < g_scratch_used; ++i) {
      if (g_scratch_cache[i].ctx_id == id) {
        *out = g_scratch_cache[i].addr;
        return MOE_OK;
      }
    }
  }
  // also makes the current device's primary context current when none is
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr)
    return MOE_ERR_CUDA;
  if (!have_id) have_id = current_context_id(&id);
  if (have_id) {
    ScratchEntry &slot = g_scratch_cache[g_scratch_next];
    slot.ctx_id = id;
    slot.addr = static_cast<int32_t *>(p);
    g_scratch_next = (g_scratch_next + 1) % kScratchCache;
    if (g_scratch_used < kScratchCache) ++g_scratch_used;
  }
  *out = static_cast<int32_t *>(p);
  return MOE_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

MOE_API moe_status_t moe_permute_noalloc(const moe_cfg_t *cfg, const void *x,
                                         const int32_t *topk_idx, int32_t *counts,
                                         int32_t *offsets, int32_t *perm, int32_t *inv,
                                         void *x_perm, moe_stream_t stream) {
  if (cfg == nullptr) return MOE_ERR_INVALID_ARG;
  const moe_cfg_t &c = *cfg;
  if (c.n_tokens < 0 || c.d_model <= 0 || c.n_experts < 1 || c.n_experts > kMaxExperts ||
      c.top_k < 1 || c.top_k > c.n_experts || c.top_k > kMaxTopK ||
      (c.dtype != MOE_DTYPE_F32 && c.dtype != MOE_DTYPE_BF16) || !isfinite(c.capacity_factor))
    return MOE_ERR_INVALID_ARG;
  const int elem = c.dtype == MOE_DTYPE_F32 ? 4 : 2;
  if (((long long)c.d_model * elem) % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if ((long long)c.n_tokens * c.top_k > INT_MAX / 2) return MOE_ERR_UNSUPPORTED;
  const void *ptrs[] = {x, topk_idx, counts, offsets, perm, inv, x_perm};
  for (const void *p : ptrs) {
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
    if (!aligned16(p)) return MOE_ERR_MISALIGNED;
  }
  const int E = c.n_experts;
  const int NT = ceil_div(c.n_tokens > 0 ? c.n_tokens : 1, router_bm(E));
  if ((long long)E * NT > kNoAllocMaxTileEntries) return MOE_ERR_WORKSPACE;  // beyond the static scratch
  int32_t *scratch = nullptr;
  moe_status_t st = scratch_in_current_context(&scratch);
  if (st != MOE_OK) return st;
  cudaStream_t s = stream;
  if (c.n_tokens == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  int32_t *tile_counts = scratch;
  int32_t *tile_base = scratch + kNoAllocMaxTileEntries;
  int32_t *mprefix = scratch + 2 * kNoAllocMaxTileEntries;
  if (launch_tile_counts(topk_idx, c.n_tokens, c.top_k, E, tile_counts, nullptr, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  ScanArgs sa{};
  sa.tile_counts = tile_counts;
  sa.tile_base = tile_base;
  sa.counts = counts;
  sa.offsets = offsets;
  sa.mprefix = mprefix;
  sa.E = E;
  sa.NT = NT;
  sa.cap = -1;
  if (c.capacity_factor > 0.f) {
    const double cap = floor((double)c.capacity_factor * (double)c.n_tokens * (double)c.top_k /
                             (double)E);
    sa.cap = cap > (double)INT_MAX ? INT_MAX : (int)cap;
  }
  sa.T = c.n_tokens;
  sa.k = c.top_k;
  if (launch_scan(sa, s) != cudaSuccess) return MOE_ERR_CUDA;
  ScatterArgs pa{};
  pa.x = x;
  pa.topk_idx = topk_idx;
  pa.tile_base = tile_base;
  pa.offsets = offsets;
  pa.perm = perm;
  pa.inv = inv;
  pa.x_perm = x_perm;
  pa.T = c.n_tokens;
  pa.d = c.d_model;
  pa.E = E;
  pa.k = c.top_k;
  pa.cap = sa.cap;
  pa.elem_bytes = elem;
  pa.err = nullptr;
  if (launch_scatter(pa, s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

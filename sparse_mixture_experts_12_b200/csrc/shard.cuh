// Token sharding of one batch over several ranks (replicated weights, each rank a
// consecutive slice of the tokens). Tokens are independent given the routing, with
// two exceptions, both handled here:
//  * the capacity drop of youngju.dev (zh) "SwitchRouter" takes each expert's pairs
//    in token-major order over the WHOLE batch, so a shard keeps at most
//    cap_e = max(0, cap - before_e) pairs for expert e, before_e being the pairs the
//    earlier shards routed to e (counted before drops; an all-gather of [E] counts);
//  * the load-balancing statistics ("load_balancing_loss", "router_z_loss") are
//    means over the whole batch: each shard produces fp64 sums, a sum all-reduce
//    adds them, and one more kernel turns the sums into the statistics.
#pragma once

#include "kernels.cuh"

namespace moe {

struct ShardCaps {
  const int32_t *counts_all;  // [W, E] pre-drop counts of every shard, shard-major
  int32_t *cap_e;             // [E] out: pairs this shard may keep per expert
  int W, rank;
};

// The scan of launch_scan with per-expert capacities cap_e (ScanArgs::cap is the
// capacity of the whole batch; < 0: unlimited, cap_e then unused).
cudaError_t launch_scan_shard(const ScanArgs &a, const ShardCaps &sc, cudaStream_t st);
// The scatter of launch_scatter keeping a pair iff its rank < cap_e[e].
cudaError_t launch_scatter_shard(const ScatterArgs &a, const int32_t *cap_e, cudaStream_t st);

// Sums of one shard for the statistics, fp64 part[1 + 2E]:
//   { sum_t logsumexp(z_t)^2, count[0..E), sum_t softmax(z_t)[0..E) }
// from the router's per-tile sums (tile_p [E, NT], tile_z [NT]) and per-tile
// counts (tile_counts [E, NT]), in a fixed order.
cudaError_t launch_aux_partials(const int32_t *tile_counts, const float *tile_p,
                                const float *tile_z, int E, int NT, double *part,
                                cudaStream_t st);
// The statistics vector out[3 + 2E] of moe_aux_stats from summed parts over T
// tokens in total.
cudaError_t launch_aux_finalize(const double *part, int E, long long T, int k, float alpha,
                                float *out, cudaStream_t st);

}  // namespace moe

// msa_merge_partials: combine n partial attentions over disjoint key sets by
// their log-sum-exp ("LSE fusion" / "Two-phase forward" tags, inteligile
// "MiniMax-M3" model page):
//   L = log sum_s exp(lse_s),  out = sum_s exp(lse_s - L) out_s,
// each out_s already normalised over its own keys; a partial with lse = -inf
// (no keys) weighs nothing.  Used to join the per-rank results of a sequence
// whose KV blocks are spread over several GPUs.  A warp per (row, head), lane =
// 4 output dimensions; HBM-bound (reads n partial rows, writes one).
#pragma once
#include "common.cuh"

namespace msa {

constexpr int MRG_THREADS = 256;

__global__ void __launch_bounds__(MRG_THREADS)
merge_partials_kernel(const __nv_bfloat16* __restrict__ outs, const float* __restrict__ lses,
                      __nv_bfloat16* __restrict__ out, float* __restrict__ lse, int n, long units) {
  const int lane = threadIdx.x & 31;
  const long u = static_cast<long>(blockIdx.x) * (MRG_THREADS / 32) + (threadIdx.x >> 5);
  if (u >= units) return;                        // whole warp
  float mx = -INFINITY;
  for (int s = 0; s < n; ++s) mx = fmaxf(mx, __ldg(lses + static_cast<long>(s) * units + u));
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (mx > -INFINITY) {
    for (int s = 0; s < n; ++s) {
      const float w = __expf(__ldg(lses + static_cast<long>(s) * units + u) - mx);
      const uint2 x = __ldg(reinterpret_cast<const uint2*>(outs + (static_cast<long>(s) * units + u) * 128) + lane);
      wsum += w;
      acc[0] = fmaf(w, bf16lo(x.x), acc[0]);
      acc[1] = fmaf(w, bf16hi(x.x), acc[1]);
      acc[2] = fmaf(w, bf16lo(x.y), acc[2]);
      acc[3] = fmaf(w, bf16hi(x.y), acc[3]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint2 y;
  y.x = pack_bf16(acc[0] * inv, acc[1] * inv);
  y.y = pack_bf16(acc[2] * inv, acc[3] * inv);
  reinterpret_cast<uint2*>(out + u * 128)[lane] = y;
  if (lse && lane == 0) lse[u] = wsum > 0.f ? mx + __logf(wsum) : -INFINITY;
}

}  // namespace msa

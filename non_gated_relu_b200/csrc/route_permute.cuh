// route_permute.cuh -- router and token permute of a decode-sized batch in one
// launch: block e computes expert e's logits for the T <= 32 tokens, and the
// last block to finish selects every token (grouped top-k) and then runs the
// whole permute (histogram, scan, tile table, stable ranking, gather) on the
// routing it has just produced, without a second kernel.
#pragma once

#include "permute.cuh"
#include "route.cuh"

namespace nh {

// Dynamic smem (floats): 8 warps x 2E (selection) + E + 3 T k (permute and
// the staged routing).  blockDim.x = 256 (>= E): small enough in registers to
// share an SM with the GEMM CTAs of the concurrent shared-expert stream.
template <typename Tin>
__global__ void __launch_bounds__(256) route_permute_small(const Tin* __restrict__ x,
                                                           const float* __restrict__ wr,
                                                           SelectArgs a, int H, unsigned int* done,
                                                           PermuteOut o) {
  extern __shared__ float smf[];
  __shared__ float red[8][32];
  __shared__ int warp_sums[33];
  __shared__ unsigned int ticket;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int T = a.T, E = a.E, k = a.k;
  float* logits = const_cast<float*>(a.logits);
  pdl_wait();
  pdl_trigger();
  router_block_logits(x, wr, (int)blockIdx.x, T, E, H, logits, red);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) ticket = atomicAdd(done, 1u);
  __syncthreads();
  if (ticket != gridDim.x - 1) return;
  __threadfence();
  float* sel = smf;                                      // 8 x 2E
  int* cnt = reinterpret_cast<int*>(smf + 16 * E);       // E
  int* pos = cnt + E;                                    // T k
  int32_t* s_idx = pos + T * k;                          // T k
  float* s_w = reinterpret_cast<float*>(s_idx + T * k);  // T k
  for (int t = wib; t < T; t += 8)
    select_token(a, t, logits + (size_t)t * E, sel + (size_t)wib * 2 * E, lane, s_idx, s_w);
  __syncthreads();
  permute_block(s_idx, s_w, x, T, k, E, H, o.tile_rows, o.max_tiles, o.counts, o.offsets, o.tiles,
                o.num_tiles, o.perm_token, o.perm_w, o.inv_row, static_cast<Tin*>(o.x_perm),
                o.status, o.sched_zero, cnt, pos, warp_sums, o.gather != 0, o.ready, o.n_ready);
  if (threadIdx.x == 0) *done = 0u;
}

}  // namespace nh

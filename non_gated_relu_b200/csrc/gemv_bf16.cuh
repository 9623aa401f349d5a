// gemv_bf16.cuh -- dense bf16 GEMM for decode-sized token counts (at most 32
// rows of activations): the shared expert and the latent projections.
//
// These layers have one "tile entry" (all tokens) and N / 128 weight tiles,
// so the tcgen05 kernel runs on N / 128 CTAs (29 for the shared up
// projection) and cannot draw full HBM bandwidth.  Here a CTA task is 16
// weight rows; its 8 warps split K in 128-feature blocks, load the weights
// with 16-byte global loads straight into the A fragments of mma.sync
// m16n8k16 (bf16 in, f32 accumulate; tokens on N = 8) and add their partial
// tiles through shared memory in warp order (deterministic).  The feature
// permutation inside a block is the one of gemv_q4.cuh: thread tq's 32
// features are one contiguous run of 64 bytes per row.
#pragma once

#include "gemv_q4.cuh"

namespace nh {
namespace dgv {

constexpr int WARPS = 8;
constexpr int MT = 16;

struct Args {
  tc::TcArgs g;            // dense rows (tile_rows, dense_rows), N, K, epilogue, out, ldo
  const void* A;           // activations [rows, K] bf16
  const void* W;           // weights [N, K] bf16
};

// One block of BK features for one n-tile: the weight runs of rows gq (wa)
// and gq + 8 (wb), BK/32 uint4 each (one uint4 = 8 features = two k-tiles),
// and the activation run of token gq.
template <int BK>
__device__ __forceinline__ void block_mma(const uint4* wa, const uint4* wb,
                                          const __nv_bfloat16* act, float* c0, float* c1) {
  constexpr int KT = BK / 16;
  uint2 bv[KT];
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) bv[kt] = __ldg(reinterpret_cast<const uint2*>(act + 4 * kt));
#pragma unroll
  for (int u = 0; u < KT / 2; ++u) {
    // k-tile 2u: run features 8u + {0,1} (.x) and {2,3} (.y); k-tile 2u + 1: .z, .w
    q4v::mma_bf16_16816(c0, wa[u].x, wb[u].x, wa[u].y, wb[u].y, bv[2 * u].x, bv[2 * u].y);
    q4v::mma_bf16_16816(c1, wa[u].z, wb[u].z, wa[u].w, wb[u].w, bv[2 * u + 1].x,
                        bv[2 * u + 1].y);
  }
}

template <int NT>
__global__ void __launch_bounds__(WARPS * 32, 2) bf16_gemv_splitk(const Args a) {
  __shared__ float red[WARPS][32][4];
  const tc::TcArgs& g = a.g;
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int num_m = (g.dense_rows + g.tile_rows - 1) / g.tile_rows;
  const int n_rb = g.N / MT;
  const int total = num_m * n_rb;
  const int K = g.K;
  const int nkb = K / 128, tail = K % 128;
  const __nv_bfloat16* A = static_cast<const __nv_bfloat16*>(a.A);
  const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(a.W);
  for (int task = blockIdx.x; task < total; task += gridDim.x) {
    const int m = task / n_rb, rb = task - m * n_rb;
    const int r0 = rb * MT;
    const int4 ent = tc::tile_entry_of(g, m);
    const int count = ent.z;
    const __nv_bfloat16* wa_p = W + (size_t)(r0 + gq) * K;
    const __nv_bfloat16* wb_p = wa_p + 8 * (size_t)K;
    for (int n0 = 0; n0 < count; n0 += 8) {
      const int j = min(n0 + gq, count - 1);
      const __nv_bfloat16* act = A + (size_t)(ent.y + j) * K;
      float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
      for (int kb = warp; kb < nkb; kb += WARPS) {
        uint4 wa[4], wb[4];
        const uint4* pa = reinterpret_cast<const uint4*>(wa_p + kb * 128 + 32 * tq);
        const uint4* pb = reinterpret_cast<const uint4*>(wb_p + kb * 128 + 32 * tq);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          wa[u] = __ldg(pa + u);
          wb[u] = __ldg(pb + u);
        }
        block_mma<128>(wa, wb, act + kb * 128 + 32 * tq, c0, c1);
      }
      if (tail && warp == nkb % WARPS) {
        // 64-feature tail: thread tq's run is features [16 tq, 16 tq + 16)
        uint4 wa[2], wb[2];
        const uint4* pa = reinterpret_cast<const uint4*>(wa_p + nkb * 128 + 16 * tq);
        const uint4* pb = reinterpret_cast<const uint4*>(wb_p + nkb * 128 + 16 * tq);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          wa[u] = __ldg(pa + u);
          wb[u] = __ldg(pb + u);
        }
        block_mma<64>(wa, wb, act + nkb * 128 + 16 * tq, c0, c1);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp][lane][i] = c0[i] + c1[i];
      __syncthreads();
      if (warp == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < WARPS; ++w) v += red[w][lane][i];
          const int jj = n0 + 2 * tq + (i & 1);
          const int f = r0 + gq + (i >> 1) * 8;
          if (jj < count) tc::epi_elem(g, ent.y + jj, f, v);
        }
      }
      __syncthreads();
    }
  }
}

}  // namespace dgv
}  // namespace nh

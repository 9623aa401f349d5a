// gemv_bf16.cuh -- dense bf16 GEMM for decode-sized token counts (at most 32
// rows of activations): the shared expert and the latent projections.
//
// These layers have one "tile entry" (all tokens) and N / 128 weight tiles,
// so the tcgen05 kernel runs on N / 128 CTAs (29 for the shared up
// projection) and cannot draw full HBM bandwidth.  Here a CTA task is 16
// weight rows, which reach shared memory by untiled bulk copies; the warps
// feed them to mma.sync m16n8k16 (bf16 in, f32 accumulate; tokens on N = 8)
// and add their partial tiles through shared memory in warp order
// (deterministic).
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

// A CTA task is 16 weight rows over the whole K, split over the 8 warps in
// units of 32 features (4 lanes x 8 bf16): warp w owns units
// [w U / 8, (w + 1) U / 8) of the U = K / 32.  Each warp streams its share in
// chunks of up to CH units through NBUF private buffers: one bulk copy per row
// and chunk (row r's units are contiguous in W), completing on the buffer's
// mbarrier.  One chunk of 11 units holds a warp's whole share for K up to
// 2816, so for the shared expert's up projection (K = 2688) one round trip to
// memory brings all of it; its down projection (K = 3712) takes a chunk of 11
// and one of up to 4.  The first chunks of the CTA's first task are issued
// before the grid waits on its predecessor (weights are inputs, never produced
// by an earlier kernel), so a dependent launch streams its weights while the
// kernel before it finishes.  Inside a unit, lane (gq, tq) reads the 16 bytes
// at 16 tq of rows gq and gq + 8 -- features 8 tq .. 8 tq + 7 of the unit --
// and the same features of its token's activations: k-tile 2u takes features
// 8 tq + {0,1} / {2,3}, k-tile 2u + 1 takes 8 tq + {4,5} / {6,7}, a bijection
// of the unit's 32 features onto the two k-tiles' slots.  Rows are PITCH bytes
// apart in a buffer, 64 modulo 128, so the eight lanes of one shared-memory
// wavefront (rows gq, gq + 1) hit disjoint banks.  K must be a multiple of 32
// and W 16-byte aligned (both hold for every weight this library takes).
constexpr int UNIT = 32;
constexpr int CH = 11;
constexpr int NBUF = 1;
constexpr int PITCH = CH * UNIT * 2;
constexpr int BUF_BYTES = MT * PITCH;
constexpr int STAGED_SMEM = WARPS * NBUF * BUF_BYTES;
static_assert(PITCH % 128 == 64, "rows gq and gq + 1 must use disjoint banks");
static_assert(BUF_BYTES % 16 == 0, "bulk copy destinations are 16-byte aligned");

template <int NT>
__global__ void __launch_bounds__(WARPS * 32, 2) bf16_gemv_staged(const Args a) {
  extern __shared__ __align__(128) uint8_t stage_smem[];
  __shared__ float red[WARPS][32][4];
  __shared__ __align__(8) uint64_t bars[WARPS][NBUF];
  __shared__ int abort_flag;
  const tc::TcArgs& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int num_m = (g.dense_rows + g.tile_rows - 1) / g.tile_rows;
  const int n_rb = g.N / MT;
  const int total = num_m * n_rb;
  const int K = g.K;
  const int U = K / UNIT;
  const int u_lo = warp * U / WARPS, u_hi = (warp + 1) * U / WARPS;
  const int nch = (u_hi - u_lo + CH - 1) / CH;
  const uint8_t* const bufp = stage_smem + warp * NBUF * BUF_BYTES;
  const uint32_t buf = smem_u32(bufp);
  const uint32_t bar = smem_u32(&bars[warp][0]);
  const __nv_bfloat16* A = static_cast<const __nv_bfloat16*>(a.A);
  const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(a.W);
  if (threadIdx.x == 0) abort_flag = 0;
  if (lane == 0)
    for (int b = 0; b < NBUF; ++b) mbar_init(bar + 8u * b, 1);
  fence_barrier_init();
  __syncthreads();
  const WaitCtl wc{&abort_flag, g.status, g.timeout_ns};
  uint32_t phase = 0u, pending = 0u;  // bit b: buffer b's next parity / a copy in flight
  // chunk c of the task at weight row r0 into buffer c % NBUF
  auto issue = [&](int r0, int c) {
    const int b = c % NBUF;
    const int ua = u_lo + c * CH, ub = min(ua + CH, u_hi);
    const uint32_t bytes = (uint32_t)(ub - ua) * UNIT * 2;
    if (lane == 0) mbar_arrive_expect_tx(bar + 8u * b, bytes * MT);
    __syncwarp();
    if (lane < MT)
      bulk_load(buf + (uint32_t)(b * BUF_BYTES + lane * PITCH),
                W + (size_t)(r0 + lane) * K + (size_t)ua * UNIT, bytes, bar + 8u * b);
    pending |= 1u << b;
  };
  if ((int)blockIdx.x < total)
    for (int c = 0; c < min(NBUF, nch); ++c) issue(((int)blockIdx.x % n_rb) * MT, c);
  pdl_wait();
  pdl_trigger();
  bool ok = true;
  for (int task = blockIdx.x; task < total; task += gridDim.x) {
    const int m = task / n_rb, rb = task - m * n_rb;
    const int r0 = rb * MT;
    const int4 ent = tc::tile_entry_of(g, m);
    const int count = ent.z;
    if (task != (int)blockIdx.x && ok)
      for (int c = 0; c < min(NBUF, nch); ++c) issue(r0, c);
    float c0[NT / 8][4], c1[NT / 8][4];
#pragma unroll
    for (int p = 0; p < NT / 8; ++p)
#pragma unroll
      for (int i = 0; i < 4; ++i) c0[p][i] = c1[p][i] = 0.f;
    for (int c = 0; c < nch; ++c) {
      const int b = c % NBUF;
      if (ok) ok = mbar_wait(bar + 8u * b, (phase >> b) & 1u, wc, SITE_GEMV_STAGE);
      if (ok) {
        phase ^= 1u << b;
        pending &= ~(1u << b);
        const int ua = u_lo + c * CH, nu = min(CH, u_hi - ua);
        const uint8_t* bp = bufp + b * BUF_BYTES + tq * 16;
#pragma unroll
        for (int p = 0; p < NT / 8; ++p) {
          if (p * 8 >= count) break;
          // token p * 8 + gq (lanes past count re-read the last token; their
          // columns are never stored)
          const int j = min(p * 8 + gq, count - 1);
          const __nv_bfloat16* act = A + (size_t)(ent.y + j) * K + (size_t)ua * UNIT + tq * 8;
          uint4 xv[CH];
#pragma unroll
          for (int uu = 0; uu < CH; ++uu)
            if (uu < nu) xv[uu] = __ldg(reinterpret_cast<const uint4*>(act + uu * UNIT));
#pragma unroll
          for (int uu = 0; uu < CH; ++uu) {
            if (uu < nu) {
              const uint4 wa = *reinterpret_cast<const uint4*>(bp + gq * PITCH + uu * 64);
              const uint4 wb = *reinterpret_cast<const uint4*>(bp + (gq + 8) * PITCH + uu * 64);
              q4v::mma_bf16_16816(c0[p], wa.x, wb.x, wa.y, wb.y, xv[uu].x, xv[uu].y);
              q4v::mma_bf16_16816(c1[p], wa.z, wb.z, wa.w, wb.w, xv[uu].z, xv[uu].w);
            }
          }
        }
      }
      // every lane is done with the buffer before it is refilled
      __syncwarp();
      if (ok && c + NBUF < nch) {
        fence_proxy_async_smem();
        issue(r0, c + NBUF);
      }
    }
#pragma unroll
    for (int p = 0; p < NT / 8; ++p) {
      if (p * 8 >= count) break;
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp][lane][i] = c0[p][i] + c1[p][i];
      __syncthreads();
      if (warp == 0 && !abort_flag) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < WARPS; ++w) v += red[w][lane][i];
          const int jj = p * 8 + 2 * tq + (i & 1);
          const int f = r0 + gq + (i >> 1) * 8;
          if (jj < count) tc::epi_elem(g, ent.y + jj, f, v);
        }
      }
      __syncthreads();
    }
  }
  // copies still in flight after a wait ran out land before the CTA exits
  for (int b = 0; b < NBUF; ++b)
    if (pending & (1u << b)) tc::mbar_drain(bar + 8u * b, (phase >> b) & 1u, g.timeout_ns, g.status);
}

}  // namespace dgv
}  // namespace nh

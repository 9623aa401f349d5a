// gemm_simt.cuh -- grouped expert GEMM on CUDA cores (float32 path).
//
// out[rows of tile, n] = epi( A[rows, :] . W[e][n, :] ) for each tile entry
// (expert e, first row, rows) of the permute's tile table.  Used for the
// float32 dtype, where tensor-core tf32 cannot hold the 1e-4 relative bar.
#pragma once

#include "common.cuh"

namespace nh {

enum Epilogue : int {
  EPI_UP_RELU2 = 0,      // out (dtype) [rows, N] = relu(acc)^2
  EPI_DOWN_COMBINE = 1,  // out (float32) [T, N]: out[dst_row[r]] += perm_w[r] * acc
                         //   (routed down projection: the weighted combine of a
                         //   token's k experts, float32 atomic adds)
  EPI_STORE_F32 = 2,     // out (float32) [rows, N] = acc
  EPI_STORE = 3,         // out (dtype) [rows, N] = acc             (latent fc1 projection)
  EPI_ADD_F32 = 4,       // out (float32) [rows, N] += acc          (latent fc2 projection;
                         //   each element has one owner tile: no atomics)
  EPI_ACC_F32 = 5,       // out (float32) [rows, N] += acc, atomic adds (shared expert,
                         //   which may run beside the routed combine)
};

struct GemmArgs {
  const void* A;          // activations [rows, K] (dtype)
  const void* B;          // weights [n_experts][N][K] (dtype)
  int K, N;
  const int4* tiles;      // (expert, first row, rows, 0) or null: dense rows
  const int32_t* num_tiles;
  int dense_rows;         // rows when tiles == null
  int tile_rows;
  int epi;
  void* out;
  int64_t ldo;            // row stride of out, elements
  const float* perm_w;
  const int32_t* dst_row; // EPI_DOWN_COMBINE: output row (token) of each permuted row
};

__device__ __forceinline__ bool tile_entry(const GemmArgs& g, int m, int4& ent) {
  if (g.tiles) {
    if (m >= *g.num_tiles) return false;
    ent = g.tiles[m];
    return true;
  }
  const int r0 = m * g.tile_rows;
  if (r0 >= g.dense_rows) return false;
  ent = make_int4(0, r0, min(g.tile_rows, g.dense_rows - r0), 0);
  return true;
}

constexpr int SG_BM = 64, SG_BN = 64, SG_BK = 16, SG_PAD = 68;

template <typename Tin>
__global__ void __launch_bounds__(256) simt_grouped_gemm(GemmArgs g) {
  __shared__ __align__(16) float As[SG_BK][SG_PAD];
  __shared__ __align__(16) float Bs[SG_BK][SG_PAD];
  pdl_wait();
  pdl_trigger();
  int4 ent;
  if (!tile_entry(g, blockIdx.y, ent)) return;
  const int e = ent.x, r0 = ent.y, nrows = ent.z;
  const int n0 = blockIdx.x * SG_BN;
  const Tin* A = static_cast<const Tin*>(g.A);
  const Tin* B = static_cast<const Tin*>(g.B) + (size_t)e * g.N * g.K;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < g.K; k0 += SG_BK) {
    for (int i = threadIdx.x; i < SG_BM * SG_BK; i += 256) {
      const int r = i / SG_BK, kk = i - r * SG_BK;
      const int kc = k0 + kk;
      As[kk][r] = (r < nrows && kc < g.K) ? to_f32(A[(size_t)(r0 + r) * g.K + kc]) : 0.f;
      const int n = n0 + r;
      Bs[kk][r] = (n < g.N && kc < g.K) ? to_f32(B[(size_t)n * g.K + kc]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = ty * 4 + i;
    if (rr >= nrows) continue;
    const int r = r0 + rr;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= g.N) continue;
      const float v = acc[i][j];
      if (g.epi == EPI_UP_RELU2) {
        static_cast<Tin*>(g.out)[(size_t)r * g.ldo + n] = from_f32<Tin>(relu2(v));
      } else if (g.epi == EPI_DOWN_COMBINE) {
        red_add_f32(static_cast<float*>(g.out) + (size_t)g.dst_row[r] * g.ldo + n,
                    g.perm_w[r] * v);
      } else if (g.epi == EPI_STORE) {
        static_cast<Tin*>(g.out)[(size_t)r * g.ldo + n] = from_f32<Tin>(v);
      } else if (g.epi == EPI_ADD_F32) {
        static_cast<float*>(g.out)[(size_t)r * g.ldo + n] += v;
      } else if (g.epi == EPI_ACC_F32) {
        red_add_f32(static_cast<float*>(g.out) + (size_t)r * g.ldo + n, v);
      } else {
        static_cast<float*>(g.out)[(size_t)r * g.ldo + n] = v;
      }
    }
  }
}

}  // namespace nh

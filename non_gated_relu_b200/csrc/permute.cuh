// permute.cuh -- token permute of the routed experts.
//
// The (token, slot) assignments are grouped per expert, in (token, slot)
// order inside each expert: a per-chunk histogram, one scan over experts
// and chunks (which also writes the tile table the expert GEMMs walk), and a
// stable scatter that gathers x into the permuted row order.  The routed
// experts are applied per expert id, as in MLX's SwitchMLP (fc1/fc2 indexed
// by the router's expert ids; exo commit "Add support for Nemotron
// sharding").
#pragma once

#include "common.cuh"

namespace nh {

constexpr int PERM_CHUNK = 256;  // tokens per histogram chunk
constexpr int PAIR_TILE_ROWS = 256;
constexpr int PAIR_ATTACH_ROWS = 64;  // largest remainder that rides on a full pair tile

// Tiles of an expert with `total` rows.  Tiles never cross an expert
// boundary.  For the CTA-pair GEMM (256-row tiles) an expert's rows past its
// full tiles form its partial last tile; a partial tile of at most
// PAIR_ATTACH_ROWS rows is attached to the expert's last full tile instead,
// so the expert's weights are streamed once per feature block for both.
__device__ __forceinline__ int expert_tile_count(int total, int tile_rows) {
  int nt = (total + tile_rows - 1) / tile_rows;
  if (tile_rows == PAIR_TILE_ROWS) {
    const int r = total % tile_rows;
    if (r > 0 && r <= PAIR_ATTACH_ROWS && total > tile_rows) --nt;
  }
  return nt;
}

// Tile i of nt of an expert: (expert, first row, rows, kind).  Kinds of the
// CTA-pair GEMM: 0 a full tile, 1 a partial tile (computed swapped), 2 a full
// tile plus an attached partial tile of rows - 256 rows.  Other tile heights
// use kind 0 only.
__device__ __forceinline__ int4 expert_tile(int e, int off, int total, int tile_rows, int i,
                                            int nt) {
  const int r0 = i * tile_rows;
  const int rows = (i == nt - 1) ? total - r0 : tile_rows;
  int kind = 0;
  if (tile_rows == PAIR_TILE_ROWS) kind = rows < tile_rows ? 1 : (rows > tile_rows ? 2 : 0);
  return make_int4(e, off + r0, rows, kind);
}

// per-chunk expert histogram: chunk_counts[c][e]
__global__ void __launch_bounds__(256) permute_hist(const int32_t* __restrict__ idx, int T, int k,
                                                    int E, int32_t* __restrict__ chunk_counts,
                                                    int* status) {
  extern __shared__ int hist[];
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * PERM_CHUNK;
  const int n = min(PERM_CHUNK, T - t0) * k;
  const int32_t* src = idx + (size_t)t0 * k;
  for (int a = threadIdx.x; a < n; a += blockDim.x) {
    const int e = src[a];
    if (e < 0 || e >= E) {
      record_status(status, NH_ERR_DEVICE_CHECK, SITE_PERMUTE_HIST, e);
      continue;
    }
    atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    chunk_counts[(size_t)blockIdx.x * E + e] = hist[e];
}

// block-wide exclusive scan of one int per thread (blockDim.x <= 1024)
__device__ __forceinline__ int block_exclusive_scan(int v, int* smem_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) smem_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? smem_warp[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < nw) smem_warp[lane] = wi - w;
    if (lane == nw - 1) smem_warp[32] = wi;
  }
  __syncthreads();
  const int res = smem_warp[warp] + inc - v;
  *total = smem_warp[32];
  __syncthreads();
  return res;
}

// One block, blockDim.x >= E (rounded to a warp multiple).  Turns the chunk
// histograms into absolute chunk bases (in place), writes counts, offsets,
// the tile table (expert, first row, rows, kind) of expert_tile, and the
// number of tiles.
__global__ void permute_scan(int32_t* __restrict__ chunk_counts, int n_chunks, int E,
                             int tile_rows, int32_t* __restrict__ counts,
                             int32_t* __restrict__ offsets, int4* __restrict__ tiles,
                             int32_t* __restrict__ num_tiles, int max_tiles,
                             unsigned int* sched_zero) {
  __shared__ int warp_sums[33];
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x < 4) sched_zero[threadIdx.x] = 0u;  // up/down GEMM tile schedulers
  const int e = threadIdx.x;
  int total = 0;
  if (e < E)
    for (int c = 0; c < n_chunks; ++c) total += chunk_counts[(size_t)c * E + e];
  int all_rows;
  const int off = block_exclusive_scan(e < E ? total : 0, warp_sums, &all_rows);
  const int nt = (e < E) ? expert_tile_count(total, tile_rows) : 0;
  int all_tiles;
  const int toff = block_exclusive_scan(nt, warp_sums, &all_tiles);
  if (e < E) {
    counts[e] = total;
    offsets[e] = off;
    int run = off;
    for (int c = 0; c < n_chunks; ++c) {
      const int v = chunk_counts[(size_t)c * E + e];
      chunk_counts[(size_t)c * E + e] = run;
      run += v;
    }
    for (int i = 0; i < nt && toff + i < max_tiles; ++i)
      tiles[toff + i] = expert_tile(e, off, total, tile_rows, i, nt);
  }
  if (e == 0) {
    offsets[E] = all_rows;
    *num_tiles = min(all_tiles, max_tiles);
  }
}

// Stable scatter of one chunk's assignments + gather of x rows into x_perm.
// Warp 0 ranks the assignments in (t, j) order 32 at a time; then every warp
// copies rows.  Dynamic smem: int run[E] + int pos[PERM_CHUNK * k].
template <typename Tin>
__global__ void __launch_bounds__(256) permute_scatter(
    const int32_t* __restrict__ idx, const float* __restrict__ w, const Tin* __restrict__ x,
    int T, int k, int E, int H, const int32_t* __restrict__ chunk_base,
    int32_t* __restrict__ perm_token, float* __restrict__ perm_w, int32_t* __restrict__ inv_row,
    Tin* __restrict__ x_perm, int* status, int do_gather) {
  extern __shared__ int sm[];
  pdl_wait();
  pdl_trigger();
  int* run = sm;
  int* pos = sm + E;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = blockIdx.x;
  const int t0 = c * PERM_CHUNK;
  const int n = min(PERM_CHUNK, T - t0) * k;
  const size_t a0 = (size_t)t0 * k;
  if (warp == 0) {
    for (int e = lane; e < E; e += 32) run[e] = chunk_base[(size_t)c * E + e];
    __syncwarp();
    const unsigned lt = (1u << lane) - 1u;
    // eight rounds of 32 assignments at a time: their loads are issued
    // together, then the rounds rank in order (the ranking is sequential)
    for (int b0 = 0; b0 < n; b0 += 8 * 32) {
      int ev[8];
      float wv[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int a = b0 + 32 * r + lane;
        ev[r] = (a < n) ? idx[a0 + a] : -1;
        wv[r] = (a < n) ? w[a0 + a] : 0.f;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int a = b0 + 32 * r + lane;
        int e = ev[r];
        if (e >= E) e = -1;  // already reported by the histogram
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int start = (e >= 0) ? run[e] : 0;
        __syncwarp();
        const int p = start + __popc(peers & lt);
        if (e >= 0 && lane == __ffs(peers) - 1) run[e] = start + __popc(peers);
        __syncwarp();
        if (a < n) {
          pos[a] = (e >= 0) ? p : -1;
          if (e >= 0) {
            perm_token[p] = t0 + a / k;
            perm_w[p] = wv[r];
            inv_row[a0 + a] = p;
          } else {
            inv_row[a0 + a] = -1;
          }
        }
      }
    }
  }
  __syncthreads();
  if (!do_gather) return;
  // gather rows: one warp per assignment
  const int nw = blockDim.x >> 5;
  const size_t row_bytes = (size_t)H * sizeof(Tin);
  const bool vec = (row_bytes % 16) == 0;
  for (int a = warp; a < n; a += nw) {
    const int p = pos[a];
    if (p < 0) continue;
    const int t = t0 + a / k;
    if (vec) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
      uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)p * H);
      const int nv = (int)(row_bytes / 16);
      for (int i = lane; i < nv; i += 32) dst[i] = src[i];
    } else {
      for (int i = lane; i < H; i += 32) x_perm[(size_t)p * H + i] = x[(size_t)t * H + i];
    }
  }
}

// copy one row of H elements with 16-byte vectors when possible
template <typename Tin>
__device__ __forceinline__ void copy_row(const Tin* __restrict__ src, Tin* __restrict__ dst, int H,
                                         int lane) {
  const size_t row_bytes = (size_t)H * sizeof(Tin);
  if ((row_bytes % 16) == 0) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    const int nv = (int)(row_bytes / 16);
    int i = lane;
    for (; i + 32 < nv; i += 64) {
      const uint4 a = s4[i], b = s4[i + 32];
      d4[i] = a;
      d4[i + 32] = b;
    }
    for (; i < nv; i += 32) d4[i] = s4[i];
  } else {
    for (int i = lane; i < H; i += 32) dst[i] = src[i];
  }
}

// x_perm[inv_row[t k + j]] = x[t] for every token t and choice j: one warp per
// token reads the row once, GATHER_CH 16-byte words per lane at a time, and
// stores it to each of the token's permuted rows (rows of dropped choices,
// inv_row < 0, do not exist).  Every permuted row is written exactly once.
constexpr int GATHER_CH = 8;

template <typename Tin>
__global__ void __launch_bounds__(256) permute_gather(const Tin* __restrict__ x,
                                                      const int32_t* __restrict__ inv_row, int T,
                                                      int k, int H, Tin* __restrict__ x_perm) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const size_t row_bytes = (size_t)H * sizeof(Tin);
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nw) {
    const Tin* src = x + (size_t)t * H;
    for (int j0 = 0; j0 < k; j0 += 32) {
      const int nj = min(32, k - j0);
      const int dst = lane < nj ? inv_row[(size_t)t * k + j0 + lane] : -1;
      if (row_bytes % 16 == 0) {
        const int nv = (int)(row_bytes / 16);
        const uint4* s4 = reinterpret_cast<const uint4*>(src);
        for (int v0 = 0; v0 < nv; v0 += 32 * GATHER_CH) {
          uint4 r[GATHER_CH];
#pragma unroll
          for (int u = 0; u < GATHER_CH; ++u) {
            const int i = v0 + 32 * u + lane;
            if (i < nv) r[u] = s4[i];
          }
          for (int j = 0; j < nj; ++j) {
            const int p = __shfl_sync(0xffffffffu, dst, j);
            if (p < 0) continue;
            uint4* d4 = reinterpret_cast<uint4*>(x_perm + (size_t)p * H);
#pragma unroll
            for (int u = 0; u < GATHER_CH; ++u) {
              const int i = v0 + 32 * u + lane;
              if (i < nv) d4[i] = r[u];
            }
          }
        }
      } else {
        for (int j = 0; j < nj; ++j) {
          const int p = __shfl_sync(0xffffffffu, dst, j);
          if (p >= 0)
            for (int i = lane; i < H; i += 32) x_perm[(size_t)p * H + i] = src[i];
        }
      }
    }
  }
}

// Whole permute of T <= PERM_CHUNK tokens by one block of blockDim.x >= E
// threads: histogram, scan, tile table, stable ranking and gather.  idx / w
// may live in global or shared memory; cnt [E] and pos [T * k] are shared
// memory; warp_sums [33] is shared memory.
template <typename Tin>
__device__ __forceinline__ void permute_block(
    const int32_t* idx, const float* w, const Tin* __restrict__ x, int T, int k, int E, int H,
    int tile_rows, int max_tiles, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int4* __restrict__ tiles, int32_t* __restrict__ num_tiles, int32_t* __restrict__ perm_token,
    float* __restrict__ perm_w, int32_t* __restrict__ inv_row, Tin* __restrict__ x_perm,
    int* status, unsigned int* sched_zero, int* cnt, int* pos, int* warp_sums, bool gather,
    int* ready_zero, int n_ready) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = T * k;
  if (threadIdx.x < 4) sched_zero[threadIdx.x] = 0u;  // up/down GEMM tile schedulers
  // per-tile-entry counters of a fused up + down launch
  for (int i = threadIdx.x; i < n_ready; i += blockDim.x) ready_zero[i] = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int a = threadIdx.x; a < n; a += blockDim.x) {
    const int e = idx[a];
    if (e < 0 || e >= E) {
      record_status(status, NH_ERR_DEVICE_CHECK, SITE_PERMUTE_HIST, e);
      continue;
    }
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  const int e = threadIdx.x;
  const int total = e < E ? cnt[e] : 0;
  int all_rows, all_tiles;
  const int off = block_exclusive_scan(total, warp_sums, &all_rows);
  const int nt = expert_tile_count(total, tile_rows);
  const int toff = block_exclusive_scan(nt, warp_sums, &all_tiles);
  if (e < E) {
    counts[e] = total;
    offsets[e] = off;
    for (int i = 0; i < nt && toff + i < max_tiles; ++i)
      tiles[toff + i] = expert_tile(e, off, total, tile_rows, i, nt);
    cnt[e] = off;  // running position for the ranking
  }
  if (e == 0) {
    offsets[E] = all_rows;
    *num_tiles = min(all_tiles, max_tiles);
  }
  __syncthreads();
  if (warp == 0) {
    const unsigned lt = (1u << lane) - 1u;
    for (int b = 0; b < n; b += 32) {
      const int a = b + lane;
      int ee = (a < n) ? idx[a] : -1;
      if (ee >= E) ee = -1;
      const unsigned peers = __match_any_sync(0xffffffffu, ee);
      const int start = (ee >= 0) ? cnt[ee] : 0;
      __syncwarp();
      const int p = start + __popc(peers & lt);
      if (ee >= 0 && lane == __ffs(peers) - 1) cnt[ee] = start + __popc(peers);
      __syncwarp();
      if (a < n) {
        pos[a] = (ee >= 0) ? p : -1;
        inv_row[a] = (ee >= 0) ? p : -1;
        if (ee >= 0) {
          perm_token[p] = a / k;
          perm_w[p] = w[a];
        }
      }
    }
  }
  if (!gather) return;  // decode: the up projection reads x itself
  __syncthreads();
  const int nw = blockDim.x >> 5;
  for (int a = warp; a < n; a += nw) {
    const int p = pos[a];
    if (p >= 0) copy_row(x + (size_t)(a / k) * H, x_perm + (size_t)p * H, H, lane);
  }
}

struct PermuteOut {
  int tile_rows, max_tiles;
  int32_t *counts, *offsets;
  int4* tiles;
  int32_t *num_tiles, *perm_token;
  float* perm_w;
  int32_t* inv_row;
  void* x_perm;
  int* status;
  unsigned int* sched_zero;
  int gather;   // 0: no x_perm (decode orientation reads x directly)
  int* ready;   // [n_ready] zeroed: the fused decode GEMM's per-entry counters
  int n_ready;
};

// Whole permute in one block for T <= PERM_CHUNK tokens (decode).
// blockDim.x = 512 (>= E).  Dynamic smem: int cnt[E] + int pos[T * k].
template <typename Tin>
__global__ void __launch_bounds__(512) permute_small(const int32_t* __restrict__ idx,
                                                     const float* __restrict__ w,
                                                     const Tin* __restrict__ x, int T, int k, int E,
                                                     int H, PermuteOut o) {
  extern __shared__ int sm[];
  __shared__ int warp_sums[33];
  pdl_wait();
  pdl_trigger();
  permute_block(idx, w, x, T, k, E, H, o.tile_rows, o.max_tiles, o.counts, o.offsets, o.tiles,
                o.num_tiles, o.perm_token, o.perm_w, o.inv_row, static_cast<Tin*>(o.x_perm),
                o.status, o.sched_zero, sm, sm + E, warp_sums, o.gather != 0, o.ready, o.n_ready);
}

}  // namespace nh

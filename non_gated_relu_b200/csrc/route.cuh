// route.cuh -- the MoE router of the Nemotron-H block on CUDA cores.
//
// logits l[t, e] = sum_h x[t, h] * Wr[e, h] (float32 accumulate, the router
// weight stays float32), then per token: selection score (the logit itself,
// or sigmoid(l) + correction bias), group score (max of the group, or the
// sum of its two largest), the topk_group best groups, the top-k experts of
// those groups with ties to the lower id, weights alpha * s / sum(s).
// (baseRT issue #46, "MoE: ... grouped top-k (n_groups=8, topk_group=1),
// routed_scaling_factor=2.5, norm_topk_prob"; ModelArgs fields of the exo
// commit "Add support for Nemotron sharding".)
#pragma once

#include "common.cuh"

namespace nh {

// ----- logits, small T: one warp per (expert, block of up to 8 tokens) ------
template <typename Tin>
__global__ void __launch_bounds__(256) router_logits_warp(const Tin* __restrict__ x,
                                                          const float* __restrict__ wr,
                                                          float* __restrict__ logits, int T, int H,
                                                          int E) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int tblocks = (T + 7) >> 3;
  const int e = warp / tblocks, tb = warp - e * tblocks;
  if (e >= E) return;
  const int t0 = tb * 8;
  const int nt = min(8, T - t0);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const float* w = wr + (size_t)e * H;
  const Tin* xb = x + (size_t)t0 * H;
  for (int h = lane; h < H; h += 32) {
    const float wv = w[h];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i < nt) acc[i] = fmaf(to_f32(xb[(size_t)i * H + h]), wv, acc[i]);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float v = acc[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0 && i < nt) logits[(size_t)(t0 + i) * E + e] = v;
  }
}

// ----- logits, large T: 64 tokens x 64 experts per block, 4x4 per thread ----
constexpr int RT_BT = 64, RT_BE = 64, RT_BK = 32, RT_PAD = 68;

template <typename Tin>
__global__ void __launch_bounds__(256) router_logits_tiled(const Tin* __restrict__ x,
                                                           const float* __restrict__ wr,
                                                           float* __restrict__ logits, int T,
                                                           int H, int E) {
  __shared__ __align__(16) float xs[RT_BK][RT_PAD];
  __shared__ __align__(16) float ws[RT_BK][RT_PAD];
  const int t0 = blockIdx.x * RT_BT, e0 = blockIdx.y * RT_BE;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < H; k0 += RT_BK) {
    for (int i = threadIdx.x; i < RT_BT * RT_BK; i += 256) {
      const int r = i / RT_BK, kk = i - r * RT_BK;
      const int t = t0 + r, h = k0 + kk;
      xs[kk][r] = (t < T && h < H) ? to_f32(x[(size_t)t * H + h]) : 0.f;
      const int e = e0 + r;
      ws[kk][r] = (e < E && h < H) ? wr[(size_t)e * H + h] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < RT_BK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
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
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < E) logits[(size_t)t * E + e] = acc[i][j];
    }
  }
}

// ----- selection: one thread per token --------------------------------------
struct SelectArgs {
  const float* logits;  // [T, E]
  const float* bias;    // [E] or null
  int32_t* topk_idx;    // [T, k]
  float* topk_w;        // [T, k]
  int* status;
  int T, E, G, tg, k;
  int norm;
  float alpha;
  int group_score;  // 0 max, 1 top-2 sum
  int use_sigma;    // select on sigmoid(l) + bias instead of l
};

__device__ __forceinline__ float sigmoid_f32(float l) { return 1.0f / (1.0f + expf(-l)); }

// total order of the selection: larger value first, equal values by lower id
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__global__ void __launch_bounds__(128) router_select(SelectArgs a) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= a.T) return;
  const float* l = a.logits + (size_t)t * a.E;
  const int g = a.E / a.G;
  auto sel = [&](int e) -> float {
    if (!a.use_sigma) return l[e];
    return sigmoid_f32(l[e]) + (a.bias ? a.bias[e] : 0.f);
  };

  // group scores (G <= 64)
  float gs[64];
  for (int q = 0; q < a.G; ++q) {
    float m1 = -INFINITY, m2 = -INFINITY;
    for (int i = 0; i < g; ++i) {
      const float v = sel(q * g + i);
      if (v > m1) {
        m2 = m1;
        m1 = v;
      } else if (v > m2) {
        m2 = v;
      }
    }
    gs[q] = a.group_score ? m1 + m2 : m1;
  }
  // keep the tg best groups: each pass takes the best group ranked after the previous pick
  uint64_t keep = 0;
  int pq = -1;
  float pv = 0.f;
  for (int r = 0; r < a.tg; ++r) {
    int bq = -1;
    float bv = 0.f;
    for (int q = 0; q < a.G; ++q) {
      if (pq >= 0 && !ranks_before(pv, pq, gs[q], q)) continue;
      if (bq < 0 || ranks_before(gs[q], q, bv, bq)) {
        bq = q;
        bv = gs[q];
      }
    }
    if (bq < 0) {
      record_status(a.status, NH_ERR_DEVICE_CHECK, SITE_ROUTE_SELECT, t);
      bq = r;
    }
    keep |= 1ull << bq;
    pq = bq;
    pv = bv;
  }
  // top-k among the kept groups' experts, in (score desc, id asc) order
  int32_t* out_i = a.topk_idx + (size_t)t * a.k;
  float* out_w = a.topk_w + (size_t)t * a.k;
  int pe = -1;
  float pev = 0.f, ssum = 0.f;
  float sj[32];
  for (int j = 0; j < a.k; ++j) {
    int be = -1;
    float bv = 0.f;
    for (int q = 0; q < a.G; ++q) {
      if (!((keep >> q) & 1ull)) continue;
      for (int i = 0; i < g; ++i) {
        const int e = q * g + i;
        const float v = sel(e);
        if (pe >= 0 && !ranks_before(pev, pe, v, e)) continue;
        if (be < 0 || ranks_before(v, e, bv, be)) {
          be = e;
          bv = v;
        }
      }
    }
    if (be < 0) {
      record_status(a.status, NH_ERR_DEVICE_CHECK, SITE_ROUTE_SELECT, t);
      be = 0;
    }
    out_i[j] = be;
    sj[j] = sigmoid_f32(l[be]);
    ssum += sj[j];
    pe = be;
    pev = bv;
  }
  for (int j = 0; j < a.k; ++j)
    out_w[j] = a.norm ? a.alpha * sj[j] / ssum : a.alpha * sj[j];
}

}  // namespace nh

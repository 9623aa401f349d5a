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

// ----- logits, large T: 64 tokens x 64 experts per block, 4x4 per thread ----
constexpr int RT_BT = 64, RT_BE = 64, RT_BK = 32, RT_PAD = 68;

template <typename Tin>
__global__ void __launch_bounds__(256) router_logits_tiled(const Tin* __restrict__ x,
                                                           const float* __restrict__ wr,
                                                           float* __restrict__ logits, int T,
                                                           int H, int E) {
  __shared__ __align__(16) float xs[RT_BK][RT_PAD];
  __shared__ __align__(16) float ws[RT_BK][RT_PAD];
  pdl_wait();
  pdl_trigger();
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

// warp-wide argmax under ranks_before (larger value, then lower id)
__device__ __forceinline__ void warp_best(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (oi >= 0 && (i < 0 || ranks_before(ov, oi, v, i))) {
      v = ov;
      i = oi;
    }
  }
}

// Selection of one token by one warp; `sel` holds the token's E selection
// scores in shared memory (written by the caller).
__device__ __forceinline__ void select_token(const SelectArgs& a, int t, const float* l,
                                             float* sel, int lane, int32_t* idx_out = nullptr,
                                             float* w_out = nullptr) {
  const int E = a.E, G = a.G, g = E / G;
  float* lraw = sel + E;  // the token's logits, staged next to its selection scores
  // produced by another block or kernel: read at L2, four loads in flight
  for (int e0 = lane; e0 < E; e0 += 128) {
    float le[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) le[i] = __ldcg(l + min(e0 + 32 * i, E - 1));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = e0 + 32 * i;
      if (e < E) {
        lraw[e] = le[i];
        sel[e] = a.use_sigma ? sigmoid_f32(le[i]) + (a.bias ? a.bias[e] : 0.f) : le[i];
      }
    }
  }
  __syncwarp();
  // group scores: lane q (and q + 32) reduces its group
  float gsv[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int q = lane + 32 * r;
    float m1 = -INFINITY, m2 = -INFINITY;
    if (q < G) {
      for (int i = 0; i < g; ++i) {
        const float v = sel[q * g + i];
        if (v > m1) {
          m2 = m1;
          m1 = v;
        } else if (v > m2) {
          m2 = v;
        }
      }
    }
    gsv[r] = a.group_score ? m1 + m2 : m1;
  }
  // keep the tg best groups (each pass: best group ranked after the previous pick)
  uint64_t keep = 0;
  int pq = -1;
  float pv = 0.f;
  for (int r = 0; r < a.tg; ++r) {
    float bv = 0.f;
    int bq = -1;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int q = lane + 32 * h;
      if (q >= G) continue;
      if (pq >= 0 && !ranks_before(pv, pq, gsv[h], q)) continue;
      if (bq < 0 || ranks_before(gsv[h], q, bv, bq)) {
        bq = q;
        bv = gsv[h];
      }
    }
    warp_best(bv, bq);
    if (bq < 0) {
      if (lane == 0) record_status(a.status, NH_ERR_DEVICE_CHECK, SITE_ROUTE_SELECT, t);
      bq = r;
    }
    keep |= 1ull << bq;
    pq = bq;
    pv = bv;
  }
  float ssum = 0.f, my_s = 0.f;
  int my_e = 0;
  const int n_cand = a.tg * g;   // experts of the kept groups
  if (n_cand <= 128) {
    // Rank every candidate against all candidates under the same total order
    // (score desc, id asc): a candidate of rank r < k is the r-th pick.  All
    // ranks are independent, so this is one pass instead of k argmax rounds.
    int c_e[4], c_r[4];
    float c_s[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = lane + 32 * r;
      c_r[r] = a.k;
      c_e[r] = 0;
      c_s[r] = 0.f;
      if (j < n_cand) {
        uint64_t kk = keep;          // j-th candidate: kept groups ascending, ids ascending
        for (int m = j / g; m > 0; --m) kk &= kk - 1;
        if (kk == 0) continue;       // fewer kept groups (a recorded selection error)
        const int e = (__ffsll((long long)kk) - 1) * g + j % g;
        const float v = sel[e];
        int rank = 0;
        for (uint64_t k2 = keep; k2; k2 &= k2 - 1) {
          const int e0 = (__ffsll((long long)k2) - 1) * g;
          for (int i = 0; i < g; ++i) rank += ranks_before(sel[e0 + i], e0 + i, v, e) ? 1 : 0;
        }
        c_e[r] = e;
        c_r[r] = rank;
        if (rank < a.k) c_s[r] = sigmoid_f32(lraw[e]);
      }
    }
    __syncwarp();
    // picks by rank into this warp's scratch (sel / lraw are no longer read);
    // a slot no candidate fills (only after a selection error) keeps expert 0
    if (lane < a.k) {
      sel[lane] = 0.f;
      lraw[lane] = __int_as_float(0);
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      if (c_r[r] < a.k) {
        sel[c_r[r]] = c_s[r];
        lraw[c_r[r]] = __int_as_float(c_e[r]);
      }
    }
    __syncwarp();
    for (int j = 0; j < a.k; ++j) ssum += sel[j];   // pick order, as the scores are summed below
    if (lane < a.k) {
      my_s = sel[lane];
      my_e = __float_as_int(lraw[lane]);
    }
  } else {
  // which of this lane's experts (e = lane + 32 i, E <= 512) lie in kept groups
  uint32_t mine = 0;
  for (int i = 0, e = lane; e < E; ++i, e += 32)
    if ((keep >> (e / g)) & 1ull) mine |= 1u << i;
  // top-k experts of the kept groups in (score desc, id asc) order
  int pe = -1;
  float pev = 0.f;
  for (int j = 0; j < a.k; ++j) {
    float bv = 0.f;
    int be = -1;
    for (int i = 0, e = lane; e < E; ++i, e += 32) {
      if (!((mine >> i) & 1u)) continue;
      const float v = sel[e];
      if (pe >= 0 && !ranks_before(pev, pe, v, e)) continue;
      if (be < 0 || ranks_before(v, e, bv, be)) {
        be = e;
        bv = v;
      }
    }
    warp_best(bv, be);
    if (be < 0) {
      if (lane == 0) record_status(a.status, NH_ERR_DEVICE_CHECK, SITE_ROUTE_SELECT, t);
      be = 0;
    }
    const float sj = sigmoid_f32(lraw[be]);
    ssum += sj;
    if (lane == j) {
      my_e = be;
      my_s = sj;
    }
    pe = be;
    pev = bv;
  }
  }
  if (lane < a.k) {
    const float wj = a.norm ? a.alpha * my_s / ssum : a.alpha * my_s;
    a.topk_idx[(size_t)t * a.k + lane] = my_e;
    a.topk_w[(size_t)t * a.k + lane] = wj;
    if (idx_out) {
      idx_out[t * a.k + lane] = my_e;
      w_out[t * a.k + lane] = wj;
    }
  }
}

// one warp per token; dynamic smem: warps_per_block * 2E floats
__global__ void __launch_bounds__(256) router_select(SelectArgs a) {
  extern __shared__ float sel_smem[];
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= a.T) return;
  select_token(a, t, a.logits + (size_t)t * a.E, sel_smem + (size_t)warp * 2 * a.E, lane);
}

// x[t, h .. h+3] as floats (h a multiple of 4, rows 8-byte aligned for bf16)
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}
__device__ __forceinline__ float4 load4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}

// Logits of expert e for T <= TB tokens, by one block: threads split H four
// elements at a time.  The token loads are unconditional (rows past T re-read
// row T - 1), so a thread issues its loads for eight tokens back to back
// instead of one dependent round trip per token; then a block reduction.
// red: [blockDim/32][32].
template <int TB, typename Tin>
__device__ __forceinline__ void router_block_logits_t(const Tin* __restrict__ x,
                                                      const float* __restrict__ wr, int e, int T,
                                                      int E, int H, float* logits,
                                                      float (*red)[32]) {
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int step = blockDim.x * 4;
  float acc[TB];
#pragma unroll
  for (int t = 0; t < TB; ++t) acc[t] = 0.f;
  const float* w = wr + (size_t)e * H;
  if ((H & 3) == 0) {
#pragma unroll 2
    for (int h = threadIdx.x * 4; h < H; h += step) {
      const int hh = h;
      const float4 wv = __ldg(reinterpret_cast<const float4*>(w + hh));
#pragma unroll
      for (int t0 = 0; t0 < TB; t0 += 8) {
        float4 xv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int tt = min(t0 + i, T - 1);
          xv[i] = load4(x + (size_t)tt * H + hh);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
          acc[t0 + i] = fmaf(xv[i].x, wv.x,
                             fmaf(xv[i].y, wv.y, fmaf(xv[i].z, wv.z, fmaf(xv[i].w, wv.w, acc[t0 + i]))));
      }
    }
  } else {
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
      const float wv = w[h];
#pragma unroll
      for (int t = 0; t < TB; ++t)
        acc[t] = fmaf(to_f32(x[(size_t)min(t, T - 1) * H + h]), wv, acc[t]);
    }
  }
#pragma unroll
  for (int t = 0; t < TB; ++t) {
    float v = acc[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[wib][t] = v;
  }
  __syncthreads();
  if (wib == 0 && lane < T) {
    float v = 0.f;
    for (int i = 0; i < nw; ++i) v += red[i][lane];
    logits[(size_t)lane * E + e] = v;
  }
}

template <typename Tin>
__device__ __forceinline__ void router_block_logits(const Tin* __restrict__ x,
                                                    const float* __restrict__ wr, int e, int T,
                                                    int E, int H, float* logits,
                                                    float (*red)[32]) {
  if (T <= 8) router_block_logits_t<8>(x, wr, e, T, E, H, logits, red);
  else if (T <= 16) router_block_logits_t<16>(x, wr, e, T, E, H, logits, red);
  else router_block_logits_t<32>(x, wr, e, T, E, H, logits, red);
}

// Decode-sized T (<= 32): block e computes expert e's logits for every token
// (its 256 threads split H four elements at a time, then reduce), and the
// last block to finish selects every token.  `done` is a counter that is
// zero on entry; the last block resets it.
template <typename Tin>
__global__ void __launch_bounds__(256) router_fused_small(const Tin* __restrict__ x,
                                                          const float* __restrict__ wr,
                                                          SelectArgs a, int H,
                                                          unsigned int* done) {
  extern __shared__ float sel_smem[];
  __shared__ float red[16][32];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int T = a.T, E = a.E;
  const int e = blockIdx.x;
  float* logits = const_cast<float*>(a.logits);
  pdl_wait();
  pdl_trigger();
  router_block_logits(x, wr, e, T, E, H, logits, red);
  // last-block-done: the block that finishes last sees every logit
  __shared__ unsigned int ticket;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) ticket = atomicAdd(done, 1u);
  __syncthreads();
  if (ticket != gridDim.x - 1) return;
  __threadfence();
  for (int t = wib; t < T; t += 8)
    select_token(a, t, logits + (size_t)t * E, sel_smem + (size_t)wib * 2 * E, lane);
  if (threadIdx.x == 0) *done = 0u;
}

// fp32 router weight -> three bf16 planes [E][3H] (hi | mid | lo) with
// w = hi + mid + lo to 24 significant bits, so that a bf16 tensor-core GEMM
// over K = 3H reproduces the fp32-weight logits.
__global__ void router_split(const float* __restrict__ wr, __nv_bfloat16* __restrict__ out, int E,
                             int H) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = (int64_t)E * H;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int e = (int)(i / H), h = (int)(i - (int64_t)e * H);
    const float w = wr[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    __nv_bfloat16* row = out + (size_t)e * 3 * H;
    row[h] = hi;
    row[H + h] = mid;
    row[2 * H + h] = lo;
  }
}

}  // namespace nh

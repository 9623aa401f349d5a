// gemm_q4.cuh -- expert GEMM with NVFP4 weights (W4A16, group size 16) on the
// sm_100a tensor cores, decode orientation.
//
// "NVFP4 W4A16 group_size 16 on the experts, shared experts" (vllm.cpp PR
// #518): every weight is an E2M1 code times an E4M3 scale shared by 16
// consecutive input features, times a float32 scale per matrix; activations
// stay bf16.  The kernel streams the 4-bit codes and the scale bytes with TMA
// (0.5625 bytes per weight instead of 2), dequantizes each stage in shared
// memory to bf16 (code x block scale, which bf16 holds exactly), multiplies
// with tcgen05.mma kind::f16 (weights on the M side, 128 rows; tokens on N),
// and applies the float32 matrix scale in the epilogue.
//
// Roles (448 threads): warp 0 lane 0 TMA producer + tile scheduler; warp 1
// tensor memory owner and MMA issuer; warps 2..5 epilogue (one TMEM lane
// quarter each); warps 6..13 dequantize (thread = half a weight row).
#pragma once

#include "gemm_tc.cuh"

namespace nh {
namespace q4 {

constexpr int BK = 64;        // K per stage (one 128-byte bf16 row after dequantization)
constexpr int UMMA_K = 16;
constexpr int M = 128;        // weight rows per tile
constexpr int DQ_WARPS = 8;
constexpr int THREADS = (6 + DQ_WARPS) * 32;
constexpr int CODE_BYTES = M * BK / 2;      // 4 KB of E2M1 pairs
constexpr int SCALE_BOX = 16;               // bytes of scales per row staged (4 stages' worth)
constexpr int SCALE_BYTES = M * SCALE_BOX;  // 2 KB

template <int NT, int STAGES>
struct Shape {
  static constexpr int A_BYTES = M * BK * 2;       // dequantized weights (bf16, 128B swizzle)
  static constexpr int B_BYTES = NT * BK * 2;      // activations
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + CODE_BYTES + SCALE_BYTES;
  static constexpr int TX_BYTES = B_BYTES + CODE_BYTES + SCALE_BYTES;
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static constexpr int TMEM_COLS = (2 * NT < 32) ? 32 : 2 * NT;
  static constexpr int NBAR = 3 * STAGES + 5 + 2 * tc::TQ;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + NBAR * 8 + 16 + 4 * tc::TQ + 4 * STAGES;
};

struct Q4Args {
  tc::TcArgs g;          // tiles, N, K, epilogue, status, scheduler (as the bf16 kernel)
  const float* gscale;   // float32 scale of each weight matrix [n_mat]
};

// E2M1 pair (one byte) and an f16x2 copy of the block scale -> bf16x2 of
// code x scale (exact: at most 6 significant bits)
__device__ __forceinline__ uint32_t dq_pair(uint32_t byte, uint32_t scale2) {
  uint32_t h;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h) : "r"(byte));
  uint32_t p;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p) : "r"(h), "r"(scale2));
  const __half2 hp = *reinterpret_cast<const __half2*>(&p);
  const float2 f = __half22float2(hp);
  return pack_bf16x2(f.x, f.y);
}

// E4M3 byte -> f16x2 holding the scale in both halves
__device__ __forceinline__ uint32_t scale_f16x2(uint32_t byte) {
  uint32_t h;
  const uint16_t b2 = (uint16_t)(byte | (byte << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(b2));
  return h;
}

template <int NT, int STAGES>
__global__ void __launch_bounds__(THREADS, 1)
    tc_q4_gemm(const __grid_constant__ CUtensorMap map_act,
               const __grid_constant__ CUtensorMap map_codes,
               const __grid_constant__ CUtensorMap map_scales, const Q4Args qa) {
  using S = Shape<NT, STAGES>;
  const tc::TcArgs& g = qa.g;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const uint32_t bar0 = base + STAGES * S::STAGE_BYTES;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto dq_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (3 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (3 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (3 * STAGES + 4);
  auto tq_full_bar = [&](int i) { return bar0 + 8u * (3 * STAGES + 5 + i); };
  auto tq_empty_bar = [&](int i) { return bar0 + 8u * (3 * STAGES + 5 + tc::TQ + i); };
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + STAGES * S::STAGE_BYTES + S::NBAR * 8);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* const tile_q = reinterpret_cast<volatile int*>(tmem_slot + 4);
  volatile int* const stage_kb = reinterpret_cast<volatile int*>(tmem_slot + 4 + tc::TQ);
  auto a_tile = [&](int s) { return base + s * S::STAGE_BYTES; };
  auto b_tile = [&](int s) { return a_tile(s) + S::A_BYTES; };
  auto c_tile = [&](int s) { return b_tile(s) + S::B_BYTES; };
  auto s_tile = [&](int s) { return c_tile(s) + CODE_BYTES; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(dq_bar(s), DQ_WARPS);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 128);
    }
    mbar_init(drain_bar, 1);
    for (int i = 0; i < tc::TQ; ++i) {
      mbar_init(tq_full_bar(i), 1);
      mbar_init(tq_empty_bar(i), 1 + 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&map_act);
    tma_prefetch_map(&map_codes);
    tma_prefetch_map(&map_scales);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();
  const WaitCtl wc{abort_flag, g.status, g.timeout_ns};

  const int num_m = g.tiles ? *g.num_tiles : (g.dense_rows + g.tile_rows - 1) / g.tile_rows;
  const int n_blocks = (g.N + M - 1) / M;
  const int total = num_m * n_blocks;
  const int nk = g.K / BK;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer + tile scheduler ----------------
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int q = i % tc::TQ;
      if (!mbar_wait(tq_empty_bar(q), ((i / tc::TQ) & 1) ^ 1u, wc, SITE_TC_PRODUCER)) {
        ok = false;
        break;
      }
      int tile = (int)atomicAdd(g.sched, 1u);
      if (tile >= total) tile = -1;
      tile_q[q] = tile;
      mbar_arrive(tq_full_bar(q));
      if (tile < 0) break;
      const int m = tile / n_blocks, nb = tile - m * n_blocks;
      const int4 ent = tc::tile_entry_of(g, m);
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc, SITE_TC_PRODUCER)) {
          ok = false;
          break;
        }
        const int ka = g.a_kwrap ? (kb * BK) % g.a_kwrap : kb * BK;
        stage_kb[stage] = kb;
        mbar_arrive_expect_tx(full_bar(stage), S::TX_BYTES);
        tma_load_3d(c_tile(stage), &map_codes, full_bar(stage), kb * (BK / 2), nb * M, ent.x);
        tma_load_3d(s_tile(stage), &map_scales, full_bar(stage), (kb / 4) * SCALE_BOX, nb * M, ent.x);
        tma_load_2d(b_tile(stage), &map_act, full_bar(stage), ka, g.row_token ? 0 : ent.y);
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (ok && mbar_wait(empty_bar(stage), phase ^ 1u, wc, SITE_TC_PRODUCER)) {
      // end marker for the dequantize warps: a stage with no copies and kb = -1
      stage_kb[stage] = -1;
      mbar_arrive(full_bar(stage));
    } else {
      const long first = issued > STAGES ? issued - STAGES : 0;
      for (long i = first; i < issued; ++i)
        tc::mbar_drain(full_bar((int)(i % STAGES)), (uint32_t)((i / STAGES) & 1), g.timeout_ns,
                       g.status);
    }
  } else if (warp >= 6) {
    // ---------------- dequantize: thread = half of a weight row ----------------
    const int t = threadIdx.x - 6 * 32;
    const int row = t & (M - 1), half = t >> 7;    // 256 threads: 128 rows x 2 halves
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    while (ok) {
      int st = 1;
      if (lane == 0) st = mbar_wait(full_bar(stage), phase, wc, SITE_TC_EPILOGUE) ? 1 : 0;
      st = __shfl_sync(0xffffffffu, st, 0);
      if (!st) break;
      const int kb = stage_kb[stage];
      if (kb < 0) break;                               // no more stages
      const uint4 c = *reinterpret_cast<const uint4*>(base_ptr + (c_tile(stage) - base) + row * 32 + half * 16);
      const uint8_t* sp = base_ptr + (s_tile(stage) - base) + row * SCALE_BOX + (kb & 3) * 4 + half * 2;
      const uint32_t s0 = scale_f16x2(sp[0]), s1 = scale_f16x2(sp[1]);
      const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
      uint32_t o[16];
#pragma unroll
      for (int wd = 0; wd < 4; ++wd)
#pragma unroll
        for (int b = 0; b < 4; ++b) o[wd * 4 + b] = dq_pair((cw[wd] >> (8 * b)) & 0xffu, wd < 2 ? s0 : s1);
      uint8_t* arow = base_ptr + (a_tile(stage) - base) + row * 128;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        const int chunk = (half * 4 + ch) ^ (row & 7);   // 128-byte swizzle of the bf16 row
        *reinterpret_cast<uint4*>(arow + chunk * 16) =
            make_uint4(o[ch * 4], o[ch * 4 + 1], o[ch * 4 + 2], o[ch * 4 + 3]);
      }
      // generic-proxy stores -> visible to the tensor core's async proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_bar(stage));
      if (++stage == STAGES) {
        stage = 0;
        phase ^= 1u;
      }
      if (*abort_flag) ok = false;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true, any = false;
    for (int i = 0; ok; ++i) {
      const int q = i % tc::TQ;
      if (!mbar_wait(tq_full_bar(q), (i / tc::TQ) & 1, wc, SITE_TC_MMA)) {
        ok = false;
        break;
      }
      const int tile = tile_q[q];
      mbar_arrive(tq_empty_bar(q));
      if (tile < 0) break;
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      if (!mbar_wait(tempty_bar(acc), aph ^ 1u, wc, SITE_TC_MMA)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t idesc = make_idesc_bf16(M, NT);
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * NT);
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(full_bar(stage), phase, wc, SITE_TC_MMA) ||
            !mbar_wait(dq_bar(stage), phase, wc, SITE_TC_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BK / UMMA_K; ++kk)
          umma_bf16(d_tmem, make_sdesc_sw128(a_tile(stage) + kk * UMMA_K * 2),
                    make_sdesc_sw128(b_tile(stage) + kk * UMMA_K * 2), idesc, (kb | kk) != 0);
        any = true;
        umma_commit(empty_bar(stage));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      umma_commit(tfull_bar(acc));
      ++it;
    }
    if (!ok && any) {
      umma_commit(drain_bar);
      tc::mbar_drain(drain_bar, 0, g.timeout_ns, g.status);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ---------------- epilogue ----------------
    const int qd = warp & 3;
    int it = 0;
    for (int i = 0;; ++i) {
      int tile = -1;
      int ok = 1;
      if (lane == 0) {
        const int slot = i % tc::TQ;
        ok = mbar_wait(tq_full_bar(slot), (i / tc::TQ) & 1, wc, SITE_TC_EPILOGUE) ? 1 : 0;
        if (ok) {
          tile = tile_q[slot];
          mbar_arrive(tq_empty_bar(slot));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (!ok || tile < 0) break;
      const int m = tile / n_blocks, nb = tile - m * n_blocks;
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      if (lane == 0) ok = mbar_wait(tfull_bar(acc), aph, wc, SITE_TC_EPILOGUE) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int4 ent = tc::tile_entry_of(g, m);
      const float gs = qa.gscale[ent.x];
      const uint32_t tq = tmem_base + ((uint32_t)(qd * 32) << 16) + (uint32_t)(acc * NT);
      const int f = nb * M + qd * 32 + lane;
      const bool valid = f < g.N;
#pragma unroll
      for (int c = 0; c < NT; c += 16) {
        float v[16];
        tmem_ld_x16(tq + (uint32_t)c, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] *= gs;
        if (g.row_token) {
          for (int j = 0; j < ent.z; ++j) {
            const int tt = g.row_token[ent.y + j] - c;
            if (tt < 0 || tt >= 16) continue;
            float val = 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) val = (u == tt) ? v[u] : val;
            if (valid) tc::epi_elem(g, ent.y + j, f, val);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (valid && c + j < ent.z) tc::epi_elem(g, ent.y + c + j, f, v[j]);
        }
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      ++it;
    }
  }
  __syncthreads();
  tc_fence_before();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(g.sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(g.sched, 0u);
      atomicExch(g.sched + 1, 0u);
    }
  }
}

}  // namespace q4
}  // namespace nh

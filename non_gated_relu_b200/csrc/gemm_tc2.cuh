// gemm_tc2.cuh -- the prefill expert GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same computation and epilogues as tc_grouped_gemm in its prefill
// orientation (gemm_tc.cuh), but each output tile is 256 rows x up to 256
// features and is computed by a cluster of two CTAs on two SMs: the leader
// CTA issues tcgen05.mma.cta_group::2 with M = 256, each CTA holds half of the
// A rows (128) and half of the B rows (N / 2) in its own shared memory, and
// each CTA's tensor memory receives its 128 rows of the accumulator.  Per SM
// this halves the B operand that has to be staged and read for the same
// number of MMA cycles, which is what limits the one-CTA 128 x 256 tile.
//
// An expert's last, partial tile (fewer than 256 rows) is computed swapped:
// 256 weight rows (128 per CTA) on the MMA M side and the remaining token rows
// (rounded up to 16) on N, so the tensor cores do not multiply padding rows.
// Both tile kinds use the same tensor maps and the same accumulator layout;
// only the operand roles, the MMA shape and the epilogue's indexing change.
//
// Roles per CTA (192 threads), as in the one-CTA kernel:
//   warp 0 lane 0  TMA producer (both CTAs; the leader also runs the tile
//                  scheduler and forwards each tile id to the peer);
//   warp 1         tensor memory owner; lane 0 of the leader issues the MMAs;
//   warps 2..5     epilogue of the CTA's 128 accumulator rows.
// Both CTAs' TMA loads complete on the leader's stage barrier; the leader's
// MMA completion is committed to the stage / accumulator barriers of both
// CTAs (two plain commits, no multicast); the peer's epilogue and scheduler
// hand-backs arrive on the leader's barriers through shared::cluster
// addresses.  All waits are bounded like the one-CTA kernel's.
#pragma once

#include "gemm_tc.cuh"

namespace nh {
namespace tc2 {

constexpr int BK = 64;
constexpr int UMMA_K = 16;
constexpr int MP = 256;       // tile rows (MMA M across the pair)
constexpr int NT = 256;       // tile features (MMA N)
constexpr int HALF = 128;     // rows of A and of B staged per CTA
constexpr int STAGES = 7;
constexpr int THREADS = 192;
constexpr int A_BYTES = HALF * BK * 2;
constexpr int B_BYTES = HALF * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * NT;
constexpr int TQ = 4;
constexpr int NBAR = 2 * STAGES + 5 + 2 * TQ;
constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + NBAR * 8 + 16 + 4 * TQ;
static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");

// MMA N of a swapped remainder tile of `rows` token rows
__device__ __forceinline__ int swap_n(int rows) { return (rows + 15) & ~15; }

// tile entry (expert, first row, rows, kind); kind 1 = swapped remainder tile
__device__ __forceinline__ int4 pair_entry(const tc::TcArgs& g, int m) {
  if (g.tiles) return g.tiles[m];
  const int r0 = m * g.tile_rows;
  const int rows = min(g.tile_rows, g.dense_rows - r0);
  return make_int4(0, r0, rows, rows < g.tile_rows ? 1 : 0);
}

__global__ void __launch_bounds__(THREADS, 1)
    tc2_grouped_gemm(const __grid_constant__ CUtensorMap map_act,
                     const __grid_constant__ CUtensorMap map_w, const tc::TcArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const uint32_t bar0 = base + STAGES * STAGE_BYTES;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  auto tq_full_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + 5 + i); };
  auto tq_empty_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + 5 + TQ + i); };
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + STAGES * STAGE_BYTES + NBAR * 8);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* const tile_q = reinterpret_cast<volatile int*>(tmem_slot + 4);

  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * 4);       // 4 epilogue warps in each CTA
    }
    mbar_init(drain_bar, 1);
    for (int i = 0; i < TQ; ++i) {
      mbar_init(tq_full_bar(i), 1);
      mbar_init(tq_empty_bar(i), 2 * 5);     // MMA (leader) / producer (peer) + 4 epilogue warps, x2
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&map_act);
    tma_prefetch_map(&map_w);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // peers' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // everything above overlaps the previous kernel; inputs are read from here on
  pdl_wait();
  pdl_trigger();
  const WaitCtl wc{abort_flag, g.status, g.timeout_ns};

  const int num_m = g.tiles ? *g.num_tiles : (g.dense_rows + g.tile_rows - 1) / g.tile_rows;
  const int n_blocks = (g.N + NT - 1) / NT;
  const int total = num_m * n_blocks;
  const int nk = g.K / BK;

  if (warp == 0 && lane == 0) {
    // ---------------- producer (+ scheduler on the leader) ----------------
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int q = i % TQ;
      const uint32_t ph = (uint32_t)((i / TQ) & 1);
      int tile;
      if (leader) {
        if (!mbar_wait_cluster(tq_empty_bar(q), ph ^ 1u, wc, SITE_TC_PRODUCER)) {
          ok = false;
          break;
        }
        tile = (int)atomicAdd(g.sched, 1u);
        if (tile >= total) tile = -1;
        tile_q[q] = tile;
        st_cluster_u32(map_to_rank(smem_u32((const void*)&tile_q[q]), 1), (uint32_t)tile);
        mbar_arrive(tq_full_bar(q));
        mbar_arrive_cluster(map_to_rank(tq_full_bar(q), 1));
      } else {
        if (!mbar_wait_cluster(tq_full_bar(q), ph, wc, SITE_TC_PRODUCER)) {
          ok = false;
          break;
        }
        tile = tile_q[q];
        mbar_arrive_cluster(map_to_rank(tq_empty_bar(q), 0));
      }
      if (tile < 0) break;
      const int m = tile / n_blocks, nb = tile - m * n_blocks;
      const int4 ent = pair_entry(g, m);
      const int n0 = nb * NT;
      // operand rows staged by this CTA: slot A (M side) and slot B (N side)
      int a_row, b_row;
      if (ent.w == 0) {                                     // activations x weights
        a_row = ent.y + (int)rank * HALF;
        b_row = n0 + (int)rank * (min(NT, g.N - n0) / 2);
      } else {                                              // weights x remainder rows
        a_row = n0 + (int)rank * HALF;
        b_row = ent.y + (int)rank * (swap_n(ent.z) / 2);
      }
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait_cluster(empty_bar(stage), phase ^ 1u, wc, SITE_TC_PRODUCER)) {
          ok = false;
          break;
        }
        const uint32_t sa = base + stage * STAGE_BYTES, sb = sa + A_BYTES;
        const uint32_t fb = map_to_rank(full_bar(stage), 0);
        const int ka = g.a_kwrap ? (kb * BK) % g.a_kwrap : kb * BK;
        if (leader) mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
        if (ent.w == 0) {
          tma_load_2d_pair(sa, &map_act, fb, ka, a_row);
          tma_load_3d_pair(sb, &map_w, fb, kb * BK, b_row, ent.x);
        } else {
          tma_load_3d_pair(sa, &map_w, fb, kb * BK, a_row, ent.x);
          tma_load_2d_pair(sb, &map_act, fb, ka, b_row);
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && leader) {
      // the leader's stage barriers count both CTAs' copies: wait for those in flight
      const long first = issued > STAGES ? issued - STAGES : 0;
      for (long i = first; i < issued; ++i)
        tc::mbar_drain(full_bar((int)(i % STAGES)), (uint32_t)((i / STAGES) & 1), g.timeout_ns,
                       g.status);
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------- MMA issuer (leader only) ----------------
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true, any = false;
    for (int i = 0; ok; ++i) {
      const int q = i % TQ;
      if (!mbar_wait_cluster(tq_full_bar(q), (uint32_t)((i / TQ) & 1), wc, SITE_TC_MMA)) {
        ok = false;
        break;
      }
      const int tile = tile_q[q];
      mbar_arrive(tq_empty_bar(q));
      if (tile < 0) break;
      const int nb = tile % n_blocks;
      const int4 ent = pair_entry(g, tile / n_blocks);
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      if (!mbar_wait_cluster(tempty_bar(acc), aph ^ 1u, wc, SITE_TC_MMA)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int n_mma = ent.w == 0 ? min(NT, g.N - nb * NT) : swap_n(ent.z);
      const uint32_t idesc = make_idesc_bf16(MP, n_mma);
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * NT);
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait_cluster(full_bar(stage), phase, wc, SITE_TC_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = base + stage * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / UMMA_K; ++kk)
          umma_bf16_pair(d_tmem, make_sdesc_sw128(sa + kk * UMMA_K * 2),
                         make_sdesc_sw128(sb + kk * UMMA_K * 2), idesc, (kb | kk) != 0);
        any = true;
        umma_commit_pair(empty_bar(stage));
        umma_commit_pair(map_to_rank(empty_bar(stage), 1));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      umma_commit_pair(tfull_bar(acc));
      umma_commit_pair(map_to_rank(tfull_bar(acc), 1));
      ++it;
    }
    if (!ok && any) {
      umma_commit_pair(drain_bar);
      tc::mbar_drain(drain_bar, 0, g.timeout_ns, g.status);
    }
  } else if (warp >= 2) {
    // ---------------- epilogue: this CTA's 128 rows of the tile ----------------
    const int qw = warp & 3;
    int it = 0;
    for (int i = 0;; ++i) {
      int tile = -1;
      int ok = 1;
      if (lane == 0) {
        const int slot = i % TQ;
        ok = mbar_wait_cluster(tq_full_bar(slot), (uint32_t)((i / TQ) & 1), wc, SITE_TC_EPILOGUE)
                 ? 1 : 0;
        if (ok) {
          tile = tile_q[slot];
          if (leader)
            mbar_arrive(tq_empty_bar(slot));
          else
            mbar_arrive_cluster(map_to_rank(tq_empty_bar(slot), 0));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (!ok || tile < 0) break;
      const int m = tile / n_blocks, nb = tile - m * n_blocks;
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      if (lane == 0) ok = mbar_wait_cluster(tfull_bar(acc), aph, wc, SITE_TC_EPILOGUE) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int4 ent = pair_entry(g, m);
      const int n0 = nb * NT;
      const uint32_t tq = tmem_base + ((uint32_t)(qw * 32) << 16) + (uint32_t)(acc * NT);
      if (ent.w == 0) {
        // accumulator lane = token row, column = output feature
        const int row = (int)rank * HALF + qw * 32 + lane;
        const bool valid = row < ent.z;
        const int n_eff = min(NT, g.N - n0);
        for (int c = 0; c < n_eff; c += 32) {
          float v[32];
          tmem_ld_x32(tq + (uint32_t)c, v);
          if (valid) tc::epi_row32(g, ent.y + row, n0 + c, v);
        }
      } else {
        // accumulator lane = output feature, column = token row of the remainder
        const int f = n0 + (int)rank * HALF + qw * 32 + lane;
        const bool valid = f < g.N;
        const int n_mma = swap_n(ent.z);
        for (int c = 0; c < n_mma; c += 16) {
          float v[16];
          tmem_ld_x16(tq + (uint32_t)c, v);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (valid && c + j < ent.z) tc::epi_elem(g, ent.y + c + j, f, v[j]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(tempty_bar(acc));
        else
          mbar_arrive_cluster(map_to_rank(tempty_bar(acc), 0));
      }
      ++it;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // no CTA leaves while its peer may still touch its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && leader) {
    __threadfence();
    if (atomicAdd(g.sched + 1, 1u) == gridDim.x / 2 - 1) {
      atomicExch(g.sched, 0u);
      atomicExch(g.sched + 1, 0u);
    }
  }
}

}  // namespace tc2
}  // namespace nh

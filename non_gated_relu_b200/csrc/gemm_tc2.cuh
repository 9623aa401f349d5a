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
// A partial tile of at most 64 rows rides on the expert's last full tile
// instead (kind 2): each K step also stages those rows (32 per CTA) and
// issues a second, swapped MMA whose A operand is the weight tile already in
// shared memory, into the other tensor-memory accumulator.  The expert's
// weights then cross from L2 once per feature block for both parts; a
// separate small tile would stream them again for a few rows of work.
// All tile kinds use the same tensor maps and accumulator layout; only the
// operand roles, the MMA shapes and the epilogue's indexing change.
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
// addresses.  The per-stage waits (producer on empty, MMA on full) are
// CTA-scope polls; the tile-id and accumulator hand-offs between the CTAs use
// cluster-scope acquire.  All waits are bounded like the one-CTA kernel's.
#pragma once

#include "gemm_tc.cuh"
#include "permute.cuh"  // PAIR_ATTACH_ROWS

namespace nh {
namespace tc2 {

constexpr int BK = 64;
constexpr int UMMA_K = 16;
constexpr int MP = 256;       // tile rows (MMA M across the pair)
constexpr int NT = 256;       // tile features (MMA N)
constexpr int HALF = 128;     // rows of A and of B staged per CTA
constexpr int C_ROWS = PAIR_ATTACH_ROWS / 2;   // attached remainder rows staged per CTA
constexpr int STAGES = 6;
constexpr int THREADS = 192;
constexpr int A_BYTES = HALF * BK * 2;
constexpr int B_BYTES = HALF * BK * 2;
constexpr int C_BYTES = C_ROWS * BK * 2;
constexpr int AB_BYTES = A_BYTES + B_BYTES;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES;
constexpr int TMEM_COLS = 2 * NT;
constexpr int TQ = 4;
constexpr int NBAR = 2 * STAGES + 5 + 2 * TQ;
constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + NBAR * 8 + 16 + 4 * TQ;
static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");

// MMA N of a swapped remainder tile of `rows` token rows
__device__ __forceinline__ int swap_n(int rows) { return (rows + 15) & ~15; }

// tile entry (expert, first row, rows, kind); kind 1 = swapped remainder tile,
// kind 2 = a full tile plus rows - MP attached remainder rows
__device__ __forceinline__ int4 pair_entry(const tc::TcArgs& g, int m) {
  if (g.tiles) return g.tiles[m];
  const int r0 = m * g.tile_rows;
  const int rows = min(g.tile_rows, g.dense_rows - r0);
  return make_int4(0, r0, rows, rows < g.tile_rows ? 1 : 0);
}

__global__ void __launch_bounds__(THREADS, 1)
    tc2_grouped_gemm(const __grid_constant__ CUtensorMap map_act,
                     const __grid_constant__ CUtensorMap map_w,
                     const __grid_constant__ CUtensorMap map_rem, const tc::TcArgs g) {
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
    tma_prefetch_map(&map_rem);
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
      // operand rows staged by this CTA: slot A (M side), slot B (N side) and,
      // for kind 2, slot C (the attached remainder rows)
      const bool swapped = ent.w == 1, attached = ent.w == 2;
      int a_row, b_row;
      if (!swapped) {                                       // activations x weights
        a_row = ent.y + (int)rank * HALF;
        b_row = n0 + (int)rank * (min(NT, g.N - n0) / 2);
      } else {                                              // weights x remainder rows
        a_row = n0 + (int)rank * HALF;
        b_row = ent.y + (int)rank * (swap_n(ent.z) / 2);
      }
      const int c_row = ent.y + MP + (int)rank * (attached ? swap_n(ent.z - MP) / 2 : 0);
      const uint32_t tx_bytes = 2u * (attached ? STAGE_BYTES : AB_BYTES);
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait_spin(empty_bar(stage), phase ^ 1u, wc, SITE_TC_PRODUCER)) {
          ok = false;
          break;
        }
        const uint32_t sa = base + stage * STAGE_BYTES, sb = sa + A_BYTES, sc = sb + B_BYTES;
        const uint32_t fb = map_to_rank(full_bar(stage), 0);
        const int ka = g.a_kwrap ? (kb * BK) % g.a_kwrap : kb * BK;
        if (leader) mbar_arrive_expect_tx(full_bar(stage), tx_bytes);
        if (!swapped) {
          tma_load_2d_pair(sa, &map_act, fb, ka, a_row);
          tma_load_3d_pair(sb, &map_w, fb, kb * BK, b_row, ent.x);
          if (attached) tma_load_2d_pair(sc, &map_rem, fb, ka, c_row);
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
      const bool attached = ent.w == 2;
      // a kind-2 tile takes both accumulators: the full tile, then the remainder
      const int acc = it & 1, acc2 = (it + 1) & 1;
      if (!mbar_wait_cluster(tempty_bar(acc), (uint32_t)((it >> 1) & 1) ^ 1u, wc, SITE_TC_MMA) ||
          (attached && !mbar_wait_cluster(tempty_bar(acc2), (uint32_t)(((it + 1) >> 1) & 1) ^ 1u,
                                          wc, SITE_TC_MMA))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int n_mma = ent.w == 1 ? swap_n(ent.z) : min(NT, g.N - nb * NT);
      const uint32_t idesc = make_idesc_bf16(MP, n_mma);
      const uint32_t idesc2 = make_idesc_bf16(MP, attached ? swap_n(ent.z - MP) : 16);
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * NT);
      const uint32_t d2_tmem = tmem_base + (uint32_t)(acc2 * NT);
      // Two copies of the K loop: the MMA stream of an ordinary tile keeps no
      // branch between its MMAs (a conditional second MMA in the same loop cost
      // about 15 % of throughput on every tile, measured)
      if (!attached) {
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_spin(full_bar(stage), phase, wc, SITE_TC_MMA)) {
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
      } else {
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_spin(full_bar(stage), phase, wc, SITE_TC_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + stage * STAGE_BYTES, sb = sa + A_BYTES, sc = sb + B_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            umma_bf16_pair(d_tmem, make_sdesc_sw128(sa + kk * UMMA_K * 2),
                           make_sdesc_sw128(sb + kk * UMMA_K * 2), idesc, (kb | kk) != 0);
          // attached partial tile: the staged weight rows on M, its rows on N
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            umma_bf16_pair(d2_tmem, make_sdesc_sw128(sb + kk * UMMA_K * 2),
                           make_sdesc_sw128(sc + kk * UMMA_K * 2), idesc2, (kb | kk) != 0);
          any = true;
          umma_commit_pair(empty_bar(stage));
          umma_commit_pair(map_to_rank(empty_bar(stage), 1));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) break;
      umma_commit_pair(tfull_bar(acc));
      umma_commit_pair(map_to_rank(tfull_bar(acc), 1));
      if (attached) {
        umma_commit_pair(tfull_bar(acc2));
        umma_commit_pair(map_to_rank(tfull_bar(acc2), 1));
      }
      it += attached ? 2 : 1;
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
      const int4 ent = pair_entry(g, m);
      const int n0 = nb * NT;
      const int n_eff = min(NT, g.N - n0);
      // wait for accumulator use `u` (slot u & 1), or give up with the CTA
      auto acquire = [&](int u) {
        int r = 1;
        if (lane == 0)
          r = mbar_wait_cluster(tfull_bar(u & 1), (uint32_t)((u >> 1) & 1), wc, SITE_TC_EPILOGUE)
                  ? 1 : 0;
        r = __shfl_sync(0xffffffffu, r, 0);
        if (r) tc_fence_after();
        return r != 0;
      };
      auto release = [&](int u) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(tempty_bar(u & 1));
          else
            mbar_arrive_cluster(map_to_rank(tempty_bar(u & 1), 0));
        }
      };
      // accumulator lane = output feature, column = token row: the rows
      // [r0, r0 + rows) of a swapped MMA; this CTA's lanes hold features
      // f0 + lane index, valid below f_end
      auto swapped_rows = [&](uint32_t tq, int r0, int rows, int f0, int f_end) {
        const int f = f0 + qw * 32 + lane;
        const bool valid = f < f_end;
        const int n_mma = swap_n(rows);
        for (int c = 0; c < n_mma; c += 16) {
          float v[16];
          tmem_ld_x16(tq + (uint32_t)c, v);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (valid && c + j < rows) tc::epi_elem(g, r0 + c + j, f, v[j]);
        }
      };
      // a kind-2 tile holds two accumulator uses: the full tile, then the
      // attached partial tile; one loop keeps a single copy of each path
      const int parts = ent.w == 2 ? 2 : 1;
      bool live = true;
      for (int part = 0; part < parts; ++part) {
        const int u = it + part;
        if (!acquire(u)) {
          live = false;
          break;
        }
        const uint32_t tq = tmem_base + ((uint32_t)(qw * 32) << 16) + (uint32_t)((u & 1) * NT);
        if (part == 0 && ent.w != 1) {
          // accumulator lane = token row, column = output feature
          const int row = (int)rank * HALF + qw * 32 + lane;
          const bool valid = row < min(ent.z, MP);
          for (int c = 0; c < n_eff; c += 32) {
            float v[32];
            tmem_ld_x32(tq + (uint32_t)c, v);
            if (valid) tc::epi_row32(g, ent.y + row, n0 + c, v);
          }
        } else {
          // kind 1: weights on M, this CTA's 128 weight rows start at
          // n0 + rank * 128.  Attached partial tile: the weight rows of the B
          // slot on M (this CTA's n_eff / 2 rows start at n0 + rank * n_eff / 2)
          const int f0 = n0 + (int)rank * (part == 0 ? HALF : n_eff / 2);
          const int f_end = part == 0 ? g.N : min(g.N, f0 + n_eff / 2);
          swapped_rows(tq, part == 0 ? ent.y : ent.y + MP, part == 0 ? ent.z : ent.z - MP, f0,
                       f_end);
        }
        release(u);
      }
      if (!live) break;
      it += parts;
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

// gemm_tc.cuh -- persistent grouped expert GEMM on the sm_100a tensor cores.
//
// For every tile entry (expert e, first row r0, rows) of the permute's tile
// table and every block of output features, D = A[r0 : r0+rows, :] . W[e]^T
// is accumulated in tensor memory by tcgen05.mma (bf16 in, f32 accumulate)
// from operand tiles that TMA stages in shared memory with 128-byte swizzle,
// and a fused epilogue turns it into
//   up_proj:   h = relu(D)^2 stored in bf16              (non-gated expert:
//              no gate projection, squared relu between the two
//              projections; vllm.cpp PR #518)
//   down_proj: y_acc[token of row] += routing weight * D    (the weighted
//              combine of a token's k experts, float32 atomic adds)
//   shared:    y_acc += D                                   (always-on expert)
//
// Two orientations:
//   prefill (SWAP = false): MMA M = 128 activation rows, N = NT weight rows;
//   decode  (SWAP = true):  MMA M = 128 weight rows, N = NT activation rows,
//     so that a handful of tokens per expert still fill the 128-row side and
//     the kernel streams each expert's weights once.
//
// Warp roles (192 threads): warp 0 lane 0 issues TMA loads into a STAGES-deep
// ring; warp 1 owns tensor memory and lane 0 issues the MMAs; warps 2..5 read
// the accumulator (each its 32-lane quarter) and run the epilogue.  Two
// accumulators in tensor memory let the epilogue of one tile overlap the
// main loop of the next.  Every mbarrier wait is bounded: when one runs out
// the CTA records NH_ERR_TIMEOUT, drains its copies and MMAs in flight, frees
// its tensor memory and returns.
#pragma once

#include "common.cuh"
#include "gemm_simt.cuh"  // Epilogue codes

namespace nh {
namespace tc {

constexpr int BK = 64;       // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int UMMA_K = 16;   // K of one kind::f16 MMA
constexpr int M = 128;       // MMA M (one CTA)
constexpr int THREADS = 192;

struct TcArgs {
  const int4* tiles;          // (expert, first row, rows, 0) or null: dense rows
  const int32_t* num_tiles;
  int dense_rows;
  int tile_rows;
  int N;                      // output features (weight rows)
  int K;                      // multiple of 64
  int a_kwrap;                // >0: the activation's K coordinate wraps at this value
  int epi;                    // Epilogue
  void* out;
  int64_t ldo;                // row stride of out, elements
  const float* perm_w;
  const int32_t* dst_row;     // EPI_DOWN_COMBINE: output row (token) of each permuted row
  const int32_t* row_token;   // decode up projection: activations are x itself (rows
                              // 0..NT-1) and permuted row r takes accumulator column
                              // row_token[r]; null otherwise
  int* status;
  uint64_t timeout_ns;
  unsigned int* sched;        // [2]: next tile, CTAs finished; zero on entry, reset on exit
  int k_split;                // >1: each output tile is computed as k_split K slices by
                              // separate tiles (additive epilogues only); 0 or 1: whole K
  int* ready;                 // fused launch: per tile entry, epilogue warps done with its
                              // first-GEMM tiles (zeroed by the permute); null otherwise
  int ready_need;             // second GEMM: count that makes a tile entry's rows ready
};

constexpr int TQ = 4;         // depth of the tile-id ring between the roles

template <bool SWAP, int NT, int STAGES>
struct Shape {
  static constexpr int A_BYTES = M * BK * 2;     // M-side tile
  static constexpr int B_BYTES = NT * BK * 2;    // N-side tile
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment");
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= 256, "MMA N");
  static constexpr int ACC_COLS = NT;
  static constexpr int TMEM_COLS = (2 * NT < 32) ? 32 : 2 * NT;
  static_assert((TMEM_COLS & (TMEM_COLS - 1)) == 0 && TMEM_COLS <= 512, "TMEM alloc");
  static constexpr int BAR_BYTES = (2 * STAGES + 5 + 2 * TQ) * 8 + 16 + 4 * TQ;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + BAR_BYTES;
};

__device__ __forceinline__ int4 tile_entry_of(const TcArgs& g, int m) {
  if (g.tiles) return g.tiles[m];
  const int r0 = m * g.tile_rows;
  return make_int4(0, r0, min(g.tile_rows, g.dense_rows - r0), 0);
}

// Wait that ignores the abort flag: used only to drain work already issued.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                           int* status) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) {
      record_status(status, NH_ERR_TIMEOUT, SITE_TC_DRAIN, 0);
      return;
    }
  }
}

// epilogue of 32 consecutive output features of one row (prefill orientation)
__device__ __forceinline__ void epi_row32(const TcArgs& g, int r, int n, const float* v) {
  if (g.epi == EPI_DOWN_COMBINE || g.epi == EPI_ACC_F32) {
    // float32 adds into the accumulator row of the token: 16 bytes per add
    const bool down = g.epi == EPI_DOWN_COMBINE;
    const float w = down ? g.perm_w[r] : 1.f;
    const int64_t row = down ? g.dst_row[r] : r;
    float* dst = static_cast<float*>(g.out) + (size_t)row * g.ldo + n;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      red_add_f32x4(dst + 4 * i, w * v[4 * i], w * v[4 * i + 1], w * v[4 * i + 2],
                    w * v[4 * i + 3]);
    return;
  }
  if (g.epi == EPI_STORE_F32 || g.epi == EPI_ADD_F32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(g.out) + (size_t)r * g.ldo + n);
    const bool add = g.epi == EPI_ADD_F32;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 o = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      if (add) {
        const float4 a = dst[i];
        o.x += a.x; o.y += a.y; o.z += a.z; o.w += a.w;
      }
      dst[i] = o;
    }
    return;
  }
  const bool up = g.epi == EPI_UP_RELU2;
  float o[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) o[i] = up ? relu2(v[i]) : v[i];
  uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + (size_t)r * g.ldo + n);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 p;
    p.x = pack_bf16x2(o[8 * i + 0], o[8 * i + 1]);
    p.y = pack_bf16x2(o[8 * i + 2], o[8 * i + 3]);
    p.z = pack_bf16x2(o[8 * i + 4], o[8 * i + 5]);
    p.w = pack_bf16x2(o[8 * i + 6], o[8 * i + 7]);
    dst[i] = p;
  }
}

// epilogue of one element (decode orientation: feature f of row r)
__device__ __forceinline__ void epi_elem(const TcArgs& g, int r, int f, float v) {
  if (g.epi == EPI_UP_RELU2) {
    static_cast<__nv_bfloat16*>(g.out)[(size_t)r * g.ldo + f] = __float2bfloat16_rn(relu2(v));
  } else if (g.epi == EPI_DOWN_COMBINE) {
    red_add_f32(static_cast<float*>(g.out) + (size_t)g.dst_row[r] * g.ldo + f, g.perm_w[r] * v);
  } else if (g.epi == EPI_STORE) {
    static_cast<__nv_bfloat16*>(g.out)[(size_t)r * g.ldo + f] = __float2bfloat16_rn(v);
  } else if (g.epi == EPI_ADD_F32) {
    static_cast<float*>(g.out)[(size_t)r * g.ldo + f] += v;
  } else if (g.epi == EPI_ACC_F32) {
    red_add_f32(static_cast<float*>(g.out) + (size_t)r * g.ldo + f, v);
  } else {
    static_cast<float*>(g.out)[(size_t)r * g.ldo + f] = v;
  }
}

// Wait until a fused launch's first GEMM has finished every tile of tile entry
// m (its epilogue warps have stored those rows and counted them), then order
// those generic-proxy stores before this thread's tensor-memory-access loads.
__device__ __forceinline__ bool wait_ready(const int* ready, int m, int need, const WaitCtl& w) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 0;; ++i) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ready + m) : "memory");
    if (v >= need) break;
    if ((i & 63u) == 63u) {
      // another CTA's wait already ran out (the status word holds an error): stop
      if (*w.abort_flag || (w.status && *reinterpret_cast<volatile int*>(w.status) != 0)) {
        *w.abort_flag = 1;
        return false;
      }
      if (globaltimer_ns() - t0 > w.timeout_ns) {
        *w.abort_flag = 1;
        record_status(w.status, NH_ERR_TIMEOUT, SITE_TC_PRODUCER, m);
        return false;
      }
    }
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// map_act2 / map_w2 / g2: a second GEMM in the same launch (g2.N > 0), over the
// same tile entries, whose activations are the first GEMM's output: the decode
// up projection and down projection as one persistent grid.  Its tiles come
// after all of the first GEMM's in the scheduler's order, and its producer
// waits per tile entry until the first GEMM's epilogues have written those
// rows (g.ready); since every CTA is resident and tiles are handed out in
// order, the tiles waited on are already running.  The SMs that finish the
// first GEMM's last tiles early go on to the second GEMM's instead of idling.
template <bool SWAP, int NT, int STAGES>
__global__ void __launch_bounds__(THREADS, 1)
    tc_grouped_gemm(const __grid_constant__ CUtensorMap map_act,
                    const __grid_constant__ CUtensorMap map_w, const TcArgs g,
                    const __grid_constant__ CUtensorMap map_act2,
                    const __grid_constant__ CUtensorMap map_w2, const TcArgs g2) {
  using S = Shape<SWAP, NT, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const uint32_t bar0 = base + STAGES * S::STAGE_BYTES;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  auto tq_full_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + 5 + i); };
  auto tq_empty_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + 5 + TQ + i); };
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + STAGES * S::STAGE_BYTES +
                                                          (2 * STAGES + 5 + 2 * TQ) * 8);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* const tile_q = reinterpret_cast<volatile int*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 128);
    }
    mbar_init(drain_bar, 1);
    for (int i = 0; i < TQ; ++i) {
      mbar_init(tq_full_bar(i), 1);
      mbar_init(tq_empty_bar(i), 1 + 4);   // MMA issuer + one lane per epilogue warp
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_map(&map_act);
    tma_prefetch_map(&map_w);
    if (g2.N > 0) {
      tma_prefetch_map(&map_act2);
      tma_prefetch_map(&map_w2);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // everything above overlaps the previous kernel; inputs are read from here on
  pdl_wait();
  pdl_trigger();
  const WaitCtl wc{abort_flag, g.status, g.timeout_ns};

  const int num_m = g.tiles ? *g.num_tiles : (g.dense_rows + g.tile_rows - 1) / g.tile_rows;
  const bool fused = g2.N > 0;
  auto n_blocks_of = [&](const TcArgs& a) { return SWAP ? (a.N + M - 1) / M : (a.N + NT - 1) / NT; };
  auto ks_of = [&](const TcArgs& a) { return a.k_split > 1 ? a.k_split : 1; };
  const int total1 = num_m * n_blocks_of(g) * ks_of(g);
  const int total = total1 + (fused ? num_m * n_blocks_of(g2) * ks_of(g2) : 0);
  // tile id -> (GEMM ph, tile entry m, feature block nb, K slice [kb_lo, kb_hi))
  auto decode_tile = [&](int tile, int& ph, int& m, int& nb, int& kb_lo, int& kb_hi) {
    ph = tile >= total1 ? 1 : 0;
    const TcArgs& a = ph ? g2 : g;
    if (ph) tile -= total1;
    const int ks_n = ks_of(a), n_blocks = n_blocks_of(a), nk = a.K / BK;
    const int ks = tile % ks_n, rest = tile / ks_n;
    m = rest / n_blocks;
    nb = rest - m * n_blocks;
    kb_lo = ks * nk / ks_n;
    kb_hi = (ks + 1) * nk / ks_n;
  };

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer + tile scheduler ----------------
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int q = i % TQ;
      if (!mbar_wait(tq_empty_bar(q), ((i / TQ) & 1) ^ 1u, wc, SITE_TC_PRODUCER)) {
        ok = false;
        break;
      }
      int tile = (int)atomicAdd(g.sched, 1u);
      if (tile >= total) tile = -1;
      tile_q[q] = tile;
      mbar_arrive(tq_full_bar(q));
      if (tile < 0) break;
      int ph, m, nb, kb_lo, kb_hi;
      decode_tile(tile, ph, m, nb, kb_lo, kb_hi);
      const TcArgs& a = ph ? g2 : g;
      const CUtensorMap* mact = ph ? &map_act2 : &map_act;
      const CUtensorMap* mw = ph ? &map_w2 : &map_w;
      const int4 ent = tile_entry_of(a, m);
      if (ph && !wait_ready(g.ready, m, g2.ready_need, wc)) {
        ok = false;
        break;
      }
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc, SITE_TC_PRODUCER)) {
          ok = false;
          break;
        }
        const uint32_t sa = base + stage * S::STAGE_BYTES, sb = sa + S::A_BYTES;
        const int ka = a.a_kwrap ? (kb * BK) % a.a_kwrap : kb * BK;
        mbar_arrive_expect_tx(full_bar(stage), S::STAGE_BYTES);
        if (!SWAP) {
          tma_load_2d(sa, mact, full_bar(stage), ka, ent.y);
          tma_load_3d(sb, mw, full_bar(stage), kb * BK, nb * NT, ent.x);
        } else {
          tma_load_3d(sa, mw, full_bar(stage), kb * BK, nb * M, ent.x);
          tma_load_2d(sb, mact, full_bar(stage), ka, a.row_token ? 0 : ent.y);
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      // let the copies already issued land before the CTA exits
      const long first = issued > STAGES ? issued - STAGES : 0;
      for (long i = first; i < issued; ++i)
        mbar_drain(full_bar((int)(i % STAGES)), (uint32_t)((i / STAGES) & 1), g.timeout_ns,
                   g.status);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true, any = false;
    for (int i = 0; ok; ++i) {
      const int q = i % TQ;
      if (!mbar_wait(tq_full_bar(q), (i / TQ) & 1, wc, SITE_TC_MMA)) {
        ok = false;
        break;
      }
      const int tile = tile_q[q];
      mbar_arrive(tq_empty_bar(q));
      if (tile < 0) break;
      int ph, m, nb, kb_lo, kb_hi;
      decode_tile(tile, ph, m, nb, kb_lo, kb_hi);
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      if (!mbar_wait(tempty_bar(acc), aph ^ 1u, wc, SITE_TC_MMA)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int n_mma = SWAP ? NT : min(NT, (ph ? g2 : g).N - nb * NT);
      const uint32_t idesc = make_idesc_bf16(M, n_mma);
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * S::ACC_COLS);
      (void)m;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(full_bar(stage), phase, wc, SITE_TC_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = base + stage * S::STAGE_BYTES, sb = sa + S::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / UMMA_K; ++kk) {
          umma_bf16(d_tmem, make_sdesc_sw128(sa + kk * UMMA_K * 2),
                    make_sdesc_sw128(sb + kk * UMMA_K * 2), idesc, (kb != kb_lo) | kk);
        }
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
      // all MMAs issued so far must finish before tensor memory is released
      umma_commit(drain_bar);
      mbar_drain(drain_bar, 0, g.timeout_ns, g.status);
    }
  } else if (warp >= 2) {
    // ---------------- epilogue: 4 warps, one TMEM lane quarter each ----------------
    const int q = warp & 3;
    int it = 0;
    for (int i = 0;; ++i) {
      int tile = -1;
      int ok = 1;
      if (lane == 0) {
        const int slot = i % TQ;
        ok = mbar_wait(tq_full_bar(slot), (i / TQ) & 1, wc, SITE_TC_EPILOGUE) ? 1 : 0;
        if (ok) {
          tile = tile_q[slot];
          mbar_arrive(tq_empty_bar(slot));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (!ok || tile < 0) break;
      int ph, m, nb, kb_lo, kb_hi;
      decode_tile(tile, ph, m, nb, kb_lo, kb_hi);
      const TcArgs& a = ph ? g2 : g;
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      if (lane == 0) ok = mbar_wait(tfull_bar(acc), aph, wc, SITE_TC_EPILOGUE) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int4 ent = tile_entry_of(a, m);
      const uint32_t tq = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * S::ACC_COLS);
      if (!SWAP) {
        const int row = q * 32 + lane;
        const bool valid = row < ent.z;
        const int n0 = nb * NT;
        const int n_eff = min(NT, a.N - n0);
        for (int c = 0; c < n_eff; c += 32) {
          float v[32];
          tmem_ld_x32(tq + (uint32_t)c, v);
          if (valid) epi_row32(a, ent.y + row, n0 + c, v);
        }
      } else {
        const int f = nb * M + q * 32 + lane;
        const bool valid = f < a.N;
#pragma unroll
        for (int c = 0; c < NT; c += 16) {
          float v[16];
          tmem_ld_x16(tq + (uint32_t)c, v);
          if (a.row_token) {
            // accumulator columns are tokens: row r of the expert takes column row_token[r]
            for (int j = 0; j < ent.z; ++j) {
              const int t = a.row_token[ent.y + j] - c;
              if (t < 0 || t >= 16) continue;
              float val = 0.f;
#pragma unroll
              for (int u = 0; u < 16; ++u) val = (u == t) ? v[u] : val;
              if (valid) epi_elem(a, ent.y + j, f, val);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (valid && c + j < ent.z) epi_elem(a, ent.y + c + j, f, v[j]);
          }
        }
      }
      if (fused && ph == 0) {
        // this warp's rows of the tile are stored: count them for the second GEMM
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(g.ready + m, 1);
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      ++it;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
  if (threadIdx.x == 0) {
    // the last CTA to finish resets the scheduler (and a fused launch's ready
    // counters) for the next launch
    __threadfence();
    if (atomicAdd(g.sched + 1, 1u) == gridDim.x - 1) {
      atomicExch(g.sched, 0u);
      atomicExch(g.sched + 1, 0u);
      if (fused)
        for (int i = 0; i < num_m; ++i) g.ready[i] = 0;
    }
  }
}

}  // namespace tc
}  // namespace nh

// gemm_q4.cuh -- expert GEMM with NVFP4 weights (W4A16, group size 16) on the
// sm_100a tensor cores, weights on the MMA M side; used for tile entries of 64
// tokens (tiles of at most 32 tokens go to the register GEMV of gemv_q4.cuh).
//
// Weight storage (vllm.cpp PR #518 names it for the checkpoint's routed and
// shared experts): every weight is an E2M1 code times an E4M3 scale shared by
// 16 consecutive input features, times a float32 scale per matrix;
// activations stay bf16.
//
// Data path of one 128-row weight tile (weights on the MMA M side, tokens on N):
//   HBM --TMA--> shared memory: 4-bit codes (128-byte swizzle), scale bytes
//                and the bf16 activation tiles, 256 input features per stage;
//   shared memory --dequantize warps--> tensor memory: bf16 weights written
//                with tcgen05.st straight into the MMA's A operand;
//   tcgen05.mma kind::f16 with A in tensor memory, B (activations) in shared
//                memory, f32 accumulator in tensor memory;
//   epilogue:    the float32 matrix scale, then the relu^2 / weighted store.
// The dequantized weights never pass through shared memory, so its traffic
// per weight is the half byte of the code; HBM sees only the NVFP4 bytes.
//
// Exact dequantization without the conversion pipe: an E2M1 code s.e1e0.m
// placed at bf16 bits 15 and 8..6 reads as the bf16 number code * 2^-126
// (code 0.5 becomes the subnormal 2^-127, the others normal numbers), so one
// bf16 multiply by scale * 2^118 gives code * scale * 2^-8 exactly (at most
// six significant bits, inside the normal range).  The epilogue multiplies
// by global * 2^8.
//
// Roles (704 threads): warp 0 lane 0 TMA producer + tile scheduler; warp 1
// tensor memory owner and MMA issuer; warps 2..5 epilogue (TMEM lane quarter
// warp % 4); warps 6..21 dequantize, in two groups of eight that take
// alternate 128-feature A tiles (thread = 64 weights of one row).
#pragma once

#include "gemm_tc.cuh"

namespace nh {
namespace q4 {

constexpr int BK = 128;             // input features of one A tile in tensor memory
constexpr int RK = 2 * BK;          // input features of one TMA stage
constexpr int SUB_TILES = RK / 64;  // 64-feature activation tiles per stage
constexpr int UMMA_K = 16;
constexpr int M = 128;              // weight rows per tile
constexpr int GROUPS = 2;           // dequantize groups (8 warps each), alternate A tiles
constexpr int DQ_WARPS = 8 * GROUPS;
constexpr int THREADS = (6 + DQ_WARPS) * 32;
constexpr int CODE_ROW = RK / 2;            // 128 bytes of codes per row and stage
constexpr int CODE_BYTES = M * CODE_ROW;    // 16 KB
constexpr int SCALE_BOX = RK / 16;          // 16 scale bytes per row and stage
constexpr int SCALE_BYTES = M * SCALE_BOX;  // 2 KB
constexpr int DQ = 2 * GROUPS;              // A tiles in tensor memory
constexpr int A_COLS = BK / 2;              // 64 columns (two bf16 per column)
constexpr int A_COL0 = 128;                 // accumulators use columns [0, 2 NT)
constexpr int TMEM_COLS = 512;
constexpr float DQ_UNSCALE = 256.0f;        // undoes the 2^-8 of the dequantized weights

template <int NT, int RAW>
struct Shape {
  static constexpr int ACT_SUB = NT * 64 * 2;
  static constexpr int RAW_BYTES = CODE_BYTES + SUB_TILES * ACT_SUB + SCALE_BYTES;
  static constexpr int RAW_STRIDE = (RAW_BYTES + 1023) / 1024 * 1024;
  static constexpr int NBAR = 2 * RAW + 2 * DQ + 5 + 2 * tc::TQ;
  static constexpr int SMEM = RAW * RAW_STRIDE + 1024 + NBAR * 8 + 16 + 4 * tc::TQ + 4 * RAW;
  static_assert(2 * NT <= A_COL0, "accumulators overlap the A tiles");
  static_assert(A_COL0 + DQ * A_COLS <= TMEM_COLS, "tensor memory");
  static_assert(ACT_SUB % 1024 == 0, "activation tiles must stay 1024-byte aligned");
  static_assert(SMEM <= 232448, "shared memory");
};

struct Q4Args {
  tc::TcArgs g;          // tiles, N, K, epilogue, status, scheduler (as the bf16 kernel)
  const float* gscale;   // float32 scale of each weight matrix [n_mat]
};

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (bf16 inputs, f32 accumulate)
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive columns from registers (one row per thread), then
// wait until the stores are complete
__device__ __forceinline__ void tmem_st_x32_wait(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Two E4M3 scale bytes (low byte first) -> two bf16x2 multipliers, each holding
// its scale * 2^118 in both halves (exact): one conversion for both bytes, the
// same arithmetic as scale_mult byte by byte.
__device__ __forceinline__ void scale_mult2(uint32_t two, uint32_t* m) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)two));
  const float s0 = __half2float(__ushort_as_half((uint16_t)(h & 0xffffu))) * 0x1p118f;
  const float s1 = __half2float(__ushort_as_half((uint16_t)(h >> 16))) * 0x1p118f;
  m[0] = pack_bf16x2(s0, s0);
  m[1] = pack_bf16x2(s1, s1);
}

// E4M3 scale byte -> bf16x2 holding scale * 2^118 in both halves (exact)
__device__ __forceinline__ uint32_t scale_mult(uint32_t byte) {
  uint32_t h;
  const uint16_t b2 = (uint16_t)(byte | (byte << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(b2));
  const float s = __half2float(__ushort_as_half((uint16_t)(h & 0xffffu))) * 0x1p118f;
  return pack_bf16x2(s, s);
}

// The four weight pairs of code word w (byte j holds columns 2j and 2j + 1,
// the even column in the low nibble) times the scale multiplier: bf16x2 each,
// value code * scale * 2^-8.
__device__ __forceinline__ void dq_word(uint32_t w, uint32_t mult, uint32_t* o) {
  const uint32_t lo = w & 0x0F0F0F0Fu;          // even columns, one code per byte
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;   // odd columns
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    // p = [lo byte k, 0, hi byte k, 0]: selector 0xF copies the sign bit of
    // hi byte 3, which is 0.  p * (2^6 + 2^12) puts each code at bits 9..6
    // and a copy at 15..12 without carries; the mask keeps the magnitude from
    // the first copy and the sign from the second.
    uint32_t p;
    asm("prmt.b32 %0, %1, %2, %3;"
        : "=r"(p)
        : "r"(lo), "r"(hi), "r"((uint32_t)(k | 0xF0 | ((4 + k) << 8) | 0xF000)));
    const uint32_t bits = (p * 4160u) & 0x81C081C0u;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(o[k]) : "r"(bits), "r"(mult));
  }
}

template <int NT, int RAW>
__global__ void __launch_bounds__(THREADS, 1)
    tc_q4_gemm(const __grid_constant__ CUtensorMap map_act,
               const __grid_constant__ CUtensorMap map_codes,
               const __grid_constant__ CUtensorMap map_scales, const Q4Args qa) {
  using S = Shape<NT, RAW>;
  const tc::TcArgs& g = qa.g;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw0 = smem_u32(smem_raw);
  const uint32_t base = (raw0 + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw0);
  // stage r: [codes 16 KB, 128-byte swizzle][activation tiles][scale bytes]
  auto code_tile = [&](int r) { return base + r * S::RAW_STRIDE; };
  auto act_tile = [&](int r, int sub) { return code_tile(r) + CODE_BYTES + sub * S::ACT_SUB; };
  auto scale_tile = [&](int r) { return code_tile(r) + CODE_BYTES + SUB_TILES * S::ACT_SUB; };
  const uint32_t bar0 = base + RAW * S::RAW_STRIDE;
  auto raw_full = [&](int r) { return bar0 + 8u * r; };
  auto raw_empty = [&](int r) { return bar0 + 8u * (RAW + r); };
  auto dq_full = [&](int d) { return bar0 + 8u * (2 * RAW + d); };
  auto dq_empty = [&](int d) { return bar0 + 8u * (2 * RAW + DQ + d); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * RAW + 2 * DQ + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * RAW + 2 * DQ + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * RAW + 2 * DQ + 4);
  auto tq_full_bar = [&](int i) { return bar0 + 8u * (2 * RAW + 2 * DQ + 5 + i); };
  auto tq_empty_bar = [&](int i) { return bar0 + 8u * (2 * RAW + 2 * DQ + 5 + tc::TQ + i); };
  uint32_t* const tmem_slot =
      reinterpret_cast<uint32_t*>(base_ptr + RAW * S::RAW_STRIDE + S::NBAR * 8);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* const tile_q = reinterpret_cast<volatile int*>(tmem_slot + 4);
  // A tiles in each stage (1 or 2; 0 marks the end of the work)
  volatile int* const raw_nd = reinterpret_cast<volatile int*>(tmem_slot + 4 + tc::TQ);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int r = 0; r < RAW; ++r) {
      mbar_init(raw_full(r), 1);
      mbar_init(raw_empty(r), DQ_WARPS + 1);   // every dequantize warp + the MMAs
    }
    for (int d = 0; d < DQ; ++d) {
      mbar_init(dq_full(d), 8);                // the eight warps of one group
      mbar_init(dq_empty(d), 1);
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
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
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
  const int nd_tile = (g.K + BK - 1) / BK;         // A tiles per weight tile
  const int nraw = (nd_tile + 1) / 2;              // TMA stages per weight tile

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer + tile scheduler ----------------
    int r = 0;
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
      for (int kr = 0; kr < nraw; ++kr) {
        if (!mbar_wait(raw_empty(r), phase ^ 1u, wc, SITE_TC_PRODUCER)) {
          ok = false;
          break;
        }
        const int nd = min(2, nd_tile - 2 * kr);
        const int nsub = min(SUB_TILES, (g.K - kr * RK) / 64);
        raw_nd[r] = nd;
        mbar_arrive_expect_tx(raw_full(r), CODE_BYTES + SCALE_BYTES + nsub * S::ACT_SUB);
        tma_load_3d(code_tile(r), &map_codes, raw_full(r), kr * CODE_ROW, nb * M, ent.x);
        tma_load_3d(scale_tile(r), &map_scales, raw_full(r), kr * SCALE_BOX, nb * M, ent.x);
        for (int sub = 0; sub < nsub; ++sub)
          tma_load_2d(act_tile(r, sub), &map_act, raw_full(r), kr * RK + sub * 64,
                      g.row_token ? 0 : ent.y);
        ++issued;
        if (++r == RAW) {
          r = 0;
          phase ^= 1u;
        }
      }
    }
    if (ok && mbar_wait(raw_empty(r), phase ^ 1u, wc, SITE_TC_PRODUCER)) {
      // end marker for the dequantize warps: a stage with no copies
      raw_nd[r] = 0;
      mbar_arrive(raw_full(r));
    } else {
      const long first = issued > RAW ? issued - RAW : 0;
      for (long i = first; i < issued; ++i)
        tc::mbar_drain(raw_full((int)(i % RAW)), (uint32_t)((i / RAW) & 1), g.timeout_ns,
                       g.status);
    }
  } else if (warp >= 6) {
    // ---------------- dequantize: codes (smem) -> bf16 A tiles (tmem) ----------------
    const int dw = warp - 6;
    const int group = dw >> 3;               // takes A tiles j with j % GROUPS == group
    const int khalf = (dw >> 2) & 1;         // features [64 khalf, 64 khalf + 64) of a tile
    const int quarter = warp & 3;            // the TMEM lanes this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16);
    int r = 0;
    uint32_t rphase = 0;
    long j = 0;                              // A tile sequence number
    bool ok = true;
    while (ok) {
      int st = 1;
      if (lane == 0) st = mbar_wait(raw_full(r), rphase, wc, SITE_TC_EPILOGUE) ? 1 : 0;
      st = __shfl_sync(0xffffffffu, st, 0);
      if (!st) break;
      const int nd = raw_nd[r];
      if (nd == 0) break;                    // end marker
      for (int t = 0; t < nd; ++t, ++j) {
        if ((int)(j % GROUPS) != group) continue;
        const int d = (int)(j % DQ);
        const uint32_t dph = (uint32_t)((j / DQ) & 1);
        if (lane == 0) st = mbar_wait(dq_empty(d), dph ^ 1u, wc, SITE_TC_EPILOGUE) ? 1 : 0;
        st = __shfl_sync(0xffffffffu, st, 0);
        if (!st) {
          ok = false;
          break;
        }
        tc_fence_after();
        // 32 code bytes = 16-byte chunks c, c + 1 of the row (128-byte swizzle)
        const int c = t * 4 + khalf * 2;
        const uint8_t* crow = base_ptr + (code_tile(r) - base) + row * CODE_ROW;
        const uint4 c0 = *reinterpret_cast<const uint4*>(crow + ((c ^ (row & 7)) << 4));
        const uint4 c1 = *reinterpret_cast<const uint4*>(crow + (((c + 1) ^ (row & 7)) << 4));
        const uint32_t sc = *reinterpret_cast<const uint32_t*>(
            base_ptr + (scale_tile(r) - base) + row * SCALE_BOX + t * 8 + khalf * 4);
        uint32_t o[32];
        {
          const uint32_t m0 = scale_mult(sc & 0xffu), m1 = scale_mult((sc >> 8) & 0xffu);
          const uint32_t m2 = scale_mult((sc >> 16) & 0xffu), m3 = scale_mult(sc >> 24);
          dq_word(c0.x, m0, o + 0);
          dq_word(c0.y, m0, o + 4);
          dq_word(c0.z, m1, o + 8);
          dq_word(c0.w, m1, o + 12);
          dq_word(c1.x, m2, o + 16);
          dq_word(c1.y, m2, o + 20);
          dq_word(c1.z, m3, o + 24);
          dq_word(c1.w, m3, o + 28);
        }
        tmem_st_x32_wait(t_row + (uint32_t)(A_COL0 + d * A_COLS + khalf * 32), o);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_full(d));
      }
      if (!ok) break;
      // this warp is done with the stage's codes and scales
      __syncwarp();
      if (lane == 0) mbar_arrive(raw_empty(r));
      if (++r == RAW) {
        r = 0;
        rphase ^= 1u;
      }
      if (*abort_flag) ok = false;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    int r = 0;
    uint32_t rphase = 0;
    long j = 0;
    int it = 0;
    bool ok = true, any = false;
    const uint32_t idesc = make_idesc_bf16(M, NT);
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
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * NT);
      for (int kr = 0; kr < nraw && ok; ++kr) {
        if (!mbar_wait(raw_full(r), rphase, wc, SITE_TC_MMA)) {
          ok = false;
          break;
        }
        const int nd = min(2, nd_tile - 2 * kr);
        for (int t = 0; t < nd; ++t, ++j) {
          const int d = (int)(j % DQ);
          if (!mbar_wait(dq_full(d), (uint32_t)((j / DQ) & 1), wc, SITE_TC_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int kd = 2 * kr + t;
          const int nsteps = min(BK, g.K - kd * BK) / UMMA_K;
          const uint32_t a_tmem = tmem_base + (uint32_t)(A_COL0 + d * A_COLS);
          for (int kk = 0; kk < nsteps; ++kk)
            umma_bf16_ta(d_tmem, a_tmem + (uint32_t)(kk * (UMMA_K / 2)),
                         make_sdesc_sw128(act_tile(r, t * 2 + (kk >> 2)) + (kk & 3) * UMMA_K * 2),
                         idesc, (kd | kk) != 0);
          any = true;
          umma_commit(dq_empty(d));
        }
        if (!ok) break;
        umma_commit(raw_empty(r));    // the stage's activations are consumed
        if (++r == RAW) {
          r = 0;
          rphase ^= 1u;
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
      const float gs = qa.gscale[ent.x] * DQ_UNSCALE;
      const uint32_t tq = tmem_base + ((uint32_t)(qd * 32) << 16) + (uint32_t)(acc * NT);
      const int f = nb * M + qd * 32 + lane;
      const bool valid = f < g.N;
#pragma unroll
      for (int c = 0; c < NT; c += 16) {
        float v[16];
        tmem_ld_x16(tq + (uint32_t)c, v);
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] *= gs;
        if (g.row_token) {
          for (int jj = 0; jj < ent.z; ++jj) {
            const int tt = g.row_token[ent.y + jj] - c;
            if (tt < 0 || tt >= 16) continue;
            float val = 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) val = (u == tt) ? v[u] : val;
            if (valid) tc::epi_elem(g, ent.y + jj, f, val);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 16; ++u)
            if (valid && c + u < ent.z) tc::epi_elem(g, ent.y + c + u, f, v[u]);
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
    tmem_dealloc(tmem_base, TMEM_COLS);
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

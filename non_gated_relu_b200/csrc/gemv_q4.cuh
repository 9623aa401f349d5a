// gemv_q4.cuh -- NVFP4 expert GEMM for decode-sized tiles (at most 32 tokens
// per expert) with warp-level MMAs fed straight from registers.
//
// With one or two tokens per expert a 128-row tcgen05.mma pays a fixed cost per
// 128 x 16 block of weights whatever N is (about 90 SM cycles, measured), which
// caps the tensor-memory kernel (gemm_q4.cuh) near a quarter of HBM speed.
// Here each warp owns 16 weight rows of one tile entry (one warp task): it
// loads the rows' 4-bit codes with 16-byte global loads, turns them into bf16 in registers
// (the exact bit construction of gemm_q4.cuh: code * scale * 2^-8) and issues
// mma.sync m16n8k16 (bf16 in, f32 accumulate) with the tokens on N = 8; the
// float32 matrix scale * 2^8 is applied in the epilogue.  Nothing goes
// through shared or tensor memory.
//
// Feature order inside the MMA.  The MMA sums over its 16 k slots in any
// order, so weights and activations may use one common permutation of the
// features.  In a block of BK (128, or a 64-feature tail) features, k-tile kt
// (of BK/16), slot kappa = 8h + 2 tq + p (tq = lane % 4, h, p in {0, 1}) holds
// feature (BK/4) tq + 4 kt + 2h + p.  Thread tq's features are then the
// contiguous run [(BK/4) tq, (BK/4)(tq + 1)) -- BK/8 bytes of codes per row,
// one 16-byte (or 8-byte) load -- and its activation values come four
// consecutive bf16 at a time.  The permutation is a bijection of the block,
// so every product is summed exactly once.
#pragma once

#include "gemm_q4.cuh"

namespace nh {
namespace q4v {

constexpr int WARPS = 8;   // per CTA
constexpr int MT = 16;     // weight rows per warp task

struct Args {
  tc::TcArgs g;            // tiles / dense rows, N, K, epilogue, out, perm_w, row_token, status
  const void* A;           // activations [*, K] bf16 (x, x_perm, h)
  const uint8_t* codes;    // [n_mat, N, K / 2]
  const uint8_t* scales;   // [n_mat, N, pitch]
  const float* gscale;     // [n_mat]
  int pitch;               // scale bytes per row
};

__device__ __forceinline__ void mma_bf16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One block of BK features for one n-tile (8 tokens): codes of rows gq (ca)
// and gq + 8 (cb) of this thread's run (BK/8 bytes = BK/32 words each), the
// scale multipliers of the run's groups, and the activation row of token gq.
// Word w of the run holds k-tiles 2w and 2w + 1; even and odd k-tiles go to
// two accumulators (c0, c1) so consecutive MMAs do not wait on each other.
// Activation loads: through the read-only path, or (`coherent`) from L2 for
// activations that an earlier part of the same launch wrote.
__device__ __forceinline__ uint2 ld_act2(const __nv_bfloat16* p, bool coherent) {
  if (!coherent) return __ldg(reinterpret_cast<const uint2*>(p));
  uint2 v;
  asm volatile("ld.global.cg.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ld_act4(const __nv_bfloat16* p, bool coherent) {
  if (!coherent) return __ldg(reinterpret_cast<const uint4*>(p));
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <int BK>
__device__ __forceinline__ void block_mma(const uint32_t* ca, const uint32_t* cb,
                                          const uint32_t* ma, const uint32_t* mb,
                                          const __nv_bfloat16* act, float* c0, float* c1,
                                          bool coherent = false) {
  constexpr int KT = BK / 16;
  uint2 bv[KT];
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) bv[kt] = ld_act2(act + 4 * kt, coherent);
#pragma unroll
  for (int w = 0; w < KT / 2; ++w) {
    uint32_t pa[4], pb[4];
    // a 16-feature scale group is 8 bytes = 2 words of the run
    q4::dq_word(ca[w], ma[w / 2], pa);
    q4::dq_word(cb[w], mb[w / 2], pb);
    // k-tile kt: slots 2tq + {0,1} = byte 2kt, slots 2tq + 8 + {0,1} = byte 2kt + 1
    mma_bf16_16816(c0, pa[0], pb[0], pa[1], pb[1], bv[2 * w].x, bv[2 * w].y);
    mma_bf16_16816(c1, pa[2], pb[2], pa[3], pb[3], bv[2 * w + 1].x, bv[2 * w + 1].y);
  }
}

// Few tasks (dense rows: the shared expert, the latent projections).
// block_mma with the activation run already in registers: run features
// 8u .. 8u + 7 in bv[u] (.x: 8u + {0,1}, .y: {2,3}, .z: {4,5}, .w: {6,7}).
__device__ __forceinline__ void block_mma_b(const uint32_t* ca, const uint32_t* cb,
                                            const uint32_t* ma, const uint32_t* mb,
                                            const uint4* bv, float* c0, float* c1) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t pa[4], pb[4];
    q4::dq_word(ca[w], ma[w / 2], pa);
    q4::dq_word(cb[w], mb[w / 2], pb);
    // word w = k-tiles 2w (features 8w + 0..3) and 2w + 1 (8w + 4..7)
    mma_bf16_16816(c0, pa[0], pb[0], pa[1], pb[1], bv[w].x, bv[w].y);
    mma_bf16_16816(c1, pa[2], pb[2], pa[3], pb[3], bv[w].z, bv[w].w);
  }
}

// NT: tokens per tile entry (16 or 32).  A CTA task is (tile entry, 16 weight
// rows); its 8 warps split the 128-feature blocks of K round-robin (the
// 64-feature tail goes to the next warp in turn) and their partial tiles are
// added through shared memory in warp order (deterministic), then warp 0
// applies the epilogue.  An entry with more than 8 tokens takes one pass per
// 8 tokens.  Tasks are dealt round-robin over the grid.
template <int NT>
__global__ void __launch_bounds__(WARPS * 32, 3) q4_gemv_splitk(const Args a) {
  __shared__ float red[WARPS][32][4];
  const tc::TcArgs& g = a.g;
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int num_m = g.tiles ? *g.num_tiles : (g.dense_rows + g.tile_rows - 1) / g.tile_rows;
  const int n_rb = g.N / MT;                        // N is a multiple of 64
  const int total = num_m * n_rb;
  const int K = g.K;
  const int nkb = K / 128, tail = K % 128;          // tail: 0 or 64 (K is a multiple of 64)
  const size_t row_bytes = (size_t)K / 2;
  const __nv_bfloat16* A = static_cast<const __nv_bfloat16*>(a.A);
  for (int task = blockIdx.x; task < total; task += gridDim.x) {
    const int m = task / n_rb, rb = task - m * n_rb;
    const int r0 = rb * MT;
    const int4 ent = tc::tile_entry_of(g, m);
    const int count = ent.z;
    const size_t wrow_a = (size_t)ent.x * g.N + r0 + gq;   // rows gq and gq + 8
    const uint8_t* ca_p = a.codes + wrow_a * row_bytes;
    const uint8_t* cb_p = ca_p + 8 * row_bytes;
    const uint8_t* sa_p = a.scales + wrow_a * a.pitch;
    const uint8_t* sb_p = sa_p + 8 * (size_t)a.pitch;
    for (int n0 = 0; n0 < count; n0 += 8) {
      // activation row of token n0 + gq (rows past count re-read the last
      // token; their columns are never stored)
      const int j = min(n0 + gq, count - 1);
      const int arow = g.row_token ? g.row_token[ent.y + j] : ent.y + j;
      const __nv_bfloat16* act = A + (size_t)arow * K;
      float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
      // the warp's blocks kb, kb + WARPS, ...: the next one's codes are in flight
      // while one is used, in two register sets taken in turn (no copies)
      int kb = warp;
      uint4 qa = make_uint4(0, 0, 0, 0), qb = qa, qa2 = qa, qb2 = qa;
      auto load = [&](int k, uint4& fa, uint4& fb) {
        fa = __ldg(reinterpret_cast<const uint4*>(ca_p + (size_t)k * 64 + 16 * tq));
        fb = __ldg(reinterpret_cast<const uint4*>(cb_p + (size_t)k * 64 + 16 * tq));
      };
      auto use = [&](int k, const uint4& fa, const uint4& fb) {
        // thread tq's 32 features are scale groups 8 k + 2 tq and + 1
        const uint32_t sa2 = *reinterpret_cast<const uint16_t*>(sa_p + k * 8 + 2 * tq);
        const uint32_t sb2 = *reinterpret_cast<const uint16_t*>(sb_p + k * 8 + 2 * tq);
        uint32_t ma[2], mb[2];
        q4::scale_mult2(sa2, ma);
        q4::scale_mult2(sb2, mb);
        const uint32_t cwa[4] = {fa.x, fa.y, fa.z, fa.w}, cwb[4] = {fb.x, fb.y, fb.z, fb.w};
        block_mma<128>(cwa, cwb, ma, mb, act + k * 128 + 32 * tq, c0, c1);
      };
      if (kb < nkb) load(kb, qa, qb);
      for (; kb < nkb; kb += 2 * WARPS) {
        if (kb + WARPS < nkb) load(kb + WARPS, qa2, qb2);
        use(kb, qa, qb);
        if (kb + WARPS < nkb) {
          if (kb + 2 * WARPS < nkb) load(kb + 2 * WARPS, qa, qb);
          use(kb + WARPS, qa2, qb2);
        }
      }
      if (tail && warp == nkb % WARPS) {
        // 64-feature tail: thread tq's run is features [16 tq, 16 tq + 16), one group
        const size_t off = (size_t)nkb * 64 + 8 * tq;
        const uint2 ta = __ldg(reinterpret_cast<const uint2*>(ca_p + off));
        const uint2 tb = __ldg(reinterpret_cast<const uint2*>(cb_p + off));
        const uint32_t ma[1] = {q4::scale_mult(sa_p[nkb * 8 + tq])};
        const uint32_t mb[1] = {q4::scale_mult(sb_p[nkb * 8 + tq])};
        const uint32_t cwa[2] = {ta.x, ta.y}, cwb[2] = {tb.x, tb.y};
        block_mma<64>(cwa, cwb, ma, mb, act + nkb * 128 + 16 * tq, c0, c1);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp][lane][i] = c0[i] + c1[i];
      __syncthreads();
      if (warp == 0) {
        // c: rows (gq, gq + 8) x tokens (n0 + 2 tq, n0 + 2 tq + 1)
        const float gs = a.gscale[ent.x] * q4::DQ_UNSCALE;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < WARPS; ++w) v += red[w][lane][i];
          const int jj = n0 + 2 * tq + (i & 1);
          const int f = r0 + gq + (i >> 1) * 8;
          if (jj < count) tc::epi_elem(g, ent.y + jj, f, v * gs);
        }
      }
      __syncthreads();
    }
  }
}

// Wait until every up-projection warp task of tile entry m has counted itself
// (a fused launch); false if the launch's status word already holds an error
// or the wait runs out (then it records NH_ERR_TIMEOUT).
__device__ __forceinline__ bool wait_entry_ready(const int* ready, int m, int need, int* status,
                                                 uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 0;; ++i) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ready + m) : "memory");
    if (v >= need) return true;
    if ((i & 63u) == 63u) {
      if (status && *reinterpret_cast<volatile int*>(status) != 0) return false;
      if (globaltimer_ns() - t0 > timeout_ns) {
        record_status(status, NH_ERR_TIMEOUT, SITE_GEMV_STAGE, m);
        return false;
      }
    }
  }
}

// Many tasks (the routed experts).  Warp tasks (tile entry, 16 weight rows)
// are dealt round-robin over all warps of the grid; each warp runs the whole
// K with the next block's codes, scale bytes and activation run in flight.  An entry with more than 8 tokens
// takes one pass per 8 tokens (the codes are re-read from L1/L2).
//
// With a2.g.N > 0 the launch also runs a second GEMM over the same tile
// entries whose activations are the first one's output (the decode up and
// down projections): warps then fetch tasks from a counter (a.g.sched), all
// of the first GEMM's before any of the second's; a warp that finishes an up
// task counts it into a.g.ready[m], and a down task of entry m first waits
// for a2.g.ready_need counts (the up tasks it waits on were handed out
// earlier, to running warps, and wait on nothing) and reads h from L2.
template <int NT>
__global__ void __launch_bounds__(WARPS * 32, 2) q4_gemv_rows(const Args a1, const Args a2) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const bool fused = a2.g.N > 0;
  const int num_m =
      a1.g.tiles ? *a1.g.num_tiles : (a1.g.dense_rows + a1.g.tile_rows - 1) / a1.g.tile_rows;
  const int total1 = num_m * (a1.g.N / MT);
  const int total = total1 + (fused ? num_m * (a2.g.N / MT) : 0);
  const int nwarps = gridDim.x * WARPS;
  int task = fused ? 0 : blockIdx.x * WARPS + (threadIdx.x >> 5);
  for (;; task += nwarps) {
    if (fused) {
      int t = 0;
      if (lane == 0) t = (int)atomicAdd(a1.g.sched, 1u);
      task = __shfl_sync(0xffffffffu, t, 0);
    }
    if (task >= total) break;
    const bool second = task >= total1;
    const Args& a = second ? a2 : a1;
    const tc::TcArgs& g = a.g;
    const int t = second ? task - total1 : task;
    const int n_rb = g.N / MT;
    const int m = t / n_rb, rb = t - m * n_rb;
    if (second) {
      int ok = 1;
      if (lane == 0)
        ok = wait_entry_ready(a1.g.ready, m, a2.g.ready_need, g.status, g.timeout_ns) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
    }
    const int K = g.K;
    const int nkb = K / 128, tail = K % 128;
    const size_t row_bytes = (size_t)K / 2;
    const __nv_bfloat16* A = static_cast<const __nv_bfloat16*>(a.A);
    const int r0 = rb * MT;
    const int4 ent = tc::tile_entry_of(g, m);
    const int count = ent.z;
    const size_t wrow_a = (size_t)ent.x * g.N + r0 + gq;
    const uint8_t* ca_p = a.codes + wrow_a * row_bytes;
    const uint8_t* cb_p = ca_p + 8 * row_bytes;
    const uint8_t* sa_p = a.scales + wrow_a * a.pitch;
    const uint8_t* sb_p = sa_p + 8 * (size_t)a.pitch;
    const float gs = a.gscale[ent.x] * q4::DQ_UNSCALE;
    for (int n0 = 0; n0 < count; n0 += 8) {
      const int j = min(n0 + gq, count - 1);
      const int arow = g.row_token ? g.row_token[ent.y + j] : ent.y + j;
      const __nv_bfloat16* act = A + (size_t)arow * K;
      float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
      // block kb's codes, scale bytes and activation run, loaded one block ahead
      uint4 qa = make_uint4(0, 0, 0, 0), qb = qa, xb[4] = {qa, qa, qa, qa};
      uint32_t sa2 = 0, sb2 = 0;
      auto fetch = [&](int kb, uint4& fa, uint4& fb, uint4* fx, uint32_t& fsa, uint32_t& fsb) {
        fa = __ldg(reinterpret_cast<const uint4*>(ca_p + (size_t)kb * 64 + 16 * tq));
        fb = __ldg(reinterpret_cast<const uint4*>(cb_p + (size_t)kb * 64 + 16 * tq));
        const __nv_bfloat16* xr = act + kb * 128 + 32 * tq;
#pragma unroll
        for (int u = 0; u < 4; ++u) fx[u] = ld_act4(xr + 8 * u, second);
        // thread tq's 32 features are scale groups 8 kb + 2 tq and + 1
        fsa = *reinterpret_cast<const uint16_t*>(sa_p + kb * 8 + 2 * tq);
        fsb = *reinterpret_cast<const uint16_t*>(sb_p + kb * 8 + 2 * tq);
      };
      // two register sets used in turn (blocks kb and kb + 1): no copies between them
      uint4 qa2 = qa, qb2 = qb, xb2[4] = {qa, qa, qa, qa};
      uint32_t sa2b = 0, sb2b = 0;
      auto use = [&](const uint4& fa, const uint4& fb, const uint4* fx, uint32_t fsa, uint32_t fsb) {
        uint32_t ma[2], mb[2];
        q4::scale_mult2(fsa, ma);
        q4::scale_mult2(fsb, mb);
        const uint32_t cwa[4] = {fa.x, fa.y, fa.z, fa.w}, cwb[4] = {fb.x, fb.y, fb.z, fb.w};
        block_mma_b(cwa, cwb, ma, mb, fx, c0, c1);
      };
      if (nkb > 0) fetch(0, qa, qb, xb, sa2, sb2);
      for (int kb = 0; kb < nkb; kb += 2) {
        if (kb + 1 < nkb) fetch(kb + 1, qa2, qb2, xb2, sa2b, sb2b);
        use(qa, qb, xb, sa2, sb2);
        if (kb + 1 < nkb) {
          if (kb + 2 < nkb) fetch(kb + 2, qa, qb, xb, sa2, sb2);
          use(qa2, qb2, xb2, sa2b, sb2b);
        }
      }
      if (tail) {
        const size_t off = (size_t)nkb * 64 + 8 * tq;
        const uint2 ta = __ldg(reinterpret_cast<const uint2*>(ca_p + off));
        const uint2 tb = __ldg(reinterpret_cast<const uint2*>(cb_p + off));
        const uint32_t ma[1] = {q4::scale_mult(sa_p[nkb * 8 + tq])};
        const uint32_t mb[1] = {q4::scale_mult(sb_p[nkb * 8 + tq])};
        const uint32_t cwa[2] = {ta.x, ta.y}, cwb[2] = {tb.x, tb.y};
        block_mma<64>(cwa, cwb, ma, mb, act + nkb * 128 + 16 * tq, c0, c1, second);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int jj = n0 + 2 * tq + (i & 1);
        const int f = r0 + gq + (i >> 1) * 8;
        if (jj < count) tc::epi_elem(g, ent.y + jj, f, (c0[i] + c1[i]) * gs);
      }
    }
    if (fused && !second) {
      // this warp's rows of h are stored: count the task for the down projection
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicAdd(a1.g.ready + m, 1);
    }
  }
  if (fused) {
    // the last CTA to finish resets the task counter and the ready counters
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      if (atomicAdd(a1.g.sched + 1, 1u) == gridDim.x - 1) {
        atomicExch(a1.g.sched, 0u);
        atomicExch(a1.g.sched + 1, 0u);
        for (int i = 0; i < num_m; ++i) a1.g.ready[i] = 0;
      }
    }
  }
}

}  // namespace q4v
}  // namespace nh

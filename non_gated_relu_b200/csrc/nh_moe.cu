// nh_moe.cu -- C ABI of libnhmoe: argument checks, workspace plan, tensor
// maps and kernel launches of the Nemotron-H non-gated MoE block forward.
// Declarations and the contract of every entry point: include/nh_moe.h.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "gemm_tc2.cuh"
#include "gemm_q4.cuh"
#include "gemv_q4.cuh"
#include "gemv_bf16.cuh"
#include "permute.cuh"
#include "route.cuh"
#include "route_permute.cuh"

namespace nh {

// ----------------------------------------------------------------------------
// errors
// ----------------------------------------------------------------------------
static thread_local std::string g_last_error;

static nh_status fail(nh_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

#define NH_CUDA(call)                                                                      \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess)                                                                 \
      return fail(NH_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_),    \
                  __FILE__, __LINE__);                                                     \
  } while (0)

#define NH_TRY(expr)                     \
  do {                                   \
    nh_status s_ = (expr);               \
    if (s_ != NH_OK) return s_;          \
  } while (0)

static nh_status launch_check(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(NH_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e));
  return NH_OK;
}

// ----------------------------------------------------------------------------
// configuration and workspace plan
// ----------------------------------------------------------------------------
constexpr int MAX_E = 512;
constexpr int MAX_G = 64;
constexpr int MAX_K = 32;
constexpr size_t ALIGN = 256;
// status region of a workspace: int32[16]
//   [0..2] status code, site, value   [3] router completion counter
//   [4..5] router GEMM tile scheduler  [6..7] up GEMM  [8..9] down GEMM
// (shared workspace: [4..5] shared up GEMM, [6..7] shared down GEMM)
constexpr size_t STATUS_BYTES = 64;
constexpr int SCHED_ROUTER = 4, SCHED_UP = 6, SCHED_DOWN = 8;
constexpr int ROUTE_PERMUTE_MAX_T = 32;
constexpr int ROUTE_PERMUTE_MAX_E = 256;
// fused decode router + permute: 8 warps x 2E selection floats + E + 3 T k
constexpr int ROUTE_PERMUTE_SMEM_MAX = (16 * 256 + 256 + 3 * 32 * 32) * 4;

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static nh_status validate(const nh_moe_config* c) {
  if (!c) return fail(NH_ERR_INVALID_ARG, "cfg is NULL");
  if (c->hidden_size < 1) return fail(NH_ERR_INVALID_ARG, "hidden_size must be >= 1");
  if (c->n_routed_experts < 1) return fail(NH_ERR_INVALID_ARG, "n_routed_experts must be >= 1");
  if (c->n_group < 1 || c->n_routed_experts % c->n_group != 0)
    return fail(NH_ERR_INVALID_ARG, "n_routed_experts (%d) must be a multiple of n_group (%d)",
                c->n_routed_experts, c->n_group);
  if (c->topk_group < 1 || c->topk_group > c->n_group)
    return fail(NH_ERR_INVALID_ARG, "topk_group must be in [1, n_group]");
  const int g = c->n_routed_experts / c->n_group;
  if (c->num_experts_per_tok < 1 || c->num_experts_per_tok > c->topk_group * g)
    return fail(NH_ERR_INVALID_ARG, "num_experts_per_tok must be in [1, topk_group * E / n_group]");
  if (c->moe_intermediate_size < 1) return fail(NH_ERR_INVALID_ARG, "moe_intermediate_size must be >= 1");
  if (c->n_shared_experts != 0 && c->n_shared_experts != 1)
    return fail(NH_ERR_INVALID_ARG, "n_shared_experts must be 0 or 1");
  if (c->n_shared_experts == 1 && c->moe_shared_expert_intermediate_size < 1)
    return fail(NH_ERR_INVALID_ARG, "moe_shared_expert_intermediate_size must be >= 1");
  if (c->norm_topk_prob != 0 && c->norm_topk_prob != 1)
    return fail(NH_ERR_INVALID_ARG, "norm_topk_prob must be 0 or 1");
  if (!std::isfinite(c->routed_scaling_factor))
    return fail(NH_ERR_INVALID_ARG, "routed_scaling_factor must be finite");
  if (c->dtype != NH_F32 && c->dtype != NH_BF16) return fail(NH_ERR_INVALID_ARG, "unknown dtype");
  if (c->group_score != NH_GROUP_SCORE_MAX && c->group_score != NH_GROUP_SCORE_TOP2)
    return fail(NH_ERR_INVALID_ARG, "unknown group_score");
  if (c->group_score == NH_GROUP_SCORE_TOP2 && g < 2)
    return fail(NH_ERR_INVALID_ARG, "the top-2 group score needs >= 2 experts per group");
  if (c->weight_format != NH_WEIGHTS_NATIVE && c->weight_format != NH_WEIGHTS_NVFP4)
    return fail(NH_ERR_INVALID_ARG, "unknown weight_format");
  if (c->weight_format == NH_WEIGHTS_NVFP4 && c->dtype != NH_BF16)
    return fail(NH_ERR_INVALID_ARG, "NVFP4 weights need bf16 activations (W4A16)");
  if (c->latent_size < 0) return fail(NH_ERR_INVALID_ARG, "latent_size must be >= 0");
  // valid; now what the kernels implement
  if (c->n_routed_experts > MAX_E)
    return fail(NH_ERR_UNSUPPORTED, "n_routed_experts > %d", MAX_E);
  if (c->n_group > MAX_G) return fail(NH_ERR_UNSUPPORTED, "n_group > %d", MAX_G);
  if (c->num_experts_per_tok > MAX_K) return fail(NH_ERR_UNSUPPORTED, "num_experts_per_tok > %d", MAX_K);
  if (c->dtype == NH_BF16) {
    if (c->hidden_size % 64 || c->moe_intermediate_size % 64 ||
        (c->n_shared_experts && c->moe_shared_expert_intermediate_size % 64) ||
        c->latent_size % 64)
      return fail(NH_ERR_UNSUPPORTED,
                  "bf16 tensor-core path needs hidden, intermediate, shared and latent sizes "
                  "that are multiples of 64");
  }
  return NH_OK;
}

struct Plan {
  int H, E, G, tg, k, I, S;
  int64_t T, rows;
  bool bf16;
  size_t elem;
  nh_moe_ws_layout lay;
};

// rows of one tile entry for T tokens: decode-sized T puts the weights on the
// MMA M side (swap), with all of an expert's rows in one entry
static void tile_plan(const nh_moe_config* c, int64_t T, int* tile_rows, int* swap) {
  if (c->weight_format == NH_WEIGHTS_NVFP4) {
    // weights are dequantized per stage: always weights on the MMA M side
    *tile_rows = T <= 16 ? 16 : (T <= 32 ? 32 : 64);
    *swap = 1;
  } else if (c->dtype == NH_F32) {
    *tile_rows = SG_BM;
    *swap = 0;
  } else if (T <= 16) {
    *tile_rows = 16;
    *swap = 1;
  } else if (T <= 32) {
    *tile_rows = 32;
    *swap = 1;
  } else if (T <= 64) {
    *tile_rows = 64;
    *swap = 1;
  } else {
    *tile_rows = tc2::MP;   // 256-row tiles computed by CTA pairs
    *swap = 0;
  }
}

static nh_status make_plan(const nh_moe_config* c, int64_t T, Plan* p) {
  NH_TRY(validate(c));
  if (T < 0) return fail(NH_ERR_INVALID_ARG, "T must be >= 0");
  const int64_t rows = T * c->num_experts_per_tok;
  if (rows >= (int64_t(1) << 31) - 4096) return fail(NH_ERR_UNSUPPORTED, "T * k must be < 2^31");
  p->H = c->hidden_size;
  p->E = c->n_routed_experts;
  p->G = c->n_group;
  p->tg = c->topk_group;
  p->k = c->num_experts_per_tok;
  p->I = c->moe_intermediate_size;
  p->S = c->moe_shared_expert_intermediate_size;
  p->T = T;
  p->rows = rows;
  p->bf16 = c->dtype == NH_BF16;
  p->elem = p->bf16 ? 2 : 4;
  nh_moe_ws_layout& L = p->lay;
  memset(&L, 0, sizeof L);
  int tr, sw;
  tile_plan(c, T, &tr, &sw);
  L.tile_rows = tr;
  L.swap_ab = sw;
  L.x_direct = (sw && T <= 64) ? 1 : 0;   // every token fits one activation tile
  L.max_tiles = (int)((rows + tr - 1) / tr + p->E);
  L.n_chunks = (int)((T + PERM_CHUNK - 1) / PERM_CHUNK);
  L.rows_alloc = rows;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + (bytes ? bytes : 1), ALIGN);
    return at;
  };
  L.status = take(STATUS_BYTES);
  L.logits = take((size_t)T * p->E * 4);
  L.router_w = take(p->bf16 ? (size_t)p->E * 3 * p->H * 2 : 0);
  L.counts = take((size_t)p->E * 4);
  L.offsets = take((size_t)(p->E + 1) * 4);
  L.chunk_counts = take((size_t)L.n_chunks * p->E * 4);
  L.perm_token = take((size_t)rows * 4);
  L.perm_w = take((size_t)rows * 4);
  L.inv_row = take((size_t)rows * 4);
  L.tiles = take((size_t)L.max_tiles * 16);
  L.num_tiles = take(4);
  L.x_perm = take(L.x_direct ? 0 : (size_t)rows * p->H * p->elem);
  L.h = take((size_t)rows * p->I * p->elem);
  L.ready = take((size_t)L.max_tiles * 4);
  L.total_bytes = o;
  return NH_OK;
}

static nh_status check_ptr(const void* p, const char* name) {
  if (!p) return fail(NH_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % 16)
    return fail(NH_ERR_INVALID_ARG, "%s must be 16-byte aligned", name);
  return NH_OK;
}

static nh_status check_ws(const Plan& p, void* ws, size_t ws_bytes) {
  NH_TRY(check_ptr(ws, "ws"));
  if (reinterpret_cast<uintptr_t>(ws) % ALIGN)
    return fail(NH_ERR_INVALID_ARG, "ws must be %zu-byte aligned", ALIGN);
  if (ws_bytes < p.lay.total_bytes)
    return fail(NH_ERR_INVALID_ARG, "ws holds %zu bytes, %zu needed", ws_bytes, p.lay.total_bytes);
  return NH_OK;
}

// the routed-expert calls take the expert-width config of a latent block
static nh_status no_latent(const nh_moe_config* c, const char* what) {
  if (c && c->latent_size)
    return fail(NH_ERR_INVALID_ARG,
                "%s: config has latent_size %d; pass the expert-width config of "
                "nh_moe_latent_config", what, c->latent_size);
  return NH_OK;
}

template <typename T>
static T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

static PermuteOut permute_out(void* ws, const nh_moe_ws_layout& L, int* status) {
  PermuteOut o;
  o.tile_rows = L.tile_rows;
  o.max_tiles = L.max_tiles;
  o.counts = at<int32_t>(ws, L.counts);
  o.offsets = at<int32_t>(ws, L.offsets);
  o.tiles = at<int4>(ws, L.tiles);
  o.num_tiles = at<int32_t>(ws, L.num_tiles);
  o.perm_token = at<int32_t>(ws, L.perm_token);
  o.perm_w = at<float>(ws, L.perm_w);
  o.inv_row = at<int32_t>(ws, L.inv_row);
  o.x_perm = at<void>(ws, L.x_perm);
  o.status = status;
  o.sched_zero = reinterpret_cast<unsigned int*>(status + SCHED_UP);
  o.gather = L.x_direct ? 0 : 1;
  o.ready = at<int>(ws, L.ready);
  o.n_ready = L.max_tiles;
  return o;
}

// ----------------------------------------------------------------------------
// device properties and kernel attributes (cached per device)
// ----------------------------------------------------------------------------
constexpr int MAX_DEVICES = 64;
static std::once_flag g_attr_once[MAX_DEVICES];
static int g_sm_count[MAX_DEVICES];
static int g_pair_clusters[MAX_DEVICES];  // co-resident 2-CTA clusters of tc2_grouped_gemm
static nh_status g_attr_status[MAX_DEVICES];

using TcPrefill = tc::Shape<false, 256, 4>;
using TcPrefill128 = tc::Shape<false, 128, 6>;
using TcSwap16 = tc::Shape<true, 16, 8>;
using TcSwap32 = tc::Shape<true, 32, 8>;
using TcSwap64 = tc::Shape<true, 64, 6>;

static nh_status set_attrs(int dev) {
  cudaDeviceProp prop;
  NH_CUDA(cudaGetDeviceProperties(&prop, dev));
  g_sm_count[dev] = prop.multiProcessorCount;
  if (prop.major != 10)
    return fail(NH_ERR_UNSUPPORTED, "libnhmoe is built for sm_100a; device %d is sm_%d%d", dev,
                prop.major, prop.minor);
  NH_CUDA(cudaFuncSetAttribute(tc::tc_grouped_gemm<false, 256, 4>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, TcPrefill::SMEM));
  NH_CUDA(cudaFuncSetAttribute(tc::tc_grouped_gemm<false, 128, 6>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, TcPrefill128::SMEM));
  NH_CUDA(cudaFuncSetAttribute(tc::tc_grouped_gemm<true, 16, 8>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, TcSwap16::SMEM));
  NH_CUDA(cudaFuncSetAttribute(tc::tc_grouped_gemm<true, 32, 8>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, TcSwap32::SMEM));
  NH_CUDA(cudaFuncSetAttribute(tc::tc_grouped_gemm<true, 64, 6>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, TcSwap64::SMEM));
  NH_CUDA(cudaFuncSetAttribute(tc2::tc2_grouped_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               tc2::SMEM));
  NH_CUDA(cudaFuncSetAttribute(q4::tc_q4_gemm<64, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               q4::Shape<64, 4>::SMEM));
  NH_CUDA(cudaFuncSetAttribute(dgv::bf16_gemv_staged<16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, dgv::STAGED_SMEM));
  NH_CUDA(cudaFuncSetAttribute(dgv::bf16_gemv_staged<32>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, dgv::STAGED_SMEM));
  NH_CUDA(cudaFuncSetAttribute(route_permute_small<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, ROUTE_PERMUTE_SMEM_MAX));
  NH_CUDA(cudaFuncSetAttribute(route_permute_small<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, ROUTE_PERMUTE_SMEM_MAX));
  {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(2 * (prop.multiProcessorCount / 2), 1, 1);
    lc.blockDim = dim3(tc2::THREADS, 1, 1);
    lc.dynamicSmemBytes = tc2::SMEM;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    int n = 0;
    NH_CUDA(cudaOccupancyMaxActiveClusters(&n, tc2::tc2_grouped_gemm, &lc));
    if (n < 1) return fail(NH_ERR_UNSUPPORTED, "no 2-CTA cluster of the pair GEMM fits on device %d", dev);
    g_pair_clusters[dev] = n;
  }
  return NH_OK;
}

static nh_status device_setup(int* dev_out) {
  int dev;
  NH_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= MAX_DEVICES) return fail(NH_ERR_UNSUPPORTED, "device id %d", dev);
  std::call_once(g_attr_once[dev], [dev] { g_attr_status[dev] = set_attrs(dev); });
  if (g_attr_status[dev] != NH_OK)
    return fail(g_attr_status[dev], "device %d setup failed (unsupported or CUDA error)", dev);
  *dev_out = dev;
  return NH_OK;
}

static uint64_t timeout_ns() {
  static uint64_t v = [] {
    const char* s = getenv("NH_MOE_TIMEOUT_NS");
    uint64_t t = s ? strtoull(s, nullptr, 10) : 0;
    return t ? t : 2000000000ull;  // 2 s: far above any single pipeline wait
  }();
  return v;
}

// Launch with programmatic dependent launch allowed: the kernel may start its
// prologue while the previous kernel in the stream finishes; every kernel of
// this library executes griddepcontrol.wait before it reads its inputs.
// The launching stream's priority, set again as a launch attribute so that a
// CUDA graph captured from prioritised streams keeps it per kernel node: the
// block scheduler then starts pending CTAs of the routed path (a high
// priority stream) before those of the concurrent shared expert.
static int stream_priority(cudaStream_t st) {
  int p = 0;
  if (cudaStreamGetPriority(st, &p) != cudaSuccess) {
    cudaGetLastError();
    p = 0;
  }
  return p;
}

template <typename Kern, typename... Args>
static nh_status launch_k(const char* what, Kern kernel, dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, Args... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributePriority;
  at[1].val.priority = stream_priority(st);
  lc.attrs = at;
  lc.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&lc, kernel, args...);
  if (e != cudaSuccess)
    return fail(NH_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e));
  return NH_OK;
}

// ----------------------------------------------------------------------------
// TMA tensor maps (driver entry point fetched through the runtime)
// ----------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// bf16 [rows, K] row-major, box {64, box_rows}, 128-byte swizzle
static nh_status map_2d(CUtensorMap* m, const void* base, int64_t K, int64_t rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(NH_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)tc::BK, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NH_ERR_CUDA, "cuTensorMapEncodeTiled (2d) failed: %d", (int)r);
  return NH_OK;
}

// bf16 [n_exp, N, K] row-major, box {64, box_rows, 1}, 128-byte swizzle
static nh_status map_3d(CUtensorMap* m, const void* base, int64_t K, int64_t N, int64_t n_exp,
                        int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(NH_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)N, (cuuint64_t)n_exp};
  cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)K * N * 2};
  cuuint32_t box[3] = {(cuuint32_t)tc::BK, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NH_ERR_CUDA, "cuTensorMapEncodeTiled (3d) failed: %d", (int)r);
  return NH_OK;
}

// ----------------------------------------------------------------------------
// one grouped GEMM: out = epi(A[rows] . W[e]^T) over the tile entries
// ----------------------------------------------------------------------------
struct GemmCall {
  const void* A;        // [rows, K_a] (dtype); K_a = a_kwrap when set, else K
  int a_kwrap;
  int64_t rows;         // rows of A
  const void* W;        // [n_exp, N, K] (dtype)
  int n_exp;
  int N, K;
  const int4* tiles;    // or null: dense over `rows`
  const int32_t* num_tiles;
  int max_tiles;        // grid bound when tiles != null
  int tile_rows;
  int swap;
  int epi;
  void* out;
  int64_t ldo;
  const float* perm_w;
  const int32_t* dst_row;    // routed down projection: token of each permuted row
  const int32_t* row_token;  // decode up projection reads x directly
  int* status;
  unsigned int* sched;  // tile scheduler counters (tensor-core path)
  int k_split;          // K slices per output tile (additive epilogues; 0/1 = none)
};

static tc::TcArgs tc_args(const GemmCall& c) {
  tc::TcArgs g{};
  g.tiles = c.tiles;
  g.num_tiles = c.num_tiles;
  g.dense_rows = (int)c.rows;
  g.tile_rows = c.tile_rows;
  g.N = c.N;
  g.K = c.K;
  g.a_kwrap = c.a_kwrap;
  g.epi = c.epi;
  g.out = c.out;
  g.ldo = c.ldo;
  g.perm_w = c.perm_w;
  g.dst_row = c.dst_row;
  g.row_token = c.row_token;
  g.status = c.status;
  g.timeout_ns = timeout_ns();
  g.sched = c.sched;
  g.k_split = c.k_split;
  return g;
}

static nh_status check_tc_call(const GemmCall& c) {
  if (!c.sched) return fail(NH_ERR_INVALID_ARG, "internal: no tile scheduler counters");
  if (c.k_split > 1 && c.epi != EPI_DOWN_COMBINE && c.epi != EPI_ACC_F32)
    return fail(NH_ERR_INVALID_ARG, "internal: K slices need an additive epilogue");
  return NH_OK;
}

// output tiles of one call: tile entries x feature blocks x K slices
template <bool SWAP, int NT>
static int64_t tc_work(const GemmCall& c) {
  const int n_blocks = SWAP ? (c.N + tc::M - 1) / tc::M : (c.N + NT - 1) / NT;
  const int64_t m_max = c.tiles ? c.max_tiles : (c.rows + c.tile_rows - 1) / c.tile_rows;
  return m_max * n_blocks * (c.k_split > 1 ? c.k_split : 1);
}

template <bool SWAP, int NT, int STAGES>
static nh_status launch_tc(const GemmCall& c, int dev, cudaStream_t st) {
  using S = tc::Shape<SWAP, NT, STAGES>;
  CUtensorMap ma, mw;
  NH_TRY(map_2d(&ma, c.A, c.a_kwrap ? c.a_kwrap : c.K, c.rows, SWAP ? NT : tc::M));
  NH_TRY(map_3d(&mw, c.W, c.K, c.N, c.n_exp, SWAP ? tc::M : NT));
  NH_TRY(check_tc_call(c));
  const tc::TcArgs g = tc_args(c);
  const int grid = (int)std::min<int64_t>(tc_work<SWAP, NT>(c), g_sm_count[dev]);
  if (grid <= 0) return NH_OK;
  const tc::TcArgs none{};
  NH_TRY((launch_k("tc_grouped_gemm", tc::tc_grouped_gemm<SWAP, NT, STAGES>, dim3(grid), dim3(tc::THREADS), S::SMEM, st, ma, mw, g, ma, mw, none)));
  return launch_check("tc_grouped_gemm");
}

// Decode up and down projections as one persistent launch (weights on the MMA
// M side): c1 writes h, c2 reads it; c2's tiles of a tile entry start once
// the 4 epilogue warps of each of c1's feature blocks of that entry have
// counted their rows into `ready` (zeroed by the permute).
template <int NT, int STAGES>
static nh_status launch_tc_fused(const GemmCall& c1, const GemmCall& c2, int* ready, int dev,
                                 cudaStream_t st) {
  using S = tc::Shape<true, NT, STAGES>;
  CUtensorMap ma1, mw1, ma2, mw2;
  NH_TRY(map_2d(&ma1, c1.A, c1.a_kwrap ? c1.a_kwrap : c1.K, c1.rows, NT));
  NH_TRY(map_3d(&mw1, c1.W, c1.K, c1.N, c1.n_exp, tc::M));
  NH_TRY(map_2d(&ma2, c2.A, c2.a_kwrap ? c2.a_kwrap : c2.K, c2.rows, NT));
  NH_TRY(map_3d(&mw2, c2.W, c2.K, c2.N, c2.n_exp, tc::M));
  NH_TRY(check_tc_call(c1));
  NH_TRY(check_tc_call(c2));
  if (c1.k_split > 1 || c1.tiles != c2.tiles)
    return fail(NH_ERR_INVALID_ARG, "internal: fused GEMMs share the tile table, whole-K first");
  tc::TcArgs g1 = tc_args(c1), g2 = tc_args(c2);
  g1.ready = ready;
  g2.ready = ready;
  g2.ready_need = 4 * ((c1.N + tc::M - 1) / tc::M);
  const int64_t work = tc_work<true, NT>(c1) + tc_work<true, NT>(c2);
  const int grid = (int)std::min<int64_t>(work, g_sm_count[dev]);
  if (grid <= 0) return NH_OK;
  NH_TRY((launch_k("tc_grouped_gemm", tc::tc_grouped_gemm<true, NT, STAGES>, dim3(grid),
                   dim3(tc::THREADS), S::SMEM, st, ma1, mw1, g1, ma2, mw2, g2)));
  return launch_check("tc_grouped_gemm");
}

// prefill orientation on CTA pairs: 256-row tiles, each CTA stages 128 rows of
// the activations and half of the weight rows
static nh_status launch_tc2(const GemmCall& c, int dev, cudaStream_t st) {
  CUtensorMap ma, mw, mr;
  NH_TRY(map_2d(&ma, c.A, c.a_kwrap ? c.a_kwrap : c.K, c.rows, tc2::HALF));
  NH_TRY(map_3d(&mw, c.W, c.K, c.N, c.n_exp, tc2::HALF));
  // rows of a partial tile attached to a full one (kind-2 tiles)
  NH_TRY(map_2d(&mr, c.A, c.a_kwrap ? c.a_kwrap : c.K, c.rows, tc2::C_ROWS));
  tc::TcArgs g{};
  g.tiles = c.tiles;
  g.num_tiles = c.num_tiles;
  g.dense_rows = (int)c.rows;
  g.tile_rows = c.tile_rows;
  g.N = c.N;
  g.K = c.K;
  g.a_kwrap = c.a_kwrap;
  g.epi = c.epi;
  g.out = c.out;
  g.ldo = c.ldo;
  g.perm_w = c.perm_w;
  g.dst_row = c.dst_row;
  g.row_token = nullptr;
  g.status = c.status;
  g.timeout_ns = timeout_ns();
  g.sched = c.sched;
  if (!g.sched) return fail(NH_ERR_INVALID_ARG, "internal: no tile scheduler counters");
  if (c.tile_rows != tc2::MP) return fail(NH_ERR_INVALID_ARG, "internal: pair tiles are 256 rows");
  const int n_blocks = (c.N + tc2::NT - 1) / tc2::NT;
  const int64_t m_max = c.tiles ? c.max_tiles : (c.rows + c.tile_rows - 1) / c.tile_rows;
  const int64_t pairs = std::min<int64_t>(m_max * n_blocks, g_pair_clusters[dev]);
  if (pairs <= 0) return NH_OK;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  lc.blockDim = dim3(tc2::THREADS, 1, 1);
  lc.dynamicSmemBytes = tc2::SMEM;
  lc.stream = st;
  cudaLaunchAttribute at[3];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  at[2].id = cudaLaunchAttributePriority;
  at[2].val.priority = stream_priority(st);
  lc.attrs = at;
  lc.numAttrs = 3;
  NH_CUDA(cudaLaunchKernelEx(&lc, tc2::tc2_grouped_gemm, ma, mw, mr, g));
  return launch_check("tc2_grouped_gemm");
}

// uint8 [n_mat, rows, row_bytes], box {box_bytes, 128 rows, 1}; with `swizzle`
// the box is 128 bytes wide and lands with the 128-byte swizzle
static nh_status map_u8_3d(CUtensorMap* m, const void* base, int64_t row_bytes, int64_t rows,
                           int64_t n_mat, int box_bytes, bool swizzle) {
  auto fn = encode_fn();
  if (!fn) return fail(NH_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)rows, (cuuint64_t)n_mat};
  cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)(row_bytes * rows)};
  cuuint32_t box[3] = {(cuuint32_t)box_bytes, (cuuint32_t)q4::M, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NH_ERR_CUDA, "cuTensorMapEncodeTiled (u8) failed: %d", (int)r);
  return NH_OK;
}

static int64_t nvfp4_pitch(int64_t cols) { return ((cols / 16 + 15) / 16) * 16; }

template <int NT, int STAGES>
static nh_status launch_q4(const GemmCall& c, const nh_nvfp4_weight& w, int dev, cudaStream_t st) {
  using S = q4::Shape<NT, STAGES>;
  CUtensorMap ma, mc, ms;
  NH_TRY(map_2d(&ma, c.A, c.K, c.rows, NT));
  NH_TRY(map_u8_3d(&mc, w.codes, c.K / 2, c.N, c.n_exp, q4::CODE_ROW, true));
  NH_TRY(map_u8_3d(&ms, w.scales, nvfp4_pitch(c.K), c.N, c.n_exp, q4::SCALE_BOX, false));
  q4::Q4Args qa{};
  tc::TcArgs& g = qa.g;
  g.tiles = c.tiles;
  g.num_tiles = c.num_tiles;
  g.dense_rows = (int)c.rows;
  g.tile_rows = c.tile_rows;
  g.N = c.N;
  g.K = c.K;
  g.a_kwrap = 0;
  g.epi = c.epi;
  g.out = c.out;
  g.ldo = c.ldo;
  g.perm_w = c.perm_w;
  g.dst_row = c.dst_row;
  g.row_token = c.row_token;
  g.status = c.status;
  g.timeout_ns = timeout_ns();
  g.sched = c.sched;
  qa.gscale = w.global_scale;
  const int n_blocks = (c.N + q4::M - 1) / q4::M;
  const int64_t m_max = c.tiles ? c.max_tiles : (c.rows + c.tile_rows - 1) / c.tile_rows;
  const int grid = (int)std::min<int64_t>(m_max * n_blocks, g_sm_count[dev]);
  if (grid <= 0) return NH_OK;
  return launch_k("tc_q4_gemm", q4::tc_q4_gemm<NT, STAGES>, dim3(grid), dim3(q4::THREADS), S::SMEM,
                  st, ma, mc, ms, qa);
}

static q4v::Args q4v_args(const GemmCall& c, const nh_nvfp4_weight& w) {
  q4v::Args a{};
  tc::TcArgs& g = a.g;
  g.tiles = c.tiles;
  g.num_tiles = c.num_tiles;
  g.dense_rows = (int)c.rows;
  g.tile_rows = c.tile_rows;
  g.N = c.N;
  g.K = c.K;
  g.a_kwrap = 0;
  g.epi = c.epi;
  g.out = c.out;
  g.ldo = c.ldo;
  g.perm_w = c.perm_w;
  g.dst_row = c.dst_row;
  g.row_token = c.row_token;
  g.status = c.status;
  g.timeout_ns = timeout_ns();
  g.sched = c.sched;
  a.A = c.A;
  a.codes = w.codes;
  a.scales = w.scales;
  a.gscale = w.global_scale;
  a.pitch = (int)nvfp4_pitch(c.K);
  return a;
}

static nh_status check_q4(const nh_nvfp4_weight* w) {
  if (!w || !w->codes || !w->scales || !w->global_scale)
    return fail(NH_ERR_INVALID_ARG, "NVFP4 weight with a NULL pointer");
  if (reinterpret_cast<uintptr_t>(w->codes) % 16 || reinterpret_cast<uintptr_t>(w->scales) % 16)
    return fail(NH_ERR_INVALID_ARG, "NVFP4 codes / scales must be 16-byte aligned");
  return NH_OK;
}

// decode-sized tiles: warp-level MMAs from registers (gemv_q4.cuh)
template <int NT>
static nh_status launch_q4v(const GemmCall& c, const nh_nvfp4_weight& w, int dev,
                            cudaStream_t st) {
  const q4v::Args a = q4v_args(c, w);
  // tasks: (tile entry, 16 weight rows).  Few tasks (dense rows: shared
  // expert, latent projections): one per CTA with K split over its warps;
  // many (routed experts): one per warp.
  const int64_t m_max = c.tiles ? c.max_tiles : (c.rows + c.tile_rows - 1) / c.tile_rows;
  const int64_t tasks = m_max * (c.N / q4v::MT);
  const int64_t slots = (int64_t)g_sm_count[dev] * 3;   // resident CTAs
  if (tasks <= 0) return NH_OK;
  if (!c.tiles && tasks < slots * q4v::WARPS / 2)
    return launch_k("q4_gemv_splitk", q4v::q4_gemv_splitk<NT>,
                    dim3((unsigned)std::min<int64_t>(tasks, slots)), dim3(q4v::WARPS * 32), 0, st,
                    a);
  // the rows kernel keeps two CTAs per SM (its launch bounds): one wave
  const int64_t grid = std::min<int64_t>((tasks + q4v::WARPS - 1) / q4v::WARPS,
                                         (int64_t)g_sm_count[dev] * 2);
  return launch_k("q4_gemv_rows", q4v::q4_gemv_rows<NT>, dim3((unsigned)grid),
                  dim3(q4v::WARPS * 32), 0, st, a, q4v::Args{});
}

// NVFP4 decode: the routed up and down projections as one launch of the rows
// GEMV, warps fetching tasks from a counter (up tasks first); a down task of a
// tile entry waits until the entry's up tasks have counted themselves into
// `ready` (zeroed by the permute and by each such launch).
template <int NT>
static nh_status launch_q4v_fused(const GemmCall& c1, const nh_nvfp4_weight& w1,
                                  const GemmCall& c2, const nh_nvfp4_weight& w2, int* ready,
                                  int dev, cudaStream_t st) {
  q4v::Args a1 = q4v_args(c1, w1), a2 = q4v_args(c2, w2);
  a1.g.ready = ready;
  a2.g.ready = ready;
  a2.g.ready_need = c1.N / q4v::MT;
  const int64_t tasks = (int64_t)c1.max_tiles * (c1.N / q4v::MT + c2.N / q4v::MT);
  if (tasks <= 0) return NH_OK;
  const int64_t grid = std::min<int64_t>((tasks + q4v::WARPS - 1) / q4v::WARPS,
                                         (int64_t)g_sm_count[dev] * 2);
  return launch_k("q4_gemv_rows", q4v::q4_gemv_rows<NT>, dim3((unsigned)grid),
                  dim3(q4v::WARPS * 32), 0, st, a1, a2);
}

static nh_status run_gemm_q4(const GemmCall& c, const nh_nvfp4_weight* w, int dev,
                             cudaStream_t st) {
  if (c.rows == 0) return NH_OK;
  NH_TRY(check_q4(w));
  switch (c.tile_rows) {
    case 16: return launch_q4v<16>(c, *w, dev, st);
    case 32: return launch_q4v<32>(c, *w, dev, st);
    case 64: return launch_q4<64, 4>(c, *w, dev, st);
    default: return fail(NH_ERR_UNSUPPORTED, "NVFP4 tile rows %d", c.tile_rows);
  }
}

// dense rows of decode size (shared expert, latent projections): CTA tasks of
// 16 weight rows with K split over the warps (gemv_bf16.cuh)
template <int NT>
static nh_status launch_dgv(const GemmCall& c, int dev, cudaStream_t st) {
  dgv::Args a{};
  tc::TcArgs& g = a.g;
  g.tiles = nullptr;
  g.num_tiles = nullptr;
  g.dense_rows = (int)c.rows;
  g.tile_rows = c.tile_rows;
  g.N = c.N;
  g.K = c.K;
  g.a_kwrap = 0;
  g.epi = c.epi;
  g.out = c.out;
  g.ldo = c.ldo;
  g.perm_w = c.perm_w;
  g.dst_row = c.dst_row;
  g.row_token = nullptr;
  g.status = c.status;
  g.timeout_ns = timeout_ns();
  g.sched = c.sched;
  a.A = c.A;
  a.W = c.W;
  const int64_t tasks = (c.rows + c.tile_rows - 1) / c.tile_rows * (c.N / dgv::MT);
  const int64_t grid = std::min<int64_t>(tasks, (int64_t)g_sm_count[dev] * 2);
  if (grid <= 0) return NH_OK;
  return launch_k("bf16_gemv_staged", dgv::bf16_gemv_staged<NT>, dim3((unsigned)grid),
                  dim3(dgv::WARPS * 32), dgv::STAGED_SMEM, st, a);
}

static nh_status run_gemm(const Plan& p, const GemmCall& c, int dev, cudaStream_t st) {
  if (c.rows == 0) return NH_OK;
  if (p.bf16 && !c.tiles && c.swap && c.a_kwrap == 0 && c.n_exp == 1 && !c.row_token) {
    if (c.tile_rows == 16) return launch_dgv<16>(c, dev, st);
    if (c.tile_rows == 32) return launch_dgv<32>(c, dev, st);
  }
  if (!p.bf16) {
    GemmArgs g;
    g.A = c.A;
    g.B = c.W;
    g.K = c.K;
    g.N = c.N;
    g.tiles = c.tiles;
    g.num_tiles = c.num_tiles;
    g.dense_rows = (int)c.rows;
    g.tile_rows = c.tile_rows;
    g.epi = c.epi;
    g.out = c.out;
    g.ldo = c.ldo;
    g.perm_w = c.perm_w;
    g.dst_row = c.dst_row;
    const int64_t m_max = c.tiles ? c.max_tiles : (c.rows + c.tile_rows - 1) / c.tile_rows;
    if (m_max > 65535) return fail(NH_ERR_UNSUPPORTED, "float32 path: too many row tiles");
    dim3 grid((c.N + SG_BN - 1) / SG_BN, (unsigned)m_max);
    NH_TRY((launch_k("simt_grouped_gemm", simt_grouped_gemm<float>, dim3(grid), dim3(256), 0, st, g)));
    return launch_check("simt_grouped_gemm");
  }
  if (!c.swap) return launch_tc2(c, dev, st);
  switch (c.tile_rows) {
    case 16: return launch_tc<true, 16, 8>(c, dev, st);
    case 32: return launch_tc<true, 32, 8>(c, dev, st);
    case 64: return launch_tc<true, 64, 6>(c, dev, st);
    default: return fail(NH_ERR_UNSUPPORTED, "tile rows %d", c.tile_rows);
  }
}

// ----------------------------------------------------------------------------
// small kernels
// ----------------------------------------------------------------------------
// y = dtype(y_acc): the one rounding of the block output, after the routed
// experts' weighted combine and the shared expert were added into y_acc
__global__ void cast_output_bf16x8(const float4* __restrict__ y_acc, uint4* __restrict__ y,
                                   int64_t n8) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = y_acc[2 * i], b = y_acc[2 * i + 1];
    y[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                      pack_bf16x2(b.z, b.w));
  }
}

template <typename Tout>
__global__ void cast_output(const float* __restrict__ y_acc, Tout* __restrict__ y, int64_t n) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    y[i] = from_f32<Tout>(y_acc[i]);
}

__global__ void selftest_timeout_kernel(int* status, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl w{&abort_flag, status, timeout_ns};
    // nothing ever arrives on this barrier: the bounded wait must run out
    mbar_wait(smem_u32(&bar), 0, w, SITE_SELFTEST);
  }
  __syncthreads();
}

// ----------------------------------------------------------------------------
// Router without caller-provided scratch (nh_moe_route_noalloc).
//
// Some callers cannot hand the library a workspace: serving stacks whose
// memory pool reserves all of device memory up front, or plugin hosts that
// give an op no scratch buffer and may not call cudaMalloc (not
// stream-ordered; it can synchronise the device).  For decode-sized batches the router's
// only scratch is the logits block, a status word and a completion counter,
// which fit in a fixed array compiled into the library.  Every device that
// loads the library holds this array until the process exits.
// ----------------------------------------------------------------------------
constexpr int64_t NOALLOC_MAX_T = 32;
constexpr int64_t NOALLOC_MAX_LOGITS = 16384;  // T * E floats (64 KiB)
constexpr size_t NOALLOC_HEADER = 256;          // status word + completion counter
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[NOALLOC_HEADER + NOALLOC_MAX_LOGITS * sizeof(float)];
static std::once_flag g_noalloc_once[MAX_DEVICES];
static void* g_noalloc_ptr[MAX_DEVICES];
static cudaError_t g_noalloc_err[MAX_DEVICES];

// Device address of the static scratch on `dev` (the current device).  The
// symbol's name in host code is only a host-side stand-in, so the address is
// looked up once per device with that device current.
static nh_status noalloc_scratch(int dev, void** out) {
  std::call_once(g_noalloc_once[dev], [dev] {
    g_noalloc_err[dev] = cudaGetSymbolAddress(&g_noalloc_ptr[dev], g_noalloc_scratch);
  });
  if (g_noalloc_err[dev] != cudaSuccess)
    return fail(NH_ERR_CUDA, "cudaGetSymbolAddress of the router scratch failed on device %d: %s",
                dev, cudaGetErrorString(g_noalloc_err[dev]));
  *out = g_noalloc_ptr[dev];
  return NH_OK;
}

static int grid_for(int64_t n, int per_block, int dev) {
  int64_t b = (n + per_block - 1) / per_block;
  const int64_t cap = (int64_t)g_sm_count[dev] * 8;
  if (b > cap) b = cap;
  return (int)(b < 1 ? 1 : b);
}

}  // namespace nh

using namespace nh;

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

const char* nh_last_error(void) { return g_last_error.c_str(); }

const char* nh_version(void) { return "nhmoe 0.1 (sm_100a)"; }

nh_status nh_moe_validate(const nh_moe_config* cfg) { return validate(cfg); }

nh_status nh_moe_workspace_layout(const nh_moe_config* cfg, int64_t T, nh_moe_ws_layout* out) {
  if (!out) return fail(NH_ERR_INVALID_ARG, "out is NULL");
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  *out = p.lay;
  return NH_OK;
}

nh_status nh_moe_workspace_size(const nh_moe_config* cfg, int64_t T, size_t* bytes) {
  if (!bytes) return fail(NH_ERR_INVALID_ARG, "bytes is NULL");
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  *bytes = p.lay.total_bytes;
  return NH_OK;
}

nh_status nh_moe_shared_workspace_size(const nh_moe_config* cfg, int64_t T, size_t* bytes) {
  if (!bytes) return fail(NH_ERR_INVALID_ARG, "bytes is NULL");
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  if (!cfg->n_shared_experts) return fail(NH_ERR_INVALID_ARG, "config has no shared expert");
  *bytes = ALIGN + align_up((size_t)T * p.S * p.elem + 1, ALIGN);
  return NH_OK;
}

nh_status nh_moe_route(const nh_moe_config* cfg, int64_t T, const void* x, const float* w_router,
                       const float* bias, int32_t* topk_idx, float* topk_w, void* ws,
                       size_t ws_bytes, void* stream) {
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  // routing touches only the regions before `counts` (status, logits, router_w)
  NH_TRY(check_ptr(ws, "ws"));
  if (reinterpret_cast<uintptr_t>(ws) % ALIGN)
    return fail(NH_ERR_INVALID_ARG, "ws must be %zu-byte aligned", ALIGN);
  if (ws_bytes < p.lay.counts)
    return fail(NH_ERR_INVALID_ARG, "ws holds %zu bytes, %zu needed for routing", ws_bytes,
                p.lay.counts);
  if (T == 0) return NH_OK;
  NH_TRY(check_ptr(x, "x"));
  NH_TRY(check_ptr(w_router, "w_router"));
  NH_TRY(check_ptr(topk_idx, "topk_idx"));
  NH_TRY(check_ptr(topk_w, "topk_w"));
  if (bias) NH_TRY(check_ptr(bias, "e_score_correction_bias"));
  int dev;
  NH_TRY(device_setup(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = at<int>(ws, p.lay.status);
  float* logits = at<float>(ws, p.lay.logits);
  NH_CUDA(cudaMemsetAsync(status, 0, STATUS_BYTES, st));
  SelectArgs a;
  a.logits = logits;
  a.bias = bias;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.status = status;
  a.T = (int)T;
  a.E = p.E;
  a.G = p.G;
  a.tg = p.tg;
  a.k = p.k;
  a.norm = cfg->norm_topk_prob;
  a.alpha = cfg->routed_scaling_factor;
  a.group_score = cfg->group_score;
  a.use_sigma = (bias != nullptr) || cfg->group_score == NH_GROUP_SCORE_TOP2;
  const size_t sel_smem = (size_t)8 * 2 * p.E * sizeof(float);
  if (T <= 32) {
    // decode: logits and selection in one launch (last block selects)
    const int blocks = p.E;
    unsigned int* done = reinterpret_cast<unsigned int*>(status + 3);
    if (p.bf16)
      NH_TRY((launch_k("router_fused_small", router_fused_small<__nv_bfloat16>, dim3(blocks), dim3(256), sel_smem, st, 
          static_cast<const __nv_bfloat16*>(x), w_router, a, p.H, done)));
    else
      NH_TRY((launch_k("router_fused_small", router_fused_small<float>, dim3(blocks), dim3(256), sel_smem, st, static_cast<const float*>(x),
                                                                w_router, a, p.H, done)));
    return launch_check("router_fused_small");
  }
  if (p.bf16 && p.E % 32 == 0) {
    // logits on the tensor cores: x (bf16) against the fp32 router weight split
    // into three bf16 planes, accumulated over K = 3H in fp32
    __nv_bfloat16* wsplit = at<__nv_bfloat16>(ws, p.lay.router_w);
    NH_TRY((launch_k("router_split", router_split, dim3(grid_for((int64_t)p.E * p.H, 256, dev)), dim3(256), 0, st, w_router, wsplit, p.E,
                                                                          p.H)));
    NH_TRY(launch_check("router_split"));
    GemmCall c{};
    c.A = x;
    c.a_kwrap = p.H;
    c.rows = T;
    c.W = wsplit;
    c.n_exp = 1;
    c.N = p.E;
    c.K = 3 * p.H;
    c.tiles = nullptr;
    c.tile_rows = tc::M;
    c.swap = 0;
    c.epi = EPI_STORE_F32;
    c.out = logits;
    c.ldo = p.E;
    c.status = status;
    c.sched = reinterpret_cast<unsigned int*>(status + SCHED_ROUTER);
    // up to 128 experts fit one 128-wide N tile (a 256-wide tile would spend
    // half of its MMA work on zero-filled weight rows)
    if (p.E <= 128)
      NH_TRY((launch_tc<false, 128, 6>(c, dev, st)));
    else
      NH_TRY((launch_tc<false, 256, 4>(c, dev, st)));
  } else {
    dim3 grid((unsigned)((T + RT_BT - 1) / RT_BT), (unsigned)((p.E + RT_BE - 1) / RT_BE));
    if (p.bf16)
      NH_TRY((launch_k("router_logits_tiled", router_logits_tiled<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, 
          static_cast<const __nv_bfloat16*>(x), w_router, logits, (int)T, p.H, p.E)));
    else
      NH_TRY((launch_k("router_logits_tiled", router_logits_tiled<float>, dim3(grid), dim3(256), 0, st, static_cast<const float*>(x), w_router,
                                                       logits, (int)T, p.H, p.E)));
    NH_TRY(launch_check("router_logits_tiled"));
  }
  NH_TRY((launch_k("router_select", router_select, dim3((unsigned)((T + 7) / 8)), dim3(256), sel_smem, st, a)));
  return launch_check("router_select");
}

nh_status nh_moe_route_noalloc(const nh_moe_config* cfg, int64_t T, const void* x,
                               const float* w_router, const float* bias, int32_t* topk_idx,
                               float* topk_w, void* stream) {
  NH_TRY(validate(cfg));
  if (T < 0) return fail(NH_ERR_INVALID_ARG, "T must be >= 0");
  if (T > NOALLOC_MAX_T)
    return fail(NH_ERR_INVALID_ARG,
                "nh_moe_route_noalloc takes at most %lld tokens (got %lld); use nh_moe_route",
                (long long)NOALLOC_MAX_T, (long long)T);
  // T <= 32 and n_routed_experts <= MAX_E (512) already keep T * E within the
  // scratch today; this check guards the logits block if MAX_E ever grows
  if (T * cfg->n_routed_experts > NOALLOC_MAX_LOGITS)
    return fail(NH_ERR_INVALID_ARG,
                "nh_moe_route_noalloc: T * n_routed_experts = %lld exceeds its fixed scratch of "
                "%lld logits; use nh_moe_route",
                (long long)(T * cfg->n_routed_experts), (long long)NOALLOC_MAX_LOGITS);
  if (T == 0) return NH_OK;
  NH_TRY(check_ptr(x, "x"));
  NH_TRY(check_ptr(w_router, "w_router"));
  NH_TRY(check_ptr(topk_idx, "topk_idx"));
  NH_TRY(check_ptr(topk_w, "topk_w"));
  if (bias) NH_TRY(check_ptr(bias, "e_score_correction_bias"));
  int dev;
  NH_TRY(device_setup(&dev));
  void* scratch;
  NH_TRY(noalloc_scratch(dev, &scratch));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(scratch);
  float* logits = reinterpret_cast<float*>(static_cast<char*>(scratch) + NOALLOC_HEADER);
  // the status word and the completion counter must start at zero each call
  NH_CUDA(cudaMemsetAsync(status, 0, STATUS_BYTES, st));
  SelectArgs a;
  a.logits = logits;
  a.bias = bias;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.status = status;
  a.T = (int)T;
  a.E = cfg->n_routed_experts;
  a.G = cfg->n_group;
  a.tg = cfg->topk_group;
  a.k = cfg->num_experts_per_tok;
  a.norm = cfg->norm_topk_prob;
  a.alpha = cfg->routed_scaling_factor;
  a.group_score = cfg->group_score;
  a.use_sigma = (bias != nullptr) || cfg->group_score == NH_GROUP_SCORE_TOP2;
  const size_t sel_smem = (size_t)8 * 2 * a.E * sizeof(float);
  const int blocks = a.E;
  unsigned int* done = reinterpret_cast<unsigned int*>(status + 3);
  if (cfg->dtype == NH_BF16)
    router_fused_small<__nv_bfloat16><<<blocks, 256, sel_smem, st>>>(
        static_cast<const __nv_bfloat16*>(x), w_router, a, cfg->hidden_size, done);
  else
    router_fused_small<float><<<blocks, 256, sel_smem, st>>>(static_cast<const float*>(x),
                                                              w_router, a, cfg->hidden_size, done);
  return launch_check("router_fused_small (no-alloc)");
}

nh_status nh_moe_permute(const nh_moe_config* cfg, int64_t T, const void* x,
                         const int32_t* topk_idx, const float* topk_w, void* ws, size_t ws_bytes,
                         void* stream) {
  NH_TRY(no_latent(cfg, "nh_moe_permute"));
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  NH_TRY(check_ws(p, ws, ws_bytes));
  int dev;
  NH_TRY(device_setup(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const nh_moe_ws_layout& L = p.lay;
  if (T == 0) {
    NH_CUDA(cudaMemsetAsync(at<int32_t>(ws, L.num_tiles), 0, 4, st));
    return NH_OK;
  }
  NH_TRY(check_ptr(x, "x"));
  NH_TRY(check_ptr(topk_idx, "topk_idx"));
  NH_TRY(check_ptr(topk_w, "topk_w"));
  int* status = at<int>(ws, L.status);
  if (T <= PERM_CHUNK) {
    // decode-sized: the whole permute in one block
    const PermuteOut o = permute_out(ws, L, status);
    const size_t smem = (size_t)(p.E + T * p.k) * sizeof(int);
    if (p.bf16)
      NH_TRY((launch_k("permute_small", permute_small<__nv_bfloat16>, dim3(1), dim3(512), smem, st,
                       topk_idx, topk_w, static_cast<const __nv_bfloat16*>(x), (int)T, p.k, p.E,
                       p.H, o)));
    else
      NH_TRY((launch_k("permute_small", permute_small<float>, dim3(1), dim3(512), smem, st,
                       topk_idx, topk_w, static_cast<const float*>(x), (int)T, p.k, p.E, p.H, o)));
    return NH_OK;
  }
  int32_t* chunk = at<int32_t>(ws, L.chunk_counts);
  NH_TRY((launch_k("permute_hist", permute_hist, dim3(L.n_chunks), dim3(256), p.E * sizeof(int), st, topk_idx, (int)T, p.k, p.E, chunk, status)));
  NH_TRY(launch_check("permute_hist"));
  const int scan_threads = ((p.E + 31) / 32) * 32;
  NH_TRY((launch_k("permute_scan", permute_scan, dim3(1), dim3(scan_threads), 0, st, chunk, L.n_chunks, p.E, L.tile_rows,
                                            at<int32_t>(ws, L.counts), at<int32_t>(ws, L.offsets),
                                            at<int4>(ws, L.tiles), at<int32_t>(ws, L.num_tiles),
                                            L.max_tiles,
                                            reinterpret_cast<unsigned int*>(status + SCHED_UP))));
  NH_TRY(launch_check("permute_scan"));
  const size_t smem = (size_t)(p.E + PERM_CHUNK * p.k) * sizeof(int);
  const int gather_blocks = g_sm_count[dev] * 4;
  if (p.bf16) {
    NH_TRY((launch_k("permute_scatter", permute_scatter<__nv_bfloat16>, dim3(L.n_chunks), dim3(32), smem, st, 
        topk_idx, topk_w, static_cast<const __nv_bfloat16*>(x), (int)T, p.k, p.E, p.H, chunk,
        at<int32_t>(ws, L.perm_token), at<float>(ws, L.perm_w), at<int32_t>(ws, L.inv_row),
        at<__nv_bfloat16>(ws, L.x_perm), status, 0)));
    NH_TRY(launch_check("permute_scatter"));
    NH_TRY((launch_k("permute_gather", permute_gather<__nv_bfloat16>, dim3(gather_blocks), dim3(256), 0, st, 
        static_cast<const __nv_bfloat16*>(x), at<int32_t>(ws, L.inv_row), (int)T, p.k, p.H,
        at<__nv_bfloat16>(ws, L.x_perm))));
  } else {
    NH_TRY((launch_k("permute_scatter", permute_scatter<float>, dim3(L.n_chunks), dim3(32), smem, st, 
        topk_idx, topk_w, static_cast<const float*>(x), (int)T, p.k, p.E, p.H, chunk,
        at<int32_t>(ws, L.perm_token), at<float>(ws, L.perm_w), at<int32_t>(ws, L.inv_row),
        at<float>(ws, L.x_perm), status, 0)));
    NH_TRY(launch_check("permute_scatter"));
    NH_TRY((launch_k("permute_gather", permute_gather<float>, dim3(gather_blocks), dim3(256), 0, st, 
        static_cast<const float*>(x), at<int32_t>(ws, L.inv_row), (int)T, p.k, p.H,
        at<float>(ws, L.x_perm))));
  }
  return launch_check("permute_gather");
}

nh_status nh_moe_route_permute(const nh_moe_config* cfg, int64_t T, const void* x,
                               const float* w_router, const float* bias, int32_t* topk_idx,
                               float* topk_w, void* ws, size_t ws_bytes, void* stream) {
  NH_TRY(no_latent(cfg, "nh_moe_route_permute"));
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  NH_TRY(check_ws(p, ws, ws_bytes));
  if (T > ROUTE_PERMUTE_MAX_T || p.E > ROUTE_PERMUTE_MAX_E) {
    NH_TRY(nh_moe_route(cfg, T, x, w_router, bias, topk_idx, topk_w, ws, ws_bytes, stream));
    return nh_moe_permute(cfg, T, x, topk_idx, topk_w, ws, ws_bytes, stream);
  }
  if (T == 0) return nh_moe_permute(cfg, T, x, topk_idx, topk_w, ws, ws_bytes, stream);
  NH_TRY(check_ptr(x, "x"));
  NH_TRY(check_ptr(w_router, "w_router"));
  NH_TRY(check_ptr(topk_idx, "topk_idx"));
  NH_TRY(check_ptr(topk_w, "topk_w"));
  if (bias) NH_TRY(check_ptr(bias, "e_score_correction_bias"));
  int dev;
  NH_TRY(device_setup(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const nh_moe_ws_layout& L = p.lay;
  int* status = at<int>(ws, L.status);
  NH_CUDA(cudaMemsetAsync(status, 0, STATUS_BYTES, st));
  SelectArgs a;
  a.logits = at<float>(ws, L.logits);
  a.bias = bias;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.status = status;
  a.T = (int)T;
  a.E = p.E;
  a.G = p.G;
  a.tg = p.tg;
  a.k = p.k;
  a.norm = cfg->norm_topk_prob;
  a.alpha = cfg->routed_scaling_factor;
  a.group_score = cfg->group_score;
  a.use_sigma = (bias != nullptr) || cfg->group_score == NH_GROUP_SCORE_TOP2;
  const PermuteOut o = permute_out(ws, L, status);
  const size_t smem = (size_t)(16 * p.E + p.E + 3 * T * p.k) * sizeof(float);
  unsigned int* done = reinterpret_cast<unsigned int*>(status + 3);
  if (p.bf16)
    return launch_k("route_permute_small", route_permute_small<__nv_bfloat16>, dim3(p.E), dim3(256),
                    smem, st, static_cast<const __nv_bfloat16*>(x), w_router, a, p.H, done, o);
  return launch_k("route_permute_small", route_permute_small<float>, dim3(p.E), dim3(256), smem, st,
                  static_cast<const float*>(x), w_router, a, p.H, done, o);
}

// GemmCall of one routed projection on the workspace: up (x -> h, relu^2) or
// down (h -> y_acc, the weighted combine)
static GemmCall routed_call(const Plan& p, void* ws, int64_t T, const void* x, const void* w,
                            float* y_acc, bool up_phase, bool nvfp4) {
  const nh_moe_ws_layout& L = p.lay;
  GemmCall c{};
  c.rows = p.rows;
  c.n_exp = p.E;
  c.tiles = at<int4>(ws, L.tiles);
  c.num_tiles = at<int32_t>(ws, L.num_tiles);
  c.max_tiles = L.max_tiles;
  c.tile_rows = L.tile_rows;
  c.swap = L.swap_ab;
  c.status = at<int>(ws, L.status);
  c.sched = reinterpret_cast<unsigned int*>(c.status + (up_phase ? SCHED_UP : SCHED_DOWN));
  c.W = w;
  if (up_phase) {
    if (L.x_direct) {
      // decode: the activation tile is x itself; rows map to tokens by perm_token
      c.A = x;
      c.rows = T;
      c.row_token = at<int32_t>(ws, L.perm_token);
    } else {
      c.A = at<void>(ws, L.x_perm);
    }
    c.N = p.I;
    c.K = p.H;
    c.epi = EPI_UP_RELU2;
    c.out = at<void>(ws, L.h);
    c.ldo = p.I;
  } else {
    // the weighted combine: y_acc[perm_token[r]] += perm_w[r] * (h[r] W_down[e]^T)
    c.A = at<void>(ws, L.h);
    c.N = p.H;
    c.K = p.I;
    c.epi = EPI_DOWN_COMBINE;
    c.out = y_acc;
    c.ldo = p.H;
    c.perm_w = at<float>(ws, L.perm_w);
    c.dst_row = at<int32_t>(ws, L.perm_token);
    // decode tiles stream an expert's weights for a few tokens: two K slices
    // per output block halve a tile's length (finer load balance at the end);
    // the combine adds both slices into y_acc
    if (L.swap_ab && !nvfp4 && p.I >= 2 * tc::BK) c.k_split = 2;
  }
  return c;
}

static nh_status experts_phase(const nh_moe_config* cfg, int64_t T, const void* x, const void* w,
                               void* ws, size_t ws_bytes, float* y_acc, void* stream,
                               bool up_phase, const nh_nvfp4_weight* wq = nullptr) {
  NH_TRY(no_latent(cfg, "routed experts"));
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  NH_TRY(check_ws(p, ws, ws_bytes));
  const bool nvfp4 = cfg->weight_format == NH_WEIGHTS_NVFP4;
  if (nvfp4 != (wq != nullptr))
    return fail(NH_ERR_INVALID_ARG, nvfp4 ? "config has NVFP4 weights: use the _nvfp4 entry points"
                                          : "config has native weights: use nh_moe_forward");
  if (T == 0) return NH_OK;
  if (!nvfp4) NH_TRY(check_ptr(w, up_phase ? "w_up" : "w_down"));
  if (up_phase) NH_TRY(check_ptr(x, "x"));
  else NH_TRY(check_ptr(y_acc, "y_acc"));
  int dev;
  NH_TRY(device_setup(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const GemmCall c = routed_call(p, ws, T, x, w, y_acc, up_phase, nvfp4);
  if (nvfp4) return run_gemm_q4(c, wq, dev, st);
  return run_gemm(p, c, dev, st);
}

nh_status nh_moe_experts_up(const nh_moe_config* cfg, int64_t T, const void* x, const void* w_up,
                            void* ws, size_t ws_bytes, void* stream) {
  return experts_phase(cfg, T, x, w_up, ws, ws_bytes, nullptr, stream, true);
}

nh_status nh_moe_experts_down(const nh_moe_config* cfg, int64_t T, const void* w_down, void* ws,
                              size_t ws_bytes, float* y_acc, void* stream) {
  return experts_phase(cfg, T, nullptr, w_down, ws, ws_bytes, y_acc, stream, false);
}

nh_status nh_moe_forward(const nh_moe_config* cfg, int64_t T, const void* x, const void* w_up,
                         const void* w_down, void* ws, size_t ws_bytes, float* y_acc,
                         void* stream) {
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  NH_TRY(check_ws(p, ws, ws_bytes));
  if (T == 0) return NH_OK;
  NH_TRY(check_ptr(x, "x"));
  NH_TRY(check_ptr(w_up, "w_up"));
  NH_TRY(check_ptr(w_down, "w_down"));
  NH_TRY(check_ptr(y_acc, "y_acc"));
  const nh_moe_ws_layout& L = p.lay;
  if (p.bf16 && L.x_direct && cfg->weight_format == NH_WEIGHTS_NATIVE && !cfg->latent_size &&
      (L.tile_rows == 16 || L.tile_rows == 32)) {
    // decode: both projections in one persistent launch
    int dev;
    NH_TRY(device_setup(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const GemmCall up = routed_call(p, ws, T, x, w_up, y_acc, true, false);
    const GemmCall down = routed_call(p, ws, T, x, w_down, y_acc, false, false);
    int* ready = at<int>(ws, L.ready);
    if (L.tile_rows == 16) return launch_tc_fused<16, 8>(up, down, ready, dev, st);
    return launch_tc_fused<32, 8>(up, down, ready, dev, st);
  }
  NH_TRY(nh_moe_experts_up(cfg, T, x, w_up, ws, ws_bytes, stream));
  return nh_moe_experts_down(cfg, T, w_down, ws, ws_bytes, y_acc, stream);
}

nh_status nh_moe_forward_nvfp4(const nh_moe_config* cfg, int64_t T, const void* x,
                               const nh_nvfp4_weight* w_up, const nh_nvfp4_weight* w_down,
                               void* ws, size_t ws_bytes, float* y_acc, void* stream) {
  if (!w_up || !w_down) return fail(NH_ERR_INVALID_ARG, "w_up / w_down is NULL");
  if (T > 0) NH_TRY(check_ptr(y_acc, "y_acc"));
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  const nh_moe_ws_layout& L = p.lay;
  if (T > 0 && cfg->weight_format == NH_WEIGHTS_NVFP4 && !cfg->latent_size && L.x_direct &&
      (L.tile_rows == 16 || L.tile_rows == 32)) {
    // decode: both projections in one launch of the rows GEMV
    NH_TRY(check_ws(p, ws, ws_bytes));
    NH_TRY(check_ptr(x, "x"));
    NH_TRY(check_q4(w_up));
    NH_TRY(check_q4(w_down));
    int dev;
    NH_TRY(device_setup(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const GemmCall up = routed_call(p, ws, T, x, nullptr, y_acc, true, true);
    const GemmCall down = routed_call(p, ws, T, x, nullptr, y_acc, false, true);
    int* ready = at<int>(ws, L.ready);
    if (L.tile_rows == 16) return launch_q4v_fused<16>(up, *w_up, down, *w_down, ready, dev, st);
    return launch_q4v_fused<32>(up, *w_up, down, *w_down, ready, dev, st);
  }
  NH_TRY(experts_phase(cfg, T, x, nullptr, ws, ws_bytes, nullptr, stream, true, w_up));
  return experts_phase(cfg, T, x, nullptr, ws, ws_bytes, y_acc, stream, false, w_down);
}

static nh_status shared_impl(const nh_moe_config* cfg, int64_t T, const void* x, const void* w_su,
                             const void* w_sd, const nh_nvfp4_weight* q_su,
                             const nh_nvfp4_weight* q_sd, float* y_acc, void* ws_shared,
                             size_t ws_shared_bytes, void* stream, bool store = false);

nh_status nh_moe_shared_nvfp4(const nh_moe_config* cfg, int64_t T, const void* x,
                              const nh_nvfp4_weight* w_su, const nh_nvfp4_weight* w_sd,
                              float* y_acc, void* ws_shared, size_t ws_shared_bytes,
                              void* stream) {
  if (!w_su || !w_sd) return fail(NH_ERR_INVALID_ARG, "w_shared_up / w_shared_down is NULL");
  return shared_impl(cfg, T, x, nullptr, nullptr, w_su, w_sd, y_acc, ws_shared,
                     ws_shared_bytes, stream);
}

nh_status nh_moe_shared(const nh_moe_config* cfg, int64_t T, const void* x, const void* w_su,
                        const void* w_sd, float* y_acc, void* ws_shared, size_t ws_shared_bytes,
                        void* stream) {
  return shared_impl(cfg, T, x, w_su, w_sd, nullptr, nullptr, y_acc, ws_shared,
                     ws_shared_bytes, stream);
}

nh_status nh_moe_shared_store(const nh_moe_config* cfg, int64_t T, const void* x,
                              const void* w_su, const void* w_sd, float* y_acc, void* ws_shared,
                              size_t ws_shared_bytes, void* stream) {
  return shared_impl(cfg, T, x, w_su, w_sd, nullptr, nullptr, y_acc, ws_shared,
                     ws_shared_bytes, stream, true);
}

static nh_status shared_impl(const nh_moe_config* cfg, int64_t T, const void* x, const void* w_su,
                             const void* w_sd, const nh_nvfp4_weight* q_su,
                             const nh_nvfp4_weight* q_sd, float* y_acc, void* ws_shared,
                             size_t ws_shared_bytes, void* stream, bool store) {
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  const bool nvfp4 = cfg->weight_format == NH_WEIGHTS_NVFP4;
  if (nvfp4 != (q_su != nullptr))
    return fail(NH_ERR_INVALID_ARG, nvfp4 ? "config has NVFP4 weights: use nh_moe_shared_nvfp4"
                                          : "config has native weights: use nh_moe_shared");
  size_t need;
  NH_TRY(nh_moe_shared_workspace_size(cfg, T, &need));
  NH_TRY(check_ptr(ws_shared, "ws_shared"));
  if (ws_shared_bytes < need)
    return fail(NH_ERR_INVALID_ARG, "ws_shared holds %zu bytes, %zu needed", ws_shared_bytes, need);
  if (T == 0) return NH_OK;
  NH_TRY(check_ptr(x, "x"));
  if (!nvfp4) {
    NH_TRY(check_ptr(w_su, "w_shared_up"));
    NH_TRY(check_ptr(w_sd, "w_shared_down"));
  }
  NH_TRY(check_ptr(y_acc, "y_acc"));
  int dev;
  NH_TRY(device_setup(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws_shared);
  void* h = static_cast<char*>(ws_shared) + ALIGN;
  NH_CUDA(cudaMemsetAsync(status, 0, STATUS_BYTES, st));
  GemmCall up{};
  up.A = x;
  up.rows = T;
  up.W = w_su;
  up.n_exp = 1;
  up.N = p.S;
  up.K = p.H;
  up.tiles = nullptr;
  up.tile_rows = p.lay.tile_rows;
  up.swap = p.lay.swap_ab;
  up.epi = EPI_UP_RELU2;
  up.out = h;
  up.ldo = p.S;
  up.status = status;
  up.sched = reinterpret_cast<unsigned int*>(status + 4);
  if (nvfp4) NH_TRY(run_gemm_q4(up, q_su, dev, st));
  else NH_TRY(run_gemm(p, up, dev, st));
  GemmCall dn = up;
  dn.A = h;
  dn.W = w_sd;
  dn.N = p.H;
  dn.K = p.S;
  // y_acc += shared expert, beside the routed combine; or y_acc = shared
  // expert, the accumulator's starting value (each element is written once)
  dn.epi = store ? EPI_STORE_F32 : EPI_ACC_F32;
  dn.out = y_acc;
  dn.ldo = p.H;
  dn.sched = reinterpret_cast<unsigned int*>(status + 6);
  if (nvfp4) return run_gemm_q4(dn, q_sd, dev, st);
  return run_gemm(p, dn, dev, st);
}

nh_status nh_moe_zero_acc(const nh_moe_config* cfg, int64_t T, float* y_acc, void* stream) {
  NH_TRY(validate(cfg));
  if (T < 0) return fail(NH_ERR_INVALID_ARG, "T must be >= 0");
  if (T == 0) return NH_OK;
  NH_TRY(check_ptr(y_acc, "y_acc"));
  NH_CUDA(cudaMemsetAsync(y_acc, 0, (size_t)T * cfg->hidden_size * sizeof(float),
                          static_cast<cudaStream_t>(stream)));
  return NH_OK;
}

// y = dtype(y_acc): the one rounding of the block output
nh_status nh_moe_finalize(const nh_moe_config* cfg, int64_t T, const float* y_acc, void* y,
                          void* stream) {
  NH_TRY(validate(cfg));
  if (T < 0) return fail(NH_ERR_INVALID_ARG, "T must be >= 0");
  if (T == 0) return NH_OK;
  NH_TRY(check_ptr(y_acc, "y_acc"));
  NH_TRY(check_ptr(y, "y"));
  int dev;
  NH_TRY(device_setup(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t n = T * (int64_t)cfg->hidden_size;
  if (cfg->dtype == NH_BF16 && n % 8 == 0) {
    NH_TRY((launch_k("cast_output_bf16x8", cast_output_bf16x8, dim3(grid_for(n / 8, 256, dev)),
                     dim3(256), 0, st, reinterpret_cast<const float4*>(y_acc),
                     static_cast<uint4*>(y), n / 8)));
  } else if (cfg->dtype == NH_BF16) {
    NH_TRY((launch_k("cast_output", cast_output<__nv_bfloat16>, dim3(grid_for(n, 256, dev)),
                     dim3(256), 0, st, y_acc, static_cast<__nv_bfloat16*>(y), n)));
  } else {
    NH_TRY((launch_k("cast_output", cast_output<float>, dim3(grid_for(n, 256, dev)), dim3(256), 0,
                     st, y_acc, static_cast<float*>(y), n)));
  }
  return launch_check("cast_output");
}

// ---------------------------------------------------------------------------
// latent projections around the routed experts
// ---------------------------------------------------------------------------
nh_status nh_moe_latent_config(const nh_moe_config* cfg, nh_moe_config* expert_cfg) {
  NH_TRY(validate(cfg));
  if (!expert_cfg) return fail(NH_ERR_INVALID_ARG, "expert_cfg is NULL");
  if (cfg->latent_size < 1) return fail(NH_ERR_INVALID_ARG, "config has no latent projections");
  *expert_cfg = *cfg;
  expert_cfg->hidden_size = cfg->latent_size;
  expert_cfg->latent_size = 0;
  expert_cfg->n_shared_experts = 0;
  return validate(expert_cfg);
}

nh_status nh_moe_latent_workspace_size(const nh_moe_config* cfg, int64_t T, size_t* bytes) {
  if (!bytes) return fail(NH_ERR_INVALID_ARG, "bytes is NULL");
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  if (cfg->latent_size < 1) return fail(NH_ERR_INVALID_ARG, "config has no latent projections");
  *bytes = ALIGN;   // status word and tile scheduler counters
  return NH_OK;
}

// out = x W^T for one projection: fc1 (H -> L, EPI_STORE) or fc2 (L -> H, EPI_ADD_F32)
static nh_status latent_gemm(const nh_moe_config* cfg, int64_t T, const void* a, const void* w,
                             void* out, bool fc1, void* ws, size_t ws_bytes, void* stream) {
  Plan p;
  NH_TRY(make_plan(cfg, T, &p));
  if (cfg->latent_size < 1) return fail(NH_ERR_INVALID_ARG, "config has no latent projections");
  NH_TRY(check_ptr(ws, "ws_latent"));
  if (ws_bytes < ALIGN)
    return fail(NH_ERR_INVALID_ARG, "ws_latent holds %zu bytes, %zu needed", ws_bytes, ALIGN);
  if (T == 0) return NH_OK;
  NH_TRY(check_ptr(a, fc1 ? "x" : "y_lat"));
  NH_TRY(check_ptr(w, fc1 ? "w_latent_fc1" : "w_latent_fc2"));
  NH_TRY(check_ptr(out, fc1 ? "x_lat" : "y_acc"));
  int dev;
  NH_TRY(device_setup(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(ws);
  NH_CUDA(cudaMemsetAsync(status, 0, STATUS_BYTES, st));
  // the projections are dense layers in the activation dtype: plan their tiles
  // as native-format weights
  nh_moe_config cn = *cfg;
  cn.weight_format = NH_WEIGHTS_NATIVE;
  int tr, sw;
  tile_plan(&cn, T, &tr, &sw);
  const int L = cfg->latent_size;
  GemmCall g{};
  g.A = a;
  g.rows = T;
  g.W = w;
  g.n_exp = 1;
  g.N = fc1 ? L : p.H;
  g.K = fc1 ? p.H : L;
  g.tiles = nullptr;
  g.tile_rows = tr;
  g.swap = sw;
  // fc2 adds onto y_acc (the shared expert's output, or zeros): one owner per
  // element, ordered after the shared expert by the caller
  g.epi = fc1 ? EPI_STORE : EPI_ADD_F32;
  g.out = out;
  g.ldo = g.N;
  g.status = status;
  g.sched = reinterpret_cast<unsigned int*>(status + 4);
  return run_gemm(p, g, dev, st);
}

nh_status nh_moe_latent_in(const nh_moe_config* cfg, int64_t T, const void* x,
                           const void* w_latent_fc1, void* x_lat, void* ws_latent,
                           size_t ws_latent_bytes, void* stream) {
  return latent_gemm(cfg, T, x, w_latent_fc1, x_lat, true, ws_latent, ws_latent_bytes, stream);
}

nh_status nh_moe_latent_out(const nh_moe_config* cfg, int64_t T, const void* y_lat,
                            const void* w_latent_fc2, float* y_acc, void* ws_latent,
                            size_t ws_latent_bytes, void* stream) {
  return latent_gemm(cfg, T, y_lat, w_latent_fc2, y_acc, false, ws_latent, ws_latent_bytes,
                     stream);
}

nh_status nh_moe_reset_status(void* ws, void* stream) {
  NH_TRY(check_ptr(ws, "ws"));
  NH_CUDA(cudaMemsetAsync(ws, 0, STATUS_BYTES, static_cast<cudaStream_t>(stream)));
  return NH_OK;
}

nh_status nh_moe_check_device(void* ws, void* stream) {
  NH_TRY(check_ptr(ws, "ws"));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  NH_CUDA(cudaStreamSynchronize(st));
  int h[4] = {0, 0, 0, 0};
  NH_CUDA(cudaMemcpy(h, ws, sizeof h, cudaMemcpyDeviceToHost));
  if (h[0] == NH_ERR_TIMEOUT)
    return fail(NH_ERR_TIMEOUT, "device wait ran out (site %d, value %d)", h[1], h[2]);
  if (h[0] == NH_ERR_DEVICE_CHECK)
    return fail(NH_ERR_DEVICE_CHECK, "device check failed (site %d, value %d)", h[1], h[2]);
  if (h[0] != 0) return fail((nh_status)h[0], "device status %d (site %d)", h[0], h[1]);
  return NH_OK;
}

nh_status nh_moe_selftest_timeout(void* ws, uint64_t timeout, void* stream) {
  NH_TRY(check_ptr(ws, "ws"));
  if (timeout == 0 || timeout > 10000000000ull)
    return fail(NH_ERR_INVALID_ARG, "timeout_ns must be in (0, 1e10]");
  int dev;
  NH_TRY(device_setup(&dev));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  NH_CUDA(cudaMemsetAsync(ws, 0, 16, st));
  selftest_timeout_kernel<<<1, 32, 0, st>>>(static_cast<int*>(ws), timeout);
  return launch_check("selftest_timeout");
}

}  // extern "C"

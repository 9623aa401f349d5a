/*
 * nh_moe.h -- C ABI of the B200 (sm_100a) Nemotron-H non-gated MoE block.
 *
 * The MoE block of Nemotron-H (`NemotronHMoE(config)`, `__call__(x) -> y`,
 * exo commit "Add support for Nemotron sharding", nemotron_h.pyi) is
 *
 *   y = sum_{j<k} w_j * down_e_j( relu( up_e_j(x) )^2 )  +  shared_down( relu( shared_up(x) )^2 )
 *
 * with (e_j, w_j) chosen per token by a grouped top-k sigmoid router and
 * experts that have no gate_proj ("Non-gated MoE", vllm.cpp PR #518; baseRT
 * issue #46, "Architecture (config.json)"; expert shapes in the auto-round PR
 * #1712 log).  One block call is, in stream order:
 *
 *   stream B:  nh_moe_zero_acc -> nh_moe_shared --------------------------+
 *   stream A:  nh_moe_route -> nh_moe_permute -> nh_moe_forward ----------+-> nh_moe_finalize
 *              (nh_moe_forward's down projection after nh_moe_zero_acc)
 *
 * The routed experts' down projection adds each token's k weighted expert
 * outputs straight into a float32 accumulator y_acc [T, H] (float32 atomic
 * adds in the GEMM epilogue), the shared expert adds its output into the
 * same y_acc, and nh_moe_finalize rounds y_acc once to the dtype of x.
 *
 * Conventions (every entry point):
 *   - All pointers named x, w_*, topk_*, y*, ws* are DEVICE pointers of the
 *     current CUDA device; `cfg` and `out`-structs are HOST pointers.
 *   - Arrays are dense row-major; weights use the PyTorch Linear layout
 *     [out_features, in_features].  Device pointers must be 16-byte aligned.
 *   - The caller owns every buffer and stream.  The library allocates no
 *     device memory and keeps no state across calls except a thread-local
 *     error string and per-device caches of kernel attributes.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work; nothing synchronises the host.
 *   - Errors: a non-NH_OK status is returned and nh_last_error() describes
 *     it; nothing is enqueued when an argument check fails.  Faults found on
 *     the device (bounded waits that ran out, index checks) are recorded in
 *     the workspace status word and read back by nh_moe_check_device.
 *   - dtype NH_BF16: x, expert weights and y are bf16 (uint16 bit patterns);
 *     the tensor-core path needs hidden_size, moe_intermediate_size and
 *     moe_shared_expert_intermediate_size to be multiples of 64, else the
 *     call returns NH_ERR_UNSUPPORTED.  dtype NH_F32: everything float32,
 *     any size.  The router weight and all accumulation are float32.
 */
#ifndef NH_MOE_H
#define NH_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NH_OK = 0,
    NH_ERR_INVALID_ARG = 1,   /* config or argument fails validation            */
    NH_ERR_UNSUPPORTED = 2,   /* valid, but outside what the kernels implement  */
    NH_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed              */
    NH_ERR_TIMEOUT = 4,       /* a bounded device-side wait ran out             */
    NH_ERR_DEVICE_CHECK = 5   /* a device-side index/shape check failed         */
} nh_status;

typedef enum { NH_F32 = 0, NH_BF16 = 1 } nh_dtype;

/* Group score of the router's group stage. */
typedef enum {
    NH_GROUP_SCORE_MAX = 0,   /* max selection score of the group's experts */
    NH_GROUP_SCORE_TOP2 = 1   /* sum of the two largest (needs >= 2 experts per group) */
} nh_group_score;

/* Storage of the routed and shared expert weights. */
typedef enum {
    NH_WEIGHTS_NATIVE = 0,    /* in the activation dtype (bf16 or float32)          */
    NH_WEIGHTS_NVFP4 = 1      /* NVFP4, see nh_nvfp4_weight (needs dtype NH_BF16)   */
} nh_weight_format;

/*
 * One stacked NVFP4 weight tensor [n_mat][rows][cols] (W4A16, group size 16:
 * vllm.cpp PR #518 names this storage for the checkpoint's routed and shared
 * expert weights).  Element (m, r, c) = e2m1(code) * e4m3(scale) * global[m] where
 *   codes  [n_mat][rows][cols/2]: two E2M1 codes per byte, column 2j in the
 *          low nibble of byte j;
 *   scales [n_mat][rows][pitch]: E4M3 scale of columns 16b .. 16b+15 in byte
 *          b; pitch = ceil(cols/16) rounded up to a multiple of 16 bytes;
 *   global [n_mat]: float32.
 * All three are device pointers, 16-byte aligned.  The struct itself is a
 * host struct.
 */
typedef struct {
    const uint8_t *codes;
    const uint8_t *scales;
    const float *global_scale;
} nh_nvfp4_weight;

/*
 * Block configuration.  Field names are the model's config.json / MLX
 * ModelArgs names (exo commit "Add support for Nemotron sharding",
 * nemotron_h.pyi, ModelArgs.moe_intermediate_size .. routed_scaling_factor).
 * `n_group` is the router's group count, which the baseRT issue #46 summary
 * writes as "n_groups=8" (in ModelArgs, n_groups is the Mamba-2 field).
 */
typedef struct {
    int32_t hidden_size;                          /* H                            */
    int32_t n_routed_experts;                     /* E, at most 512               */
    int32_t n_group;                              /* G, E % G == 0                */
    int32_t topk_group;                           /* tg, 1 <= tg <= G             */
    int32_t num_experts_per_tok;                  /* k, 1 <= k <= tg * E / G, <= 32 */
    int32_t moe_intermediate_size;                /* I                            */
    int32_t moe_shared_expert_intermediate_size;  /* S (ignored if no shared)     */
    int32_t n_shared_experts;                     /* 0 or 1                       */
    int32_t norm_topk_prob;                       /* bool                         */
    float routed_scaling_factor;                  /* alpha, finite                */
    int32_t dtype;                                /* nh_dtype                     */
    int32_t group_score;                          /* nh_group_score               */
    int32_t weight_format;                        /* nh_weight_format             */
    int32_t latent_size;                          /* L: 0, or the routed experts'
                                                     width between the latent
                                                     projections (see
                                                     nh_moe_latent_in)           */
} nh_moe_config;

/* Byte offsets of the regions inside the routed-path workspace `ws`. */
typedef struct {
    size_t total_bytes;
    size_t status;        /* int32[16]: status, site, value, scheduler counters */
    size_t logits;        /* float [T, E] router logits                         */
    size_t router_w;      /* bf16 [E, 3H] router weight as three bf16 planes    */
    size_t counts;        /* int32 [E] assignments per expert                   */
    size_t offsets;       /* int32 [E + 1] exclusive scan of counts             */
    size_t chunk_counts;  /* int32 [n_chunks, E] per-chunk histograms           */
    size_t perm_token;    /* int32 [T * k] token of each permuted row           */
    size_t perm_w;        /* float [T * k] routing weight of each permuted row  */
    size_t inv_row;       /* int32 [T, k] permuted row of assignment (t, j)     */
    size_t tiles;         /* int32 [max_tiles, 4] (expert, first row, rows,
                             kind: 1 = an expert's partial last tile of the
                             CTA-pair GEMM, computed with weights on M)        */
    size_t num_tiles;     /* int32 [1] number of valid tile entries             */
    size_t x_perm;        /* dtype [rows_alloc, H] x gathered in permuted order
                             (empty when x_direct: the GEMM reads x itself)   */
    size_t h;             /* dtype [rows_alloc, I] relu^2(up) in permuted order */
    size_t ready;         /* int32 [max_tiles] per tile entry: up-projection tiles
                             finished, when nh_moe_forward runs both projections
                             of a decode batch as one launch; zero between
                             launches (the permute zeroes it, and each such
                             launch leaves it zero)                            */
    int64_t rows_alloc;   /* T * k rounded up to the tile height                */
    int32_t tile_rows;    /* rows per tile entry of this (cfg, T)               */
    int32_t max_tiles;
    int32_t n_chunks;     /* token chunks of the permute histogram              */
    int32_t swap_ab;      /* 1: weights on the MMA M side (small T, or NVFP4)   */
    int32_t x_direct;     /* 1: the up projection reads x itself (no x_perm)    */
} nh_moe_ws_layout;

/* Validate a configuration (no device work). */
nh_status nh_moe_validate(const nh_moe_config *cfg);

/* Size of the routed-path workspace for T tokens (T >= 0). */
nh_status nh_moe_workspace_size(const nh_moe_config *cfg, int64_t T, size_t *bytes);

/* Region offsets of the routed-path workspace (for inspection and tests). */
nh_status nh_moe_workspace_layout(const nh_moe_config *cfg, int64_t T, nh_moe_ws_layout *out);

/* Size of the shared-expert workspace (relu^2 hidden [T, S] in dtype). */
nh_status nh_moe_shared_workspace_size(const nh_moe_config *cfg, int64_t T, size_t *bytes);

/*
 * Router: logits l = x Wr^T (float32 accumulate), scores s = sigmoid(l),
 * selection score s + e_score_correction_bias (bias may be NULL = 0; with
 * no bias and the max group score the selection runs on the logits, which
 * the sigmoid orders identically), group score, topk_group groups kept,
 * top-k experts among them, ties to the lower group / expert id, output in
 * (score desc, id asc) order; weights alpha * s_j / sum s (norm_topk_prob)
 * or alpha * s_j, from the unbiased s.  (baseRT issue #46 MoE summary;
 * ModelArgs.n_group .. routed_scaling_factor; the router correction bias is
 * a float32 tensor of the checkpoint, auto-round PR #1712.)
 *   x [T, H] dtype; w_router [E, H] float32; bias [E] float32 or NULL;
 *   topk_idx [T, k] int32 (out); topk_w [T, k] float32 (out);
 *   ws / ws_bytes: routed-path workspace (holds the status word and logits).
 * The status word is cleared here: nh_moe_route starts a block call.
 */
nh_status nh_moe_route(const nh_moe_config *cfg, int64_t T, const void *x, const float *w_router,
                       const float *e_score_correction_bias, int32_t *topk_idx, float *topk_w,
                       void *ws, size_t ws_bytes, void *stream);

/*
 * nh_moe_route followed by nh_moe_permute, as one call with the same
 * arguments and results (topk_idx / topk_w written, workspace filled for
 * nh_moe_forward).  For T <= 32 and n_routed_experts <= 256 both run in a
 * single kernel: the block that finishes the router logits last selects every
 * token and then permutes the routing it produced; otherwise it makes the two
 * calls.
 */
nh_status nh_moe_route_permute(const nh_moe_config *cfg, int64_t T, const void *x,
                               const float *w_router, const float *e_score_correction_bias,
                               int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes,
                               void *stream);

/*
 * nh_moe_route_noalloc: the router of nh_moe_route for decode-sized batches,
 * for callers that cannot allocate device memory or pass a workspace: serving
 * stacks whose memory pool has already claimed the device's free memory, and
 * plugin hosts that hand an op its inputs and outputs but no scratch buffer
 * and whose op code may not call cudaMalloc (it is not stream-ordered and can
 * synchronise the device).  None of the cited sources has such a call: it is
 * a packaging choice of this library.
 *   Same arguments and results as nh_moe_route, without ws / ws_bytes.
 *   Limits: T <= 32 and T * n_routed_experts <= 16384; larger sizes return
 *   NH_ERR_INVALID_ARG with a message naming the limit (use nh_moe_route).
 *   Scratch: a fixed 64 KiB + 256 B array compiled into the library, held by
 *   every device that loads it until the process exits.  Nothing is
 *   allocated: no cudaMalloc / cudaFree, no allocating library call.
 *   The first call on a device looks up that array's device address (a
 *   one-time set-up per device); make that first call before any stream
 *   capture.  The array is shared by all calls on a device and keeps the last
 *   call's contents; each call clears its status word and counter first.
 *   Calls that overlap on the GPU (different streams, no ordering) race on
 *   that array: order them on one stream.  Device-side status of these calls
 *   is not reported through nh_moe_check_device.
 */
nh_status nh_moe_route_noalloc(const nh_moe_config *cfg, int64_t T, const void *x,
                               const float *w_router, const float *e_score_correction_bias,
                               int32_t *topk_idx, float *topk_w, void *stream);

/*
 * Token permute: per-expert histogram, exclusive scan, stable scatter of the
 * (t, j) assignments in (t, j) order, the tile table of the expert GEMMs and
 * (unless the layout's x_direct is set) the gather
 * x_perm[row] = x[perm_token[row]].  It also zeroes the layout's `ready`
 * counters and the expert GEMMs' tile schedulers.  The routed experts are
 * applied per expert id (MLX SwitchMLP fc1/fc2 indexed by the router's
 * expert ids, exo commit "Add support for Nemotron sharding").
 *   topk_idx / topk_w as produced by nh_moe_route (any valid ids in [0, E)
 *   are accepted; an id out of range sets NH_ERR_DEVICE_CHECK on the device).
 */
nh_status nh_moe_permute(const nh_moe_config *cfg, int64_t T, const void *x,
                         const int32_t *topk_idx, const float *topk_w, void *ws, size_t ws_bytes,
                         void *stream);

/*
 * Routed experts with the weighted combine (exo commit "Add support for
 * Nemotron sharding": switch_layers.pyi SwitchMLP fc1 / fc2 per expert id,
 * and nemotron_h.pyi NemotronHMoE.__call__, which sums the k experts of a
 * token weighted by the router):
 *   h[r] = relu(x[perm_token[r]] W_up[e]^T)^2      (float32 accumulate, h in
 *                                                   dtype, in the workspace)
 *   y_acc[perm_token[r]] += perm_w[r] * (h[r] W_down[e]^T)      (float32)
 * for every permuted row r of expert e.  The adds are float32 atomic adds
 * issued by the down projection's epilogue, so the order in which a token's
 * k contributions (and the shared expert's) are summed is not fixed: results
 * can differ between runs in the last float32 bits.
 *   x [T, H] dtype (the same x that nh_moe_permute saw); w_up [E, I, H] dtype;
 *   w_down [E, H, I] dtype; y_acc [T, H] float32, read and added to: it must
 *   hold its starting value (zeros from nh_moe_zero_acc, optionally plus the
 *   shared expert) before the down projection runs, and no other stream may
 *   write it meanwhile except nh_moe_shared's adds.
 * Needs nh_moe_permute's workspace contents.  For bf16 batches of at most 32
 * tokens both projections run as one launch (down tiles of a tile entry start
 * once its up tiles have stored h); larger batches take one launch each.  The
 * call may be repeated after one permute.
 */
nh_status nh_moe_forward(const nh_moe_config *cfg, int64_t T, const void *x, const void *w_up,
                         const void *w_down, void *ws, size_t ws_bytes, float *y_acc,
                         void *stream);

/*
 * nh_moe_forward with NVFP4 routed-expert weights (cfg->weight_format ==
 * NH_WEIGHTS_NVFP4): w_up [E][I][H], w_down [E][H][I] as nh_nvfp4_weight.
 * Each weight is dequantized in registers (code x block scale, exact in
 * bf16): for tiles of up to 32 tokens per expert straight into warp-level MMA
 * fragments, for 64-token tiles into tensor memory as the A operand of
 * tcgen05.mma.  The float32 matrix scale is applied in the epilogue.  Adds
 * into y_acc exactly like nh_moe_forward; batches of at most 32 tokens run
 * both projections as one launch, as there.
 */
nh_status nh_moe_forward_nvfp4(const nh_moe_config *cfg, int64_t T, const void *x,
                               const nh_nvfp4_weight *w_up, const nh_nvfp4_weight *w_down,
                               void *ws, size_t ws_bytes, float *y_acc, void *stream);

/*
 * The two phases of nh_moe_forward, for callers that schedule or time them
 * separately (same arguments and requirements):
 *   nh_moe_experts_up:   h = relu(x[perm_token] W_up[e]^T)^2 into the workspace;
 *   nh_moe_experts_down: y_acc[perm_token[r]] += perm_w[r] * (h[r] W_down[e]^T).
 */
nh_status nh_moe_experts_up(const nh_moe_config *cfg, int64_t T, const void *x, const void *w_up,
                            void *ws, size_t ws_bytes, void *stream);
nh_status nh_moe_experts_down(const nh_moe_config *cfg, int64_t T, const void *w_down, void *ws,
                              size_t ws_bytes, float *y_acc, void *stream);

/*
 * Shared expert (NemotronHMLP up_proj / down_proj, always on, unscaled; exo
 * commit "Add support for Nemotron sharding", nemotron_h.pyi):
 *   y_acc += relu(x W_su^T)^2 W_sd^T      (float32 atomic adds)
 *   w_shared_up [S, H]; w_shared_down [H, S] (dtype); y_acc [T, H] float32,
 *   the accumulator nh_moe_forward adds into; ws_shared:
 *   nh_moe_shared_workspace_size bytes.
 * Independent of the routed path: may run on a second stream, concurrently
 * with nh_moe_forward, once y_acc holds its starting value.
 */
nh_status nh_moe_shared(const nh_moe_config *cfg, int64_t T, const void *x, const void *w_shared_up,
                        const void *w_shared_down, float *y_acc, void *ws_shared,
                        size_t ws_shared_bytes, void *stream);

/*
 * The shared expert as the accumulator's starting value instead of an add:
 *   y_acc = relu(x W_su^T)^2 W_sd^T      (float32 stores, each element once)
 * Same arguments as nh_moe_shared.  It replaces nh_moe_zero_acc plus
 * nh_moe_shared when it completes before any routed add into y_acc (the
 * caller orders them, e.g. nh_moe_experts_down after an event of this call's
 * stream), saving the zero fill and the read half of the shared adds.
 */
nh_status nh_moe_shared_store(const nh_moe_config *cfg, int64_t T, const void *x,
                              const void *w_shared_up, const void *w_shared_down, float *y_acc,
                              void *ws_shared, size_t ws_shared_bytes, void *stream);

/* nh_moe_shared with NVFP4 shared-expert weights: w_shared_up [1][S][H],
 * w_shared_down [1][H][S]. */
nh_status nh_moe_shared_nvfp4(const nh_moe_config *cfg, int64_t T, const void *x,
                              const nh_nvfp4_weight *w_shared_up,
                              const nh_nvfp4_weight *w_shared_down, float *y_acc,
                              void *ws_shared, size_t ws_shared_bytes, void *stream);

/*
 * y_acc = 0: the starting value of the float32 accumulator [T, H] (H =
 * cfg->hidden_size) that nh_moe_shared and nh_moe_forward add into.  An
 * asynchronous memset on `stream`; no kernel.
 */
nh_status nh_moe_zero_acc(const nh_moe_config *cfg, int64_t T, float *y_acc, void *stream);

/*
 * y = dtype(y_acc): the block output, rounded once (float32 dtype: a copy).
 *   y_acc [T, H] float32 after nh_moe_forward and nh_moe_shared; y [T, H]
 *   dtype (out).  H = cfg->hidden_size.
 *
 * Tensor-parallel shards (exo commit "Add support for Nemotron sharding",
 * the NemotronHMoE branch of the sharding strategy: the routed fc1 and the
 * shared up_proj are split over their output features, the routed fc2 and the
 * shared down_proj over their input features, the router is replicated, and
 * one all-reduce sums the block output): a rank runs the whole path with the
 * config of its shard (moe_intermediate_size and
 * moe_shared_expert_intermediate_size set to its share of I and S, each a
 * multiple of 64) and its slices of the weights.  Its y_acc is then its
 * float32 contribution; the caller sums y_acc over the ranks (an all-reduce)
 * and calls nh_moe_finalize on the sum, so the output is rounded once.
 */
nh_status nh_moe_finalize(const nh_moe_config *cfg, int64_t T, const float *y_acc, void *y,
                          void *stream);

/*
 * Latent MoE projections (ModelOpt descriptor NemotronHMoELayerDescriptor:
 * latent_fc1_name='fc1_latent_proj', latent_fc2_name='fc2_latent_proj'; the
 * descriptor names the two modules and gives no formula).  Reading used, with
 * L = cfg->latent_size > 0:
 *   x_lat = dtype(x W_fc1^T)                     W_fc1 [L, H]   (nh_moe_latent_in)
 *   routed experts on x_lat, in width L: W_up [E, I, L], W_down [E, L, I],
 *     routing on x (nh_moe_route with cfg), combined as usual into a zeroed
 *     float32 y_lat_acc [T, L] and rounded to y_lat [T, L] (nh_moe_zero_acc,
 *     nh_moe_forward, nh_moe_finalize with the expert-width config)
 *   y_acc += y_lat W_fc2^T                       W_fc2 [H, L]   (nh_moe_latent_out)
 *     where y_acc holds zeros plus the shared expert (nh_moe_zero_acc and
 *     nh_moe_shared with cfg), complete before this call
 *   y = dtype(y_acc)                                            (nh_moe_finalize)
 * The routed-expert calls (nh_moe_permute, nh_moe_forward[_nvfp4],
 * nh_moe_experts_*) take the expert-width config
 * that nh_moe_latent_config writes (hidden_size = L, latent_size = 0,
 * n_shared_experts = 0) and return NH_ERR_INVALID_ARG for a config with
 * latent_size > 0; nh_moe_route and nh_moe_shared take cfg itself.
 * nh_moe_route needs only the first `counts` bytes of its workspace layout.
 *   x [T, H], x_lat [T, L], y_lat [T, L]: dtype; W_fc1, W_fc2: dtype (also
 *   with NVFP4 expert weights); y_acc [T, H] float32 (read and written; each
 *   element by one thread); ws_latent:
 *   nh_moe_latent_workspace_size bytes.  Device pointers, 16-byte aligned.
 */
nh_status nh_moe_latent_config(const nh_moe_config *cfg, nh_moe_config *expert_cfg);
nh_status nh_moe_latent_workspace_size(const nh_moe_config *cfg, int64_t T, size_t *bytes);
nh_status nh_moe_latent_in(const nh_moe_config *cfg, int64_t T, const void *x,
                           const void *w_latent_fc1, void *x_lat, void *ws_latent,
                           size_t ws_latent_bytes, void *stream);
nh_status nh_moe_latent_out(const nh_moe_config *cfg, int64_t T, const void *y_lat,
                            const void *w_latent_fc2, float *y_acc, void *ws_latent,
                            size_t ws_latent_bytes, void *stream);

/*
 * Clear the status word at the start of workspace `ws` (any of the
 * library's workspaces), asynchronously on `stream`.  nh_moe_route,
 * nh_moe_route_permute, nh_moe_shared and the latent projections clear their
 * own workspace; a sequence that starts on a routed workspace with
 * nh_moe_permute (the experts of a latent block) calls this first.
 */
nh_status nh_moe_reset_status(void *ws, void *stream);

/*
 * Synchronises `stream`, reads the workspace status word and returns it
 * (NH_OK, NH_ERR_TIMEOUT or NH_ERR_DEVICE_CHECK); a pending CUDA error is
 * returned as NH_ERR_CUDA.  `ws` is any of the library's workspaces
 * (routed, shared or latent): each starts with its own status word.
 */
nh_status nh_moe_check_device(void *ws, void *stream);

/*
 * Failure-detection self test: launches one kernel whose bounded wait on an
 * mbarrier that nothing arrives on runs out after `timeout_ns`; the kernel
 * records NH_ERR_TIMEOUT in the status word of `ws` and returns, leaving the
 * context usable.  Read the result with nh_moe_check_device.
 */
nh_status nh_moe_selftest_timeout(void *ws, uint64_t timeout_ns, void *stream);

/* Message of the last non-OK status returned on this host thread. */
const char *nh_last_error(void);

/* Library version string. */
const char *nh_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NH_MOE_H */

/*
 * flint_moe.h -- C ABI of libflint_moe.so: one Flint MoE layer's decode step on
 * B200 (sm_100a), with NVFP4 weight-only (W4A16) experts.
 *
 * What the layer computes (sources, by page title and section):
 *  - Routing: every MoE layer has 256 routed experts, picks 6 per token, and
 *    adds one always-on shared expert ("Recursive Flint: 40B Local Coding
 *    Model, Benchmarks", architecture table, row "Experts"; "Run the Flint
 *    coding model on a CPU VPS", section "What Flint is, from the model card").
 *  - A fused top-k router and expert-indexed GEMVs for small-batch decode, and a
 *    grouped-GEMM path for larger batches ("[Model] Add Flint
 *    (RecursiveSI/flint)", section "What happened", third paragraph).
 *  - Weight-only NVFP4 serving, W4A16 ("[Model] Add Flint (RecursiveSI/flint)",
 *    section "What happened", first paragraph).
 *  - The pages fix no gating function, FFN type, shapes or bit layout; the layer
 *    contract this library implements fixes them:
 *      logits = x . W_r; softmax over the E logits; the top_k largest (ties to
 *      the lower expert index); gates = their probabilities renormalised to 1;
 *      each selected expert and each shared expert (weight 1) is a SwiGLU FFN
 *        FFN(x) = W_down (silu(W_gate x) * (W_up x)),  silu(g) = g / (1 + e^-g);
 *      out = sum_j gate_j FFN_{id_j}(x) + sum_s FFN_shared_s(x) (+ residual).
 *    NVFP4 weights: E2M1 codes, one E4M3 scale per 16 consecutive elements
 *    along K, one FP32 scale per (expert, matrix):
 *        w = e2m1(q) * e4m3(sb) * s_t.
 *
 * Conventions for every entry point:
 *  - Returns flint_status (0 = FLINT_OK). Nothing throws across the ABI.
 *    flint_last_error() gives a message for the calling thread's last failure.
 *  - Host-side validation happens before any launch; on a validation error no
 *    work is enqueued.
 *  - Device pointers are cudaMalloc'd (or equivalent) memory on the current
 *    device, owned by the caller; the library never allocates or frees device
 *    memory and never synchronises, except flint_moe_get_status (which reads
 *    the device status word) and flint_debug_* helpers.
 *  - All work is enqueued on `stream` (a cudaStream_t passed as void*; NULL =
 *    the legacy default stream).
 *  - bf16 tensors are raw 16-bit patterns (uint16_t); 16-byte alignment is
 *    required for every device pointer (FLINT_ERR_MISALIGNED otherwise).
 *
 * Packed HBM layout of the expert weights (flint_pack_nvfp4 writes it):
 *  Experts are stored expert-major: routed experts 0..E-1, then the shared
 *  expert(s). Within an expert, the gate and up projections are row-interleaved
 *  ("units"): unit u = [gate row u | up row u], u = 0..I-1, followed by the d
 *  rows of the down projection.
 *    packed (codes):  per expert 3*I*d/2 bytes. Unit u at byte u*d: gate row u
 *                     (d/2 bytes) then up row u (d/2 bytes). Down row n at byte
 *                     I*d + n*I/2. Within a row, byte j holds element 2j in its
 *                     low nibble and element 2j+1 in its high nibble.
 *    block_scales:    per expert 3*I*d/16 bytes, same rows in the same order:
 *                     unit u at byte u*d/8 (gate row's d/16 scales, then up
 *                     row's); down row n at byte I*d/8 + n*I/16. Scale byte b of
 *                     a row covers elements 16b..16b+15.
 *    tensor_scales:   float [E+S][3] = {gate, up, down} per expert.
 *  So every row is a whole number of 16-byte vectors (d, I multiples of 32),
 *  and any run of consecutive units or down rows is one contiguous span in
 *  each of the two arrays.
 *  BF16 weights (wdtype FLINT_W_BF16) use the same row order with bf16
 *  elements in `packed` (per expert 3*I*d*2 bytes); block_scales and
 *  tensor_scales are then ignored (NULL allowed).
 *
 * Supported shapes: d one of {512, 1024, 2048, 4096}; inter one of
 * {128, 256, 512, 1024}; 1 <= n_experts <= 512; 1 <= top_k <= 8, top_k <=
 * n_experts; n_shared 0 or 1. Others return FLINT_ERR_UNSUPPORTED_SHAPE.
 */
#ifndef FLINT_MOE_H
#define FLINT_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum flint_status {
  FLINT_OK = 0,
  FLINT_ERR_INVALID_ARG = -1,       /* null pointer, negative size, bad enum */
  FLINT_ERR_UNSUPPORTED_SHAPE = -2, /* shape outside the supported set */
  FLINT_ERR_MISALIGNED = -3,        /* a device pointer not 16-byte aligned */
  FLINT_ERR_WORKSPACE = -4,         /* workspace NULL or smaller than required */
  FLINT_ERR_CUDA = -5,              /* a CUDA runtime call failed (message kept) */
  FLINT_ERR_DEVICE_CHECK = -6,      /* a kernel recorded a failed check */
  FLINT_ERR_TIMEOUT = -7            /* a bounded device-side wait ran out */
} flint_status;

typedef enum flint_wdtype { FLINT_W_NVFP4 = 0, FLINT_W_BF16 = 1 } flint_wdtype;

typedef struct flint_moe_shape {
  int32_t d;         /* hidden size */
  int32_t inter;     /* expert intermediate width I */
  int32_t n_experts; /* routed experts E */
  int32_t top_k;     /* experts selected per token */
  int32_t n_shared;  /* always-on shared experts (0 or 1), gate weight 1 */
  int32_t wdtype;    /* flint_wdtype of the expert weights */
} flint_moe_shape;

typedef struct flint_moe_weights {
  const void* packed;          /* device; NVFP4 codes or bf16 weights, layout above */
  const uint8_t* block_scales; /* device; E4M3 block scales (NVFP4 only) */
  const float* tensor_scales;  /* device; float [E+S][3] (NVFP4 only) */
} flint_moe_weights;

/* Device-side check codes recorded in the workspace status word. */
enum {
  FLINT_DEVCHECK_EXPERT_ID = 1,   /* an expert id outside [0, E) reached a kernel */
  FLINT_DEVCHECK_NONFINITE = 2,   /* a non-finite weight reached the packer */
  FLINT_DEVCHECK_WAIT = 4,        /* a bounded wait gave up (FLINT_ERR_TIMEOUT) */
  FLINT_DEVCHECK_MMA = 8,         /* the tensor-core path rejected a tile */
  FLINT_DEVCHECK_INDEX = 16       /* a position or cache slot outside its range (skipped) */
};

typedef enum flint_path {
  FLINT_PATH_AUTO = 0, /* NVFP4: GEMV kernels below 32 tokens, tensor-core path from
                          32; bf16 weights: tensor-core path */
  FLINT_PATH_GEMV = 1, /* CUDA-core dequant-GEMV kernels at any token count */
  FLINT_PATH_MMA = 2   /* TMA-staged dequant-to-tensor-memory + tcgen05 MMA at any
                          count up to 16384 tokens (above 128 tokens the pairs
                          are grouped by a counting sort and each expert's
                          tokens are cut into tiles of 128; E + S <= 1024);
                          NVFP4 weights need inter >= 256; no input_rmsnorm */
} flint_path;

typedef enum flint_layer_variant {
  FLINT_LAYER_AUTO = 0,   /* one token: the cluster kernel when the shape fits it;
                             2..8 tokens: the persistent kernel's tensor-core loops */
  FLINT_LAYER_FMA = 1,    /* persistent kernel, CUDA-core dot products (fma.rn.f32.f16) */
  FLINT_LAYER_MMA = 2,    /* persistent kernel, register-fragment mma.sync m16n8k16 */
  FLINT_LAYER_CLUSTER = 3 /* 16-CTA cluster kernels, NVFP4 weights. One token: one
                             cluster per selected expert and one for the shared
                             expert. 2..8 tokens: persistent clusters that each
                             route the batch and take the active experts in turn
                             (register-fragment mma.sync, d in {512, 1024, 2048},
                             inter in {256, 512, 1024}, E <= 256). Routing, the
                             SwiGLU exchange and the down rows stay inside a
                             cluster (distributed shared memory), and the last CTA
                             to finish a block of output rows sums the experts'
                             gated partials in slot order. More than 8 tokens, or a
                             shape that does not fit on the device:
                             FLINT_ERR_UNSUPPORTED_SHAPE */
} flint_layer_variant;

typedef struct flint_moe_options {
  int32_t path;          /* flint_path */
  int32_t use_pdl;       /* 1 (default when options == NULL): chain the layer's
                            kernels with programmatic dependent launch */
  int32_t* topk_ids;     /* optional device int32 [T][top_k]: routed ids written here */
  float* topk_weights;   /* optional device float [T][top_k]: their gates */
  int32_t split_kernels; /* 1: run batch <= 8 as three kernels chained with programmatic
                            dependent launch instead of one persistent kernel */
  int32_t input_rmsnorm; /* 1: each token's x is divided by its RMS, sqrt(mean(x^2) + 1e-6)
                            (no learned weight), before the router and the experts;
                            the residual is added unnormalised. 0 (default): no norm */
  void* profile_events;  /* optional cudaEvent_t[2], recorded on `stream` just before
                            and just after the kernel that streams the expert weights
                            (the persistent layer kernel, or the gate/up kernel of the
                            three-kernel path, whose records then serialise the chain);
                            for per-kernel timing */
  int32_t layer_variant; /* flint_layer_variant: inner loops of the persistent
                            single-kernel path (batch <= 8). FLINT_LAYER_MMA
                            multiplies the in-register decoded NVFP4 weights (exact
                            in f16) with the f16-staged activations, f32
                            accumulate; other values FLINT_ERR_INVALID_ARG */
} flint_moe_options;

/* Bytes of the packed codes / block scales / tensor scales for a shape. Return 0
 * for an unsupported shape. For FLINT_W_BF16 the codes figure is the bf16 size
 * and the other two are 0. */
size_t flint_packed_bytes(const flint_moe_shape* shape);
size_t flint_block_scale_bytes(const flint_moe_shape* shape);
size_t flint_tensor_scale_bytes(const flint_moe_shape* shape);

/* flint_pack_nvfp4 -- quantise and lay out all experts' weights.
 *  w: device, [E+S][3][I*d] fp32 (w_is_bf16 = 0) or bf16 bits (w_is_bf16 = 1):
 *     matrix 0 = gate [I][d], 1 = up [I][d], 2 = down [d][I], row-major.
 *  Writes packed / block_scales / tensor_scales in the layout above, following
 *  the recipe: s_t = amax/2688 (1 if amax = 0); per block of 16 along K
 *  sb = E4M3_rne_satfinite((amax_b/6)/s_t); q = E2M1_rne_satfinite(w/(e4m3(sb)*s_t)),
 *  q = 0 when e4m3(sb) = 0; all fp32 steps round to nearest, no fused
 *  multiply-add. A non-finite weight sets FLINT_DEVCHECK_NONFINITE in the
 *  status word of `workspace` (needs flint_moe_workspace_bytes(shape, 1) bytes)
 *  and its tensor is left unspecified. shape->wdtype must be FLINT_W_NVFP4. */
int flint_pack_nvfp4(const void* w, int32_t w_is_bf16, const flint_moe_shape* shape,
                     void* packed, uint8_t* block_scales, float* tensor_scales,
                     void* workspace, size_t ws_bytes, void* stream);

/* flint_pack_bf16 -- lay out bf16 weights ([E+S][3][I*d] bf16 bits, device) in
 * the same expert-major row order, for shape->wdtype == FLINT_W_BF16. */
int flint_pack_bf16(const uint16_t* w, const flint_moe_shape* shape, uint16_t* packed,
                    void* stream);

/* Workspace bytes for calls of up to max_tokens tokens. The workspace holds the
 * status word, router logits, routing, grouping and the FFN intermediates; it
 * must not be shared by calls that may overlap on the GPU. Calls of any token
 * count up to max_tokens may alternate on one workspace; a workspace serves
 * one shape (after a shape change, flint_moe_workspace_init it again). */
size_t flint_moe_workspace_bytes(const flint_moe_shape* shape, int32_t max_tokens);

/* Zeroes the whole workspace (ws_bytes bytes): the control block at its head
 * (status word, router arrival counter, the single-kernel path's launch
 * generation) and the single-kernel path's tagged
 * router logits and SwiGLU values, which follow it at offsets that depend on
 * the shape only. Call
 * once after allocating a workspace, before its first use. Kernels only ever
 * set bits in the status word, and flint_moe_get_status reads and clears it. */
int flint_moe_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* flint_moe_route -- the router alone.
 *  x: device bf16 [T][d]; router_w: device bf16 [E][d] (W_r transposed, row e
 *  is expert e); topk_ids: device int32 [T][top_k] (descending logit, ties to
 *  the lower index); topk_weights: device float [T][top_k], summing to 1 per
 *  token. T = 0 is a no-op. */
int flint_moe_route(const uint16_t* x, int32_t T, const uint16_t* router_w,
                    const flint_moe_shape* shape, int32_t* topk_ids, float* topk_weights,
                    void* workspace, size_t ws_bytes, void* stream);

/* flint_moe_forward -- the whole layer: route, group tokens by expert, run the
 * selected and shared experts' SwiGLU FFNs from the packed weights, combine.
 *  x: device bf16 [T][d]; residual: device bf16 [T][d] or NULL (added to the
 *  combined output before rounding); out: device bf16 [T][d], round to nearest
 *  even. out may alias residual but not x. T = 0 is a no-op. */
int flint_moe_forward(const uint16_t* x, int32_t T, const uint16_t* router_w,
                      const flint_moe_weights* weights, const flint_moe_shape* shape,
                      const uint16_t* residual, uint16_t* out, void* workspace,
                      size_t ws_bytes, void* stream);

/* As flint_moe_forward, with options (path choice, PDL, routing outputs).
 * options == NULL behaves as flint_moe_forward.
 * Arithmetic: every NVFP4 path forms the exact f16 value of an e2m1 code times
 * its e4m3 block scale (at most 6 significant bits) and multiplies it with x
 * scaled per token by a power of two into f16 (h likewise per row), products
 * exact, accumulating in fp32; outputs bf16, round to nearest even. The
 * single-kernel path (batch <= 8) does so with CUDA-core fma.rn.f32.f16 or
 * register-fragment mma.sync (layer_variant). The tensor-core path
 * (FLINT_PATH_MMA, or AUTO from 32 tokens) multiplies on tcgen05 (kind::f16,
 * fp32 accumulators in tensor memory): NVFP4 weights are dequantised to f16
 * straight into tensor memory; bf16 weights multiply bf16 x directly. SwiGLU
 * intermediates are kept in fp32 and fed to the down projection as f16 (NVFP4,
 * power-of-two row scale) or bf16 (bf16 weights). Its profile events bracket
 * the gate/up kernel. */
int flint_moe_forward_ex(const uint16_t* x, int32_t T, const uint16_t* router_w,
                         const flint_moe_weights* weights, const flint_moe_shape* shape,
                         const uint16_t* residual, uint16_t* out, void* workspace,
                         size_t ws_bytes, const flint_moe_options* options, void* stream);

/* flint_moe_forward_noalloc -- the same layer forward as flint_moe_forward,
 * for callers that cannot allocate device memory when they call it: runtimes
 * that hand all device memory to their own pool up front, plug-ins hosted by
 * an application that forbids allocations on its serving path, or latency-
 * critical paths that cannot afford an allocation. (This entry point has no
 * counterpart in the pages; it is a packaging convenience.)
 *  Instead of a caller workspace it uses a scratch array of 1 MiB compiled into
 *  the library as a device global: every GPU that loads the library holds those
 *  1 MiB until the process exits. It allocates nothing: no cudaMalloc, no
 *  cudaFree, no allocating library routine.
 *  Arguments as for flint_moe_forward. A call whose scratch would exceed 1 MiB
 *  (flint_moe_workspace_bytes(shape, T) > 1048576) returns FLINT_ERR_WORKSPACE
 *  with a message, before any launch.
 *  The first call in each CUDA context (each device's primary context, or any
 *  other context the caller made current) looks up the array's device address
 *  in that context (cudaGetSymbolAddress) and caches it by the context's id;
 *  make that first call before any stream capture.
 *  The array keeps its contents between calls. Calls of one shape rely on the
 *  launch tags of the single-kernel path, so nothing is cleared; when the
 *  shape differs from the previous call's in that context, the call first
 *  zeroes the array (an asynchronous memset on `stream`) except its status
 *  word. Device check flags accumulate in that status word until
 *  flint_moe_noalloc_get_status reads and clears them.
 *  All calls share the one array:
 *  calls that may run at the same time on the GPU (different streams, or
 *  different host threads) race on it and corrupt each other's results;
 *  serialise them on one stream. */
int flint_moe_forward_noalloc(const uint16_t* x, int32_t T, const uint16_t* router_w,
                              const flint_moe_weights* weights, const flint_moe_shape* shape,
                              const uint16_t* residual, uint16_t* out, void* stream);

/* flint_moe_noalloc_get_status -- flint_moe_get_status for the built-in
 * scratch of flint_moe_forward_noalloc in the current context: synchronises
 * `stream`, reads the status word into *device_flags (may be NULL) and clears
 * it. Returns FLINT_OK, or FLINT_ERR_TIMEOUT / FLINT_ERR_DEVICE_CHECK when a
 * flag was set. (No counterpart in the pages.) */
int flint_moe_noalloc_get_status(int32_t* device_flags, void* stream);

/* Debug helper: the device address of the built-in scratch in the current
 * context (looked up as flint_moe_forward_noalloc does), e.g. to pass it to
 * flint_debug_wait_timeout. */
int flint_debug_noalloc_scratch(void** addr);

/* ---- the 4-bit output head ("Recursive Flint: 40B Local Coding Model,
 * Benchmarks": architecture table, row "Vocabulary", and section "How
 * Recursive built Flint", the 4-bit output head) ----
 * A dense NVFP4 matrix W [rows][cols] (rows = vocabulary, cols = hidden size)
 * in plain row-major planes: codes [rows][cols/2] (element 2j in the low
 * nibble of byte j), E4M3 scales [rows][cols/16] (byte b covers elements
 * 16b..16b+15), one fp32 tensor scale; w = e2m1(q) * e4m3(sb) * s_t. */

/* flint_pack_nvfp4_dense -- quantise W (device, fp32 or bf16 bits when
 * w_is_bf16, row-major [rows][cols]) with the experts' recipe (s_t =
 * amax/2688, per-16 E4M3 scale, E2M1 codes; fp32 round to nearest, no fused
 * multiply-add) into the planes above. cols one of 512, 1024, 2048, 4096;
 * workspace >= 1280 bytes (status word at byte 0; a non-finite weight sets
 * FLINT_DEVCHECK_NONFINITE there). Asynchronous on `stream`. */
int flint_pack_nvfp4_dense(const void* w, int32_t w_is_bf16, int32_t rows, int32_t cols, uint8_t* codes,
                           uint8_t* scales, float* tensor_scale, void* workspace, size_t ws_bytes, void* stream);

/* flint_lm_head -- out[t][v] = sum_c w[v][c] x[t][c] for T <= 8 decode
 * tokens. x: device bf16 [T][cols]; out: device fp32 [T][rows]. The exact
 * e2m1*e4m3 values (f16) multiply x scaled per token by a power of two into
 * f16 on the register-fragment tensor cores (mma.sync, fp32 accumulation);
 * the partial sums of a row's 512-column parts are added in part order; the
 * tensor scale and 1/sigma are applied once per logit. workspace >= 4 bytes
 * (status word; read it with flint_moe_get_status). Asynchronous on `stream`. */
int flint_lm_head(const uint16_t* x, int32_t T, const uint8_t* codes, const uint8_t* scales,
                  const float* tensor_scale, int32_t rows, int32_t cols, float* out, void* workspace,
                  size_t ws_bytes, void* stream);

/* flint_moe_forward_routed -- the layer's experts with the routing supplied
 * by the caller instead of computed: out[t] = sum_{j<top_k} topk_weights[t][j]
 * * FFN_{topk_ids[t][j]}(x_t) + shared expert(x_t) (+ residual[t]), bf16 out,
 * on the tensor-core path (T <= 16384; more than 128 tokens need E + S <= 1024;
 * NVFP4 weights need inter >= 256). The expert-parallel layer calls it with
 * top_k = 1 and n_shared = 0 over the rows it receives, the shared expert seen
 * as one more local expert (ids are validated on the device: an id outside
 * [0, E) is skipped and sets FLINT_DEVCHECK_EXPERT_ID). topk_ids device int32
 * [T][top_k], topk_weights device float [T][top_k] (4-byte aligned); the
 * other pointers and the workspace as for flint_moe_forward (workspace of
 * flint_moe_workspace_bytes(shape, >= T) bytes). Asynchronous on `stream`. */
int flint_moe_forward_routed(const uint16_t* x, int32_t T, const int32_t* topk_ids, const float* topk_weights,
                             const flint_moe_weights* weights, const flint_moe_shape* shape,
                             const uint16_t* residual, uint16_t* out, void* workspace, size_t ws_bytes,
                             void* stream);

/* flint_ep_dispatch -- expert-parallel dispatch of one layer over n_ranks
 * GPUs ("[Model] Add Flint (RecursiveSI/flint)", section "What happened":
 * expert parallelism, left on stock layers there). Rank r holds routed
 * experts [r E/R, (r+1) E/R) and the shared expert as local id E/R. Each of
 * the T (top_k + n_shared) pairs (token t, slot j) goes to the rank holding
 * its expert (the shared slot to `rank`, gate 1); pairs are ordered by
 * destination rank, then by pair index t (top_k + n_shared) + j (a stable
 * counting sort). Outputs (device, sized for P = T (top_k + n_shared) rows):
 *   send_x      bf16 [P][d]: x row of each send position (positions >= the
 *               total count are not written)
 *   send_ids    int32 [P]: local expert id on the destination rank
 *   send_gates  float [P]: the pair's gate
 *   send_token  int32 [P]: source token
 *   send_counts int32 [n_ranks]: rows for each rank (the send splits)
 *   pair_pos    int32 [T][top_k + n_shared]: send position of each pair, -1
 *               for a dropped pair (an id outside [0, E): sets
 *               FLINT_DEVCHECK_EXPERT_ID in the nullable device `status`)
 * n_ranks 1..8 dividing n_experts; top_k 1..8; n_shared 0 or 1; d a
 * multiple of 8; x and send_x 16-byte aligned. Two kernels, asynchronous on
 * `stream`. */
int flint_ep_dispatch(const int32_t* topk_ids, const float* topk_weights, int32_t T, int32_t top_k,
                      int32_t n_shared, int32_t n_experts, int32_t n_ranks, int32_t rank, const uint16_t* x,
                      int32_t d, uint16_t* send_x, int32_t* send_ids, float* send_gates, int32_t* send_token,
                      int32_t* send_counts, int32_t* pair_pos, int32_t* status, void* stream);

/* flint_ep_combine -- the expert-parallel layer's output on the home rank:
 * out[t] = bf16(sum_{j < slots, pair_pos[t][j] >= 0} y[pair_pos[t][j]] +
 * residual[t]) in fp32. y: device bf16 [rows][d], the expert rows returned
 * in send order (each already scaled by its gate); pair_pos as written by
 * flint_ep_dispatch; residual nullable. slots 1..9; d a multiple of 8; y, out,
 * residual 16-byte aligned. One kernel, asynchronous on `stream`. */
int flint_ep_combine(const uint16_t* y, const int32_t* pair_pos, int32_t T, int32_t slots, int32_t d,
                     const uint16_t* residual, uint16_t* out, void* stream);

/* flint_qk_norm_rope_kv -- the attention prologue of one layer: fused Q/K
 * normalisation + rotary embedding + KV-cache write ("[Model] Add Flint
 * (RecursiveSI/flint)", section "What happened"; heads from "Recursive Flint:
 * 125 tok/s on an M4 Pro", architecture table: 32 query, 4 key/value heads of
 * dimension 128, rotary positions on the sliding-window layers, none on the
 * full-attention layers).
 *   qkv      device bf16 [T][n_q_heads + 2*n_kv_heads][head_dim]: the fused
 *            projection, query heads, then key heads, then value heads
 *   q_norm_w, k_norm_w  device bf16 [head_dim]
 *   query/key heads: y = x / sqrt(mean(x^2) + eps) * w (fp32); with rope != 0,
 *   pairs (i, i + head_dim/2) rotated by row positions[t] of cos_sin (device
 *   fp32 [max_pos][head_dim], cos in the first half of a row, sin in the
 *   second, 16-byte aligned): first = y_i cos - y_j sin, second = y_j cos + y_i
 *   sin; outputs rounded to bf16.
 *   q_out    device bf16 [T][n_q_heads][head_dim]
 *   k_cache, v_cache  device bf16 [n_slots][n_kv_heads][head_dim]; token t's
 *            key and value heads go to row slots[t] (device int32 [T]); other
 *            rows are not touched.
 *   status   nullable device int32: a slot outside [0, n_slots) (that token's
 *            key and value are not written) or a position outside [0,
 *            max_pos) (its rotation is skipped) sets FLINT_DEVCHECK_INDEX.
 * head_dim must be 128. The caller owns all buffers; 16-byte aligned pointers.
 * One kernel, asynchronous on `stream`; T = 0 launches nothing. The pages
 * give no norm type or rotary layout: RMS normalisation with a learned weight
 * and the rotate-half pairing are the readings taken. */
int flint_qk_norm_rope_kv(const uint16_t* qkv, int32_t T, int32_t n_q_heads, int32_t n_kv_heads,
                          int32_t head_dim, const uint16_t* q_norm_w, const uint16_t* k_norm_w,
                          const float* cos_sin, int32_t max_pos, const int32_t* positions, int32_t rope,
                          float eps, const int32_t* slots, int64_t n_slots, uint16_t* q_out, uint16_t* k_cache,
                          uint16_t* v_cache, int32_t* status, void* stream);

/* flint_decode_attention -- grouped-query decode attention of one layer over
 * the bf16 KV cache flint_qk_norm_rope_kv writes ("[Model] Add Flint
 * (RecursiveSI/flint)", section "What happened": the attention step of the
 * per-layer decode chain; heads from "Recursive Flint: 125 tok/s on an M4 Pro",
 * architecture table: 32 query, 4 key/value heads of dimension 128; the
 * sliding-window layers pass a window-sized range, the full-attention layers
 * the whole history).
 *   q        device bf16 [T][n_q_heads][head_dim]: one query per token
 *   k_cache, v_cache  device bf16 [n_rows][n_kv_heads][head_dim]
 *   start    device int64 [T], len device int32 [T]: token t attends rows
 *            start[t] .. start[t] + len[t] - 1
 *   out      device bf16 [T][n_q_heads][head_dim]:
 *            out[t][h] = sum_j w_j v[start+j][g], w = softmax_j(scale *
 *            q[t][h] . k[start+j][g]), g = h / (n_q_heads / n_kv_heads);
 *            zeros for len 0. fp32 scores and sums; the weights enter the
 *            value sum rounded to bf16.
 *   max_len  host upper bound of len[t]; it sizes the split of each context
 *            into chunks (about 296 CTAs in all) and the workspace.
 *   workspace  device, 16-byte aligned, flint_decode_attention_workspace_bytes(
 *            T, n_kv_heads, max_len) bytes (0 -- NULL allowed -- when each
 *            context fits one chunk): per-chunk partial results, overwritten
 *            by every call.
 *   status   nullable device int32: len[t] > max_len (clamped to max_len) or
 *            a range outside [0, n_rows) or len < 0 (that token's output is
 *            zeros) sets FLINT_DEVCHECK_INDEX.
 * head_dim must be 128, n_q_heads a multiple of n_kv_heads with at most 8
 * query heads per kv head, T <= 65535, max_len <= 2^30, scale > 0 (1/sqrt(128) for the
 * model). q, caches, out: 16-byte aligned. The caller owns all buffers. One or
 * two kernels, asynchronous on `stream`; T = 0 launches nothing. */
size_t flint_decode_attention_workspace_bytes(int32_t T, int32_t n_kv_heads, int32_t max_len);
int flint_decode_attention(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache, int64_t n_rows,
                           const int64_t* start, const int32_t* len, int32_t T, int32_t n_q_heads,
                           int32_t n_kv_heads, int32_t head_dim, int32_t max_len, float scale, uint16_t* out,
                           void* workspace, size_t workspace_bytes, int32_t* status, void* stream);

/* Synchronises `stream`, reads the workspace status word into *device_flags
 * (FLINT_DEVCHECK_* bits, may be NULL) and clears it. Returns FLINT_OK, or
 * FLINT_ERR_TIMEOUT / FLINT_ERR_DEVICE_CHECK when a flag was set. */
int flint_moe_get_status(void* workspace, int32_t* device_flags, void* stream);

/* Message of the calling thread's last failed call ("" if none). */
const char* flint_last_error(void);

/* Debug helper: the exact products e2m1(q) * e4m3(sb) of consecutive rows of
 * one expert's weights, decoded by the same device routines the FFN kernels
 * use. matrix 0: `rows` gate/up units from unit row0, written as fp32
 * [2*rows][d] (gate row, then up row, per unit); matrix 1: `rows` down rows
 * from row0, fp32 [rows][I]. out is device memory. tensor_scale_out (host,
 * nullable) receives {gate, up} scales for matrix 0, the down scale for 1.
 * Synchronises the stream. */
int flint_debug_dequant(const flint_moe_weights* weights, const flint_moe_shape* shape,
                        int32_t expert, int32_t matrix, int32_t row0, int32_t rows,
                        float* out, float* tensor_scale_out, void* stream);

/* Debug helper: decoded weights e2m1(q) * e4m3(sb) (no tensor scale) of a
 * tile of one expert matrix, produced by the tensor-core decoders themselves:
 * decoder 0 the tcgen05 path's decode into tensor memory (dequant_slice_tmem,
 * read back with tcgen05.ld; tiles of 128 rows x 256 K), decoder 1 the
 * register-fragment decode of the persistent kernel's mma.sync variant
 * (tc_segment, extracted through the MMA with one-hot B columns; tiles of 16
 * rows x 128 K). matrix 0: the 2*inter interleaved gate/up rows of the packed
 * layout (row 2u = gate row u, 2u+1 = up row u); 1: the d down rows. Rows
 * [row0, row0+rows) and K columns [k0, k0+kn) in whole tiles; out: device fp32
 * [rows][kn]. Synchronises the stream. */
int flint_debug_decode(const flint_moe_weights* weights, const flint_moe_shape* shape, int32_t expert,
                       int32_t matrix, int32_t decoder, int32_t row0, int32_t rows, int32_t k0, int32_t kn,
                       float* out, void* stream);

/* Debug helper: the grouping of routed ids by expert (active experts in
 * ascending id order, then the shared experts; per expert its pairs
 * token << 8 | slot in ascending token order; offsets), computed on the
 * device by one of the layer's grouping routines: impl 0 the CTA grouping of
 * the persistent single-kernel path and the tensor-core path (T <= 128),
 * impl 1 the warp grouping of the three-kernel path (T * top_k <= 64), impl 2
 * its CTA grouping (T <= 32), impl 3 the counting-sort grouping the
 * tensor-core path uses above 128 tokens (T <= 16384, E + S <= 1024; its
 * scratch needs a workspace of flint_moe_workspace_bytes for T tokens). ids:
 * device int32 [T][top_k]. Outputs (device):
 * act int32 [E+S], off int32 [E+S+1], pair int32 [T*(top_k+S)], counts int32
 * [2] = {routed experts in use, active experts}. An id outside [0, E) is
 * skipped and sets FLINT_DEVCHECK_EXPERT_ID in the workspace status word (read
 * it with flint_moe_get_status). Asynchronous on `stream`. */
int flint_debug_group(const int32_t* ids, int32_t T, const flint_moe_shape* shape, int32_t impl, int32_t* act,
                      int32_t* off, int32_t* pair, int32_t* counts, void* workspace, size_t ws_bytes, void* stream);

/* Failure-detection hook: launches one kernel whose bounded wait on a
 * shared-memory barrier that nothing completes gives up after `cycles` SM clock
 * cycles (clamped to [1, 2e9]) and records FLINT_DEVCHECK_WAIT in the
 * workspace status word, the way every wait in the layer kernels does. It
 * leaves no copy in flight and the context stays usable; read the result with
 * flint_moe_get_status. */
int flint_debug_wait_timeout(void* workspace, int64_t cycles, void* stream);

/* Library version string. */
const char* flint_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FLINT_MOE_H */

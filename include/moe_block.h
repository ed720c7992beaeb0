/*
 * moe_block.h - C ABI of a B200 (sm_100a) library for one Gemma-4-26B-A4B
 * mixture-of-experts feed-forward block.
 *
 * What the block computes (the layer's statement on the pages):
 *   - gm.nn.Gemma4_26B_A4B, class docstring and TransformerConfig: every layer
 *     has "a MoE branch (128 experts, expert_dim=704)" and "a dense shared
 *     MLP branch" of width 2112 (hidden_dim = moe_dense_hidden_dim), with
 *     embed_dim 2816, num_experts 128, top_k_experts 8, dtype bfloat16;
 *   - Gemma-4-26B-A4B model card: gating "softmax" over expert logits, 8
 *     routed experts per token, "Selected expert weights are renormalized to
 *     sum to 1", one always-on expert of width 2112, FFN activation "GeGLU
 *     (tanh-approximate GELU)", no FFN biases;
 *   - G4-MeroMero-26B-A4B-NVFP4 config.json: the NVFP4 format (below).
 *
 *   logits[t, e] = sum_d x[t, d] * W_router[d, e]  (+ router_bias[e])
 *   idx[t, 0..k-1] = the k largest logits, largest first; equal logits: the
 *                    lower expert index first
 *   w[t, j]        = softmax over all experts, restricted to idx[t, .] and
 *                    renormalised (= softmax of the k kept logits)
 *   ffn(x; G, U, D) = (gelu_tanh(x G) * (x U)) D,
 *                    gelu_tanh(z) = z/2 (1 + tanh(sqrt(2/pi)(z + 0.044715 z^3)))
 *   out[t] = ffn(x[t]; Sg, Su, Sd) + sum_j w[t, j] ffn(x[t]; Wg[e], Wu[e], Wd[e]),
 *            e = idx[t, j]
 *
 * Numerics: bf16 inputs, fp32 accumulation everywhere; the GeGLU hidden rows
 * h and the routed experts' outputs y are rounded to bf16 between kernels; the
 * shared branch stays fp32; out is the round-to-nearest-even bf16 of the fp32
 * sum (s + w_0 y_0 + w_1 y_1 + ..., in slot order). Results are bitwise
 * deterministic for a given device and input.
 *
 * Conventions for every call:
 *   - all tensor pointers are DEVICE pointers, row-major, contiguous, 16-byte
 *     aligned, owned by the caller; the library never frees caller memory;
 *   - bf16 means IEEE bfloat16 bit patterns (uint16_t here);
 *   - calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream): they validate on the host, enqueue kernels and return
 *     without synchronising, except moe_get_device_status;
 *   - T == 0 is a no-op returning MOE_OK; invalid arguments return an error
 *     before anything is enqueued;
 *   - the library needs sm_100 (B200); other devices get MOE_ERR_ARCH.
 */
#ifndef MOE_BLOCK_H
#define MOE_BLOCK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, negative size, unsupported dims, aliasing */
  MOE_ERR_ALIGNMENT = 2,     /* a pointer is not 16-byte aligned */
  MOE_ERR_ARCH = 3,          /* the current device is not sm_100 */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime call failed (launch, allocation) */
  MOE_ERR_WORKSPACE = 5,     /* caller workspace smaller than moe_workspace_bytes_ex */
  MOE_ERR_DEVICE_TIMEOUT = 6, /* a kernel's bounded wait ran out (reported by moe_get_device_status) */
  MOE_ERR_GUARD = 7           /* a workspace guard word was overwritten (reported by moe_get_device_status) */
} moe_status;

/* Gemma-4-26B-A4B block constants (TransformerConfig of gm.nn.Gemma4_26B_A4B). */
#define MOE_EMBED_DIM 2816
#define MOE_NUM_EXPERTS 128
#define MOE_EXPERT_DIM 704
#define MOE_HIDDEN_DIM 2112
#define MOE_TOP_K 8

/*
 * Full parameter set. Dims left 0 take the Gemma-4-26B-A4B values above.
 * Supported dims: embed_dim, expert_dim, hidden_dim multiples of 64;
 * num_experts a multiple of 8 and <= 128; 1 <= top_k_experts <= num_experts.
 *
 * Weights (bf16, row-major, exactly as given - no repacking):
 *   w_router [embed_dim, num_experts]
 *   wg, wu   [num_experts, embed_dim, expert_dim]   (gate, up)
 *   wd       [num_experts, expert_dim, embed_dim]   (down)
 *   sg, su   [embed_dim, hidden_dim]                (shared gate, up)
 *   sd       [hidden_dim, embed_dim]                (shared down)
 * x [T, embed_dim] bf16 in; out [T, embed_dim] bf16 out, written fully; out
 * must not overlap x.
 *
 * Optional (NULL = absent):
 *   router_bias [num_experts] fp32, added to the logits before the softmax;
 *   workspace / workspace_bytes: caller scratch of at least
 *     moe_workspace_bytes_ex(p) bytes, 256-byte aligned; without it the
 *     library uses one cached allocation per device (grown on demand, kept
 *     until process exit; calls on different streams then share it, so run
 *     them one after another or give each its own workspace);
 *   out_f32 [T, embed_dim] fp32: the pre-rounding output (out == RNE(out_f32));
 *   idx_out [T, top_k] int32, w_out [T, top_k] fp32: the routing used;
 *   cnt_out [num_experts] int32: tokens per expert;
 *   logits_out [T, num_experts] fp32: the router logits the selection used
 *     (router_bias included), a debug output (also honoured by moe_route and
 *     moe_route_noalloc).
 *
 * The normalisation sandwich around the block (model card: RMSNorm layers,
 * "sandwich" = pre and post, epsilon 1e-06), each part optional:
 *   norm_pre  [embed_dim] bf16: the block computes on
 *             x_n = RNE_bf16(norm_pre * x / sqrt(mean(x^2) + 1e-6)) (router,
 *             experts and shared MLP all read x_n; kept in the workspace);
 *   norm_post [embed_dim] bf16: the block output f becomes
 *             norm_post * f / sqrt(mean(f^2) + 1e-6), in fp32;
 *   residual  nonzero: out = RNE(x + that), the raw input x added in fp32.
 * With any of the three, embed_dim must be <= 4096 (a row per CTA). out_f32
 * then holds the final pre-rounding value.
 *
 * Expert parallelism (the layer split over G devices, each holding 1/G of the
 * experts and a 1/G slice of the shared MLP's hidden units): an expert shard
 * owns experts [expert_begin, expert_begin + expert_count) of the
 * num_experts the router scores (expert_count 0 = all of them). Then wg, wu,
 * wd hold only those experts ([expert_count, ...], expert 0 of the arrays
 * being expert_begin); w_router still covers every expert, so routing and
 * weights are those of the whole layer; sg, su, sd are the shard's slice of
 * the shared MLP (hidden_dim = the slice width, sg / su its columns, sd its
 * rows). The call then computes the shard's partial sum
 *   s_slice[t] + sum over the slots j whose expert is local of w[t, j] y_j[t],
 * slots in order, in fp32; the partial sums of all shards add up to the
 * block's output (GeGLU acts per hidden unit, so the shared MLP splits
 * exactly over its hidden units). The caller sums them across devices (e.g.
 * a reduce-scatter) and rounds with moe_round_bf16. A shard may not use
 * norm_post or residual, which act on the full sum.
 * out may be NULL when out_f32 is given: only the fp32 result is written.
 *
 * Debug aid: with check_guards nonzero, the block writes a pattern into the
 * 256 guard bytes that end every workspace layout (moe_ws_layout.guard)
 * before its first kernel and checks it after its last (two extra launches);
 * a kernel that wrote past the workspace's data then shows as MOE_ERR_GUARD
 * from moe_get_device_status. The block's kernels also range-check every
 * index they read back from the workspace and record MOE_ERR_INVALID_ARG
 * instead of addressing memory out of range.
 */
typedef struct moe_params {
  int T;
  int top_k_experts;
  int embed_dim;
  int num_experts;
  int expert_dim;
  int hidden_dim;
  const void* x;
  const void* w_router;
  const float* router_bias;
  const void* wg;
  const void* wu;
  const void* wd;
  const void* sg;
  const void* su;
  const void* sd;
  void* out;
  float* out_f32;
  int32_t* idx_out;
  float* w_out;
  int32_t* cnt_out;
  void* workspace;
  size_t workspace_bytes;
  const void* norm_pre;
  const void* norm_post;
  int residual;
  float* logits_out;
  int expert_begin;
  int expert_count;
  int check_guards;
} moe_params;

/*
 * Where the block's intermediates live inside a workspace (byte offsets from
 * its start). R = T * top_k routed rows, ordered expert by expert, tokens
 * ascending within an expert.
 *   x_perm [R, embed_dim] bf16   - x gathered into routed-row order
 *   h      [R, expert_dim] bf16  - routed GeGLU hidden rows
 *   y      [R, embed_dim] bf16   - routed expert outputs (unweighted)
 *   hs     [T, hidden_dim] bf16  - shared GeGLU hidden rows
 *   s      [T, embed_dim] fp32   - shared MLP output
 *   idx [T, top_k] int32, w [T, top_k] fp32, cnt [E] int32, off [E + 1] int32,
 *   row_of [T, top_k] int32 (routed row of each (token, slot)),
 *   token_of [R] int32 (token of each routed row)
 *   x_norm [T, embed_dim] bf16   - the pre-normed block input (with norm_pre)
 */
typedef struct moe_ws_layout {
  size_t total_bytes;
  size_t x_perm, h, y, hs, s;
  size_t idx, w, cnt, off, row_of, token_of;
  size_t x_norm;
  size_t guard;  /* 256 guard bytes, the last of the layout */
} moe_ws_layout;

/* Bytes of workspace a call with these params needs (T, top_k and dims are read). */
size_t moe_workspace_bytes_ex(const moe_params* p);
/* Same for the Gemma-4-26B-A4B dims. */
size_t moe_workspace_bytes(int T, int top_k);
/* Fill *out with the workspace layout for these params; MOE_ERR_INVALID_ARG on bad dims. */
moe_status moe_workspace_layout(const moe_params* p, moe_ws_layout* out);

/*
 * The block forward pass at the Gemma-4-26B-A4B dims, top_k 8, no router
 * bias, library-owned workspace. Pointers as in moe_params.
 */
moe_status moe_block_forward(const void* x, const void* w_router, const void* wg, const void* wu, const void* wd,
                             const void* sg, const void* su, const void* sd, int T, void* out, void* stream);

/* The block forward pass with every option (see moe_params). */
moe_status moe_block_forward_ex(const moe_params* p, void* stream);

/*
 * Router only (the first step of the block): logits in fp32, top-k selection
 * and renormalised softmax weights. Uses p->T, top_k_experts, embed_dim,
 * num_experts, x, w_router, router_bias and the workspace fields;
 * writes idx [T, top_k] int32 and w [T, top_k] fp32.
 */
moe_status moe_route(const moe_params* p, int32_t* idx, float* w, void* stream);

/*
 * Expert-major permutation of the (token, slot) assignments in idx
 * [T, top_k] (values in [0, num_experts), distinct within a row, as the
 * router produces them; out-of-range values are skipped and reported by
 * moe_get_device_status): cnt [num_experts] tokens per
 * expert, off [num_experts + 1] exclusive scan of cnt, row_of [T, top_k]
 * routed row of each assignment, token_of [T * top_k] token of each row. Rows
 * of expert e are off[e] .. off[e+1]-1 in ascending token order. Integer
 * work, bit-exact. Uses p->T, top_k_experts, num_experts, workspace fields.
 */
moe_status moe_permute(const moe_params* p, const int32_t* idx, int32_t* cnt, int32_t* off, int32_t* row_of,
                       int32_t* token_of, void* stream);

/*
 * Synchronise `stream`, then read and clear the library's device error word
 * on the current device. MOE_ERR_DEVICE_TIMEOUT if any kernel gave up a
 * bounded wait since the last call (its outputs are then undefined);
 * MOE_ERR_CUDA if the stream reports a CUDA error.
 */
moe_status moe_get_device_status(void* stream);

/*
 * Failure-path check: launch one small kernel that waits, bounded by
 * timeout_us microseconds, on a barrier that nothing will complete. The wait
 * runs out, the kernel records MOE_ERR_DEVICE_TIMEOUT in the device error
 * word and returns; the context stays usable.
 */
moe_status moe_debug_timeout_probe(int timeout_us, void* stream);

/*
 * End-to-end variant of moe_block_forward_ex for callers whose activations
 * live in host memory: enqueues the copy of x_host (T * embed_dim bf16) into
 * the device buffer p->x, the forward pass, and the copy of p->out back into
 * out_host, all on `stream`. Host buffers should be pinned for the copies to
 * be asynchronous; the caller synchronises `stream` before reading out_host.
 */
moe_status moe_block_forward_hostio(const moe_params* p, const void* x_host, void* out_host, void* stream);

/*
 * Per-kernel timing. After moe_profile_begin(kernel_mask), every kernel this
 * thread enqueues whose id bit is set in kernel_mask is bracketed by two CUDA
 * events recorded on its stream (an event between two kernels also ends their
 * launch overlap, so time the whole step with a narrow mask).
 * moe_profile_end() waits for those events, writes per kernel id the summed
 * milliseconds and the number of launches into total_ms[0..n) and
 * launches[0..n), stops recording and returns the number of kernel ids.
 * moe_kernel_name(id) names a kernel id (NULL past the last one).
 */
moe_status moe_profile_begin(uint32_t kernel_mask);
int moe_profile_end(float* total_ms, int* launches, int n);
const char* moe_kernel_name(int id);

/*
 * moe_route without any device allocation (the pages have no counterpart; it
 * exists for callers of this library that are not allowed to allocate device
 * memory: applications whose memory is owned by their own allocator or
 * reserved up front, which forbid libraries to call cudaMalloc behind their
 * back, and runtimes whose allocation calls would stall or fail mid-run).
 *
 * Same arguments, kernels, split of the reduction and therefore bit-identical
 * results as moe_route (idx, w and the optional logits_out are caller memory;
 * the workspace fields of p are ignored). Its scratch - the split-K partial
 * logits and the token-expert bitmasks - lives in a fixed 10 MiB __device__
 * array inside the library, which every GPU that loads the library holds until
 * the process exits; that size holds moe_route's own split at every batch up
 * to the limit. T is limited to 4096 tokens; a larger batch returns
 * MOE_ERR_WORKSPACE before anything is enqueued. No cudaMalloc, cudaFree or
 * allocating library routine is called.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) once for that device; make that first call before
 * any stream capture. Every call on a device shares the one array, and a call
 * overwrites what the previous call left there: calls that may overlap on the
 * GPU (different streams, or different host threads) race and must be
 * serialised by the caller.
 */
moe_status moe_route_noalloc(const moe_params* p, int32_t* idx, float* w, void* stream);

/* ------------------------------------------------------------------ NVFP4
 *
 * The NVFP4 variant follows the checkpoint's quantisation_config
 * (G4-MeroMero-26B-A4B-NVFP4 config.json, config_groups.group_0): every
 * expert and shared Linear holds e2m1 values in groups of 16 along its input
 * dimension K with one float8_e4m3 scale per group and one fp32 tensor scale
 * ("tensor_group"); weights are static, input activations are quantised per
 * call under a calibrated tensor scale ("dynamic": "local", static_minmax);
 * the router stays bf16 ("ignore": layers.N.router.proj).
 *
 * Quantisation of a group under tensor scale G, in fp32 with IEEE
 * round-to-nearest operations:
 *   s = e4m3_satfinite(RN(RN(amax16 / 6) * G)); q_i = e2m1_satfinite(RN(x_i * RN(G / s)))
 *   (s = 0 makes the group 0); value x^_i = e2m1(q_i) * s / G; weights use G = 448*6/amax.
 *
 * Storage of one [K, N] Linear (or G of them, experts stacked):
 *   q  [G][N][K/2] bytes: e2m1 codes, K-major, element 2j of a row in the low
 *      nibble of byte j;
 *   sf [G][ceil(N/128)][K/64][512] bytes: the group scales of rows 128a..128a+127
 *      and K range 64b..64b+63 form one 512-byte atom, row r, 16-group c (0..3)
 *      at byte 16*(r%32) + 4*(r/32) + c; rows past N hold scale 0;
 *   g  [G] fp32 tensor scales.
 */
typedef struct moe_nvfp4_linear {
  const uint8_t* q;
  const uint8_t* sf;
  const float* g;
} moe_nvfp4_linear;

/* Sizes of q and sf for G groups of [K, N] (K a multiple of 64, N of 64). */
moe_status moe_nvfp4_weight_bytes(int groups, int K, int N, size_t* q_bytes, size_t* sf_bytes);

/*
 * Quantise bf16 weights w [groups][K][N] (N contiguous: exactly the layout the
 * bf16 block takes) into q, sf and g (caller-owned device buffers of the sizes
 * above). Deterministic; enqueued on stream.
 */
moe_status moe_nvfp4_quantize_weight(const void* w, int groups, int K, int N, uint8_t* q, uint8_t* sf, float* g,
                                     void* stream);

/*
 * Quantise activation rows x [rows][K] bf16 under tensor scale g into
 * q [rows][K/2] and sf [ceil(rows/128)][K/64][512] (the same formats; a
 * standalone entry to the quantiser the NVFP4 block applies to x).
 */
moe_status moe_nvfp4_quantize_act(const void* x, int rows, int K, float g, uint8_t* q, uint8_t* sf, void* stream);

/*
 * Parameters of one NVFP4 block. Dims, x, w_router, router_bias, out, out_f32,
 * idx_out, w_out, cnt_out and workspace as in moe_params (num_experts, the
 * shared width and embed_dim multiples of 128 are not needed; all three dims
 * multiples of 64). g_x, g_h, g_hs: static tensor scales of the block input,
 * the routed GeGLU rows and the shared GeGLU rows. rms_norm_out = 1 writes
 * out = y / sqrt(mean(y^2) + 1e-6) of the block output y (no learned scale):
 * the inter-block norm of a stack of blocks.
 */
typedef struct moe_nvfp4_params {
  int T;
  int top_k_experts;
  int embed_dim;
  int num_experts;
  int expert_dim;
  int hidden_dim;
  const void* x;
  const void* w_router;
  const float* router_bias;
  moe_nvfp4_linear wg, wu, wd;  /* G = num_experts */
  moe_nvfp4_linear sg, su, sd;  /* G = 1 */
  float g_x, g_h, g_hs;
  int rms_norm_out;
  void* out;
  float* out_f32;
  int32_t* idx_out;
  float* w_out;
  int32_t* cnt_out;
  void* workspace;
  size_t workspace_bytes;
} moe_nvfp4_params;

size_t moe_nvfp4_workspace_bytes(const moe_nvfp4_params* p);

/*
 * Where the NVFP4 block's intermediates live inside its workspace (byte
 * offsets). Routed rows are padded per expert to whole 128-row blocks
 * (routed_rows rows in all); token-order buffers have token_rows rows (T
 * rounded up to 128). Codes are e2m1 [rows][K/2] (element 2j in the low
 * nibble of byte j), group scales e4m3 in 512-byte atoms [rows/128][K/64][512]
 * (row r, 16-group c of the 64-K block at byte 16*(r%32) + 4*(r/32%4) + c):
 *   xq_perm / xsf_perm  x quantised, routed-row order (K = embed_dim)
 *   xq_tok / xsf_tok    x quantised, token order
 *   hq / hsf            routed GeGLU rows quantised under g_h (K = expert_dim)
 *   hsq / hssf          shared GeGLU rows quantised under g_hs (K = hidden_dim)
 *   y [routed_rows, embed_dim] bf16, s [T, embed_dim] fp32
 *   idx, w, cnt, off, row_of as in moe_ws_layout (row_of: the padded routed row)
 */
typedef struct moe_nvfp4_ws_layout {
  size_t total_bytes;
  size_t xq_perm, xsf_perm, xq_tok, xsf_tok;
  size_t hq, hsf, hsq, hssf;
  size_t y, s;
  size_t idx, w, cnt, off, row_of;
  long long routed_rows, token_rows;
} moe_nvfp4_ws_layout;

moe_status moe_nvfp4_workspace_layout(const moe_nvfp4_params* p, moe_nvfp4_ws_layout* out);

/* One NVFP4 block forward pass (router bf16, expert and shared Linears NVFP4). */
moe_status moe_block_forward_nvfp4(const moe_nvfp4_params* p, void* stream);

/*
 * Calibration observer for the NVFP4 activation scales (the checkpoint's
 * input_activations observer static_minmax): runs the bf16 block on p (which
 * must carry a caller workspace) and writes, in device fp32 [3] buffers,
 * amax[0] = max |x| (the block input, after norm_pre when given), amax[1] =
 * max |h| over the routed GeGLU rows, amax[2] = max |hs| over the shared
 * GeGLU rows, and the tensor scales scales[i] = RN(448 * 6 / amax[i]) (1 for
 * an all-zero tensor): g_x, g_h, g_hs of moe_nvfp4_params. amax and scales
 * must not overlap. The GeGLU rows are observed as stored, in bf16.
 */
moe_status moe_nvfp4_calibrate(const moe_params* p, float* amax, float* scales, void* stream);

/* --------------------------------------------- weight-only SFP8 / Q4_0
 *
 * The pages give a whole-model footprint for two more weight formats, SFP8
 * and Q4_0 (Gemma-4-26B-A4B record, "MEMORY IS SET BY TOTAL, NOT ACTIVE":
 * 57.7 GB bf16, 28.8 GB at SFP8, 14.4 GB at Q4_0), and print neither format.
 * Readings (weight-only: every expert and shared Linear weight quantised
 * along its input dimension K, each matrix on its own; router and
 * activations stay bf16):
 *   SFP8: sign bit and a 7-bit magnitude code m - 0 is zero, m in [1, 63] is
 *         (1 + (m & 3)/4) 2^((m >> 2) - 23), m in [64, 127] is
 *         (1 + (m & 7)/8) 2^(((m >> 3) & 7) - 7) (3 mantissa bits from 2^-7 up,
 *         2 below, largest 1.875); one fp32 scale S = amax / 1.875 per matrix;
 *         code = nearest magnitude to |w| / S (ties to the even code,
 *         saturating) with w's sign; w^ = value * S.
 *   Q4_0: the ggml block format - blocks of 32 along K, d = (the block's
 *         first element of largest magnitude, sign kept) / -8 stored as fp16,
 *         q = min(15, trunc(w / d + 8.5)) in fp32 arithmetic, w^ = (q - 8) d.
 * The block then computes as the bf16 block on the dequantised weights (h,
 * y bf16, s fp32, out bf16); SFP8 values are exact in bf16 and the matrix
 * scale multiplies the fp32 sums, while a Q4_0 weight (q - 8) d is rounded to
 * bf16 (nearest even) before the tensor cores.
 *
 * Storage of G stacked [K, N] Linears (K and N multiples of 64), the
 * transposed weight in 128-row blocks and 64-deep K blocks:
 *   SFP8: q [G][ceil(N/128)][K/64][128 rows x 64 code bytes]; scale [G] fp32
 *   Q4_0: q [G][ceil(N/128)][K/64][128 rows x 32 bytes | 128 rows x 2 fp16 d]
 *         (element 2i of a 16-byte piece in the low nibble of its byte i; the
 *         row's two scales cover K 0-31 and 32-63); scale unused (NULL)
 * A row's codes are 16-byte pieces in K order, piece j of row r stored at
 * position j ^ ((r >> 1) & 3) (SFP8) or j ^ ((r >> 2) & 1) (Q4_0) of the row.
 * Rows past N hold zeros.
 */
#define MOE_WFMT_SFP8 1
#define MOE_WFMT_Q4_0 2

typedef struct moe_wq_linear {
  const uint8_t* q;
  const float* scale;
} moe_wq_linear;

/* Bytes of q for G stacked [K, N] Linears in `format`. */
moe_status moe_wq_weight_bytes(int format, int groups, int K, int N, size_t* bytes);

/*
 * Quantise bf16 weights w [groups][K][N] (N contiguous: the bf16 block's
 * layout) into q (and, SFP8, scale [groups]); caller-owned device buffers of
 * the sizes above. Deterministic; enqueued on stream.
 */
moe_status moe_wq_quantize_weight(int format, const void* w, int groups, int K, int N, uint8_t* q, float* scale,
                                  void* stream);

/*
 * One block with weight-only SFP8 or Q4_0 expert and shared Linears. Dims,
 * x, w_router (bf16), router_bias, out, out_f32, idx_out, w_out, cnt_out and
 * workspace as in moe_params (workspace: moe_wq_workspace_bytes).
 */
typedef struct moe_wq_params {
  int T;
  int top_k_experts;
  int embed_dim;
  int num_experts;
  int expert_dim;
  int hidden_dim;
  int format;
  const void* x;
  const void* w_router;
  const float* router_bias;
  moe_wq_linear wg, wu, wd; /* G = num_experts */
  moe_wq_linear sg, su, sd; /* G = 1 */
  void* out;
  float* out_f32;
  int32_t* idx_out;
  float* w_out;
  int32_t* cnt_out;
  void* workspace;
  size_t workspace_bytes;
} moe_wq_params;

size_t moe_wq_workspace_bytes(const moe_wq_params* p);
moe_status moe_block_forward_wq(const moe_wq_params* p, void* stream);

/* -------------------------------------------------------- dense GeGLU FFN
 *
 * The feed-forward of the dense E4B sibling (gm.nn.Gemma4_E4B
 * TransformerConfig: embed_dim 2560, hidden_dim 10240, enable_moe=False) - the
 * same bias-free GeGLU, tanh GELU on the gate projection, as the 26B-A4B
 * block's shared MLP:
 *   out = RNE_bf16((gelu_tanh(x Wg) * (x Wu)) Wd), fp32 accumulation, the
 *   hidden rows stored as bf16 (RNE), as in the block.
 * Dims left 0 take embed_dim 2560 and hidden_dim 10240; both must be
 * multiples of 64. Weights bf16, row-major, exactly as given: wg, wu
 * [embed_dim, hidden_dim], wd [hidden_dim, embed_dim]. x [T, embed_dim] bf16
 * in, out [T, embed_dim] bf16 out (must not overlap x); out_f32 [T, embed_dim]
 * fp32 (optional): the pre-rounding output. workspace: at least
 * moe_dense_workspace_bytes(p) bytes, 256-byte aligned, or NULL for the
 * library's cached allocation. T = 0 is a no-op; errors as for the block.
 */
#define MOE_E4B_EMBED_DIM 2560
#define MOE_E4B_HIDDEN_DIM 10240

typedef struct moe_dense_params {
  int T;
  int embed_dim;
  int hidden_dim;
  const void* x;
  const void* wg;
  const void* wu;
  const void* wd;
  void* out;
  float* out_f32;
  void* workspace;
  size_t workspace_bytes;
} moe_dense_params;

size_t moe_dense_workspace_bytes(const moe_dense_params* p);
moe_status moe_dense_ffn_forward(const moe_dense_params* p, void* stream);

/*
 * out[i] = RNE_bf16(in[i]) for i < n (fp32 in, bf16 out; n a multiple of 8,
 * both 16-byte aligned, not overlapping): the final rounding of an output
 * summed across expert shards.
 */
moe_status moe_round_bf16(const float* in, void* out, size_t n, void* stream);

/*
 * Check the guard words of the caller workspace p->workspace (laid out for
 * p's dims) on their own: MOE_ERR_GUARD from the next moe_get_device_status
 * if they differ from the pattern a guarded call wrote.
 */
moe_status moe_workspace_guard_check(const moe_params* p, void* stream);

/* Human-readable name of a status code. */
const char* moe_status_string(moe_status s);

/* Number of kernels the last forward call on this thread enqueued. */
int moe_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_BLOCK_H */

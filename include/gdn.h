/*
 * gdn.h -- C ABI of libgdn: the Gated DeltaNet (GDN) token mixer's gated
 * delta rule on NVIDIA B200 (sm_100a).
 *
 * The operation ("Qwen3.8-Flash-Next: architecture, efficiency and technical
 * lineage", section 03 "Gated DeltaNet", update equations; product form in
 * "On the Design of Qwen3.8-Next Architecture ... close reading", section
 * 4.1), per sequence and per value head, token by token:
 *
 *     S~  = alpha_t S_{t-1}
 *     e_t = v_t - S~^T k_t
 *     S_t = S~ + beta_t k_t e_t^T      (= alpha_t (I - beta_t k k^T) S + beta_t k v^T)
 *     y_t = scale * S_t^T q_t
 *
 * with q, k L2-normalised over d_k (the same page, section 03, and the
 * hyper.ai summary, "Method": queries and keys are L2-normalised), alpha =
 * exp(log_alpha) in (0,1), beta in (0,1), and an optional output epilogue
 * (section 03, "what Qwen changed on the original GDN": zero-centred
 * RMSNorm, sigmoid output gate; normalise first, then gate):
 *
 *     out_t = y_t / sqrt(mean_j y_tj^2 + eps_norm) * (1 + w) * sigmoid(g_t)
 *
 * Conventions shared by every entry point:
 *   - All pointers are DEVICE pointers unless stated otherwise, dense and
 *     row-major, 16-byte aligned.  The caller owns every buffer; the library
 *     allocates no memory and, apart from gdn_check_device_error, never
 *     synchronises.  Work is enqueued on `stream` and runs asynchronously;
 *     a CUDA error raised by the kernel surfaces on the caller's next
 *     synchronisation.
 *   - Value head h reads QK head h / (H_v / H_qk) (contiguous groups);
 *     H_v % H_qk != 0 is GDN_ERR_INVALID_ARG.
 *   - The recurrent state of one head is S[i][j], i over d_k, j over d_v,
 *     fp32.  Prefill and decode use the same layout, so decode continues from
 *     a prefill's final state.
 *   - Supported head dims: d_k, d_v in {16, 32, 64, 128}; anything else is
 *     GDN_ERR_UNSUPPORTED.
 *   - Input dtype (q, k, v, g and the output y): GDN_BF16 or GDN_FP32.
 *     log_alpha, beta, norm_w and all states are always fp32.
 *   - Arguments are validated on the host before anything is enqueued; a
 *     rejected call enqueues nothing and leaves every output untouched.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle (same object as cudaStream_t); 0 = legacy
 * default stream. */
typedef struct CUstream_st* gdn_stream_t;

typedef enum {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = 1, /* null pointer, bad shape, bad cu_seqlens ...  */
  GDN_ERR_UNSUPPORTED = 2, /* a head dim or dtype the library does not support */
  GDN_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed         */
  GDN_ERR_TIMEOUT = 4      /* a device-side wait hit its iteration limit   */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_FP32 = 1 } gdn_dtype;

/* Which prefill kernel runs.  AUTO picks the tensor-core kernel when it
 * supports the shape (bf16, d_k = d_v = 128) and the portable CUDA-core
 * kernel otherwise.  The tensor kernel runs either one CTA per (sequence,
 * value head) or, when there are too few of those to fill the GPU, several
 * CTAs per item that split the per-chunk work: a cluster (PAIR) or, given a
 * workspace (gdn_chunk_fwd_ws), one chain CTA and two preparation CTAs per
 * item exchanging tiles through the workspace (SPLIT).  PAIR / SINGLE /
 * SPLIT force one layout (same results up to rounding).  A tensor path on an
 * unsupported shape is GDN_ERR_UNSUPPORTED. */
typedef enum {
  GDN_PATH_AUTO = 0,
  GDN_PATH_TENSOR = 1,        /* tcgen05 MMA + TMEM chunked kernel, layout chosen by size */
  GDN_PATH_SIMT = 2,          /* fp32 CUDA-core chunked kernel                           */
  GDN_PATH_TENSOR_PAIR = 3,   /* tensor kernel, two CTAs (a cluster) per sequence x head */
  GDN_PATH_TENSOR_SINGLE = 4, /* tensor kernel, one CTA per sequence x head             */
  GDN_PATH_TENSOR_SPLIT = 5   /* tensor kernel, chain + 2 prep CTAs per item; workspace  */
} gdn_prefill_path;

/*
 * gdn_chunk_fwd -- prefill over a packed batch of variable-length sequences,
 * chunkwise-parallel within each sequence (chunks of 64 tokens), the fp32
 * state carried from chunk to chunk.  The result equals the token-by-token
 * recurrence above up to rounding.
 *
 *   q, k           [total_T, H_qk, d_k]  in_dtype
 *   v              [total_T, H_v, d_v]   in_dtype
 *   log_alpha      [total_T, H_v] fp32, log of the decay gate (finite, <= 0)
 *   beta           [total_T, H_v] fp32, write gate
 *   g              [total_T, H_v, d_v] in_dtype, or NULL: no epilogue
 *   norm_w         [d_v] fp32 (applied as 1 + w), or NULL (= zeros); ignored
 *                  when g is NULL
 *   initial_state  [n_seq, H_v, d_k, d_v] fp32, or NULL (= zeros)
 *   cu_seqlens     [n_seq + 1] int32 DEVICE array of sequence offsets,
 *                  cu[0] = 0, non-decreasing, cu[n_seq] = total_T; NULL
 *                  means one sequence (n_seq must be 1).  Empty sequences
 *                  are allowed (final = initial).  The library cannot read
 *                  a device array on the host without a synchronisation, so
 *                  a malformed cu_seqlens is caught by the kernel: offending
 *                  sequences write nothing and gdn_check_device_error
 *                  reports GDN_ERR_INVALID_ARG.
 *   n_seq          number of sequences (>= 1)
 *   total_T        number of packed tokens (>= 0)
 *   l2norm_qk      1: normalise q, k in the kernel; 0: used as given
 *   eps_l2         inside the L2-norm square root (default 1e-6)
 *   eps_norm       inside the RMSNorm square root (default 1e-6)
 *   scale          multiplies y before the epilogue (default 1.0)
 *   y              [total_T, H_v, d_v] in_dtype, written
 *   final_state    [n_seq, H_v, d_k, d_v] fp32 or NULL; may alias
 *                  initial_state exactly (in-place update), must not
 *                  partially overlap it
 *   path           kernel selection (see gdn_prefill_path)
 */
gdn_status gdn_chunk_fwd_path(
    const void* q, const void* k, const void* v, const float* log_alpha,
    const float* beta, const void* g, const float* norm_w,
    const float* initial_state, const int32_t* cu_seqlens, int32_t n_seq,
    int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm,
    float scale, void* y, float* final_state, gdn_prefill_path path,
    gdn_stream_t stream);

/*
 * gdn_chunk_fwd_workspace_size -- bytes of device workspace that
 * gdn_chunk_fwd_ws can use for a batch of n_seq sequences x H_v value heads.
 * Up to 64 items: the split layout (per item a ring of eight 73,984-byte
 * hand-off slots and 128 bytes of flags, the flag block rounded up to 256
 * bytes; 28,416,000 bytes for 48 items).  More than 64 items and at most 1024
 * sequences: n_seq int32 (rounded up to 256 bytes) for the order in which
 * the one-CTA layout takes the sequences, longest first, so that long
 * sequences do not start last.  Returns 0 when neither applies: not bf16
 * with d_k = d_v = 128, or more than 64 items and more than 1024 sequences.
 * Host only; no CUDA call.
 */
size_t gdn_chunk_fwd_workspace_size(int32_t n_seq, int32_t H_v, int32_t d_k, int32_t d_v,
                                    gdn_dtype in_dtype);

/*
 * gdn_chunk_fwd_ws -- gdn_chunk_fwd_path with a caller-owned device
 * workspace that enables the split layout for small batches (and the
 * longest-first sequence order of the one-CTA layout for larger ones).
 *
 *   workspace        DEVICE pointer, 256-byte aligned, or NULL (then this is
 *                    gdn_chunk_fwd_path)
 *   workspace_bytes  its size; must be >= gdn_chunk_fwd_workspace_size(...)
 *                    when workspace is not NULL (else GDN_ERR_INVALID_ARG)
 *
 * With AUTO / TENSOR, the split layout runs when the workspace is given and
 * all 3 x n_seq x H_v CTAs fit on the device at once (one cooperative
 * launch); otherwise the call behaves as gdn_chunk_fwd_path and the
 * workspace is not touched.  SPLIT without a workspace is
 * GDN_ERR_INVALID_ARG; SPLIT on a batch that does not fit is
 * GDN_ERR_UNSUPPORTED.  The library clears the workspace's flags on `stream`
 * at the start of every call (an asynchronous memset) or rewrites the
 * sequence order (a one-CTA kernel launched before the prefill), so no
 * initialisation is needed; its contents are meaningless between calls.
 * The order changes which CTA takes which item, not the arithmetic: the
 * results equal those of a call without a workspace bit for bit.  Two calls that
 * may run at the same time (different streams) must not share a workspace.
 */
gdn_status gdn_chunk_fwd_ws(
    const void* q, const void* k, const void* v, const float* log_alpha,
    const float* beta, const void* g, const float* norm_w,
    const float* initial_state, const int32_t* cu_seqlens, int32_t n_seq,
    int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm,
    float scale, void* y, float* final_state, gdn_prefill_path path,
    void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_chunk_fwd_static_ws -- gdn_chunk_fwd_ws with GDN_PATH_TENSOR_SPLIT and
 * a workspace that is a fixed array inside the library (28,416,000 bytes of
 * device memory per device, part of the module image) instead of caller
 * memory: for callers that cannot give the library any memory.  The method's
 * description has no counterpart to this call; it is a deployment variant of
 * the split layout.  Nothing is allocated.
 *
 *   Arguments as for gdn_chunk_fwd, with the same argument errors
 *   (GDN_ERR_INVALID_ARG for bad head counts, dims or epsilons) checked first.
 *   Capacity: n_seq * H_v <= 48 items.  A larger batch, or a shape the split
 *   layout does not serve (not bf16 with d_k = d_v = 128), returns
 *   GDN_ERR_UNSUPPORTED before anything is enqueued; so does a batch whose
 *   3 x n_seq x H_v CTAs cannot all be resident on the device.
 *   The first call on each device looks the array's address up
 *   (cudaGetSymbolAddress, which may load the module) and keeps it; make that
 *   first call outside stream capture.  The kept address is not valid across
 *   a device reset (cudaDeviceReset or a destroyed primary context): do not
 *   call this entry point after one.  Each call clears the array's flags on `stream`
 *   before its kernel runs, so nothing needs initialising.
 *   All calls on a device share the one array: calls that can overlap (other
 *   streams, other host threads) race on it and must be serialised by the
 *   caller.  Calls on one stream are ordered and safe.
 */
gdn_status gdn_chunk_fwd_static_ws(
    const void* q, const void* k, const void* v, const float* log_alpha,
    const float* beta, const void* g, const float* norm_w,
    const float* initial_state, const int32_t* cu_seqlens, int32_t n_seq,
    int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm,
    float scale, void* y, float* final_state, gdn_stream_t stream);

/* gdn_chunk_fwd -- gdn_chunk_fwd_path with GDN_PATH_AUTO. */
gdn_status gdn_chunk_fwd(
    const void* q, const void* k, const void* v, const float* log_alpha,
    const float* beta, const void* g, const float* norm_w,
    const float* initial_state, const int32_t* cu_seqlens, int32_t n_seq,
    int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm,
    float scale, void* y, float* final_state, gdn_stream_t stream);

/*
 * gdn_decode_step -- one token for each of N independent sequences; the
 * state is read once and written back once, in place.
 *
 *   q, k        [N, H_qk, d_k] in_dtype
 *   v           [N, H_v, d_v]  in_dtype
 *   log_alpha   [N, H_v] fp32;  beta [N, H_v] fp32
 *   g, norm_w   optional epilogue, as for gdn_chunk_fwd
 *   state       [N, H_v, d_k, d_v] fp32, read and overwritten
 *   y           [N, H_v, d_v] in_dtype, written
 * Other arguments as for gdn_chunk_fwd.  N = 0 is a no-op.
 */
gdn_status gdn_decode_step(
    const void* q, const void* k, const void* v, const float* log_alpha,
    const float* beta, const void* g, const float* norm_w, float* state,
    int32_t N, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm,
    float scale, void* y, gdn_stream_t stream);

/*
 * gdn_decode_multi -- T_s consecutive tokens for each of N independent
 * sequences in one launch (e.g. verifying T_s speculative tokens).  The
 * result equals T_s calls of gdn_decode_step; the state is read once and
 * written once, and may be snapshotted after every token so that a caller
 * can roll back to any accepted prefix.  (A deployment variant of the decode
 * step; the update per token is the one described for gdn_decode_step.)
 *
 *   q, k        [N, T_s, H_qk, d_k] in_dtype
 *   v           [N, T_s, H_v, d_v]  in_dtype
 *   log_alpha   [N, T_s, H_v] fp32;  beta [N, T_s, H_v] fp32
 *   g, norm_w   optional epilogue: g [N, T_s, H_v, d_v], as for gdn_chunk_fwd
 *   state_in    [N, H_v, d_k, d_v] fp32, the state before the first token
 *   state_out   [N, H_v, d_k, d_v] fp32, the state after the last token; may
 *               be state_in exactly (in place), must not partially overlap
 *               it; NULL: not written (state_in is left as it was)
 *   snapshots   [T_s, N, H_v, d_k, d_v] fp32 or NULL: snapshot t holds the
 *               state after token t of every sequence (each one a valid
 *               state tensor); must not overlap state_in or state_out
 *   y           [N, T_s, H_v, d_v] in_dtype, written
 * Other arguments as for gdn_chunk_fwd.  N = 0 or T_s = 0 is a no-op;
 * T_s > 32 is GDN_ERR_UNSUPPORTED (the tokens' inputs are staged on chip).
 */
gdn_status gdn_decode_multi(
    const void* q, const void* k, const void* v, const float* log_alpha,
    const float* beta, const void* g, const float* norm_w,
    const float* state_in, float* state_out, float* snapshots, int32_t N,
    int32_t T_s, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm,
    float scale, void* y, gdn_stream_t stream);

/*
 * Front end of the mixer: a short depthwise causal convolution over time
 * (kernel 4) followed by SiLU, applied channel by channel to q, k and v
 * before the gated delta rule ("Qwen3.8-Flash-Next: architecture, efficiency
 * and technical lineage", section 02 module table, GDN row: Q/K/V pass a
 * short causal conv of kernel 4; hyper.ai summary, "Method": projections
 * followed by short depthwise causal convolutions; "On the Design of
 * Qwen3.8-Next Architecture ... close reading", section 4.1: short conv +
 * SiLU + L2 norm).  Per channel, with w[c][3] the weight of the current
 * token: u_t = w3 x_t + w2 x_{t-1} + w1 x_{t-2} + w0 x_{t-3} (no bias), and
 * the output is u_t * sigmoid(u_t).  SiLU on v as well as on q and k is a
 * reading: the pages name the activation for q and k only.
 *
 * Shared conventions of the calls below:
 *   conv_w      [2 H_qk d_k + H_v d_v, 4] fp32; channels numbered q (head
 *               major, H_qk d_k of them), then k, then v (H_v d_v)
 *   conv state  [n_seq (or N), H_v, 3, 2 d_k + d_v] fp32: for value head h,
 *               the three inputs before the next token (oldest first) of its
 *               QK head's q channels, k channels, then its own v channels.
 *               The q/k part is repeated in each value head of a group (all
 *               copies equal), so one value head's slice can be rewritten in
 *               place by the kernel that owns it.  NULL input = zeros.
 */

/*
 * gdn_conv_frontend -- the front end alone over a packed batch.
 *   q, k, v            pre-conv inputs, shapes and dtype as gdn_chunk_fwd's
 *   conv_state_in      the state before each sequence, or NULL (zeros)
 *   conv_state_out     the state after each sequence (its last three inputs,
 *                      earlier ones from conv_state_in for sequences shorter
 *                      than three), or NULL; must not overlap conv_state_in
 *   q_out, k_out, v_out  outputs, same shapes and dtype; must not overlap
 *                      the inputs
 * HBM-bound: every element read once and written once.
 */
gdn_status gdn_conv_frontend(
    const void* q, const void* k, const void* v, const float* conv_w,
    const float* conv_state_in, float* conv_state_out, const int32_t* cu_seqlens,
    int32_t n_seq, int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, void* q_out, void* k_out, void* v_out, gdn_stream_t stream);

/* Workspace bytes gdn_chunk_fwd_conv needs (0 for arguments it never accepts):
 * the front end's outputs plus gdn_chunk_fwd_workspace_size(...). */
size_t gdn_chunk_fwd_conv_workspace_size(int32_t n_seq, int64_t total_T, int32_t H_qk,
                                         int32_t H_v, int32_t d_k, int32_t d_v,
                                         gdn_dtype in_dtype);

/*
 * gdn_chunk_fwd_conv -- gdn_chunk_fwd_ws on pre-conv q, k, v (the L2 norm of
 * q and k, when l2norm_qk, follows the SiLU).  On the portable path
 * (GDN_PATH_SIMT, or GDN_PATH_AUTO for shapes the tensor-core kernel does not
 * serve) the front end is fused into the prefill kernel and the activations
 * stay in fp32 on chip.  On the tensor-core paths the front end runs first
 * (gdn_conv_frontend, its outputs written into the workspace in the input
 * dtype), then the prefill.  conv_state_in / conv_state_out as for
 * gdn_conv_frontend; everything else as for gdn_chunk_fwd_ws.  The workspace
 * (256-byte aligned, at least gdn_chunk_fwd_conv_workspace_size bytes) is
 * required.
 */
gdn_status gdn_chunk_fwd_conv(
    const void* q, const void* k, const void* v, const float* conv_w,
    const float* conv_state_in, float* conv_state_out, const float* log_alpha,
    const float* beta, const void* g, const float* norm_w, const float* initial_state,
    const int32_t* cu_seqlens, int32_t n_seq, int64_t total_T, int32_t H_qk, int32_t H_v,
    int32_t d_k, int32_t d_v, gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2,
    float eps_norm, float scale, void* y, float* final_state, gdn_prefill_path path,
    void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_decode_conv -- gdn_decode_multi on pre-conv q, k, v with the front end
 * fused into the decode kernel: each (sequence, value head) convolves its
 * staged q/k/v channels with its slice of conv_state ([N, H_v, 3,
 * 2 d_k + d_v], read, then rewritten in place with the last three inputs;
 * NULL = zeros, not written), applies SiLU, then runs the T_s decode steps.
 * conv_w is required and is laid out as for gdn_conv_frontend; conv_state
 * must not overlap state_in, state_out or snapshots.  Other arguments as for
 * gdn_decode_multi.  Continues a gdn_chunk_fwd_conv prefill exactly (same
 * state layouts).
 */
gdn_status gdn_decode_conv(
    const void* q, const void* k, const void* v, const float* conv_w, float* conv_state,
    const float* log_alpha, const float* beta, const void* g, const float* norm_w,
    const float* state_in, float* state_out, float* snapshots, int32_t N, int32_t T_s,
    int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v, gdn_dtype in_dtype,
    int32_t l2norm_qk, float eps_l2, float eps_norm, float scale, void* y,
    gdn_stream_t stream);

/*
 * Gated Residual (GR) with an FP8 residual state, around each block of the
 * layer ("Qwen3.8-Flash-Next: architecture, efficiency and technical
 * lineage", section 05 "Residual design", part 4 "GR", its "Group RMSNorm"
 * and "Low-rank router" boxes, and the inference paragraph of the same
 * section on the FP8 state and the fused read and write).  The residual
 * stream of a token is n_r branches of d channels (the model: n_r = 4,
 * d = 2560, router rank d / 8 = 320):
 *
 *   read:  R^_i = R_i / sqrt(mean(R_i^2) + eps) * gamma_i
 *          G    = sigmoid(W_u SiLU((1/n_r) W_d vec(R^)))      (n_r x d gates)
 *          x    = (1/n_r) sum_i G_i o R^_i                     (block input)
 *          s    = 2 sigmoid((1/n_r) W_w vec(R^))               (n_r write scalars)
 *   write: R'_i = R_i + s_i y                                  (block output y)
 *
 * State: codes [T, n_r, d] uint8, OCP E4M3 (finite, saturating), and one
 * fp32 scale per (token, branch) row: value = E4M3(code) * scale.  A written
 * row is requantised with scale max|R'| / 448 (1 for an all-zero row), codes
 * rounded to nearest even.  Format, scaling and eps are readings: the pages
 * say only that the state is FP8.
 */

/* Workspace bytes gdn_gr_read needs (0 for arguments it never accepts). */
size_t gdn_gr_read_workspace_size(int64_t T, int32_t n_r, int32_t d, int32_t rank);

/*
 * gdn_gr_read -- the block input x and the write scalars s from the state.
 *   codes, scales   the state, as above (read only)
 *   gamma           [n_r, d] fp32 branch gains
 *   W_d             [rank, n_r d] bf16;  W_u [n_r d, rank] bf16;
 *   W_w             [n_r, n_r d] bf16
 *   T, n_r (1..8), d (multiple of 8), rank (multiple of 8), eps (>= 0)
 *   x               [T, d] bf16, written
 *   s               [T, n_r] fp32, written (pass to gdn_gr_write)
 *   workspace       256-byte aligned, gdn_gr_read_workspace_size bytes
 * The two router products run on this library's tcgen05 GEMM (bf16
 * operands, fp32 accumulation in tensor memory, bf16 results; when its
 * tile grid is small and K long, the first is split along K into fp32
 * partials in the workspace that are summed in a fixed order, so results
 * stay deterministic); the normalisation, the router
 * activations and the gated branch mean are kernels of their own.  Five or
 * six kernel launches (six when the first GEMM splits K), after two
 * device-to-device copies and a memset that stack [W_d; W_w; 0] into the
 * workspace, all on `stream`.
 */
gdn_status gdn_gr_read(const uint8_t* codes, const float* scales, const float* gamma,
                       const void* W_d, const void* W_u, const void* W_w, int64_t T,
                       int32_t n_r, int32_t d, int32_t rank, float eps, void* x, float* s,
                       void* workspace, size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_gr_write -- R'_i = R_i + s_i y, requantised in place (codes and scales
 * are rewritten).  y [T, d] bf16; s [T, n_r] fp32 from gdn_gr_read.  One
 * kernel; each row is read twice (its maximum, then its codes) and written
 * once.
 */
gdn_status gdn_gr_write(uint8_t* codes, float* scales, const void* y, const float* s,
                        int64_t T, int32_t n_r, int32_t d, gdn_stream_t stream);

/*
 * gdn_chunk_bwd_workspace_size -- bytes of device workspace gdn_chunk_bwd
 * needs for a packed batch (0 for arguments it can never accept).  About
 * 460 KB per 64-token chunk per value head at d_k = d_v = 128 (chunk states
 * and their gradients, per-chunk matrices) plus 1.1 KB per token per value
 * head; e.g. 1.45 GB for one 4,096-token sequence with 48 value heads.
 */
size_t gdn_chunk_bwd_workspace_size(int32_t n_seq, int64_t total_T, int32_t H_qk,
                                    int32_t H_v, int32_t d_k, int32_t d_v);

/*
 * gdn_chunk_bwd -- gradients of a gdn_chunk_fwd call, for training.
 *
 * Differentiates the forward of gdn_chunk_fwd (the recurrence of
 * "Qwen3.8-Flash-Next: architecture, efficiency and technical lineage",
 * section 03 "Gated DeltaNet", update equations, with the optional RMSNorm x
 * sigmoid(g) epilogue of the same section) given the gradient of the loss
 * with respect to its outputs.  The pages describe no backward; this is the
 * exact derivative of the forward, evaluated chunkwise (C = 64) on CUDA
 * cores in fp32.  Nothing of the forward call is needed: the chunk states
 * are recomputed from the inputs.
 *
 * Inputs: every forward input, with the same meaning, shapes, dtypes and
 * defaults as for gdn_chunk_fwd (g and norm_w select the epilogue), plus
 *   dy              [total_T, H_v, d_v] in_dtype: dLoss/dy (y after the
 *                   epilogue when g is given)
 *   d_final_state   [n_seq, H_v, d_k, d_v] fp32 or NULL (zeros)
 * Outputs (fp32, caller-owned, fully overwritten):
 *   dq, dk          [total_T, H_qk, d_k]  (through the in-kernel L2 norm
 *                   when l2norm_qk; summed over the value heads of a group)
 *   dv              [total_T, H_v, d_v]
 *   dlog_alpha      [total_T, H_v]
 *   dbeta           [total_T, H_v]
 *   dg              [total_T, H_v, d_v]; required when g is given, else
 *                   must be NULL
 *   dnorm_w         [d_v] or NULL (only with g; not written when NULL)
 *   d_initial_state [n_seq, H_v, d_k, d_v] or NULL (not written)
 *   workspace       device memory, 256-byte aligned, at least
 *                   gdn_chunk_bwd_workspace_size(...) bytes; owned by the
 *                   caller and not retained; calls that may overlap must not
 *                   share one
 * Every pointer 16-byte aligned; outputs must not overlap inputs or each
 * other.  Errors as for gdn_chunk_fwd; a workspace that is missing, too
 * small or misaligned is GDN_ERR_INVALID_ARG.  Asynchronous on `stream`;
 * allocates nothing.
 */
gdn_status gdn_chunk_bwd(
    const void* q, const void* k, const void* v, const float* log_alpha,
    const float* beta, const void* g, const float* norm_w,
    const float* initial_state, const int32_t* cu_seqlens, int32_t n_seq,
    int64_t total_T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
    gdn_dtype in_dtype, int32_t l2norm_qk, float eps_l2, float eps_norm,
    float scale, const void* dy, const float* d_final_state, float* dq, float* dk,
    float* dv, float* dlog_alpha, float* dbeta, float* dg, float* dnorm_w,
    float* d_initial_state, void* workspace, size_t workspace_bytes,
    gdn_stream_t stream);

/*
 * gdn_check_device_error -- synchronise `stream`, then read and clear the
 * library's device-side error word on the current device.  Returns GDN_OK,
 * GDN_ERR_TIMEOUT (a kernel's bounded wait ran out and the kernel returned
 * early; its outputs are incomplete), GDN_ERR_INVALID_ARG (a kernel found a
 * malformed cu_seqlens) or GDN_ERR_CUDA (the synchronisation itself failed).
 * This call blocks the host; the compute entry points never do.
 */
gdn_status gdn_check_device_error(gdn_stream_t stream);

/*
 * gdn_selftest_bounded_wait -- exercises the failure path of the library's
 * bounded waits without a fault: one thread waits on a device flag that
 * nothing sets, with the same bounded poll the split-layout prefill
 * (GDN_PATH_TENSOR_SPLIT) uses for its hand-off flags, gives up after
 * `iterations` polls (each ~32 ns apart),
 * records the timeout in the device error word and returns.  A following
 * gdn_check_device_error reports GDN_ERR_TIMEOUT once, and the context stays
 * usable.  (A test entry point; the pages have no counterpart.)
 */
gdn_status gdn_selftest_bounded_wait(int32_t iterations, gdn_stream_t stream);

/* Static text for a status code. */
const char* gdn_status_string(gdn_status status);

/* Library version as an integer (major * 10000 + minor * 100 + patch). */
int32_t gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */

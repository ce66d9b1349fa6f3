/*
 * jab_dit.h -- C ABI of the B200 (sm_100a) Ideogram 4 single-stream DiT block hot path.
 *
 * The three calls of the hot path:
 *   dit_block_forward   one single-stream DiT block over the joint [text; image] sequence
 *   cond_proj_forward   the frozen llm_cond_norm / llm_cond_proj projection of the
 *                       13 concatenated 4096-wide text-encoder hidden states
 *   euler_cfg_step      dual-branch classifier-free guidance + one flow-matching Euler step
 * and the per-step kernels they are built from, exposed for parity testing.
 *
 * Conventions (all calls):
 *   - Every pointer is caller-owned DEVICE memory unless stated otherwise; the library
 *     allocates nothing per call.  Scratch comes from the caller's workspace.
 *   - bf16 data is passed as raw 16-bit patterns (uint16_t / void*), e4m3 as bytes.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous on it; the return code covers synchronous argument validation and
 *     launch errors only.  Device-side failures (a bounded wait that timed out) are
 *     reported by dit_poll_error().
 *   - Pointers must be 16-byte aligned; tensors are dense row-major.
 *   - Each call runs on the CUDA device current on the calling thread.
 */
#ifndef JAB_DIT_H
#define JAB_DIT_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DIT_API __attribute__((visibility("default")))
#else
#define DIT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DIT_OK = 0,
  DIT_ERR_INVALID_ARG = 1, /* null / misaligned pointer, inconsistent sizes */
  DIT_ERR_UNSUPPORTED = 2, /* a size this build does not handle (see each call) */
  DIT_ERR_WORKSPACE = 3,   /* workspace missing or smaller than *_workspace_bytes() */
  DIT_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed */
  DIT_ERR_TIMEOUT = 5,     /* a device-side bounded wait gave up (from dit_poll_error) */
  DIT_ERR_DEVICE = 6       /* another device-side error was recorded (from dit_poll_error) */
} dit_status;

/* Storage formats of activations, for the per-step kernels below. */
typedef enum { DIT_FMT_BF16 = 0, DIT_FMT_F16 = 1, DIT_FMT_F32 = 2 } dit_format;

/* Shape and numerics of one block.
 * rope_sections: rotary PAIRS per axis (t, h, w), laid out contiguously over the
 *   first head_dim/2 frequencies; must sum to head_dim/2.  The Ideogram 4 deep dive,
 *   section 6-3 ("3D MRoPE"), gives mrope_section = (24, 20, 20) for head_dim 128.
 * rope_theta: RoPE base (10000 by default); inv_freq_i = fp32(theta^(-2i/head_dim)).
 * eps: RMSNorm epsilon of every norm in the block.
 * gelu_tanh: 0 = exact erf GELU, 1 = tanh approximation.
 * Supported: d_model = n_heads * head_dim <= 8192, head_dim in {64, 128}, d_model and d_mlp
 * multiples of 256. */
typedef struct {
  int32_t d_model, n_heads, head_dim, d_mlp;
  int32_t rope_sections[3];
  float rope_theta, eps;
  int32_t gelu_tanh;
} dit_block_config;

/* FP8 weights of one block, as the Ideogram 4 FP8 checkpoint stores them
 * (unsloth diffusion_ideogram4.py commit log, fp8 loader commit): e4m3 bytes
 * [out, in] row-major with a per-output-row fp32 weight_scale [out]; the real weight
 * is fp8 * weight_scale[:, None].  w_qkv is the fused attention.qkv.weight [3d, d]
 * with Q, K, V rows stacked in that order; w_o is attention.o.weight [d, d];
 * w_up [d_mlp, d], w_down [d, d_mlp] are the FeedForward projections.
 * Gains are bf16: g_norm1, g_norm2 [d] (the two pre-norms), g_q, g_k [head_dim]
 * (QK-RMSNorm, shared by all heads). */
typedef struct {
  const uint8_t *w_qkv, *w_o, *w_up, *w_down;
  const float *s_qkv, *s_o, *s_up, *s_down;
  const void *g_norm1, *g_norm2, *g_q, *g_k;
} dit_block_weights;

/* Bytes of device workspace dit_block_forward needs for this shape (256-byte aligned). */
DIT_API size_t dit_block_workspace_bytes(const dit_block_config* cfg, int batch, int n_text, int grid_h, int grid_w);

/* One single-stream DiT block forward (Ideogram 4.0 announcement thread: self-attention,
 * QK-RMSNorm and 3D multimodal RoPE over one sequence of text and image tokens; deep dive
 * section 4-2: text and image tokens concatenated through the same self-attention):
 *   h  = RMSNorm(x; g_norm1)
 *   q,k,v = split(h W_qkv^T);  q,k = MRoPE(RMSNorm_head(q; g_q)), MRoPE(RMSNorm_head(k; g_k))
 *   x1 = x + Attn(q, k, v) W_o^T          (bidirectional, softmax scale 1/sqrt(head_dim))
 *   y  = x1 + GELU(RMSNorm(x1; g_norm2) W_up^T) W_down^T
 * x_in: bf16 [batch, n_text + grid_h*grid_w, d_model], text rows first, image rows in
 *   raster order (r*grid_w + c).
 * x_out: bf16, same shape; must not alias x_in.
 * t_img: temporal position of the image tokens (< 0 => n_text).  Text token j sits at
 *   (j, j, j); image cell (r, c) at (t_img, r, c).
 * pos: optional int32 [S, 3] (t, h, w) per token overriding the rule above; NULL to derive.
 * workspace: >= dit_block_workspace_bytes() bytes, 256-byte aligned.
 * Errors: INVALID_ARG (null/misaligned/aliasing), UNSUPPORTED (shape rules above),
 *   WORKSPACE, CUDA. */
DIT_API int dit_block_forward(const dit_block_config* cfg, const dit_block_weights* w, const void* x_in, void* x_out,
                      int batch, int n_text, int grid_h, int grid_w, int t_img, const int32_t* pos,
                      void* workspace, size_t ws_bytes, void* stream);

/* dit_block_forward over a padded batch of prompts of different text lengths (SimpleTuner
 * Ideogram 4 quickstart, "Text Embed Cache": text embeddings are kept at each prompt's own token
 * length and only padded when a batch is formed).  Element b of x_in [batch, n_text +
 * grid_h*grid_w, d_model] holds, in this order, its L_b text rows, its grid_h*grid_w image rows
 * (raster order) and n_text - L_b rows of padding.  Every element is computed as if it were run
 * alone: text token j at (j, j, j), image cell (r, c) at (t, r, c) with t = L_b (or t_img when
 * t_img >= 0), and its attention takes only its first L_b + grid_h*grid_w tokens as keys.  The
 * outputs of padding rows are unspecified (they are computed like any row, at position (0,0,0)).
 * text_lens: DEVICE int32 [batch], 16-byte aligned; each value is clamped to [0, n_text]; an
 *   element must have at least one token (L_b + grid_h*grid_w >= 1).
 * workspace: >= dit_block_workspace_bytes() bytes (the same size as dit_block_forward).
 * Errors: as dit_block_forward; INVALID_ARG for a null or misaligned text_lens. */
DIT_API int dit_block_forward_padded(const dit_block_config* cfg, const dit_block_weights* w, const void* x_in,
                                     void* x_out, int batch, int n_text, int grid_h, int grid_w, int t_img,
                                     const int32_t* text_lens, void* workspace, size_t ws_bytes, void* stream);

/* The W8A8 variant of dit_block_forward: the inputs of the QKV and MLP-up projections (the two
 * pre-norm outputs) are quantised to e4m3 per token (scale = amax of the row / 448, codes rounded
 * to nearest even, saturating) and multiplied with the e4m3 weights on the FP8 tensor-core path
 * (tcgen05 kind::f8f6f4, twice the 16-bit rate).  The normalised, rotated q and k are rounded to
 * e4m3 as well, with one static scale each (see dit_qknorm_mrope_e4m3), for q k^T on the same
 * path; P V, the output and the MLP-down products keep 16-bit activations.  The pages run the
 * dequantised model with 16-bit activations; this variant trades accuracy for speed (FP8 training
 * through fp8-torchao is what SimpleTuner's quickstart, "ハードウェアと精度", uses); its error
 * against the 16-bit pipeline is a few per cent per element (2.5 % mean at 1024 px).
 * Arguments, workspace and errors as dit_block_forward; UNSUPPORTED for d_model > 8192. */
DIT_API int dit_block_forward_w8a8(const dit_block_config* cfg, const dit_block_weights* w, const void* x_in,
                                   void* x_out, int batch, int n_text, int grid_h, int grid_w, int t_img,
                                   const int32_t* pos, void* workspace, size_t ws_bytes, void* stream);

/* Bytes of device workspace dit_stack_forward needs: one block's workspace plus one
 * activation buffer [batch, S, d_model] bf16 for the ping-pong between blocks. */
DIT_API size_t dit_stack_workspace_bytes(const dit_block_config* cfg, int batch, int n_text, int grid_h, int grid_w);

/* n_blocks DiT blocks back to back (the Ideogram 4 DiT stacks 34 of them: Ideogram 4.0
 * announcement thread, "four key components"; deep dive section 4-2):
 *   x_out = block[n-1]( ... block[1]( block[0](x_in) ) ... )
 * w: HOST array of n_blocks weight sets (each as for dit_block_forward; read during the call).
 * The intermediate activations alternate between x_out and a buffer in the workspace so that
 * the last block writes x_out; the result equals n_blocks successive dit_block_forward calls
 * bit for bit.  Other arguments as dit_block_forward; x_out must not alias x_in.
 * workspace: >= dit_stack_workspace_bytes() bytes, 256-byte aligned.
 * Errors: as dit_block_forward (INVALID_ARG also for n_blocks < 1 or a null w). */
DIT_API int dit_stack_forward(const dit_block_config* cfg, const dit_block_weights* w, int n_blocks, const void* x_in,
                              void* x_out, int batch, int n_text, int grid_h, int grid_w, int t_img,
                              const int32_t* pos, void* workspace, size_t ws_bytes, void* stream);

/* Bytes of device workspace dit_denoise_steps needs: the block inputs and outputs of both
 * branches ([batch, n_text + grid_h*grid_w, d_model] bf16, four buffers) plus the larger of the
 * two stacks' workspaces. */
DIT_API size_t dit_denoise_workspace_bytes(const dit_block_config* cfg, int batch, int n_text_c, int n_text_u,
                                           int grid_h, int grid_w);

/* n_steps flow-matching denoising steps with dual-branch classifier-free guidance (Ideogram 4
 * deep dive, section 4-6 pseudocode; section 4-4: asymmetric CFG with a separate unconditional
 * DiT, and a guidance weight that may change per step, e.g. V4_QUALITY_48 = 45 steps at 7 then
 * 3 steps at 3).  Per step i:
 *   v_c = stack_cond  ([text_cond;   z])   (n_blocks blocks, weights w_cond)
 *   v_u = stack_uncond([text_uncond; z])   (n_blocks blocks, weights w_uncond)
 *   z   = z + dt[i] * (v_u + guidance[i] * (v_c - v_u))    (= gw v_c + (1 - gw) v_u)
 * The pages describe neither the map from the latent to the DiT's image tokens nor the final
 * projection back to a velocity; both are taken as the identity here: z holds the image tokens
 * themselves (d_model channels), enters each branch as bf16 rows after its text rows, and the
 * velocity of a branch is the image rows of its stack's bf16 output.  The update is fp32 as in
 * euler_cfg_step.
 * text_cond: bf16 [batch, n_text_c, d_model]; text_uncond: bf16 [batch, n_text_u, d_model]
 *   (the unconditional branch's text, zeros on the pages; n_text_u may be 0).
 * z: fp32 [batch, grid_h*grid_w, d_model], updated in place.
 * w_cond, w_uncond: HOST arrays of n_blocks weight sets each.
 * guidance, dt: HOST arrays of n_steps values (dt = s - t < 0 when integrating from t=1 to 0).
 * workspace: >= dit_denoise_workspace_bytes() bytes, 256-byte aligned.
 * Errors: as dit_stack_forward; INVALID_ARG for null arrays or n_steps < 0. */
DIT_API int dit_denoise_steps(const dit_block_config* cfg, const dit_block_weights* w_cond,
                              const dit_block_weights* w_uncond, int n_blocks, const void* text_cond, int n_text_c,
                              const void* text_uncond, int n_text_u, float* z, int batch, int grid_h, int grid_w,
                              int n_steps, const float* guidance, const float* dt, void* workspace, size_t ws_bytes,
                              void* stream);

/* One branch's block input of a denoising step, the first part of each step of dit_denoise_steps
 * (for callers that run the two branches themselves, e.g. on two GPUs):
 *   x[b] = [text[b]; bf16(z[b])]
 * z: fp32 [batch, n_img, d_model]; text: bf16 [batch, n_text, d_model] (NULL when n_text = 0);
 * x: bf16 [batch, n_text + n_img, d_model].  d_model % 8 == 0. */
DIT_API int dit_tokens_from_latent(const float* z, const void* text, void* x, int batch, int n_text, int n_img,
                                   int d_model, void* stream);

/* Size of the fixed device scratch behind dit_block_forward_noalloc (32 MiB).  Every GPU
 * that loads this library holds this much device memory until the process exits. */
#define DIT_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* dit_block_forward for callers that cannot allocate device memory: hosts that reserve all
 * device memory at start-up, plugin interfaces that pass a kernel only its inputs and outputs,
 * or latency-critical paths where an allocation (which may synchronise the device) is not
 * acceptable.  The pages describe no such call; it exists for these integrators.
 * Same arguments and results as dit_block_forward, minus the workspace: the intermediates live
 * in a fixed array of DIT_NOALLOC_SCRATCH_BYTES inside the library.  No allocation happens.
 * Limits and behaviour:
 *  - shapes whose dit_block_workspace_bytes() exceeds DIT_NOALLOC_SCRATCH_BYTES return
 *    DIT_ERR_UNSUPPORTED (e.g. the tiny 16 + 8x8 block fits; the 1024 px block does not);
 *  - the first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *    with that device current and keeps it for later calls on that device;
 *  - all calls share the one array and it keeps the last call's contents; calls that
 *    overlap on the GPU (other streams, other threads) race on it, so serialise them. */
DIT_API int dit_block_forward_noalloc(const dit_block_config* cfg, const dit_block_weights* w, const void* x_in,
                                      void* x_out, int batch, int n_text, int grid_h, int grid_w, int t_img,
                                      const int32_t* pos, void* stream);

/* Bytes of device workspace cond_proj_forward needs: the normalised features (f16) and,
 * when the token count leaves SMs idle, fp32 split-K partial sums of the projection. */
DIT_API size_t cond_proj_workspace_bytes(int n_tok, int n_layers, int hidden, int d_out);

/* llm_cond_norm + llm_cond_proj (SimpleTuner Ideogram 4 quickstart, "Text Embed Cache"):
 *   out = RMSNorm(feats; g_norm, eps) (scale (.) W8)^T
 * feats: bf16 [n_tok, n_layers*hidden] (13 x 4096 = 53,248 for Ideogram 4);
 * g_norm: bf16 [n_layers*hidden]; w: e4m3 [d_out, n_layers*hidden]; scale: fp32 [d_out];
 * out: bf16 [n_tok, d_out].  n_layers*hidden and d_out must be multiples of 256. */
DIT_API int cond_proj_forward(const void* feats, int n_tok, int n_layers, int hidden, const void* g_norm, float eps,
                      const uint8_t* w, const float* scale, int d_out, void* out, void* workspace, size_t ws_bytes,
                      void* stream);

/* Dual-branch CFG + Euler (Ideogram 4 deep dive, section 4-6 pseudocode):
 *   v = v_uncond + guidance * (v_cond - v_uncond)   (= gw*v_cond + (1-gw)*v_uncond)
 *   x = x + dt * v                                  (dt = s - t < 0 from t=1 to 0)
 * x: fp32 [n], updated in place; v_cond, v_uncond: bf16 [n].  Arithmetic is fp32:
 * d = v_c - v_u; v = fma(guidance, d, v_u); x = fma(dt, v, x). */
DIT_API int euler_cfg_step(float* x, const void* v_cond, const void* v_uncond, int64_t n, float guidance, float dt,
                   void* stream);

/* ---- per-step kernels (the block is composed of these; exposed for parity tests) ---- */

/* e4m3 bytes -> bf16 [n], exact for every finite code (the FP8 dequant the GEMMs use
 * on chip, before the per-row scale). */
DIT_API int dit_e4m3_to_bf16(const uint8_t* codes, void* out, int64_t n, void* stream);

/* Row RMSNorm with gain: y = x / sqrt(mean(x^2) + eps) * g, fp32 math.
 * x: [rows, cols] in x_fmt (BF16 or F32); y: [rows, cols] in y_fmt (BF16 or F16);
 * g: bf16 [cols].  x and y may alias when the formats match.  cols % 8 == 0. */
DIT_API int dit_rmsnorm_rows(const void* x, int x_fmt, const void* g, void* y, int y_fmt, int64_t rows, int64_t cols,
                             float eps, void* stream);

/* The (t, h, w) int32 [S, 3] positions the block uses for this sequence (see dit_block_forward). */
DIT_API int dit_mrope_positions(int n_text, int grid_h, int grid_w, int t_img, int32_t* pos_out, void* stream);

/* Y[M, N] = act( A[M, K] (W8[N, K])^T * scale[N] ) + R[M, N]
 * A: a_fmt (BF16 or F16) row-major; W8: e4m3 row-major (the weight is widened on chip,
 * exactly, to A's format); scale: fp32 [N]; act: 0 = none, 1 = GELU (gelu_tanh selects
 * the form); R: optional residual in res_fmt (BF16/F16/F32), NULL for none; Y: y_fmt
 * (BF16/F16/F32).  fp32 accumulation.  N % 32 == 0, K % 16 == 0. */
DIT_API int dit_gemm_w8a16(const void* a, int a_fmt, const uint8_t* w8, const float* scale, void* y, int y_fmt,
                           const void* residual, int res_fmt, int M, int N, int K, int act, int gelu_tanh,
                           void* stream);

/* Y[M, N] = act( A8[M, K] (W8[N, K])^T * sa[m] * sw[n] ): e4m3 activations with a per-row fp32
 * scale sa [M] and e4m3 weights with their per-row weight_scale sw [N], both row-major; Y in y_fmt
 * (BF16/F16/F32); act 0 = none, 1 = GELU (gelu_tanh selects the form).  fp32 accumulation.
 * N % 32 == 0, K % 16 == 0. */
DIT_API int dit_gemm_w8a8(const uint8_t* a8, const float* sa, const uint8_t* w8, const float* sw, void* y, int y_fmt,
                          int M, int N, int K, int act, int gelu_tanh, void* stream);

/* Row RMSNorm to per-token e4m3: o = x / sqrt(mean(x^2) + eps) * g (fp32), s = amax|o| / 448
 * (1 for a zero row), y8 = e4m3(o / s) rounded to nearest even; y_scale[row] = s.
 * x: [rows, cols] in x_fmt (BF16 or F32); g: bf16 [cols]; y8: bytes [rows, cols]; y_scale: fp32
 * [rows].  cols % 8 == 0, cols <= 8192. */
DIT_API int dit_rmsnorm_rows_e4m3(const void* x, int x_fmt, const void* g, uint8_t* y8, float* y_scale, int64_t rows,
                                  int64_t cols, float eps, void* stream);

/* Per-head QK-RMSNorm + 3D M-RoPE, in place on a fused qkv buffer [batch, S, 3d] in fmt
 * (BF16 or F16; Q columns [0, d), K columns [d, 2d); V untouched).  pos: int32 [S, 3] or
 * NULL (derived from n_text/grid/t_img as in dit_block_forward).  The rotary angles are
 * computed inside the kernel (exact fp64 product, fp64 reduction modulo 2 pi, fp32 cosine and
 * sine); workspace and ws_bytes are not used and may be NULL / 0. */
DIT_API int dit_qknorm_mrope(void* qkv, int fmt, int batch, int n_text, int grid_h, int grid_w, int t_img, const int32_t* pos,
                     const dit_block_config* cfg, const void* g_q, const void* g_k, void* workspace,
                     size_t ws_bytes, void* stream);

/* The W8A8 variant's q and k (FP8 format: unsloth diffusion_ideogram4.py commit log, fp8 loader
 * commit; QK-RMSNorm and M-RoPE: Ideogram 4.0 announcement thread): per-head QK-RMSNorm + 3D
 * M-RoPE of the fused qkv buffer exactly as dit_qknorm_mrope computes them, written as e4m3
 * codes instead of back into qkv (qkv is only read).  scale[0] (q) and scale[1] (k) =
 * fp32(fp32(sqrt(hd)) * max|g|) / 448 with g = g_q or g_k: a normalised head vector's norm is at
 * most sqrt(hd) * max|g| and the rotations keep it, so no code saturates.  q8, k8: [batch, S, d]
 * bytes, codes of value * fp32(1 / scale) rounded to nearest even; 16-byte aligned, caller-owned
 * device memory; scale: fp32 [2] on the device.  Other arguments and errors as dit_qknorm_mrope. */
DIT_API int dit_qknorm_mrope_e4m3(const void* qkv, int fmt, int batch, int n_text, int grid_h, int grid_w, int t_img,
                                  const int32_t* pos, const dit_block_config* cfg, const void* g_q, const void* g_k,
                                  uint8_t* q8, uint8_t* k8, float* scale, void* stream);

/* Joint attention with e4m3 q and k (Ideogram 4 deep dive, section 4-2: one sequence, one
 * bidirectional self-attention): out = softmax(scale[0] scale[1] (q8 k8^T) / sqrt(hd)) v per head,
 * q8 k8^T accumulated in fp32 from the codes on the FP8 tensor-core path, v and P V in fmt (BF16
 * or F16) from the fused qkv buffer [batch, S, 3d] (columns [2d, 3d)).  q8, k8: [batch, S, d]
 * bytes (16-byte aligned); scale: fp32 [2] on the device; out: [batch, S, d] in fmt.  Errors as
 * dit_joint_attention. */
DIT_API int dit_joint_attention_e4m3(const uint8_t* q8, const uint8_t* k8, const float* scale, const void* qkv,
                                     void* out, int fmt, int batch, int seq, int n_heads, int head_dim, void* stream);

/* Joint bidirectional attention: out[b, s, h*hd:(h+1)*hd] = softmax(q k^T / sqrt(hd)) v
 * over all S tokens, per head, reading q, k, v from a fused qkv buffer [batch, S, 3d] in
 * fmt (BF16 or F16).  out: [batch, S, d] in the same format. */
DIT_API int dit_joint_attention(const void* qkv, void* out, int fmt, int batch, int seq, int n_heads, int head_dim, void* stream);

/* Synchronise `stream`, then report (and clear) device-side errors recorded by any
 * kernel of this library on the current device since the last poll. */
DIT_API int dit_poll_error(void* stream);

/* ---- launch instrumentation (off by default) ----
 * While enabled, each kernel launched by dit_block_forward, cond_proj_forward,
 * euler_cfg_step, dit_rmsnorm_rows and dit_qknorm_mrope is bracketed by CUDA events on
 * its stream (the standalone GEMM and attention calls are not), so the device time of
 * every launch inside a timed region can be read back.  dit_profile_enable creates
 * max_marks events (host-side handles; the only resources this library creates) and
 * starts recording; dit_profile_read synchronises on the recorded events, writes up to
 * max_records (tag, milliseconds) pairs and returns how many it wrote (negative status
 * on error), then clears the record. */
typedef enum {
  DIT_KERNEL_END = 0,
  DIT_KERNEL_ROPE_TABLE = 1, /* no longer launched: the angles are computed by the QK-norm kernel */
  DIT_KERNEL_RMSNORM = 2,
  DIT_KERNEL_GEMM_QKV = 3,
  DIT_KERNEL_QKNORM_MROPE = 4,
  DIT_KERNEL_ATTENTION = 5,
  DIT_KERNEL_GEMM_O = 6,
  DIT_KERNEL_GEMM_UP = 7,
  DIT_KERNEL_GEMM_DOWN = 8,
  DIT_KERNEL_COND_RMSNORM = 9,
  DIT_KERNEL_COND_GEMM = 10,
  DIT_KERNEL_EULER_CFG = 11,
  DIT_KERNEL_COND_REDUCE = 12
} dit_kernel_tag;
DIT_API int dit_profile_enable(int max_marks);
/* As dit_profile_enable, but only the launches whose tag t has bit (1u << t) set in tag_mask
 * are bracketed (e.g. 1u << DIT_KERNEL_GEMM_UP: two events per block, around the MLP
 * up-projection only, so the other kernels keep their back-to-back launches).  The records
 * read back are those launches alone.  INVALID_ARG for max_marks <= 0 or an empty mask. */
DIT_API int dit_profile_enable_tags(int max_marks, uint32_t tag_mask);
DIT_API int dit_profile_disable(void);
DIT_API int dit_profile_read(int* tags, float* ms, int max_records);

/* Raw device error word seen by the last dit_poll_error() that reported an error:
 * bits 0..11 name the wait that gave up (0x1xx = bounded-wait timeout), bits 12..15 the
 * CTA's rank in its cluster, bits 16..31 the k-block / loop index. */
DIT_API uint32_t dit_last_device_error(void);

/* Launch a one-thread kernel whose only wait can never complete: it gives up after the
 * configured limit (dit_set_wait_timeout_ms) and records a timeout, which the next
 * dit_poll_error() reports as DIT_ERR_TIMEOUT.  Exercises the failure path of every
 * pipelined kernel here without faulting or hanging the device. */
DIT_API int dit_wait_selftest(void* stream);

/* Set the wall-time limit of every device-side bounded wait (default 2000 ms). */
DIT_API int dit_set_wait_timeout_ms(uint32_t ms);

DIT_API const char* dit_status_str(int status);

/* The cudaError_t code behind the last DIT_ERR_CUDA status returned on any thread (0 if none). */
DIT_API int dit_last_cuda_error(void);

/* ABI version of this header (bumped on any signature change). */
DIT_API int dit_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* JAB_DIT_H */

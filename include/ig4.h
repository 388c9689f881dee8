/*
 * ig4.h - C ABI of a B200 (sm_100a) implementation of the Ideogram 4
 * single-stream DiT block forward and of the 34-block stack.
 *
 * The operation is the one described on the Ideogram 4.0 survey page
 * ("Ideogram 4.0", section "模型架构", subsections "单 block 内部",
 * "Model spec" and "条件注入方式"):  one sequence [text tokens | image latent
 * tokens] of width emb_dim (4608) flows through Ideogram4TransformerBlock
 * layers, each an AdaLN-modulated self-attention with QK-RMSNorm and 3D
 * multimodal RoPE (mrope_section (24, 20, 20), rope_theta 5e6; text tokens use
 * a 1D position broadcast to the 3 axes, image tokens use (t, h, w)), followed
 * by an AdaLN-modulated SwiGLU MLP (intermediate 12288), both with gated
 * residuals driven by a 512-d timestep embedding (adaln_dim 512).  The weights
 * are released in FP8 E4M3 (SimpleTuner quickstart page, "硬件和精度").
 *
 * Conventions fixed where the pages are silent (they match the CPU oracle):
 *   AdaLN: mod = SiLU(temb) W_ada^T + b_ada, chunks of D in the order
 *     shift_msa, scale_msa, gate_msa, shift_mlp, scale_mlp, gate_mlp;
 *   pre-norm: RMSNorm over D (weightless, eps), then (1 + scale) and + shift;
 *   QK-RMSNorm: per head over head_dim with weights g_q, g_k [head_dim];
 *   rotary: the 64 frequency pairs act on dims [0,128) of each head, pair j
 *     joining dims j and j+64; pairs [0,24) follow t, [24,44) h, [44,64) w;
 *     inv_freq[j] = theta^(-2j/128);
 *   positions: text token l -> (l, l, l); image token (t, i, j) of a
 *     row-major grid -> (T+t, T+i, T+j) after T text tokens;
 *   attention: softmax(q k^T / sqrt(head_dim)) v, no mask;
 *   SwiGLU: u = silu(h W_gate^T) * (h W_up^T);  no biases on the block linears.
 *
 * Memory: every pointer argument documented as "device" must be device
 * memory of the current device; the caller owns every buffer.  The library
 * never allocates, frees, or synchronises a stream, except
 * ig4_last_device_error and ig4_sm_clock_mhz, which synchronise the stream
 * they are given.
 * Linear weights are row-major [out, in] (K contiguous).  All calls are
 * asynchronous on the given cudaStream_t (passed as void*, NULL = legacy
 * default stream); argument errors are returned synchronously and nothing is
 * launched.  A device-side wait that runs past its limit (about 2 s) sets a
 * device error word that ig4_last_device_error reports as IG4_ERR_TIMEOUT.
 * Calls that share a workspace or output buffer must be ordered by the caller.
 */
#ifndef IG4_H
#define IG4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ig4_status {
  IG4_OK = 0,
  IG4_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer */
  IG4_ERR_UNSUPPORTED = 2,  /* a shape or dtype outside what the kernels support */
  IG4_ERR_WORKSPACE = 3,    /* workspace too small or misaligned */
  IG4_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed */
  IG4_ERR_TIMEOUT = 5       /* a device-side wait ran past its limit */
} ig4_status;

typedef enum ig4_dtype {
  IG4_F32 = 0,
  IG4_BF16 = 1,
  IG4_E4M3 = 2,  /* FP8 E4M3 "fn" (max 448), with an fp32 scale array */
  /* block / stack weights only ("2.2 NVFP4 Mixed" of the deployment article
   * cited at the NVFP4 section below): the FFN linears w_gate, w_up, w_down
   * in NVFP4 (E2M1 codes [N][K/2], packed E4M3 block scales sf_*, fp32
   * channel scales s_*), every other linear in E4M3 with its s_* scale.
   * The FFN then consumes NVFP4 activations (ig4_nvfp4_quantize of the
   * bf16 h2 and u).  Needs I % 256 == 0 and B*L > 128. */
  IG4_NVFP4_MIXED = 3
} ig4_dtype;

/* Shape and precision of one block call.  L = T_text + grid_t*grid_h*grid_w.
 * Supported: head_dim == 256, D == H*256, D % 256 == 0, I % 128 == 0,
 * adaln_dim % 8 == 0 and <= 1024, B*L >= 1, x_dtype F32 or BF16,
 * w_dtype BF16, E4M3 or NVFP4_MIXED (then also I % 256 == 0, B*L > 128). */
typedef struct ig4_config {
  int B, T_text, grid_t, grid_h, grid_w;
  int D, H, head_dim, I, adaln_dim;
  double rope_theta;   /* 5e6 */
  int sections[3];     /* (24, 20, 20): must sum to 64 */
  float eps;           /* RMSNorm epsilon, 1e-6 */
  int x_dtype;         /* residual stream storage: IG4_F32 or IG4_BF16 */
  int w_dtype;         /* linear weights: IG4_BF16, IG4_E4M3 with s_* scales, or
                          IG4_NVFP4_MIXED */
} ig4_config;

/* One block's weights (device pointers).  w_* are [out, in] row-major in
 * w_dtype: w_ada [6D, adaln_dim], w_qkv [3D, D] (rows: q | k | v, head-major,
 * column n = head*256 + d), w_o [D, D], w_gate [I, D], w_up [I, D],
 * w_down [D, I].  s_* are fp32 per-output-channel scales [out] (E4M3 and
 * NVFP4_MIXED, else ignored).  b_ada fp32 [6D], g_q / g_k fp32 [head_dim].
 * sf_gate / sf_up / sf_down: packed NVFP4 block scales of the FFN weights
 * (ig4_nvfp4_pack_scales), IG4_NVFP4_MIXED only, else ignored (zero them). */
typedef struct ig4_block_weights {
  const void *w_ada, *w_qkv, *w_o, *w_gate, *w_up, *w_down;
  const float *s_ada, *s_qkv, *s_o, *s_gate, *s_up, *s_down;
  const float *b_ada, *g_q, *g_k;
  const void *sf_gate, *sf_up, *sf_down;
} ig4_block_weights;

/* Stack weights: a host array of n_blocks block weight structs, the latent
 * in-projection w_in [D, C] + b_in [D], the final AdaLN w_f [2D, adaln_dim] +
 * b_f [2D] (chunks shift, scale), the out-projection w_out [C, D] + b_out [C].
 * Weights in cfg->w_dtype, s_* scales for E4M3 (for IG4_NVFP4_MIXED these three
 * linears are E4M3 and only the blocks' FFNs NVFP4).  C = latent_ch (128). */
typedef struct ig4_stack_weights {
  int n_blocks;
  int latent_ch;
  const ig4_block_weights *blocks;   /* HOST array of n_blocks entries */
  const void *w_in;  const float *s_in;  const float *b_in;
  const void *w_f;   const float *s_f;   const float *b_f;
  const void *w_out; const float *s_out; const float *b_out;
} ig4_stack_weights;

/* Human-readable name of a status code (static string, never NULL). */
const char *ig4_status_string(int status);

/* ABI revision of this header (increases on any incompatible change). */
int ig4_abi_version(void);

/* ------------------------------------------------------------ positions ---
 * MRoPE position table (survey page, "单 block 内部": text tokens use a 1D
 * position broadcast to the 3 axes, image tokens use (t, h, w); "条件注入方式":
 * text precedes the image).  Writes int32 pos[3][L] (rows t, h, w), with
 * text token l at (l, l, l) and image token (t, i, j), row-major over the
 * grid, at (T+t, T+i, T+j).  out_on_device = 0: pos_out is host memory and the
 * table is written by host code before the call returns (stream unused);
 * 1: pos_out is device memory, written by a kernel launched on `stream`.
 * Errors: INVALID_ARG for negative sizes, L == 0, L > 2^24, or NULL pos_out. */
ig4_status ig4_mrope_positions(int T_text, int grid_t, int grid_h, int grid_w,
                               int32_t *pos_out, int out_on_device, void *stream);

/* --------------------------------------------------------- rotary table ---
 * Rotary tables for a position table: cos_out[l][j] = cos(pos[axis(j)][l] *
 * theta^(-2j/128)), sin_out likewise, fp32 [L][64], angles evaluated in fp64.
 * axis(j) follows `sections` (contiguous chunks t, h, w).  pos: device int32
 * [3][L]; outputs device.  Errors: INVALID_ARG (NULL, L < 1, sections not
 * summing to 64, theta <= 0). */
ig4_status ig4_rope_table(int L, const int32_t *pos, double rope_theta, const int sections[3],
                          float *cos_out, float *sin_out, void *stream);

/* ----------------------------------------------------- AdaLN modulation ---
 * AdaLN modulation (survey page, "单 block 内部": AdaLN from the timestep
 * embedding gives the per-block modulation): mod[b][n] = sum_k SiLU(temb[b][k])
 * * W[n][k] (* w_scale[n] for E4M3) + bias[n], fp32 out [B][N].  temb fp32
 * [B][A]; W [N][A] in w_dtype (BF16 or E4M3); bias fp32 [N] or NULL.
 * Errors: INVALID_ARG (NULL, B < 1, B > 8, A % 8, A > 1024, N < 1). */
ig4_status ig4_adaln_modulation(int B, int A, int N, const float *temb, const void *w,
                                int w_dtype, const float *w_scale, const float *bias,
                                float *mod_out, void *stream);

/* ------------------------------------------------------ norm + modulate ---
 * Pre-norm + modulate: h[r] = x[r] * rsqrt(mean(x[r]^2) + eps) * (1 + scale[b])
 * + shift[b] for each token row r of sample b = r / L.  x [B*L][D] in x_dtype
 * (F32 or BF16); shift / scale fp32 with sample stride mod_stride (pointers into
 * an AdaLN output, e.g. mod + 0*D and mod + 1*D with stride 6D).  Output h in
 * h_dtype: BF16, or E4M3 with a per-row fp32 scale written to h_scale_out
 * (h = code * scale, scale = max|h| / 448).  D % 8 == 0, D <= 8192. */
ig4_status ig4_norm_modulate(int B, int L, int D, const void *x, int x_dtype,
                             const float *shift, const float *scale, int mod_stride, float eps,
                             void *h_out, int h_dtype, float *h_scale_out, void *stream);

/* ------------------------------------------------ QKV + QK-norm + MRoPE ---
 * Fused QKV projection with per-head QK-RMSNorm and MRoPE (survey page,
 * "单 block 内部": self-attention with QK-RMSNorm and 3D MRoPE).
 * qkv = h W_qkv^T; q and k are RMS-normalised per (token, head) with g_q / g_k
 * and rotated with the tables of ig4_rope_table; v passes through.
 * h [B*L][D] in h_dtype (BF16; or E4M3 with per-row scale h_scale when
 * w_dtype is E4M3).  Outputs (bf16, device): q_out, k_out [B][H][L][256],
 * vt_out [B][H][256][vt_ld] (v transposed, keys contiguous), vt_ld >= L and
 * vt_ld % 8 == 0.  Errors: UNSUPPORTED unless head_dim == 256 and D == 256*H. */
ig4_status ig4_qkv_project(int B, int L, int D, int H, const void *h, int h_dtype,
                           const float *h_scale, const void *w_qkv, int w_dtype,
                           const float *w_scale, const float *g_q, const float *g_k, float eps,
                           const float *rope_cos, const float *rope_sin, void *q_out,
                           void *k_out, void *vt_out, int vt_ld, void *stream);

/* ------------------------------------------------------ joint attention ---
 * Joint bidirectional attention over [text | image] (survey page: one
 * self-attention over the single sequence, no separate branches):
 * o[b, l, h*256 + d] = sum_m softmax_m(q[b,h,l] . k[b,h,m] / 16) v[b,h,m,d].
 * q, k bf16 [B][H][L][256]; vt bf16 [B][H][256][vt_ld]; o_out bf16 [B*L][H*256];
 * all device, 16-byte aligned (an o_out 32-byte aligned is written with
 * 32-byte stores, one otherwise 16-byte aligned with 16-byte stores: the same
 * values).  Errors: INVALID_ARG (NULL, misaligned, L < 1, vt_ld < L or
 * vt_ld % 8). */
ig4_status ig4_joint_attention(int B, int H, int L, const void *q, const void *k,
                               const void *vt, int vt_ld, void *o_out, void *stream);

/* ig4_joint_attention with a workspace (256-byte aligned, at least
 * ig4_joint_attention_workspace_size(B, H, L) bytes; 0 when no workspace is
 * needed).  With it, a persistent grid of one CTA per SM takes equal shares
 * of all (query tile, key tile) pairs, whatever the number of (b, h, query
 * tile) items, and the items split between CTAs are merged by a second
 * kernel (pieces in a fixed order, so the result is deterministic); the
 * block entry points work this way.  Without it (workspace NULL) every item
 * is one CTA. */
size_t ig4_joint_attention_workspace_size(int B, int H, int L);
ig4_status ig4_joint_attention_ws(int B, int H, int L, const void *q, const void *k,
                                  const void *vt, int vt_ld, void *o_out, void *workspace,
                                  size_t ws_bytes, void *stream);

/* ------------------------------------------------ gated residual linear ---
 * Gated residual linear (survey page, "单 block 内部": AdaLN gates modulate
 * the attention and MLP residual paths): x_out[r][n] = x_res[r][n] +
 * gate[b*gate_stride + n] * sum_k a[r][k] W[n][k] (scaled by a_scale[r] *
 * w_scale[n] in E4M3), b = r / L.  a [B*L][K] in a_dtype (BF16, or E4M3 +
 * a_scale when w_dtype is E4M3); x_res / x_out [B*L][N] in x_dtype and may be
 * the same buffer.  N % 128 == 0, K % 64 == 0 (bf16) / % 128 == 0 (E4M3). */
ig4_status ig4_gated_residual_linear(int B, int L, int N, int K, const void *a, int a_dtype,
                                     const float *a_scale, const void *w, int w_dtype,
                                     const float *w_scale, const float *gate, int gate_stride,
                                     const void *x_res, void *x_out, int x_dtype, void *stream);

/* --------------------------------------------------------------- SwiGLU ---
 * SwiGLU hidden state (survey page, "单 block 内部": SwiGLU MLP with a SiLU
 * gate): u[r][i] = silu(sum_k h[r][k] Wg[i][k]) * sum_k h[r][k] Wu[i][k]
 * (E4M3: each sum times h_scale[r] * s_gate[i] or s_up[i]).  h [M][K];
 * w_gate, w_up [I][K]; u_out bf16 [M][I].  I % 128 == 0, K % 64 == 0 (bf16) /
 * % 128 == 0 (E4M3). */
ig4_status ig4_swiglu(int M, int I, int K, const void *h, int h_dtype, const float *h_scale,
                      const void *w_gate, const void *w_up, int w_dtype, const float *s_gate,
                      const float *s_up, void *u_out, void *stream);

/* ------------------------------------------------------ FP8 activations ---
 * Row quantisation of an activation to FP8 E4M3 for the FP8-weight path:
 * scale[r] = max_k |x[r][k]| / 448 (1 if the row is zero), q[r][k] =
 * RNE(x[r][k] / scale[r]) saturated to +-448.  x bf16 [M][K]; q_out E4M3
 * [M][K]; scale_out fp32 [M].  K % 8 == 0, K <= 16384. */
ig4_status ig4_quantize_rows(int M, int K, const void *x, void *q_out, float *scale_out,
                             void *stream);

/* Block quantisation of an activation to MX8, the form the FP8 block feeds
 * its out- and down-projections (block-scaled E4M3, tcgen05 kind::mxf8f6f4;
 * the release weights' FP8 E4M3 format is from "Ideogram 4 快速开始",
 * hardware and precision section; the 32-element blocks are this library's
 * choice): for every 32 consecutive elements of a row with amax = max |x|,
 * e = ceil(log2(float(amax / 448))) (at least -126; 0 for a zero block),
 * codes = RNE_E4M3(x * 2^-e) saturated to +-448, scale byte = e + 127.
 * x bf16 [M][K]; codes_out E4M3 [M][K]; sf_out receives the scale bytes in
 * the tensor cores' order: the 4 scales of row r and 128-element k-block kb
 * at byte 512 ((r / 128) (K / 128) + kb) + 16 (r % 32) + 4 ((r % 128) / 32),
 * ig4_mx8_scale_bytes(M, K) bytes (rows padded to a multiple of 128; the
 * padding is not written).  K % 128 == 0, K <= 65536; x and codes_out
 * 16-byte aligned.  Errors: IG4_ERR_INVALID_ARG. */
ig4_status ig4_quantize_mx8(int M, int K, const void *x, void *codes_out, void *sf_out,
                            void *stream);
size_t ig4_mx8_scale_bytes(int M, int K);

/* --------------------------------------------------------- whole block ---
 * Bytes of workspace ig4_block_forward needs for cfg (0 if cfg is invalid). */
size_t ig4_workspace_size(const ig4_config *cfg);

/* One Ideogram4TransformerBlock forward: x_out = block(x_in).  x_in, x_out
 * [B][L][D] in cfg->x_dtype (device, must not overlap); pos device int32
 * [3][L] (see ig4_mrope_positions); temb device fp32 [B][adaln_dim];
 * workspace device, 256-byte aligned, >= ig4_workspace_size(cfg).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE (checked before any launch). */
ig4_status ig4_block_forward(const ig4_config *cfg, const ig4_block_weights *w,
                             const void *x_in, void *x_out, const int32_t *pos,
                             const float *temb, void *workspace, size_t ws_bytes, void *stream);

/* ig4_block_forward that also records the caller's CUDA events (cudaEvent_t
 * handles passed as void*) on `stream` around each kernel: events[0] before
 * the first launch and events[i+1] after launch i.  n_events must be 0 (no
 * tracing) or IG4_BLOCK_TRACE_EVENTS.  Launch order: 0 AdaLN, 1 rotary table,
 * 2 norm1, 3 QKV+norm+rope, 4 attention, 5 out-proj+residual, 6 norm2,
 * 7 gate/up+SwiGLU, 8 down+residual; the E4M3 path adds 9 quantise(o) and
 * 10 quantise(u), recorded in launch order (quantise(o) before out-proj).
 * An entry may be NULL: that boundary is not recorded (e.g. only the two
 * events around one kernel, so the other kernels keep overlapping their
 * launches with the kernel before them). */
#define IG4_BLOCK_TRACE_EVENTS 12
ig4_status ig4_block_forward_traced(const ig4_config *cfg, const ig4_block_weights *w,
                                    const void *x_in, void *x_out, const int32_t *pos,
                                    const float *temb, void *workspace, size_t ws_bytes,
                                    void *stream, void *const *events, int n_events);

/* ------------------------------------------- block without a workspace ---
 * ig4_block_forward for callers that cannot allocate device memory.  This
 * entry point has no counterpart on the pages: it exists for callers such as
 * inference runtimes that plan all device memory ahead and forbid allocation
 * while they execute, real-time loops that cannot afford cudaMalloc's
 * latency and implicit synchronisation, and hosts whose own caching allocator
 * owns the GPU's memory.  Instead of a caller workspace it uses a scratch
 * array of IG4_NOALLOC_SCRATCH_BYTES (64 MiB) that the library reserves as a
 * static device variable: every GPU that loads the library holds those bytes
 * until the process exits.  It allocates nothing and calls no allocating
 * routine.  The caller still passes inputs and outputs as for
 * ig4_block_forward (same layouts and errors).  A configuration fits when
 * ig4_workspace_size(cfg) <= IG4_NOALLOC_SCRATCH_BYTES; larger ones return
 * IG4_ERR_WORKSPACE before anything is launched.  At B = 1 that is up to 941
 * tokens of the full-width block (D 4608, I 12288) with bf16 weights, 796
 * with E4M3 weights and 750 with NVFP4 Mixed weights; 4094, 3469 and 3270
 * tokens at D 1024, I 2816.
 * The first call on a device looks up the scratch array's device address
 * (a set-up done with that device current, and done again if the device's
 * context has changed since, e.g. after a device reset); make that first call
 * before any stream capture.  All calls share the one array and it keeps the
 * previous call's contents; no part of it needs to start at zero, because
 * every byte a call reads there was written earlier in the same call.  Calls
 * whose work overlaps on the GPU (different streams, or different host
 * threads without ordering) race on the array: order them. */
#define IG4_NOALLOC_SCRATCH_BYTES (64ull << 20)
ig4_status ig4_block_forward_noalloc(const ig4_config *cfg, const ig4_block_weights *w,
                                     const void *x_in, void *x_out, const int32_t *pos,
                                     const float *temb, void *stream);

/* ---------------------------------------------------------------- stack ---
 * Bytes of workspace ig4_stack_forward needs (0 if invalid). */
size_t ig4_stack_workspace_size(const ig4_config *cfg, int latent_ch);

/* One denoiser step of the stack (survey page: 34 single-stream layers over
 * [text | image]; 128-channel latent tokens, a 1024 px image = 64 x 64 grid):
 * s = [text | x_latent W_in^T + b_in]; s = block_i(s) for each block;
 * out_latent = (RMSNorm(s) (1 + scale_f) + shift_f)[:, T:] W_out^T + b_out,
 * (shift_f, scale_f) = SiLU(temb) W_f^T + b_f.  x_latent [B][N][C], text
 * [B][T][D], out_latent [B][N][C], all in cfg->x_dtype (device); N = grid_t *
 * grid_h * grid_w; pos and temb as for ig4_block_forward. */
ig4_status ig4_stack_forward(const ig4_config *cfg, const ig4_stack_weights *sw,
                             const void *x_latent, const void *text, void *out_latent,
                             const int32_t *pos, const float *temb, void *workspace,
                             size_t ws_bytes, void *stream);

/* ig4_stack_forward that also copies the sequence [B][L][D] (bf16, the
 * stack's residual stream [text | image]) entering block tap_blocks[i] into
 * the caller's device buffer tap_out[i] (16-byte aligned, 2*B*L*D bytes),
 * for i < n_taps; tap_blocks[i] == n_blocks takes the sequence after the
 * last block (the final norm's input).  The copies are stream-ordered device
 * copies between the launches and change nothing else.  For inspecting a
 * deep stack block by block.  Errors: INVALID_ARG for a block index outside
 * [0, n_blocks], a NULL or misaligned tap buffer, n_taps < 0; otherwise as
 * for ig4_stack_forward. */
ig4_status ig4_stack_forward_tapped(const ig4_config *cfg, const ig4_stack_weights *sw,
                                    const void *x_latent, const void *text, void *out_latent,
                                    const int32_t *pos, const float *temb, void *workspace,
                                    size_t ws_bytes, void *stream, const int *tap_blocks,
                                    void *const *tap_out, int n_taps);

/* -------------------------------------------------------------- NVFP4 ---
 * Block-scaled 4-bit linear layers ("不用再充会员！Ideogram 4.0 NF4 免费本地部署"
 * deployment article, section "2.2 NVFP4 Mixed": FFN linears stored as
 * 4-bit floats sharing an E4M3 scale per block; "SGLang cookbook: Ideogram
 * 4": NVFP4 runs on B200 / Blackwell).  Operands are E2M1 codes (sign, 2
 * exponent bits with bias 1, 1 mantissa bit), two per byte with element 2i
 * in the low nibble, rows K-contiguous; each row has one UE4M3 scale per 16
 * K-elements (a 64-element block format repeats its scale over the four
 * 16-element sub-blocks) and one fp32 scale:
 *   out[m][n] = a_scale[m] * w_scale[n] * sum_k A(m,k) W(n,k) (+ bias[n]),
 *   A(m,k) = e4m3(a_sf[m][k/16]) * e2m1(a_code[m][k]), W likewise.
 *
 * ig4_nvfp4_scale_bytes: bytes of a packed scale array for `rows` rows of K
 * elements (rows rounded up to 128; 0 if K is not a multiple of 64).
 * ig4_nvfp4_pack_scales: row-major UE4M3 scales [rows][K/16] (device) ->
 * the packed order the tensor cores read (per 128 rows and 64 K-elements a
 * 512-byte block; byte 16 (r % 32) + 4 ((r % 128) / 32) + (k / 16) % 4);
 * padding rows get zero scales.
 * ig4_nvfp4_linear: M >= 1, N a multiple of 128, K a multiple of 256;
 * a_codes [M][K/2], w_codes [N][K/2] bytes; a_sf, w_sf packed scales;
 * a_scale [M], w_scale [N], bias [N] (or NULL) fp32; out [M][N] fp32 or bf16
 * (out_dtype).  All device pointers 16-byte aligned; stream-ordered.
 * Errors: IG4_ERR_INVALID_ARG.
 * ig4_nvfp4_quantize: activations x bf16 [M][K] (device, K a multiple of
 * 64) -> codes [M][K/2], packed scales (ig4_nvfp4_scale_bytes(M, K) bytes;
 * padding rows are not written) and row_scale fp32 [M], by the recipe
 *   row_scale[m] = max_k |x[m][k]| / (6 * 448)  (1 for an all-zero row),
 *   sf[m][b]     = RNE_E4M3(max over block b |x[m][.]| / (6 row_scale[m])),
 *   code[m][k]   = RNE_E2M1(x[m][k] * (1 / (row_scale[m] sf[m][k/16]))),
 * each step a float32 operation, E2M1 saturating at 6 (a block whose scale
 * rounds to 0 gets zero codes).  Errors: IG4_ERR_INVALID_ARG. */
size_t ig4_nvfp4_scale_bytes(int rows, int K);
ig4_status ig4_nvfp4_pack_scales(int rows, int K, const void *sf_rows, void *sf_packed,
                                 void *stream);
ig4_status ig4_nvfp4_linear(int M, int N, int K, const void *a_codes, const void *a_sf,
                            const float *a_scale, const void *w_codes, const void *w_sf,
                            const float *w_scale, const float *bias, void *out, int out_dtype,
                            void *stream);
ig4_status ig4_nvfp4_quantize(int M, int K, const void *x, void *codes, void *sf_packed,
                              float *row_scale, void *stream);

/* -------------------------------------------------- text conditioning ---
 * The step before the stack ("Ideogram 4 快速开始" (SimpleTuner quickstart),
 * section "Text embed cache"): the text encoder output concatenates the
 * hidden states of 13 layers, 13 * 4096 = 53248 fp32 features per token, and
 * the transformer's frozen llm_cond_norm and llm_cond_proj layers project
 * them to the conditioning the stack reads as its text prefix (4608 values
 * per token, bf16).  Readings: llm_cond_norm is one RMSNorm with a learned
 * weight over the whole concatenated feature; llm_cond_proj a linear layer
 * with bias:  text_out = (raw * rsqrt(mean(raw^2) + eps) * g_norm) W^T + b.
 *
 * raw fp32 [M][K_raw] (M = tokens of all samples), g_norm fp32 [K_raw],
 * w_proj [D][K_raw] (bf16, or E4M3 codes with the per-output-channel fp32
 * w_scale [D]; with E4M3 the normed features are quantised to E4M3 with a
 * per-token scale, as in the block's FP8 path), b_proj fp32 [D], text_out
 * bf16 [M][D]; all device, 16-byte aligned.  K_raw and D multiples of 128.
 * Workspace (256-byte aligned) of ig4_text_cond_workspace_size bytes holds
 * the normed features.  Errors: IG4_ERR_INVALID_ARG, IG4_ERR_WORKSPACE. */
size_t ig4_text_cond_workspace_size(int M, int K_raw, int w_dtype);
ig4_status ig4_text_cond_project(int M, int K_raw, int D, const float *raw, const float *g_norm,
                                 float eps, const void *w_proj, const float *w_scale, int w_dtype,
                                 const float *b_proj, void *text_out, void *workspace,
                                 size_t ws_bytes, void *stream);

/* ------------------------------------------------------------ sampler ---
 * One step of the sampler around the stack ("Ideogram 4.0" survey page,
 * section 训练方法: the DiT predicts a flow-matching velocity and inference
 * takes explicit Euler steps z_{t-dt} = z_t + v dt; the noise schedule is
 * logit-normal in (mu, std) with mu shifted by resolution,
 * mu_adjusted = mu_base + 0.5 log(num_pixels / 512^2); classifier-free
 * guidance is asymmetric: the unconditional pass drops the text tokens and
 * runs on the image tokens only, with a guidance weight that drops for the
 * last "polish" steps; section Infra: the presets V4_QUALITY_48 (45 steps at
 * gw 7 + 3 at gw 3, mu 0, std 1.5), V4_DEFAULT_20 (18 + 2, mu 0, std 1.75),
 * V4_TURBO_12 (11 + 1, mu 0.5, std 1.75); "Ideogram 4 快速开始", section
 * 验证: the unconditional branch is a separate, image-only transformer).
 *
 * Readings: t runs from 1 (noise) to 0 (clean latent); step i goes from
 * t_i to t_{i+1} with dt = t_i - t_{i+1} > 0; the log is natural; the
 * timestep embedding of each branch is an input (the pages do not describe
 * the timestep embedder).
 *
 * Host: the N + 1 times t_out[i] = sigmoid(mu_adjusted + std *
 * Phi^-1(1 - i/N)) (the (1 - i/N) quantiles of the logit-normal
 * distribution), t_out[0] = 1 and t_out[N] = 0 exactly.  num_steps 1 ..
 * 100000, std_dev > 0, finite mu_base, positive sizes; else
 * IG4_ERR_INVALID_ARG.  Caller-owned host array of num_steps + 1 doubles. */
ig4_status ig4_flow_schedule(int num_steps, double mu_base, double std_dev, int height_px,
                             int width_px, double *t_out);

/* Host: guidance weight of each step: gw_main for the first
 * num_steps - n_polish steps, gw_polish for the last n_polish (0 <= n_polish
 * <= num_steps).  Caller-owned host array of num_steps floats. */
ig4_status ig4_guidance_schedule(int num_steps, int n_polish, float gw_main, float gw_polish,
                                 float *gw_out);

/* Device: guided Euler update of n elements (n a multiple of 8):
 * z_out = z_in + dt * (v_uncond + gw * (v_cond - v_uncond)), velocities bf16,
 * latents fp32; z_out may alias z_in.  If z16_out is not NULL it also
 * receives z_out rounded to bf16 (the stack's input type).  With v_cond =
 * v_uncond = NULL it only writes z16_out = bf16(z_in) (dt, gw ignored; z_out
 * may be NULL).  All pointers 16-byte aligned; stream-ordered. */
ig4_status ig4_cfg_euler(long long n, const void *v_cond, const void *v_uncond, float gw,
                         float dt, const float *z_in, float *z_out, void *z16_out, void *stream);

/* Bytes of workspace ig4_denoise_step needs (0 if invalid): both branches'
 * velocities, the bf16 latent and one stack workspace (the two stacks run
 * one after the other on the stream). */
size_t ig4_denoise_workspace_size(const ig4_config *cfg, int latent_ch);

/* One sampler step with asymmetric CFG: v_c = stack_cond([text | z]) with
 * cfg (T_text text tokens, positions pos_cond [3][T + N]); v_u =
 * stack_uncond(z) over the image tokens alone (T_text = 0, positions
 * pos_uncond [3][N], no text); then z += (t_cur - t_next) * (v_u + gw *
 * (v_c - v_u)).  z: fp32 [B][N][C] on the device, updated in place; text as
 * for ig4_stack_forward; temb_cond, temb_uncond fp32 [B][adaln_dim];
 * cfg->x_dtype must be IG4_BF16 (the stacks run on the bf16-rounded
 * latent).  cond and uncond are two separate transformers with the same
 * width and latent_ch.  Errors as for ig4_stack_forward. */
ig4_status ig4_denoise_step(const ig4_config *cfg, const ig4_stack_weights *cond,
                            const ig4_stack_weights *uncond, float *z, const void *text,
                            const int32_t *pos_cond, const int32_t *pos_uncond,
                            const float *temb_cond, const float *temb_uncond, float t_cur,
                            float t_next, float gw, void *workspace, size_t ws_bytes,
                            void *stream);

/* ------------------------------------------------- multi-GPU layouts ---
 * Tensor parallelism over heads (TP) and Ulysses sequence parallelism over
 * the image tokens (SP) of the block ("SGLang cookbook: Ideogram 4",
 * section 3, tensor and sequence parallelism: TP shards the DiT weights and
 * its degree must divide the 18 heads; Ulysses SP keeps the weights whole on
 * every GPU and shards the image-token sequence; both validated on B200 at
 * 1024 x 1024 with 2 GPUs).  These calls compute one rank's share; the data
 * each rank must receive from the others between the calls is moved by the
 * caller (a collective, or peer-mapped pointers for ig4_tp_reduce).  At most
 * 8 ranks.  All calls are stream-ordered; argument errors are returned before
 * anything is launched.
 *
 * TP, tp_size P dividing H and with (I / P) % 128 == 0, weights BF16 or E4M3
 * (IG4_NVFP4_MIXED: UNSUPPORTED).  Rank r holds heads [r H/P, (r+1) H/P) and
 * FFN columns [r I/P, (r+1) I/P); its ig4_block_weights hold: w_ada, s_ada,
 * b_ada, g_q, g_k whole; w_qkv [3 D/P][D] = the q rows, then the k rows, then
 * the v rows of its heads (s_qkv likewise); w_o [D][D/P] = the columns of
 * W_o for its heads (s_o [D] whole); w_gate, w_up [I/P][D] = its rows
 * (s_gate, s_up [I/P]); w_down [D][I/P] = its columns (s_down [D] whole).
 * One block on rank r, with y = x_out:
 *   ig4_block_tp_attention -> partial_r = [r == 0] x + gate_msa * (o_r W_o,r^T)
 *   x1 = sum over ranks of partial_r         (all-reduce; ig4_tp_reduce)
 *   ig4_block_tp_mlp       -> partial_r = [r == 0] x1 + gate_mlp * (u_r W_down,r^T)
 *   y  = sum over ranks of partial_r         (all-reduce; ig4_tp_reduce)
 * partials are fp32 [B*L][D] (device, 16-byte aligned); the gates commute
 * with the sum, so the reduced partials are exactly the block's x1 and y up
 * to fp32 rounding.  ig4_block_tp_mlp reads the AdaLN output that
 * ig4_block_tp_attention left in the workspace: pass the same workspace,
 * unchanged in between.  The FP8 path quantises each rank's attention
 * output and SwiGLU output over its own columns.
 * ig4_tp_reduce: out[i] = sum_{k < n_src} src[k][i] (fp32, in index order,
 * so every rank computes the same bits), stored as out_dtype (IG4_F32 or
 * IG4_BF16); src is a HOST array of n_src device-accessible fp32 pointers
 * (this GPU's memory, or peer memory mapped into it), n % 8 == 0.
 *
 * SP, sp_size P dividing H, at least P image tokens.  Rank r holds the T text
 * tokens and the image tokens [off_r, off_r + N_r) of the row-major grid
 * (contiguous shares, the first N % P ranks one token more;
 * ig4_sp_image_range): its local sequence x_local is [B][T + N_r][D], text
 * first, with the positions of ig4_sp_positions.  One block on rank r:
 *   ig4_block_sp_pre       AdaLN, norm, QKV (+QK-norm, MRoPE) of the local
 *                          tokens; packs the phase-0 send buffer;
 *   all-to-all, phase 0    (rank s sends chunk (s -> d) to every d)
 *   ig4_block_sp_attention unpacks q, k, v of head group r
 *                          [r H/P, (r+1) H/P) over all L tokens (text rows
 *                          from its own QKV, image rows from every rank),
 *                          attention, packs the phase-1 send buffer;
 *   all-to-all, phase 1
 *   ig4_block_sp_post      unpacks o of the local tokens (all heads),
 *                          out-projection + gated residual, norm, SwiGLU,
 *                          down-projection + gated residual -> x_out_local.
 * The text tokens are computed on every rank, with the same result there.
 * Chunk (s -> d), bf16, ig4_sp_exchange_bytes(cfg, P, phase, s, d) bytes:
 *   phase 0: q [B][H/P][N_s][256], then k likewise, then v^T
 *            [B][H/P][256][N_s], of head group d over s's image tokens;
 *   phase 1: o [B][T + N_d][H/P * 256] of head group s over d's text and
 *            image tokens.
 * A send buffer holds the chunks to d = 0 .. P-1 in order, a receive buffer
 * the chunks from s = 0 .. P-1 in order (16-byte aligned).  The workspace
 * (ig4_sp_workspace_size) must be the same for the three calls of a block. */
size_t ig4_tp_workspace_size(const ig4_config *cfg, int tp_size);
ig4_status ig4_block_tp_attention(const ig4_config *cfg, int tp_rank, int tp_size,
                                  const ig4_block_weights *w, const void *x_in,
                                  const int32_t *pos, const float *temb, float *partial,
                                  void *workspace, size_t ws_bytes, void *stream);
ig4_status ig4_block_tp_mlp(const ig4_config *cfg, int tp_rank, int tp_size,
                            const ig4_block_weights *w, const void *x1, float *partial,
                            void *workspace, size_t ws_bytes, void *stream);
ig4_status ig4_tp_reduce(long long n, int n_src, const float *const *src, void *out,
                         int out_dtype, void *stream);
ig4_status ig4_sp_image_range(const ig4_config *cfg, int sp_size, int sp_rank, int *img_off,
                              int *img_count);
/* int32 [3][T + N_r] positions of rank r's local tokens (host memory written
 * before returning if out_on_device == 0, else device memory by a kernel). */
ig4_status ig4_sp_positions(const ig4_config *cfg, int sp_size, int sp_rank, int32_t *pos_out,
                            int out_on_device, void *stream);
size_t ig4_sp_workspace_size(const ig4_config *cfg, int sp_size, int sp_rank);
size_t ig4_sp_exchange_bytes(const ig4_config *cfg, int sp_size, int phase, int src_rank,
                             int dst_rank);
ig4_status ig4_block_sp_pre(const ig4_config *cfg, int sp_rank, int sp_size,
                            const ig4_block_weights *w, const void *x_local,
                            const int32_t *pos_local, const float *temb, void *send,
                            void *workspace, size_t ws_bytes, void *stream);
ig4_status ig4_block_sp_attention(const ig4_config *cfg, int sp_rank, int sp_size,
                                  const void *recv, void *send_o, void *workspace,
                                  size_t ws_bytes, void *stream);
ig4_status ig4_block_sp_post(const ig4_config *cfg, int sp_rank, int sp_size,
                             const ig4_block_weights *w, const void *x_local, void *x_out_local,
                             const void *recv_o, void *workspace, size_t ws_bytes,
                             void *stream);

/* ------------------------------------------------------------ failure ---
 * Synchronises `stream`, then reads and clears the device error word that the
 * kernels set when a bounded wait times out: IG4_ERR_TIMEOUT if set,
 * IG4_ERR_CUDA if the synchronisation itself failed, else IG4_OK. */
ig4_status ig4_last_device_error(void *stream);

/* Failure-detection self test: launches a one-CTA kernel that waits on an
 * mbarrier nothing will ever complete, with a wait limit of wait_us
 * microseconds (1 .. 5,000,000).  The kernel gives up at the limit, sets the
 * device error word and returns, so a following ig4_last_device_error()
 * returns IG4_ERR_TIMEOUT and the context stays usable.  No paper
 * counterpart: it exercises the timeout path every other kernel relies on. */
ig4_status ig4_selftest_timeout(int wait_us, void *stream);

/* ---------------------------------------------------------- measurement ---
 * SM clock as a kernel sees it: launches a one-thread kernel on `stream`
 * that counts SM cycles over window_us microseconds (1 .. 100,000) of the
 * GPU's global timer, synchronises the stream and writes cycles / time in
 * MHz to *mhz (host).  Queued after other work it reads the clock at the
 * moment that work ends, e.g. a power-capped clock after sustained tensor
 * work.  IG4_ERR_INVALID_ARG for a window out of range or a null mhz;
 * IG4_ERR_CUDA if the launch or the synchronisation fails.  No paper
 * counterpart: an instrument for reading timings. */
ig4_status ig4_sm_clock_mhz(int window_us, void *stream, double *mhz);

#ifdef __cplusplus
}
#endif

#endif /* IG4_H */

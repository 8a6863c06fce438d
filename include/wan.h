/*
 * wan.h -- C ABI of libwan: the Wan2.1 / Wan2.2 video DiT block forward and
 * the CFG-combined flow-matching Euler step on one NVIDIA B200 (sm_100a).
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - All tensor pointers are DEVICE pointers unless stated; the caller owns
 *    every buffer. The library never allocates or frees device memory: the
 *    block forward takes a caller-supplied workspace.
 *  - Work is enqueued on the caller's stream (`wan_stream_t` is the same
 *    type as `cudaStream_t`; NULL is the legacy default stream) and returns
 *    without synchronising. Results are valid once the stream reaches them.
 *  - Row-major, densely packed layouts. A "row" of an activation tensor is
 *    one token. Matrices of `nn.Linear`-style projections are stored
 *    [out_features, in_features] and applied as y = a W^T + b.
 *  - Return value: WAN_OK (0) or a negative WAN_E* code; a human-readable
 *    message for the calling thread is available from wan_last_error().
 *    Argument errors are detected on the host before anything is launched.
 *  - Every pointer must be 16-byte aligned (WAN_EALIGN otherwise).
 *
 * Sources (the pages that define the computation):
 *  [WALK]   "Wan2.2 code walkthrough" (newtid.com/chuangyezixun/14194.html):
 *           WanAttentionBlock core-logic snippet, 3D RoPE snippet,
 *           self-attention snippet, sampling-loop (CFG) snippet.
 *  [DIGEST] "Wan paper deep dive" (charles2530.github.io), section
 *           "Video DiT and Flow Matching": shared AdaLN MLP with per-block
 *           bias, flow-matching interpolation and velocity; its
 *           inference-optimisation table ("FP8 GEMM": per-tensor weight,
 *           per-token activation quantization).
 */
#ifndef WAN_H_
#define WAN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *wan_stream_t;

/* status codes */
#define WAN_OK            0
#define WAN_EINVAL       -1   /* bad argument: sizes, NULL pointer, inconsistent dims   */
#define WAN_EALIGN       -2   /* a pointer is not 16-byte aligned                       */
#define WAN_EUNSUPPORTED -3   /* dtype / head_dim combination not implemented           */
#define WAN_ECUDA        -4   /* a CUDA runtime or driver call failed                   */
#define WAN_ETIMEOUT     -5   /* a kernel's bounded wait gave up (see wan_device_status) */
#define WAN_EBOUNDS      -6   /* debug builds: a kernel's store fell outside its buffer */

/* element types */
#define WAN_F32  0
#define WAN_BF16 1
#define WAN_FP8  2   /* block mode: FP8 GEMMs, bf16 everything else (see wan_dims) */
#define WAN_FP8_ATTN 3  /* block mode: WAN_FP8 plus the 8-bit self-attention      */

/* Problem statement of one block call ([WALK]: grid sizes after the (1,2,2)
 * patch embedding, dim, heads, ffn_dim, text length, eps). */
typedef struct {
  int F, H, W;      /* token grid; L = F*H*W tokens per sequence, token i at
                       t = i/(H*W), h = (i/W)%H, w = i%W                      */
  int dim;          /* D, model width                                         */
  int heads;        /* n; head_dim d = dim/heads                              */
  int ffn_dim;      /* FFN hidden width                                       */
  int text_len;     /* T, text tokens per sequence (context rows)             */
  float eps;        /* LayerNorm / RMSNorm epsilon (1e-6 in Wan)              */
  int dtype;        /* WAN_F32: every matrix, bias, context and intermediate
                       in float32 with exact fp32 FMA arithmetic.
                       WAN_BF16: matrices, biases, context and intermediates
                       in bfloat16, tensor-core products accumulated in fp32;
                       norms, softmax, residual stream in fp32.
                       WAN_FP8 ([DIGEST] "FP8 GEMM"): as WAN_BF16, except
                       that the ten projection matrices are e4m3 codes with
                       one scale each (wan_block_weights.w_scales) and every
                       projection's input is quantized to e4m3 per token
                       inside the block; the products run on the FP8 tensor
                       cores and are accumulated in fp32.
                       WAN_FP8_ATTN: WAN_FP8 with the self-attention run as
                       wan_attention_8bit ([DIGEST] "8-bit FlashAttention");
                       the cross-attention stays bf16.                       */
  int e0_per_token; /* 0: e0 is [B, 6, dim] (one timestep per sequence);
                       1: e0 is [B, L, 6, dim], one timestep per token
                       ([WALK] time-projection snippet: the embedding is
                       unflattened to (batch, seq_len); TI2V)                */
} wan_dims;

/* Parameters of one WanAttentionBlock ([WALK] block snippet). Pointers marked
 * (dt) are in wan_dims.dtype, the others float32. All [dim] unless noted. */
typedef struct {
  const float *modulation;                 /* [6, dim] per-block bias added to e0      */
  const void *wq, *bq, *wk, *bk, *wv, *bv; /* (dt) self-attn q/k/v: [dim,dim], [dim]   */
  const void *wo, *bo;                     /* (dt) self-attn output projection         */
  const float *gq, *gk;                    /* self-attn q/k RMSNorm gains              */
  const float *g3, *b3;                    /* norm3 (affine LayerNorm) gain and bias   */
  const void *cwq, *cbq, *cwk, *cbk, *cwv, *cbv; /* (dt) cross-attn projections       */
  const void *cwo, *cbo;                   /* (dt) cross-attn output projection        */
  const float *cgq, *cgk;                  /* cross-attn q/k RMSNorm gains             */
  const void *w1, *b1;                     /* (dt) FFN in:  [ffn_dim, dim], [ffn_dim]  */
  const void *w2, *b2;                     /* (dt) FFN out: [dim, ffn_dim], [dim]      */
  const float *w_scales;                   /* WAN_FP8 only (NULL otherwise): [10] scales
                                              of wq, wk, wv, wo, cwq, cwk, cwv, cwo, w1,
                                              w2, whose codes (uint8 e4m3) replace the
                                              matrices above; biases stay bf16          */
} wan_block_weights;

/* Message describing the last error on the calling thread ("" if none). */
const char *wan_last_error(void);

/* wan_rope_freqs -- the precomputed 3D RoPE table ([WALK] 3D RoPE snippet:
 * a 1024-position table split into t / h / w sections).
 *   head_dim  d, even, 2..256. The d/2 complex pairs are split
 *             [c - 2(c/3), c/3, c/3] (c = d/2) between the t, h, w axes; an
 *             axis owning p pairs uses omega_j = theta^(-2j/(2p)), j < p.
 *   max_pos   rows of the table (1024 in Wan); grid sizes must not exceed it.
 *   theta     base (1e4 in Wan).
 *   table     out, device, float32 [max_pos][d/2][2] = (cos, sin) of
 *             pos * omega_j; angles are formed in fp64, stored rounded.
 * Errors: WAN_EINVAL for odd / out-of-range head_dim, max_pos < 1, NULL. */
int wan_rope_freqs(int head_dim, int max_pos, double theta, float *table,
                   wan_stream_t stream);

/* Bytes of workspace wan_block_forward needs for `B` sequences of `dims`
 * (0 on invalid dims). The workspace holds, at the offsets returned by
 * wan_block_workspace_offset, the intermediates of the last call. */
size_t wan_block_workspace_bytes(const wan_dims *dims, int B);

/* Workspace buffers (for inspection after a call; all row-major):          */
#define WAN_WS_ACT   0  /* (dt) [B*L, dim]   last normalised branch input (FFN's)  */
#define WAN_WS_QKV   1  /* (dt) [B*L, 3*dim] self q | k | v: k normalised and rotated; q rotated
                           (on the bf16 path q's RMS factor is applied inside the attention) */
#define WAN_WS_O     2  /* (dt) [B*L, dim]   self-attention output (before W_o)     */
#define WAN_WS_QC    3  /* (dt) [B*L, dim]   cross-attention q (normalised)         */
#define WAN_WS_KVC   4  /* (dt) [B*T, 2*dim] cross k | v (k normalised)             */
#define WAN_WS_OC    5  /* (dt) [B*L, dim]   cross-attention output (before W_o)    */
#define WAN_WS_H     6  /* (dt) [B*L, ffn]   FFN hidden after GELU                  */
#define WAN_WS_MOD   7  /* f32  [B, 6, dim]  modulation + e0                        */
#define WAN_WS_STATS 8  /* f32  [max(B*L, B*T), 4, dim/256] per-row partial sums of squares of
                           q, k, cross q, cross k (bf16 path) */
#define WAN_WS_A8     9  /* u8 [max(B*L*ffn, B*T*dim)] e4m3 codes of the last quantized GEMM input
                           (WAN_FP8 only; empty otherwise)                              */
#define WAN_WS_ASCALE 10 /* f32 [max(B*L, B*T)] their per-row scales (WAN_FP8 only)       */
#define WAN_WS_ATTN8  11 /* scratch of the 8-bit self-attention (WAN_FP8_ATTN only)         */
#define WAN_WS_COUNT 12
/* Byte offset of buffer `which` inside the workspace, or (size_t)-1. */
size_t wan_block_workspace_offset(const wan_dims *dims, int B, int which);

/* wan_block_forward -- one WanAttentionBlock on B sequences, in place on x
 * ([WALK] WanAttentionBlock core-logic snippet):
 *     m  = modulation + e0[b]                      (chunks m0..m5)
 *     x += m2 * SelfAttn(LN(x) * (1 + m1) + m0)
 *     x += CrossAttn(LN(x) * g3 + b3, ctx)         (ungated)
 *     x += m5 * FFN(LN(x) * (1 + m4) + m3)
 *   SelfAttn: q,k = RMSNorm_dim(a W^T + b) * gain, v = a W^T + b, q and k
 *   rotated by 3D RoPE, softmax(q k^T / sqrt(d)) v over all L tokens of the
 *   same sequence, output projection. CrossAttn: the same without RoPE,
 *   keys/values from ctx, first ctx_lens[b] text tokens valid. FFN: Linear,
 *   GELU(tanh), Linear. LayerNorm without affine uses eps inside the sqrt.
 *
 *   dims      problem statement; head_dim must be 128 for WAN_BF16 and
 *             WAN_FP8, and one of 32, 64, 128 for WAN_F32. dim % 64 == 0,
 *             ffn_dim % 64 == 0; WAN_BF16 and WAN_FP8 also need
 *             dim % 256 == 0 (WAN_FP8: ffn_dim % 128 == 0).
 *             The dtype picks the kernels: WAN_F32 runs every product on
 *             the exact-fp32 CUDA-core kernels, WAN_BF16 / WAN_FP8 on the
 *             tcgen05 tensor-core kernels; a shape outside a kernel's rules
 *             is refused with WAN_EUNSUPPORTED, never run on another kernel.
 *   B         sequences (2 for a CFG pair: same x, two contexts), >= 1.
 *   x         in/out float32 [B, L, dim], the residual stream.
 *   ctx       (dt) [B, T, dim] projected text tokens.
 *   ctx_lens  device int32 [B] valid text tokens (0..T), or NULL (all T).
 *   e0        float32 [B, 6, dim] time projection (shift, scale, gate,
 *             shift2, scale2, gate2), shared by all blocks of a step; with
 *             dims->e0_per_token, [B, L, 6, dim], one per token.
 *   w         block parameters (host struct of device pointers).
 *   rope      table from wan_rope_freqs(head_dim, max_pos >= max(F,H,W)).
 *   rope_max_pos  rows in that table.
 *   workspace device buffer of ws_bytes >= wan_block_workspace_bytes().
 * Errors: WAN_EINVAL (dims, NULLs, small workspace, grid beyond the table),
 * WAN_EUNSUPPORTED (head_dim/dtype), WAN_EALIGN, WAN_ECUDA. */
int wan_block_forward(const wan_dims *dims, int B, float *x, const void *ctx,
                      const int *ctx_lens, const float *e0,
                      const wan_block_weights *w, const float *rope,
                      int rope_max_pos, void *workspace, size_t ws_bytes,
                      wan_stream_t stream);

/* wan_block_forward_noalloc -- wan_block_forward without a caller-supplied
 * workspace, for callers that cannot allocate device memory: a plug-in that
 * only receives buffers from a host framework which owns the GPU's memory
 * pool, a serving process whose memory budget is fixed up front, or a
 * latency-critical loop where an allocation (which can synchronise the
 * device) is not allowed. The pages have no counterpart to this entry point;
 * it exists only for such callers.
 *   Same arguments and results as wan_block_forward, minus workspace and
 *   ws_bytes. The workspace is a built-in device array of
 *   WAN_NOALLOC_WORKSPACE_BYTES bytes that every GPU loading the library
 *   holds until the process exits; the entry point itself allocates nothing.
 *   Problems with wan_block_workspace_bytes(dims, B) above that size are
 *   rejected (WAN_EINVAL, message names both sizes).
 *   The array's device address is looked up on every call made while the
 *   stream is not capturing (a device reset moves the array); the first call
 *   with a given device current must come before any stream capture.
 *   B == 0 and invalid dims give the same status as wan_block_forward.
 *   All calls on a device share the array and it keeps the previous call's
 *   contents (the block writes every byte it reads, so no clearing is
 *   needed); calls that may overlap on the GPU race on it. */
#define WAN_NOALLOC_WORKSPACE_BYTES (16u << 20)
int wan_block_forward_noalloc(const wan_dims *dims, int B, float *x, const void *ctx,
                              const int *ctx_lens, const float *e0,
                              const wan_block_weights *w, const float *rope,
                              int rope_max_pos, wan_stream_t stream);

/* ---------------------------------------------------------------------------
 * Sequence-parallel (head-parallel, "Ulysses") phases of the block
 * ([DIGEST] training/inference-system section, 2D context parallelism:
 * Ulysses inside Ring; [WALK] CLI, --ulysses). N ranks each hold a token
 * shard of the sequence; around the self-attention an all-to-all gives every
 * rank all tokens of n/N heads and a second one returns the outputs:
 *   wan_block_sp_qkv     LN1 + modulate, QKV projection, q / k RMSNorm and
 *                        3D RoPE on the rank's rows -> q | k | v per row
 *   (caller) all-to-all  token shards -> head shards (wan_permute_chunks
 *                        packs and unpacks the exchanged buffers)
 *   wan_attention        all tokens, the rank's n/N heads
 *   (caller) all-to-all  head shards -> token shards
 *   wan_block_sp_finish  output projection + gated residual, cross-attention
 *                        branch, FFN branch on the rank's rows
 * With N = 1 (one shard = the whole sequence) the phases compute the block of
 * wan_block_forward; bf16 differs only in rounding q after its RMS factor
 * (wan_block_forward applies that factor inside the attention). WAN_F32 and
 * WAN_BF16 only.
 * ------------------------------------------------------------------------- */

/* Workspace bytes of wan_block_sp_qkv / wan_block_sp_finish for B sequences
 * of `rows` token rows each (0 on invalid arguments). */
size_t wan_block_sp_workspace_bytes(const wan_dims *dims, int B, int rows);

/* wan_block_sp_qkv -- the self-attention inputs of a token shard.
 *   dims      the whole problem (grid (F, H, W) gives the RoPE positions).
 *   rows      tokens of each sequence held here; row r is token tok0 + r of
 *             the grid (tok0 + rows <= F*H*W).
 *   x         float32 [B, rows, dim]; e0 as in wan_block_forward (per token:
 *             [B, rows, 6, dim], the shard's rows).
 *   qkv       out, (dt) [B, rows, 3*dim]: q | k | v of each row; q and k
 *             RMS-normalised with their gains and rotated by the 3D RoPE.
 *   workspace ws_bytes >= wan_block_sp_workspace_bytes(dims, B, rows).
 * Errors as wan_block_forward; WAN_EINVAL for a shard outside the grid,
 * WAN_EUNSUPPORTED for WAN_FP8 modes. */
int wan_block_sp_qkv(const wan_dims *dims, int B, int rows, int tok0, const float *x,
                     const float *e0, const wan_block_weights *w, const float *rope,
                     int rope_max_pos, void *qkv, void *workspace, size_t ws_bytes,
                     wan_stream_t stream);

/* wan_block_sp_finish -- the rest of the block on a token shard:
 *   x += m2 * (o W_o^T + b_o); x += CrossAttn(norm3 x, ctx); x += m5 * FFN(...)
 *   x         in/out float32 [B, rows, dim] (the shard's rows).
 *   ctx, ctx_lens, e0, w  as in wan_block_forward (e0 per token: the shard's rows).
 *   o         (dt) [B, rows, dim] self-attention output of the shard's rows,
 *             all heads (heads in order within a row).
 * Errors as wan_block_sp_qkv. */
int wan_block_sp_finish(const wan_dims *dims, int B, int rows, float *x, const void *ctx,
                        const int *ctx_lens, const float *e0, const wan_block_weights *w,
                        const void *o, void *workspace, size_t ws_bytes, wan_stream_t stream);

/* wan_permute_chunks -- dst = src with its axes permuted, in units of
 * chunk_bytes: src is row-major [dims[0]]...[dims[ndim-1]] chunks, dst is
 * row-major over axes perm[0], ..., perm[ndim-1] of src (dst axis k runs over
 * src axis perm[k]). Used to pack and unpack the all-to-all buffers of the
 * sequence-parallel attention, e.g. q|k|v rows [B][rows][3][N][n/N*d] ->
 * per-destination [N][B][rows][3][n/N*d] with perm (3, 0, 1, 2).
 *   ndim 1..5; chunk_bytes a positive multiple of 16; src and dst device
 *   buffers of prod(dims) * chunk_bytes bytes each, 16-byte aligned, not
 *   overlapping.
 * Errors: WAN_EINVAL (bad ndim / perm / chunk size, overlap, NULL),
 * WAN_EALIGN. */
int wan_permute_chunks(const void *src, void *dst, int ndim, const int *dims,
                       const int *perm, size_t chunk_bytes, wan_stream_t stream);

/* ---------------------------------------------------------------------------
 * Whole-model forward on latents ([WALK] WanModel structure and forward
 * snippets, time-projection snippet; [DIFFUSERS] "3D Patchify", "Unpatchify").
 *   x   = Conv3d(C_in, dim, kernel = stride = (1,2,2))(latent), flattened to
 *         tokens (t, h, w order)
 *   e   = Linear(SiLU(Linear(sinusoid(t))))  (freq_dim features: cos | sin of
 *         t * 10000^(-j/(freq_dim/2)))
 *   e0  = Linear(SiLU(e)) as [B, 6, dim]
 *   ctx = Linear(GELU_tanh(Linear(text)))   (text_dim -> dim -> dim)
 *   x   = blocks[0..n-1](x, ctx, e0)        (wan_block_forward)
 *   y   = Linear(LN(x) (1 + m1) + m0), m = head_modulation + e  (C_out * 4 outputs)
 *   out = y folded back to [C_out, F, H, W] (token features ordered
 *         (kt, kh, kw, c), channel fastest)
 * ------------------------------------------------------------------------- */
typedef struct {
  int C_in, C_out;      /* latent channels in / out (16 / 16 for T2V)           */
  int F, H, W;          /* latent grid before patching; H and W even; the token
                           grid is (F, H/2, W/2)                                 */
  int dim, heads, ffn_dim;
  int text_len;         /* T text tokens per sequence                            */
  int text_dim;         /* width of the text encoder features (4096 for umT5)   */
  int freq_dim;         /* sinusoidal time features (256)                        */
  float eps;
  int dtype;            /* WAN_F32 | WAN_BF16 | WAN_FP8, as in wan_dims; with
                           WAN_FP8 the blocks run their FP8 GEMMs and the
                           embeddings and head are bf16                           */
  int t_per_token;      /* 0: t is [B]; 1: t is [B, L] (L = F (H/2) (W/2)), one
                           timestep per token; the blocks then get e0 per token */
} wan_model_dims;

/* (dt) = wan_model_dims.dtype; others float32. */
typedef struct {
  const void *patch_w, *patch_b;      /* (dt) [dim, C_in*4] (Conv3d weight [dim, C_in, 1, 2, 2]), [dim] */
  const void *text_w1, *text_b1;      /* (dt) [dim, text_dim], [dim]           */
  const void *text_w2, *text_b2;      /* (dt) [dim, dim], [dim]                */
  const float *time_w1, *time_b1;     /* [dim, freq_dim], [dim]                */
  const float *time_w2, *time_b2;     /* [dim, dim], [dim]                     */
  const float *proj_w, *proj_b;       /* [6*dim, dim], [6*dim]                 */
  const float *head_mod;              /* [2, dim] (shift, scale) bias           */
  const void *head_w, *head_b;        /* (dt) [C_out*4, dim], [C_out*4]        */
} wan_model_weights;

/* Workspace bytes for wan_model_forward (0 on invalid dims). */
size_t wan_model_workspace_bytes(const wan_model_dims *dims, int B);

/* wan_model_forward -- the model above for B sequences.
 *   latent  float32 [B, C_in, F, H, W]; t float32 [B] (device) timesteps.
 *   text    (dt) [B, T, text_dim] text encoder features; ctx_lens as in
 *           wan_block_forward (device int32 [B] or NULL).
 *   w       model weights; blocks: HOST array of num_blocks block weights.
 *   rope    table from wan_rope_freqs(dim/heads, rope_max_pos >= the token grid).
 *   out     float32 [B, C_out, F, H, W] (the predicted velocity).
 * Constraints: wan_dims rules for the token grid (F, H/2, W/2) and dim / heads /
 * ffn_dim; H, W even; C_in * 4 and freq_dim multiples of 8; text_dim a multiple
 * of 64 (when text_len > 0); num_blocks >= 0; every pointer 16-byte aligned.
 * Kernels: the blocks as in wan_block_forward; the time MLP (fp32, B rows)
 * on a small-M weight-streaming kernel; with WAN_BF16 the patch embedding,
 * text MLP and head on the tensor-core GEMM, except a patch embedding whose
 * 4 * C_in is not a multiple of 64 (I2V's 36 channels), which runs on the
 * CUDA-core GEMM (K = 144: a negligible share of the model's work).
 * The workspace holds the token stream, the embeddings and one block
 * workspace; the head's normalised tokens reuse the block's ACT buffer.
 * Errors: as wan_block_forward. */
int wan_model_forward(const wan_model_dims *dims, int B, const float *latent, const float *t,
                      const void *text, const int *ctx_lens, const wan_model_weights *w,
                      const wan_block_weights *blocks, int num_blocks, const float *rope,
                      int rope_max_pos, float *out, void *workspace, size_t ws_bytes,
                      wan_stream_t stream);

/* wan_quantize_fp8 -- e4m3 quantization ([DIGEST] "FP8 GEMM"), per row (one
 * scale per token) or per tensor (one scale for all, as for weights).
 *   src       (src_dtype: WAN_F32 or WAN_BF16) [rows, cols], dense.
 *   per_row   1: scale[r] for every row; 0: one scale for the whole tensor.
 *   q         out uint8 [rows, cols] e4m3 codes ("fn" encoding: 1 sign,
 *             4 exponent bits biased by 7, 3 mantissa bits, largest 448).
 *   scale     out float32 [rows] (per_row) or [1]: amax / 448.
 * Rule: code = e4m3(x * (448 / amax)), nearest value with ties to even,
 * saturating at +-448; 448 / amax, the product and amax / 448 each rounded to
 * fp32. An all-zero row (or tensor) gets codes 0 and scale 0.
 * Constraints: cols % 4 == 0 (per row) or rows * cols % 4 == 0 (per tensor).
 * Errors: WAN_EINVAL (sizes, NULL), WAN_EALIGN, WAN_EUNSUPPORTED. */
int wan_quantize_fp8(const void *src, int src_dtype, int rows, int cols, int per_row, uint8_t *q,
                     float *scale, wan_stream_t stream);

/* wan_linear_fp8 -- FP8 linear layer on the tensor cores ([DIGEST] "FP8 GEMM"):
 *   out[m, n] = (sum_k a[m, k] w[n, k]) * a_scale[m] * w_scale[0] + bias[n]
 *   a        uint8 e4m3 [M, K], a_scale float32 [M] (per token);
 *   w        uint8 e4m3 [N, K], w_scale float32 [1] (per tensor), both as
 *            written by wan_quantize_fp8; bias bf16 [N] or NULL.
 *   out      float32 [M, N].
 * Products of codes are exact and accumulated in fp32.
 * Constraints: K % 128 == 0, N % 32 == 0, M >= 1.
 * Errors: WAN_EINVAL, WAN_EALIGN, WAN_EUNSUPPORTED. */
int wan_linear_fp8(int M, int N, int K, const uint8_t *a, const float *a_scale, const uint8_t *w,
                   const float *w_scale, const void *bias, float *out, wan_stream_t stream);

/* UniPC multistep sampler for the latent ("Wan2.2 I2V inference trace",
 * section 4 "DIT": the latent update "UniPC: x_noise <- step(v, t, x_noise)";
 * the method of Zhao et al., 2023, "UniPC: A Unified Predictor-Corrector
 * Framework for Fast Sampling of Diffusion Models", data-prediction form,
 * B(h) = e^h - 1). With alpha = 1 - sigma, lambda = log(alpha / sigma) and
 * the data prediction m_i = x_i - sigma_i v_i of evaluation i, one step
 * corrects the sample reached by step i - 1 with m_i (UniC) and predicts the
 * sample at sigma_{i+1} (UniP); orders 1 and 2, the first step first order.
 *
 * wan_unipc_coefficients (host only) -- the step's eight coefficients
 *   x_c    = c[0] x + c[1] last + c[2] m_{i-1} + c[3] m_{i-2} + c[4] m_i
 *   x_next = c[5] x_c + c[6] m_i + c[7] m_{i-1}
 *   sigmas  host double [num_sigmas], decreasing in [0, 1), only the last 0;
 *           num_sigmas - 1 model evaluations, step in [0, num_sigmas - 2].
 *   order   1 or 2; lower_order_final: the last step first order (a last
 *           step onto sigma = 0 is always first order).
 * wan_unipc_step -- applies one step in place, n float32 elements:
 *   v = v_uncond + guide_scale (v_cond - v_uncond) (v_uncond NULL: v_cond),
 *   m_out = x - sigma_i v, last = x_c, x = x_next (coef from the call above
 *   with the same step). m_prev1 / m_prev2 are m_{i-1} / m_{i-2} (may be
 *   NULL where their coefficients are 0); last is read only when c[1] != 0.
 *   m_out, m_prev1, m_prev2 must be distinct buffers (the caller rotates 3).
 * Errors: WAN_EINVAL (schedule, step, NULL), WAN_EUNSUPPORTED (order > 2,
 *         dtype), WAN_EALIGN. */
int wan_unipc_coefficients(const double *sigmas, int num_sigmas, int step, int order,
                           int lower_order_final, double coef[8]);
int wan_unipc_step(float *x, float *last, float *m_out, const float *m_prev1,
                   const float *m_prev2, const void *v_cond, const void *v_uncond, int v_dtype,
                   size_t n, float guide_scale, float sigma, const double coef[8],
                   wan_stream_t stream);

/* wan_attention_8bit -- 8-bit flash attention ([DIGEST] inference-optimisation
 * table, "8-bit FlashAttention": int8 for S = Q K^T, FP8 for O = P V, fp32
 * accumulation across key blocks), non-causal, head_dim 128.
 *   q, k, v   bf16 [B, Lq|Lk, heads, 128]; o out bf16 [B, Lq, heads, 128].
 *   k_lens    as in wan_attention (device int32 [B] or NULL).
 *   scale     logit scale; 0 for 1/sqrt(128).
 *   workspace device scratch of wan_attention_8bit_workspace_bytes() bytes.
 * Quantization inside the call (decisions in fp32): q to int8 per (token,
 * head) with scale amax/127, k to int8 per (sequence, head) over all Lk keys,
 * v to e4m3 per (sequence, head, channel) over all Lk keys (amax/448); int8
 * codes are round-half-even of x * (127 / amax), clamped to +-127. S is
 * accumulated exactly in int32, P = exp(S c - m) is rounded to e4m3 before
 * the P V product (fp32 accumulation), the row sum uses the unrounded P.
 * Errors: WAN_EINVAL, WAN_EALIGN, WAN_EUNSUPPORTED (Lk == 0 included). */
size_t wan_attention_8bit_workspace_bytes(int B, int heads, int Lq, int Lk);
int wan_attention_8bit(int B, int heads, int Lq, int Lk, const void *q, const void *k, const void *v,
                       void *o, const int *k_lens, float scale, void *workspace, size_t ws_bytes,
                       wan_stream_t stream);

/* wan_attention -- softmax attention, non-causal, every head
 * ([WALK] self-attention snippet: global window, key lengths).
 *   B, heads, Lq, Lk, head_dim   sizes (head_dim 128 for WAN_BF16; 32, 64
 *                                or 128 for WAN_F32).
 *   q         (dt) [B, Lq, heads, head_dim]; k, v (dt) [B, Lk, heads, head_dim].
 *   o         out (dt) [B, Lq, heads, head_dim]; must not alias q, k or v.
 *   k_lens    device int32 [B] valid keys per sequence (0..Lk), or NULL (Lk);
 *             a sequence with 0 valid keys gets o = 0.
 *   scale     logit scale; pass 0 for 1/sqrt(head_dim).
 *   grid      HOST int[3] = (F, H, W) with F*H*W == Lq == Lk: q and k are
 *             first rotated IN PLACE by the 3D RoPE of their token index
 *             (using `rope`, rope_max_pos rows); NULL: q, k are read only.
 *   rope, rope_max_pos  ignored when grid is NULL. */
int wan_attention(int B, int heads, int Lq, int Lk, int head_dim, int dtype,
                  void *q, void *k, const void *v, void *o,
                  const int *k_lens, float scale, const int *grid,
                  const float *rope, int rope_max_pos, wan_stream_t stream);

/* wan_euler_cfg_step -- classifier-free guidance followed by one explicit
 * Euler step of the flow-matching ODE ([WALK] sampling-loop snippet;
 * [DIGEST] "Video DiT and Flow Matching"):
 *     v = v_uncond + guide_scale * (v_cond - v_uncond)   (v = v_cond if v_uncond NULL)
 *     x = x + (sigma_next - sigma) * v
 *   x         in/out float32 [n].
 *   v_cond, v_uncond  [n] in v_dtype (WAN_F32 or WAN_BF16); may alias each
 *             other, not x.
 * Arithmetic in fp32 (one FMA chain per element). n may be 0. */
int wan_euler_cfg_step(float *x, const void *v_cond, const void *v_uncond,
                       int v_dtype, size_t n, float guide_scale, float sigma,
                       float sigma_next, wan_stream_t stream);

/* wan_device_status -- synchronise `stream`, then report and clear the
 * library's device-side watchdog word for the current device: WAN_OK, or
 * WAN_ETIMEOUT if a kernel gave up a bounded wait since the last call (its
 * outputs are then invalid), WAN_EBOUNDS if a debug build's bounds check
 * caught a store outside its buffer (the store was skipped), or WAN_ECUDA if
 * the stream holds a CUDA error. */
int wan_device_status(wan_stream_t stream);

/* wan_debug_bounds -- 1 in a debug build (compiled with WAN_DEBUG_BOUNDS:
 * every plain global store of the block's kernels -- the GEMM epilogue's
 * q / k sums of squares, LayerNorm, RMSNorm / RoPE, the k / q row scaling,
 * the chunk permutation, CFG-Euler, the CUDA-core GEMM and attention -- is
 * checked against its buffer's extent before it is made; the tensor-core
 * GEMM and attention write their outputs with TMA stores and reduce-adds,
 * which the tensor maps clip), 0 otherwise. */
int wan_debug_bounds(void);

/* wan_selftest_watchdog -- enqueue a one-CTA kernel whose bounded wait on an
 * mbarrier can never complete, so the wait gives up after its limit (about
 * 2 s), records its code in the watchdog word and returns without trapping.
 * A following wan_device_status(stream) reports WAN_ETIMEOUT (and clears the
 * word); the CUDA context stays usable. Test support for the failure path of
 * every tcgen05 kernel's waits; the pages have no counterpart. While the word
 * is set, tensor-core kernels launched afterwards skip their work. */
int wan_selftest_watchdog(wan_stream_t stream);

/* Launch instrumentation. While enabled, every kernel the library launches is
 * bracketed by two CUDA events recorded on its stream (a few microseconds of
 * host overhead per launch). wan_profile_enable(on) also clears the record;
 * wan_profile_read waits for the recorded events and returns, for one kernel
 * class, the number of launches and their summed device time in ms. Events
 * are created on first use and reused; at most 65536 launches are recorded.
 * Not thread-safe against concurrent enable/read. */
#define WAN_K_GEMM_TC      0  /* tensor-core GEMM (any epilogue)              */
#define WAN_K_GEMM_SIMT    1  /* CUDA-core GEMM                               */
#define WAN_K_ATTN_SELF    2  /* tensor-core attention, self (block)          */
#define WAN_K_ATTN_CROSS   3  /* tensor-core attention, cross (block)         */
#define WAN_K_ATTN_SIMT    4  /* CUDA-core attention                          */
#define WAN_K_LAYERNORM    5  /* LayerNorm + modulation / affine              */
#define WAN_K_QKNORM_ROPE  6  /* q/k RMSNorm and/or 3D RoPE                   */
#define WAN_K_EULER        7  /* CFG + Euler update                           */
#define WAN_K_MISC         8  /* modulation combine, RoPE table               */
#define WAN_K_ATTN_TC      9  /* tensor-core attention via wan_attention      */
#define WAN_K_MODEL       10  /* patchify, embeddings, head, unpatchify       */
#define WAN_K_QUANT       11  /* e4m3 quantization of GEMM inputs / weights   */
#define WAN_K_COUNT       12
int wan_profile_enable(int on);
int wan_profile_read(int kernel_class, int *launches, double *total_ms);

#ifdef __cplusplus
}
#endif
#endif /* WAN_H_ */

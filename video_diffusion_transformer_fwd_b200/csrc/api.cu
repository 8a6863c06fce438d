// C ABI of libwan: argument checking, workspace layout and the launch
// sequence of one WanAttentionBlock ("Wan2.2 code walkthrough" (newtid.com),
// WanAttentionBlock core-logic snippet) and the CFG-Euler step (sampling-loop
// snippet; "Wan paper deep dive" (charles2530.github.io), "Video DiT and
// Flow Matching").
#include "common.cuh"

#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <climits>
#include <mutex>

namespace wan {

static thread_local char g_msg[512] = "";

int set_error(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_error(cudaError_t e, const char *what) {
  return set_error(WAN_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Watchdog word: kernels with bounded waits write a nonzero code here when a
// wait runs out (they never trap).
__device__ int g_watchdog_word;

int *watchdog_ptr() {
  static int *ptrs[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_watchdog_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int *>(p);
  }
  return ptrs[dev];
}

// ---------------------------------------------------------------- dispatch
// The kernel is chosen by dtype alone: WAN_F32 runs the exact-fp32 CUDA-core
// kernels, WAN_BF16 the tcgen05 tensor-core kernels. A bf16 problem outside
// the tensor-core kernels' shape rules is refused (WAN_EUNSUPPORTED, with the
// rule in the message); it never falls back to another kernel.
static int run_gemm(const GemmArgs &g, int dtype, cudaStream_t s) {
  if (dtype == WAN_F32) return WAN_PROF(WAN_K_GEMM_SIMT, s, gemm_simt(g, dtype, s));
  if (dtype != WAN_BF16) return set_error(WAN_EUNSUPPORTED, "GEMM dtype %d", dtype);
  if (!gemm_tc_supported(g))
    return set_error(WAN_EUNSUPPORTED,
                     "bf16 GEMM M=%d N=%d K=%d outside the tensor-core kernel's rules (K %% 64 == 0, N %% 32 == 0, "
                     "256-column weight segments, 16-byte aligned rows)", g.M, g.N, g.K);
  return WAN_PROF(WAN_K_GEMM_TC, s, gemm_tc(g, s));
}

// cls: profiling class of the tensor-core launch
static int run_attention(const AttnArgs &a, int dtype, cudaStream_t s, int cls) {
  if (dtype == WAN_F32) return WAN_PROF(WAN_K_ATTN_SIMT, s, attention_simt(a, dtype, s));
  if (dtype != WAN_BF16) return set_error(WAN_EUNSUPPORTED, "attention dtype %d", dtype);
  if (!attention_tc_supported(a))
    return set_error(WAN_EUNSUPPORTED,
                     "bf16 attention (B=%d heads=%d Lq=%d Lk=%d d=%d) outside the tensor-core kernel's rules "
                     "(head_dim 128, row strides %% 8 == 0, 16-byte aligned, B and heads <= 65535)",
                     a.B, a.heads, a.Lq, a.Lk, a.d);
  return WAN_PROF(cls, s, attention_tc(a, s));
}

// ---------------------------------------------------------------- workspace
struct WsLayout {
  size_t off[WAN_WS_COUNT];
  size_t total;
};

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }
static bool is_fp8(int dt) { return dt == WAN_FP8 || dt == WAN_FP8_ATTN; }

// Modulation source of a block call: the combined [B, 6, D] (one timestep per
// sequence) or the caller's per-token e0 [B*L, 6, D] plus the block's
// modulation, added where they are read.
struct ModSrc {
  bool ptok;
  const float *e0, *mod, *modulation;
  int L, D;
};
static LnMod ln_of(const ModSrc &m, int shift_chunk, int scale_chunk) {
  return m.ptok ? ln_mod_tok(m.e0, m.modulation, m.D, shift_chunk, scale_chunk)
                : ln_mod_seq(m.mod, m.L, m.D, shift_chunk, scale_chunk);
}
static void gate_of(const ModSrc &m, GemmArgs &g, int chunk) {
  g.gate_stride = 6 * m.D;
  if (m.ptok) {
    g.gate = m.e0 + chunk * m.D; g.rows_per_gate = 1; g.gate_bias = m.modulation + chunk * m.D;
  } else {
    g.gate = m.mod + chunk * m.D; g.rows_per_gate = m.L;
  }
}

static int check_dims(const wan_dims *d, int B) {
  if (!d) return set_error(WAN_EINVAL, "dims is NULL");
  if (B < 0) return set_error(WAN_EINVAL, "B=%d < 0", B);
  if (d->F < 1 || d->H < 1 || d->W < 1) return set_error(WAN_EINVAL, "grid %dx%dx%d", d->F, d->H, d->W);
  if (d->dim < 64 || d->dim % 64) return set_error(WAN_EINVAL, "dim %d must be a positive multiple of 64", d->dim);
  if (d->dim > 8192) return set_error(WAN_EUNSUPPORTED, "dim %d > 8192", d->dim);
  if (d->heads < 1 || d->dim % d->heads) return set_error(WAN_EINVAL, "dim %d not divisible by heads %d", d->dim, d->heads);
  if (d->ffn_dim < 64 || d->ffn_dim % 64) return set_error(WAN_EINVAL, "ffn_dim %d must be a positive multiple of 64", d->ffn_dim);
  if (d->text_len < 0) return set_error(WAN_EINVAL, "text_len %d < 0", d->text_len);
  if (!(d->eps >= 0.f)) return set_error(WAN_EINVAL, "eps must be >= 0");
  if (d->e0_per_token != 0 && d->e0_per_token != 1) return set_error(WAN_EINVAL, "e0_per_token must be 0 or 1");
  if (d->dtype != WAN_F32 && d->dtype != WAN_BF16 && !is_fp8(d->dtype))
    return set_error(WAN_EUNSUPPORTED, "dtype %d", d->dtype);
  const int hd = d->dim / d->heads;
  if (d->dtype != WAN_F32 && hd != 128) return set_error(WAN_EUNSUPPORTED, "bf16 / fp8 paths need head_dim 128 (got %d)", hd);
  if (d->dtype != WAN_F32 && B > 65535)
    return set_error(WAN_EUNSUPPORTED, "bf16 / fp8 paths take at most 65535 sequences a call (got %d)", B);
  if (d->dtype != WAN_F32 && d->dim % 256)
    return set_error(WAN_EUNSUPPORTED, "bf16 / fp8 paths need dim %% 256 == 0 (got %d): the QKV epilogue "
                                       "normalises q and k over whole 256-column tiles", d->dim);
  if (is_fp8(d->dtype) && d->ffn_dim % 128)
    return set_error(WAN_EUNSUPPORTED, "fp8 path needs ffn_dim %% 128 == 0");
  if (d->dtype == WAN_F32 && hd != 32 && hd != 64 && hd != 128)
    return set_error(WAN_EUNSUPPORTED, "fp32 path needs head_dim 32, 64 or 128 (got %d)", hd);
  const long long L = (long long)d->F * d->H * d->W;
  if (L * (long long)(B > 0 ? B : 1) > INT_MAX / 4) return set_error(WAN_EINVAL, "B*L too large");
  if ((long long)d->text_len * (B > 0 ? B : 1) > INT_MAX / 4) return set_error(WAN_EINVAL, "B*T too large");
  return WAN_OK;
}

// Workspace of a block call on `rows` token rows per sequence (the whole
// sequence, or one rank's shard in the sequence-parallel phases).
static WsLayout layout_rows(const wan_dims *d, int B, int rows) {
  WsLayout w;
  const size_t es = dtype_size(d->dtype);
  const size_t BL = (size_t)B * rows, D = d->dim, T = d->text_len, Fh = d->ffn_dim;
  const size_t sz[WAN_WS_COUNT] = {
      BL * D * es,            // ACT
      BL * 3 * D * es,        // QKV
      BL * D * es,            // O
      BL * D * es,            // QC
      (size_t)B * T * 2 * D * es,  // KVC
      BL * D * es,            // OC
      BL * Fh * es,           // H
      (size_t)B * 6 * D * 4,  // MOD
      (BL > (size_t)B * T ? BL : (size_t)B * T) * 4 * (D >= 256 ? D / 256 : 1) * 4,   // STATS: per-row partial sums of squares
      is_fp8(d->dtype) ? (BL * Fh > (size_t)B * T * D ? BL * Fh : (size_t)B * T * D) : 0,   // A8
      is_fp8(d->dtype) ? (BL > (size_t)B * T ? BL : (size_t)B * T) * 4 : 0,                // ASCALE
      d->dtype == WAN_FP8_ATTN && B > 0 ? attention_8bit_ws_bytes(B, d->heads, rows, rows) : 0,
  };
  size_t o = 0;
  for (int i = 0; i < WAN_WS_COUNT; ++i) {
    w.off[i] = o;
    o += align256(sz[i]);
  }
  w.total = o;
  return w;
}
static WsLayout layout_of(const wan_dims *d, int B) { return layout_rows(d, B, d->F * d->H * d->W); }

// ---------------------------------------------------------------- FP8 block
// The fused bf16 block with every projection on the FP8 tensor cores
// ("Wan paper deep dive" (charles2530.github.io), inference-optimisation
// table, "FP8 GEMM"): each projection's input is quantized per token to e4m3
// (inside the LayerNorm for the three normalised branch inputs, by a row pass
// for the attention outputs, the FFN hidden and the context), the weights are
// e4m3 with one scale per matrix, and the GEMM epilogue multiplies by both
// scales before the bias, q/k-norm, GELU or gated residual.
static int block_forward_fp8(const wan_dims &d, int B, float *x, const void *ctx, const int *ctx_lens,
                             const wan_block_weights *w, const float *rope, char *ws, const WsLayout &lay,
                             const ModSrc &ms, cudaStream_t s) {
  const int L = d.F * d.H * d.W, D = d.dim, T = d.text_len, Fh = d.ffn_dim, hd = D / d.heads, BL = B * L;
  const size_t es = 2;
  char *qkv = ws + lay.off[WAN_WS_QKV];
  void *o = ws + lay.off[WAN_WS_O];
  void *qc = ws + lay.off[WAN_WS_QC];
  char *kvc = ws + lay.off[WAN_WS_KVC];
  void *oc = ws + lay.off[WAN_WS_OC];
  void *hbuf = ws + lay.off[WAN_WS_H];
  float *stats = reinterpret_cast<float *>(ws + lay.off[WAN_WS_STATS]);
  uint8_t *a8 = reinterpret_cast<uint8_t *>(ws + lay.off[WAN_WS_A8]);
  float *asc = reinterpret_cast<float *>(ws + lay.off[WAN_WS_ASCALE]);
  const float *wsc = w->w_scales;
  const int parts = D / 256, sstride = 4 * parts;
  const float scale = 1.0f / sqrtf((float)hd);
  int rc;
  auto gemm8 = [&](GemmArgs &g) -> int {
    g.fp8 = 1; g.A = a8; g.lda = g.K; g.a_scale = asc;
    if (!gemm_tc_supported(g)) return set_error(WAN_EUNSUPPORTED, "fp8 GEMM M=%d N=%d K=%d", g.M, g.N, g.K);
    return WAN_PROF(WAN_K_GEMM_TC, s, gemm_tc(g, s));
  };
  auto quant_rows = [&](const void *src, int rows, int cols) -> int {
    return WAN_PROF(WAN_K_QUANT, s, launch_quant_rows(src, WAN_BF16, (size_t)cols, rows, cols, a8, asc, s));
  };

  // ---- self-attention
  if ((rc = WAN_PROF(WAN_K_LAYERNORM, s, launch_layernorm_mod_fp8(x, a8, asc, BL, D, ln_of(ms, 0, 1), nullptr, nullptr, d.eps, s)))) return rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = 3 * D; g.K = D;
    g.Bseg[0] = w->wq; g.Bseg[1] = w->wk; g.Bseg[2] = w->wv;
    g.bias[0] = w->bq; g.bias[1] = w->bk; g.bias[2] = w->bv;
    g.b_scale[0] = wsc + 0; g.b_scale[1] = wsc + 1; g.b_scale[2] = wsc + 2;
    g.segN = D; g.nseg = 3; g.C = qkv; g.ldc = 3 * D; g.epi = EPI_QKNORM;
    g.gamma[0] = w->gq; g.gamma[1] = w->gk; g.gamma[2] = nullptr;
    g.ss = stats; g.ss_stride = sstride; g.ss_col[0] = 0; g.ss_col[1] = 1; g.ss_col[2] = -1;
    g.rope = rope; g.rope_mask = 3; g.F = d.F; g.H = d.H; g.W = d.W; g.head_dim = hd;
    if ((rc = gemm8(g))) return rc;
  }
  if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, s, launch_scale_rows(qkv + D * es, BL, 3 * D, D, stats + parts, sstride, parts, d.eps, s)))) return rc;
  {
    AttnArgs a = {};
    a.B = B; a.heads = d.heads; a.Lq = L; a.Lk = L; a.d = hd;
    a.q = qkv; a.ldq = 3 * D; a.k = qkv + D * es; a.ldk = 3 * D; a.v = qkv + 2 * D * es; a.ldv = 3 * D;
    a.o = o; a.ldo = D; a.scale = scale;
    a.q_ss = stats; a.q_ss_stride = sstride; a.q_ss_parts = parts; a.q_ss_n = (float)D; a.q_ss_eps = d.eps;
    if (!attention_tc_supported(a)) return set_error(WAN_EUNSUPPORTED, "fp8 block: self-attention shape");
    if (d.dtype == WAN_FP8_ATTN) {
      if (!attention_8bit_supported(a)) return set_error(WAN_EUNSUPPORTED, "fp8 block: 8-bit self-attention shape");
      if ((rc = WAN_PROF(WAN_K_ATTN_SELF, s, attention_8bit(a, ws + lay.off[WAN_WS_ATTN8], s)))) return rc;
    } else if ((rc = WAN_PROF(WAN_K_ATTN_SELF, s, attention_tc(a, s)))) {
      return rc;
    }
  }
  if ((rc = quant_rows(o, BL, D))) return rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = D; g.Bseg[0] = w->wo; g.bias[0] = w->bo; g.b_scale[0] = wsc + 3;
    g.segN = D; g.nseg = 1;
    g.epi = EPI_RESID; g.X = x; g.ldx = D;
    gate_of(ms, g, 2);
    if ((rc = gemm8(g))) return rc;
  }

  // ---- cross-attention (ungated)
  if ((rc = WAN_PROF(WAN_K_LAYERNORM, s, launch_layernorm_mod_fp8(x, a8, asc, BL, D, LnMod{}, w->g3, w->b3, d.eps, s)))) return rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = D; g.Bseg[0] = w->cwq; g.bias[0] = w->cbq; g.b_scale[0] = wsc + 4;
    g.segN = D; g.nseg = 1; g.C = qc; g.ldc = D; g.epi = EPI_QKNORM;
    g.gamma[0] = w->cgq; g.ss = stats; g.ss_stride = sstride; g.ss_col[0] = 2; g.ss_col[1] = g.ss_col[2] = -1;
    if ((rc = gemm8(g))) return rc;
  }
  if (T > 0) {
    if ((rc = quant_rows(ctx, B * T, D))) return rc;
    GemmArgs g = {};
    g.M = B * T; g.N = 2 * D; g.K = D;
    g.Bseg[0] = w->cwk; g.Bseg[1] = w->cwv; g.bias[0] = w->cbk; g.bias[1] = w->cbv;
    g.b_scale[0] = wsc + 5; g.b_scale[1] = wsc + 6;
    g.segN = D; g.nseg = 2; g.C = kvc; g.ldc = 2 * D; g.epi = EPI_QKNORM;
    g.gamma[0] = w->cgk; g.gamma[1] = nullptr; g.ss = stats; g.ss_stride = sstride;
    g.ss_col[0] = 3; g.ss_col[1] = -1; g.ss_col[2] = -1;
    if ((rc = gemm8(g))) return rc;
    if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, s, launch_scale_rows(kvc, B * T, 2 * D, D, stats + 3 * parts, sstride, parts, d.eps, s)))) return rc;
  }
  {
    AttnArgs a = {};
    a.B = B; a.heads = d.heads; a.Lq = L; a.Lk = T; a.d = hd;
    a.q = qc; a.ldq = D; a.k = kvc; a.ldk = 2 * D; a.v = kvc + D * es; a.ldv = 2 * D;
    a.o = oc; a.ldo = D; a.k_lens = ctx_lens; a.scale = scale;
    a.q_ss = stats + 2 * parts; a.q_ss_stride = sstride; a.q_ss_parts = parts; a.q_ss_n = (float)D; a.q_ss_eps = d.eps;
    if ((rc = run_attention(a, WAN_BF16, s, WAN_K_ATTN_CROSS))) return rc;
  }
  if ((rc = quant_rows(oc, BL, D))) return rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = D; g.Bseg[0] = w->cwo; g.bias[0] = w->cbo; g.b_scale[0] = wsc + 7;
    g.segN = D; g.nseg = 1;
    g.epi = EPI_RESID; g.X = x; g.ldx = D; g.gate = nullptr; g.rows_per_gate = L;
    if ((rc = gemm8(g))) return rc;
  }

  // ---- FFN
  if ((rc = WAN_PROF(WAN_K_LAYERNORM, s, launch_layernorm_mod_fp8(x, a8, asc, BL, D, ln_of(ms, 3, 4), nullptr, nullptr, d.eps, s)))) return rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = Fh; g.K = D; g.Bseg[0] = w->w1; g.bias[0] = w->b1; g.b_scale[0] = wsc + 8;
    g.segN = Fh; g.nseg = 1; g.epi = EPI_GELU; g.C = hbuf; g.ldc = Fh;
    if ((rc = gemm8(g))) return rc;
  }
  if ((rc = quant_rows(hbuf, BL, Fh))) return rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = Fh; g.Bseg[0] = w->w2; g.bias[0] = w->b2; g.b_scale[0] = wsc + 9;
    g.segN = D; g.nseg = 1;
    g.epi = EPI_RESID; g.X = x; g.ldx = D;
    gate_of(ms, g, 5);
    if ((rc = gemm8(g))) return rc;
  }
  return WAN_OK;
}

// ---------------------------------------------------------------- block stages
// One block call on `rows` token rows of each of B sequences; row r of a
// sequence is token tok0 + r of its (F, H, W) grid. wan_block_forward runs the
// stages on whole sequences; the sequence-parallel entry points run the first
// and the last on one rank's token shard, the attention between them running
// on a head shard of the whole sequence after an all-to-all.
struct BlockCall {
  const wan_dims *d;
  int B, rows, tok0;
  float *x;
  const void *ctx;
  const int *ctx_lens;
  const float *e0;
  const wan_block_weights *w;
  const float *rope;
  int rope_max_pos;
  char *ws;
  WsLayout lay;
  cudaStream_t s;
  ModSrc ms;
};

static int parts_of(int D) { return D >= 256 ? D / 256 : 1; }

// m = modulation + e0 (shift, scale, gate, shift2, scale2, gate2) into the
// workspace, unless e0 is per token (then read in place)
static int stage_mod(const BlockCall &c) {
  if (c.ms.ptok) return WAN_OK;
  return WAN_PROF(WAN_K_MISC, c.s, launch_mod_combine(c.w->modulation, c.e0, const_cast<float *>(c.ms.mod),
                                                      c.B, c.d->dim, c.s));
}

// LN1 + modulate, the QKV projection, q / k RMSNorm and 3D RoPE into qkv
// [B * rows, 3 * dim] (q | k | v per row). bf16: the GEMM epilogue leaves
// the rows' sums of squares in the workspace statistics; k is scaled by its
// RMS factor here, q too when `normalize_q` (otherwise the attention folds
// q's factor into its logit scale).
static int stage_self_qkv(const BlockCall &c, void *qkv, bool normalize_q) {
  const wan_dims &d = *c.d;
  const int D = d.dim, hd = D / d.heads, BL = c.B * c.rows, dt = d.dtype;
  const size_t es = dtype_size(dt);
  void *act = c.ws + c.lay.off[WAN_WS_ACT];
  float *stats = reinterpret_cast<float *>(c.ws + c.lay.off[WAN_WS_STATS]);
  const int parts = parts_of(D), sstride = 4 * parts;
  int rc;
  if ((rc = WAN_PROF(WAN_K_LAYERNORM, c.s, launch_layernorm_mod(c.x, act, dt, BL, D, ln_of(c.ms, 0, 1), nullptr,
                                                                nullptr, d.eps, c.s)))) return rc;
  GemmArgs g = {};
  g.M = BL; g.N = 3 * D; g.K = D; g.A = act; g.lda = D;
  g.Bseg[0] = c.w->wq; g.Bseg[1] = c.w->wk; g.Bseg[2] = c.w->wv;
  g.bias[0] = c.w->bq; g.bias[1] = c.w->bk; g.bias[2] = c.w->bv;
  g.segN = D; g.nseg = 3; g.C = qkv; g.ldc = 3 * D;
  g.rope = c.rope; g.F = d.F; g.H = d.H; g.W = d.W; g.head_dim = hd; g.rows_per_seq = c.rows; g.tok0 = c.tok0;
  char *q = static_cast<char *>(qkv);
  if (dt == WAN_BF16) {
    g.epi = EPI_QKNORM;
    g.gamma[0] = c.w->gq; g.gamma[1] = c.w->gk; g.gamma[2] = nullptr;
    g.ss = stats; g.ss_stride = sstride; g.ss_col[0] = 0; g.ss_col[1] = 1; g.ss_col[2] = -1;
    g.rope_mask = 3;
    if ((rc = run_gemm(g, dt, c.s))) return rc;
    if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, c.s, launch_scale_rows(q + D * es, BL, 3 * D, D, stats + parts, sstride,
                                                                 parts, d.eps, c.s)))) return rc;
    if (normalize_q &&
        (rc = WAN_PROF(WAN_K_QKNORM_ROPE, c.s, launch_scale_rows(q, BL, 3 * D, D, stats, sstride, parts, d.eps, c.s))))
      return rc;
    return WAN_OK;
  }
  g.epi = EPI_STORE;
  if ((rc = run_gemm(g, dt, c.s))) return rc;
  if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, c.s, launch_rmsnorm_rope(q, dt, BL, 3 * D, D, hd, c.w->gq, d.eps, c.rope,
                                                                 c.rope_max_pos, d.F, d.H, d.W, c.s, c.rows,
                                                                 c.tok0)))) return rc;
  return WAN_PROF(WAN_K_QKNORM_ROPE, c.s, launch_rmsnorm_rope(q + D * es, dt, BL, 3 * D, D, hd, c.w->gk, d.eps, c.rope,
                                                              c.rope_max_pos, d.F, d.H, d.W, c.s, c.rows, c.tok0));
}

// Self-attention of whole sequences (rows == L) from the stage_self_qkv
// output; bf16 folds q's RMS factor into the logit scale.
static int stage_self_attention(const BlockCall &c, const void *qkv, void *o) {
  const wan_dims &d = *c.d;
  const int D = d.dim, hd = D / d.heads;
  const size_t es = dtype_size(d.dtype);
  const char *q = static_cast<const char *>(qkv);
  AttnArgs a = {};
  a.B = c.B; a.heads = d.heads; a.Lq = c.rows; a.Lk = c.rows; a.d = hd;
  a.q = q; a.ldq = 3 * D; a.k = q + D * es; a.ldk = 3 * D; a.v = q + 2 * D * es; a.ldv = 3 * D;
  a.o = o; a.ldo = D; a.k_lens = nullptr; a.scale = 1.0f / sqrtf((float)hd);
  if (d.dtype == WAN_BF16) {
    const int parts = parts_of(D);
    a.q_ss = reinterpret_cast<const float *>(c.ws + c.lay.off[WAN_WS_STATS]); a.q_ss_stride = 4 * parts;
    a.q_ss_parts = parts; a.q_ss_n = (float)D; a.q_ss_eps = d.eps;
  }
  return run_attention(a, d.dtype, c.s, WAN_K_ATTN_SELF);
}

// The rest of the block on the call's rows: x += m2 * (o W_o^T + b_o), the
// cross-attention branch (ungated) and the FFN branch.
static int stage_finish(const BlockCall &c, const void *o) {
  const wan_dims &d = *c.d;
  const int D = d.dim, T = d.text_len, Fh = d.ffn_dim, hd = D / d.heads, BL = c.B * c.rows, dt = d.dtype;
  const size_t es = dtype_size(dt);
  const bool tc = dt == WAN_BF16;
  void *act = c.ws + c.lay.off[WAN_WS_ACT];
  void *qc = c.ws + c.lay.off[WAN_WS_QC];
  char *kvc = c.ws + c.lay.off[WAN_WS_KVC];
  void *oc = c.ws + c.lay.off[WAN_WS_OC];
  void *hbuf = c.ws + c.lay.off[WAN_WS_H];
  float *stats = reinterpret_cast<float *>(c.ws + c.lay.off[WAN_WS_STATS]);
  const int parts = parts_of(D), sstride = 4 * parts;
  int rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = D; g.A = o; g.lda = D;
    g.Bseg[0] = c.w->wo; g.bias[0] = c.w->bo; g.segN = D; g.nseg = 1;
    g.epi = EPI_RESID; g.X = c.x; g.ldx = D;
    gate_of(c.ms, g, 2);
    if ((rc = run_gemm(g, dt, c.s))) return rc;
  }

  // ---- cross-attention branch (ungated): x += Wco . Attn(q(norm3 x), k(ctx), v(ctx))
  if ((rc = WAN_PROF(WAN_K_LAYERNORM, c.s, launch_layernorm_mod(c.x, act, dt, BL, D, LnMod{}, c.w->g3, c.w->b3,
                                                                d.eps, c.s)))) return rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = D; g.A = act; g.lda = D;
    g.Bseg[0] = c.w->cwq; g.bias[0] = c.w->cbq; g.segN = D; g.nseg = 1;
    g.C = qc; g.ldc = D;
    g.epi = tc ? EPI_QKNORM : EPI_STORE;
    g.gamma[0] = c.w->cgq; g.ss = stats; g.ss_stride = sstride; g.ss_col[0] = 2; g.ss_col[1] = g.ss_col[2] = -1;
    if ((rc = run_gemm(g, dt, c.s))) return rc;
  }
  if (!tc && (rc = WAN_PROF(WAN_K_QKNORM_ROPE, c.s, launch_rmsnorm_rope(qc, dt, BL, D, D, hd, c.w->cgq, d.eps, nullptr,
                                                                        0, 1, 1, 1, c.s)))) return rc;
  if (T > 0) {
    GemmArgs g = {};
    g.M = c.B * T; g.N = 2 * D; g.K = D; g.A = c.ctx; g.lda = D;
    g.Bseg[0] = c.w->cwk; g.Bseg[1] = c.w->cwv; g.bias[0] = c.w->cbk; g.bias[1] = c.w->cbv;
    g.segN = D; g.nseg = 2; g.C = kvc; g.ldc = 2 * D;
    g.epi = tc ? EPI_QKNORM : EPI_STORE;
    g.gamma[0] = c.w->cgk; g.gamma[1] = nullptr; g.ss = stats; g.ss_stride = sstride;
    g.ss_col[0] = 3; g.ss_col[1] = -1; g.ss_col[2] = -1;
    if ((rc = run_gemm(g, dt, c.s))) return rc;
    if (tc) {
      if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, c.s, launch_scale_rows(kvc, c.B * T, 2 * D, D, stats + 3 * parts, sstride,
                                                                   parts, d.eps, c.s)))) return rc;
    } else if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, c.s, launch_rmsnorm_rope(kvc, dt, c.B * T, 2 * D, D, hd, c.w->cgk,
                                                                          d.eps, nullptr, 0, 1, 1, 1, c.s)))) {
      return rc;
    }
  }
  {
    AttnArgs a = {};
    a.B = c.B; a.heads = d.heads; a.Lq = c.rows; a.Lk = T; a.d = hd;
    a.q = qc; a.ldq = D; a.k = kvc; a.ldk = 2 * D; a.v = kvc + D * es; a.ldv = 2 * D;
    a.o = oc; a.ldo = D; a.k_lens = c.ctx_lens; a.scale = 1.0f / sqrtf((float)hd);
    if (tc) {
      a.q_ss = stats + 2 * parts; a.q_ss_stride = sstride; a.q_ss_parts = parts;
      a.q_ss_n = (float)D; a.q_ss_eps = d.eps;
    }
    if ((rc = run_attention(a, dt, c.s, WAN_K_ATTN_CROSS))) return rc;
  }
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = D; g.A = oc; g.lda = D;
    g.Bseg[0] = c.w->cwo; g.bias[0] = c.w->cbo; g.segN = D; g.nseg = 1;
    g.epi = EPI_RESID; g.X = c.x; g.ldx = D; g.gate = nullptr; g.rows_per_gate = c.rows;
    if ((rc = run_gemm(g, dt, c.s))) return rc;
  }

  // ---- FFN branch: x += m5 * W2 . gelu_tanh(W1 . (LN(x)(1 + m4) + m3))
  if ((rc = WAN_PROF(WAN_K_LAYERNORM, c.s, launch_layernorm_mod(c.x, act, dt, BL, D, ln_of(c.ms, 3, 4), nullptr,
                                                                nullptr, d.eps, c.s)))) return rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = Fh; g.K = D; g.A = act; g.lda = D;
    g.Bseg[0] = c.w->w1; g.bias[0] = c.w->b1; g.segN = Fh; g.nseg = 1;
    g.epi = EPI_GELU; g.C = hbuf; g.ldc = Fh;
    if ((rc = run_gemm(g, dt, c.s))) return rc;
  }
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = Fh; g.A = hbuf; g.lda = Fh;
    g.Bseg[0] = c.w->w2; g.bias[0] = c.w->b2; g.segN = D; g.nseg = 1;
    g.epi = EPI_RESID; g.X = c.x; g.ldx = D;
    gate_of(c.ms, g, 5);
    if ((rc = run_gemm(g, dt, c.s))) return rc;
  }
  return WAN_OK;
}

// Checks shared by the block entry points; fills the call on success.
// `need_ctx` / `need_rope`: the call runs the cross-attention / the RoPE.
static int prepare_call(BlockCall &c, const wan_dims *dims, int B, int rows, int tok0, float *x, const void *ctx,
                        const int *ctx_lens, const float *e0, const wan_block_weights *w, const float *rope,
                        int rope_max_pos, void *workspace, size_t ws_bytes, cudaStream_t s, bool need_ctx,
                        bool need_rope) {
  const wan_dims &d = *dims;
  if (!w) return set_error(WAN_EINVAL, "weights is NULL");
  const void *ptrs[] = {x, e0, workspace, w->modulation, w->wq, w->bq, w->wk, w->bk, w->wv,
                        w->bv, w->wo, w->bo, w->gq, w->gk, w->g3, w->b3, w->cwq, w->cbq, w->cwk,
                        w->cbk, w->cwv, w->cbv, w->cwo, w->cbo, w->cgq, w->cgk, w->w1, w->b1,
                        w->w2, w->b2, need_rope ? rope : x};
  for (size_t i = 0; i < sizeof(ptrs) / sizeof(ptrs[0]); ++i) {
    if (!ptrs[i]) return set_error(WAN_EINVAL, "pointer argument #%zu is NULL", i);
    if (!aligned16(ptrs[i])) return set_error(WAN_EALIGN, "pointer argument #%zu not 16-byte aligned", i);
  }
  if (is_fp8(d.dtype)) {
    if (!w->w_scales) return set_error(WAN_EINVAL, "WAN_FP8 needs w_scales");
    if (!aligned16(w->w_scales)) return set_error(WAN_EALIGN, "w_scales not 16-byte aligned");
  }
  if (need_ctx && d.text_len > 0 && !ctx) return set_error(WAN_EINVAL, "ctx is NULL");
  if (ctx && !aligned16(ctx)) return set_error(WAN_EALIGN, "ctx not 16-byte aligned");
  if (ctx_lens && !aligned16(ctx_lens)) return set_error(WAN_EALIGN, "ctx_lens not 16-byte aligned");
  if (need_rope) {
    const int gmax = d.F > d.H ? (d.F > d.W ? d.F : d.W) : (d.H > d.W ? d.H : d.W);
    if (rope_max_pos < gmax) return set_error(WAN_EINVAL, "rope table has %d rows, grid needs %d", rope_max_pos, gmax);
  }
  c.lay = layout_rows(dims, B, rows);
  if (ws_bytes < c.lay.total) return set_error(WAN_EINVAL, "workspace %zu bytes < %zu needed", ws_bytes, c.lay.total);
  c.d = dims; c.B = B; c.rows = rows; c.tok0 = tok0; c.x = x; c.ctx = ctx; c.ctx_lens = ctx_lens; c.e0 = e0;
  c.w = w; c.rope = rope; c.rope_max_pos = rope_max_pos; c.ws = static_cast<char *>(workspace); c.s = s;
  c.ms = ModSrc{d.e0_per_token != 0, e0, reinterpret_cast<float *>(c.ws + c.lay.off[WAN_WS_MOD]), w->modulation,
                rows, d.dim};
  return WAN_OK;
}

// Rows and first token of a sequence-parallel call, and its dtype.
static int check_shard(const wan_dims *dims, int B, int rows, int tok0) {
  int rc = check_dims(dims, B);
  if (rc) return rc;
  const long long L = (long long)dims->F * dims->H * dims->W;
  if (rows < 1 || tok0 < 0 || tok0 + (long long)rows > L)
    return set_error(WAN_EINVAL, "token shard [%d, %d + %d) outside the %lld-token grid", tok0, tok0, rows, L);
  if (is_fp8(dims->dtype)) return set_error(WAN_EUNSUPPORTED, "the sequence-parallel phases run WAN_F32 or WAN_BF16");
  return WAN_OK;
}

}  // namespace wan

using namespace wan;

extern "C" {

const char *wan_last_error(void) { return g_msg; }

int wan_rope_freqs(int head_dim, int max_pos, double theta, float *table, wan_stream_t stream) {
  g_msg[0] = 0;
  if (head_dim < 2 || head_dim > 256 || head_dim % 2) return set_error(WAN_EINVAL, "head_dim %d", head_dim);
  if (max_pos < 1) return set_error(WAN_EINVAL, "max_pos %d", max_pos);
  if (!(theta > 0.0)) return set_error(WAN_EINVAL, "theta must be > 0");
  if (!table) return set_error(WAN_EINVAL, "table is NULL");
  if (!aligned16(table)) return set_error(WAN_EALIGN, "table not 16-byte aligned");
  return WAN_PROF(WAN_K_MISC, (cudaStream_t)stream, launch_rope_table(head_dim, max_pos, theta, table, (cudaStream_t)stream));
}

size_t wan_block_workspace_bytes(const wan_dims *dims, int B) {
  if (check_dims(dims, B) != WAN_OK) return 0;
  return layout_of(dims, B).total;
}

size_t wan_block_workspace_offset(const wan_dims *dims, int B, int which) {
  if (check_dims(dims, B) != WAN_OK || which < 0 || which >= WAN_WS_COUNT) return (size_t)-1;
  return layout_of(dims, B).off[which];
}

int wan_block_forward(const wan_dims *dims, int B, float *x, const void *ctx, const int *ctx_lens,
                      const float *e0, const wan_block_weights *w, const float *rope,
                      int rope_max_pos, void *workspace, size_t ws_bytes, wan_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_dims(dims, B);
  if (rc) return rc;
  if (B == 0) return WAN_OK;
  const wan_dims &d = *dims;
  const int L = d.F * d.H * d.W;
  BlockCall c;
  if ((rc = prepare_call(c, dims, B, L, 0, x, ctx, ctx_lens, e0, w, rope, rope_max_pos, workspace, ws_bytes,
                         (cudaStream_t)stream, true, true))) return rc;
  if ((rc = stage_mod(c))) return rc;
  if (is_fp8(d.dtype)) return block_forward_fp8(d, B, x, ctx, ctx_lens, w, rope, c.ws, c.lay, c.ms, c.s);
  void *qkv = c.ws + c.lay.off[WAN_WS_QKV];
  void *o = c.ws + c.lay.off[WAN_WS_O];
  if ((rc = stage_self_qkv(c, qkv, false))) return rc;
  if ((rc = stage_self_attention(c, qkv, o))) return rc;
  return stage_finish(c, o);
}

size_t wan_block_sp_workspace_bytes(const wan_dims *dims, int B, int rows) {
  if (check_shard(dims, B, rows, 0) != WAN_OK) return 0;
  return layout_rows(dims, B, rows).total;
}

int wan_block_sp_qkv(const wan_dims *dims, int B, int rows, int tok0, const float *x, const float *e0,
                     const wan_block_weights *w, const float *rope, int rope_max_pos, void *qkv,
                     void *workspace, size_t ws_bytes, wan_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_shard(dims, B, rows, tok0);
  if (rc) return rc;
  if (B == 0) return WAN_OK;
  if (!qkv) return set_error(WAN_EINVAL, "qkv is NULL");
  if (!aligned16(qkv)) return set_error(WAN_EALIGN, "qkv not 16-byte aligned");
  BlockCall c;
  if ((rc = prepare_call(c, dims, B, rows, tok0, const_cast<float *>(x), nullptr, nullptr, e0, w, rope,
                         rope_max_pos, workspace, ws_bytes, (cudaStream_t)stream, false, true))) return rc;
  if ((rc = stage_mod(c))) return rc;
  return stage_self_qkv(c, qkv, true);
}

int wan_block_sp_finish(const wan_dims *dims, int B, int rows, float *x, const void *ctx, const int *ctx_lens,
                        const float *e0, const wan_block_weights *w, const void *o, void *workspace,
                        size_t ws_bytes, wan_stream_t stream) {
  g_msg[0] = 0;
  int rc = check_shard(dims, B, rows, 0);
  if (rc) return rc;
  if (B == 0) return WAN_OK;
  if (!o) return set_error(WAN_EINVAL, "o is NULL");
  if (!aligned16(o)) return set_error(WAN_EALIGN, "o not 16-byte aligned");
  BlockCall c;
  if ((rc = prepare_call(c, dims, B, rows, 0, x, ctx, ctx_lens, e0, w, nullptr, 0, workspace, ws_bytes,
                         (cudaStream_t)stream, true, false))) return rc;
  if ((rc = stage_mod(c))) return rc;
  return stage_finish(c, o);
}

int wan_permute_chunks(const void *src, void *dst, int ndim, const int *dims, const int *perm, size_t chunk_bytes,
                       wan_stream_t stream) {
  g_msg[0] = 0;
  if (ndim < 1 || ndim > 5 || !dims || !perm) return set_error(WAN_EINVAL, "ndim %d must be 1..5 with dims and perm", ndim);
  if (chunk_bytes == 0 || chunk_bytes % 16) return set_error(WAN_EINVAL, "chunk_bytes %zu must be a positive multiple of 16", chunk_bytes);
  bool seen[5] = {false, false, false, false, false};
  long long n = 1;
  for (int k = 0; k < ndim; ++k) {
    if (dims[k] < 0) return set_error(WAN_EINVAL, "dims[%d] = %d < 0", k, dims[k]);
    if (perm[k] < 0 || perm[k] >= ndim || seen[perm[k]]) return set_error(WAN_EINVAL, "perm is not a permutation");
    seen[perm[k]] = true;
    n *= dims[k];
  }
  if (n == 0) return WAN_OK;
  if (!src || !dst) return set_error(WAN_EINVAL, "NULL buffer");
  if (!aligned16(src) || !aligned16(dst)) return set_error(WAN_EALIGN, "buffers must be 16-byte aligned");
  const size_t bytes = (size_t)n * chunk_bytes;
  const char *a = static_cast<const char *>(src), *b = static_cast<const char *>(dst);
  if (a < b + bytes && b < a + bytes) return set_error(WAN_EINVAL, "src and dst overlap");
  cudaStream_t s = (cudaStream_t)stream;
  return WAN_PROF(WAN_K_MISC, s, launch_permute_chunks(src, dst, ndim, dims, perm, chunk_bytes, s));
}

int wan_quantize_fp8(const void *src, int src_dtype, int rows, int cols, int per_row, uint8_t *q,
                     float *scale, wan_stream_t stream) {
  g_msg[0] = 0;
  if (rows < 0 || cols < 0) return set_error(WAN_EINVAL, "rows %d cols %d", rows, cols);
  if (src_dtype != WAN_F32 && src_dtype != WAN_BF16) return set_error(WAN_EUNSUPPORTED, "src dtype %d", src_dtype);
  if (!scale && !(per_row && rows == 0)) return set_error(WAN_EINVAL, "scale is NULL");
  const size_t n = (size_t)rows * cols;
  if (n > 0 && (!src || !q)) return set_error(WAN_EINVAL, "NULL tensor");
  const void *ps[] = {src, q, scale};
  for (const void *p : ps)
    if (p && !aligned16(p)) return set_error(WAN_EALIGN, "pointer not 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  if (per_row) {
    if (cols % 4) return set_error(WAN_EUNSUPPORTED, "per-row quantization needs cols %% 4 == 0");
    return WAN_PROF(WAN_K_QUANT, s, launch_quant_rows(src, src_dtype, (size_t)cols, rows, cols, q, scale, s));
  }
  if (n % 4) return set_error(WAN_EUNSUPPORTED, "per-tensor quantization needs rows * cols %% 4 == 0");
  return WAN_PROF(WAN_K_QUANT, s, launch_quant_tensor(src, src_dtype, n, q, scale, s));
}

int wan_linear_fp8(int M, int N, int K, const uint8_t *a, const float *a_scale, const uint8_t *w,
                   const float *w_scale, const void *bias, float *out, wan_stream_t stream) {
  g_msg[0] = 0;
  if (M < 0 || N < 0 || K < 0) return set_error(WAN_EINVAL, "M %d N %d K %d", M, N, K);
  if (M == 0 || N == 0) return WAN_OK;
  if (K % 128 || K == 0 || N % 32) return set_error(WAN_EUNSUPPORTED, "fp8 linear needs K %% 128 == 0, N %% 32 == 0");
  if ((long long)M * N > (long long)INT_MAX * 4) return set_error(WAN_EINVAL, "M * N too large");
  const void *ps[] = {a, a_scale, w, w_scale, out};
  for (const void *p : ps) {
    if (!p) return set_error(WAN_EINVAL, "NULL pointer");
    if (!aligned16(p)) return set_error(WAN_EALIGN, "pointer not 16-byte aligned");
  }
  if (bias && !aligned16(bias)) return set_error(WAN_EALIGN, "bias not 16-byte aligned");
  GemmArgs g = {};
  g.M = M; g.N = N; g.K = K; g.A = a; g.lda = K;
  g.Bseg[0] = w; g.bias[0] = bias; g.segN = N; g.nseg = 1;
  g.epi = EPI_RESID; g.X = out; g.ldx = N; g.gate = nullptr; g.rows_per_gate = 1; g.x_store = 1;
  g.fp8 = 1; g.a_scale = a_scale; g.b_scale[0] = w_scale;
  if (!gemm_tc_supported(g)) return set_error(WAN_EUNSUPPORTED, "fp8 linear M=%d N=%d K=%d", M, N, K);
  cudaStream_t s = (cudaStream_t)stream;
  return WAN_PROF(WAN_K_GEMM_TC, s, gemm_tc(g, s));
}

size_t wan_attention_8bit_workspace_bytes(int B, int heads, int Lq, int Lk) {
  if (B < 1 || heads < 1 || Lq < 1 || Lk < 1) return 0;
  return attention_8bit_ws_bytes(B, heads, Lq, Lk);
}

int wan_attention_8bit(int B, int heads, int Lq, int Lk, const void *q, const void *k, const void *v,
                       void *o, const int *k_lens, float scale, void *workspace, size_t ws_bytes,
                       wan_stream_t stream) {
  g_msg[0] = 0;
  if (B < 0 || heads < 1 || Lq < 0 || Lk < 0) return set_error(WAN_EINVAL, "bad sizes");
  if (B == 0 || Lq == 0) return WAN_OK;
  if (Lk == 0) return set_error(WAN_EUNSUPPORTED, "8-bit attention needs Lk >= 1");
  if ((long long)B * Lq * heads > INT_MAX / 32 || (long long)B * Lk * heads > INT_MAX / 32)
    return set_error(WAN_EINVAL, "sizes too large");
  const void *ps[] = {q, k, v, o, workspace};
  for (const void *p : ps) {
    if (!p) return set_error(WAN_EINVAL, "NULL pointer");
    if (!aligned16(p)) return set_error(WAN_EALIGN, "pointer not 16-byte aligned");
  }
  if (k_lens && !aligned16(k_lens)) return set_error(WAN_EALIGN, "k_lens not 16-byte aligned");
  if (ws_bytes < attention_8bit_ws_bytes(B, heads, Lq, Lk)) return set_error(WAN_EINVAL, "workspace too small");
  AttnArgs a = {};
  a.B = B; a.heads = heads; a.Lq = Lq; a.Lk = Lk; a.d = 128;
  a.q = q; a.ldq = heads * 128; a.k = k; a.ldk = heads * 128; a.v = v; a.ldv = heads * 128;
  a.o = o; a.ldo = heads * 128; a.k_lens = k_lens; a.scale = scale > 0.f ? scale : 1.0f / sqrtf(128.f);
  if (!attention_8bit_supported(a)) return set_error(WAN_EUNSUPPORTED, "8-bit attention shape");
  cudaStream_t s = (cudaStream_t)stream;
  return WAN_PROF(WAN_K_ATTN_TC, s, attention_8bit(a, workspace, s));
}

int wan_attention(int B, int heads, int Lq, int Lk, int head_dim, int dtype, void *q, void *k,
                  const void *v, void *o, const int *k_lens, float scale, const int *grid,
                  const float *rope, int rope_max_pos, wan_stream_t stream) {
  g_msg[0] = 0;
  if (B < 0 || heads < 1 || Lq < 0 || Lk < 0) return set_error(WAN_EINVAL, "bad sizes");
  if (dtype != WAN_F32 && dtype != WAN_BF16) return set_error(WAN_EUNSUPPORTED, "dtype %d", dtype);
  if (dtype == WAN_BF16 && head_dim != 128) return set_error(WAN_EUNSUPPORTED, "bf16 attention needs head_dim 128");
  if (dtype == WAN_F32 && head_dim != 32 && head_dim != 64 && head_dim != 128)
    return set_error(WAN_EUNSUPPORTED, "fp32 attention needs head_dim 32, 64 or 128");
  if ((long long)B * Lq * heads * head_dim > (long long)INT_MAX * 8 || (long long)B * Lq > INT_MAX / 4 ||
      (long long)B * Lk > INT_MAX / 4)
    return set_error(WAN_EINVAL, "sizes too large");
  if (B == 0 || Lq == 0) return WAN_OK;
  if (!q || !o || (Lk > 0 && (!k || !v))) return set_error(WAN_EINVAL, "NULL tensor");
  const void *ps[] = {q, k, v, o, k_lens};
  for (const void *p : ps)
    if (p && !aligned16(p)) return set_error(WAN_EALIGN, "pointer not 16-byte aligned");
  const size_t es = dtype_size(dtype);
  const size_t qbytes = (size_t)B * Lq * heads * head_dim * es;
  const size_t kbytes = (size_t)B * Lk * heads * head_dim * es;
  const char *oc = static_cast<const char *>(o);
  auto overlap = [&](const void *p, size_t n) {
    const char *c = static_cast<const char *>(p);
    return p && c < oc + qbytes && oc < c + n;
  };
  if (overlap(q, qbytes) || overlap(k, kbytes) || overlap(v, kbytes)) return set_error(WAN_EINVAL, "o aliases q, k or v");
  cudaStream_t s = (cudaStream_t)stream;
  const int D = heads * head_dim;
  int rc;
  if (grid) {
    const int F = grid[0], H = grid[1], W = grid[2];
    if (q == k) return set_error(WAN_EINVAL, "q and k must be distinct buffers when grid is given");
    if (F < 1 || H < 1 || W < 1 || (long long)F * H * W != Lq || Lq != Lk)
      return set_error(WAN_EINVAL, "grid %dx%dx%d does not match Lq=%d Lk=%d", F, H, W, Lq, Lk);
    const int gmax = F > H ? (F > W ? F : W) : (H > W ? H : W);
    if (!rope || rope_max_pos < gmax) return set_error(WAN_EINVAL, "rope table missing or too short");
    if (!aligned16(rope)) return set_error(WAN_EALIGN, "rope not 16-byte aligned");
    if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, s, launch_rope_only(q, dtype, B * Lq, D, D, head_dim, rope, rope_max_pos, F, H, W, s)))) return rc;
    if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, s, launch_rope_only(k, dtype, B * Lk, D, D, head_dim, rope, rope_max_pos, F, H, W, s)))) return rc;
  }
  AttnArgs a = {};
  a.B = B; a.heads = heads; a.Lq = Lq; a.Lk = Lk; a.d = head_dim;
  a.q = q; a.ldq = D; a.k = k; a.ldk = D; a.v = v; a.ldv = D; a.o = o; a.ldo = D;
  a.k_lens = k_lens; a.scale = scale != 0.f ? scale : 1.0f / sqrtf((float)head_dim);
  return run_attention(a, dtype, s, WAN_K_ATTN_TC);
}

int wan_euler_cfg_step(float *x, const void *v_cond, const void *v_uncond, int v_dtype, size_t n,
                       float guide_scale, float sigma, float sigma_next, wan_stream_t stream) {
  g_msg[0] = 0;
  if (n == 0) return WAN_OK;
  if (!x || !v_cond) return set_error(WAN_EINVAL, "NULL tensor");
  if (v_dtype != WAN_F32 && v_dtype != WAN_BF16) return set_error(WAN_EUNSUPPORTED, "v_dtype %d", v_dtype);
  if (!aligned16(x) || !aligned16(v_cond) || (v_uncond && !aligned16(v_uncond)))
    return set_error(WAN_EALIGN, "pointer not 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  return WAN_PROF(WAN_K_EULER, s, launch_euler_cfg(x, v_cond, v_uncond, v_dtype, n, guide_scale,
                                                    sigma_next - sigma, s));
}

int wan_debug_bounds(void) { return kDebugBounds ? 1 : 0; }

int wan_device_status(wan_stream_t stream) {
  g_msg[0] = 0;
  WAN_TRY_CUDA(cudaStreamSynchronize((cudaStream_t)stream), "stream synchronize");
  int *p = watchdog_ptr();
  if (!p) return set_error(WAN_ECUDA, "watchdog symbol unavailable");
  int v = 0;
  WAN_TRY_CUDA(cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost), "read watchdog");
  if (v != 0) {
    const int zero = 0;
    WAN_TRY_CUDA(cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice), "clear watchdog");
    if (v >= WAN_DBG_CODE_BASE)
      return set_error(WAN_EBOUNDS, "debug bounds check: a store fell outside its buffer (site %d)",
                       v - WAN_DBG_CODE_BASE);
    return set_error(WAN_ETIMEOUT, "a kernel gave up a bounded wait (code %d)", v);
  }
  return WAN_OK;
}

}  // extern "C"

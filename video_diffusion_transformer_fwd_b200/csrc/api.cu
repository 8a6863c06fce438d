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

static WsLayout layout_of(const wan_dims *d, int B) {
  WsLayout w;
  const size_t es = dtype_size(d->dtype);
  const size_t BL = (size_t)B * d->F * d->H * d->W, D = d->dim, T = d->text_len, Fh = d->ffn_dim;
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
      d->dtype == WAN_FP8_ATTN && B > 0 ? attention_8bit_ws_bytes(B, d->heads, d->F * d->H * d->W, d->F * d->H * d->W) : 0,
  };
  size_t o = 0;
  for (int i = 0; i < WAN_WS_COUNT; ++i) {
    w.off[i] = o;
    o += align256(sz[i]);
  }
  w.total = o;
  return w;
}

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
  if (!w) return set_error(WAN_EINVAL, "weights is NULL");
  const wan_dims &d = *dims;
  const int L = d.F * d.H * d.W, D = d.dim, T = d.text_len, Fh = d.ffn_dim, hd = D / d.heads;
  const int dt = d.dtype;
  const size_t es = dtype_size(dt);
  cudaStream_t s = (cudaStream_t)stream;

  const void *ptrs[] = {x, e0, rope, workspace, w->modulation, w->wq, w->bq, w->wk, w->bk, w->wv,
                        w->bv, w->wo, w->bo, w->gq, w->gk, w->g3, w->b3, w->cwq, w->cbq, w->cwk,
                        w->cbk, w->cwv, w->cbv, w->cwo, w->cbo, w->cgq, w->cgk, w->w1, w->b1,
                        w->w2, w->b2};
  for (size_t i = 0; i < sizeof(ptrs) / sizeof(ptrs[0]); ++i) {
    if (!ptrs[i]) return set_error(WAN_EINVAL, "pointer argument #%zu is NULL", i);
    if (!aligned16(ptrs[i])) return set_error(WAN_EALIGN, "pointer argument #%zu not 16-byte aligned", i);
  }
  if (is_fp8(dt)) {
    if (!w->w_scales) return set_error(WAN_EINVAL, "WAN_FP8 needs w_scales");
    if (!aligned16(w->w_scales)) return set_error(WAN_EALIGN, "w_scales not 16-byte aligned");
  }
  if (T > 0 && !ctx) return set_error(WAN_EINVAL, "ctx is NULL");
  if (ctx && !aligned16(ctx)) return set_error(WAN_EALIGN, "ctx not 16-byte aligned");
  if (ctx_lens && !aligned16(ctx_lens)) return set_error(WAN_EALIGN, "ctx_lens not 16-byte aligned");
  const int gmax = d.F > d.H ? (d.F > d.W ? d.F : d.W) : (d.H > d.W ? d.H : d.W);
  if (rope_max_pos < gmax) return set_error(WAN_EINVAL, "rope table has %d rows, grid needs %d", rope_max_pos, gmax);
  const WsLayout lay = layout_of(dims, B);
  if (ws_bytes < lay.total) return set_error(WAN_EINVAL, "workspace %zu bytes < %zu needed", ws_bytes, lay.total);

  char *ws = static_cast<char *>(workspace);
  void *act = ws + lay.off[WAN_WS_ACT];
  char *qkv = ws + lay.off[WAN_WS_QKV];
  void *o = ws + lay.off[WAN_WS_O];
  void *qc = ws + lay.off[WAN_WS_QC];
  char *kvc = ws + lay.off[WAN_WS_KVC];
  void *oc = ws + lay.off[WAN_WS_OC];
  void *hbuf = ws + lay.off[WAN_WS_H];
  float *mod = reinterpret_cast<float *>(ws + lay.off[WAN_WS_MOD]);
  const int BL = B * L;

  // m = modulation + e0  (shift, scale, gate, shift2, scale2, gate2)
  const ModSrc ms{d.e0_per_token != 0, e0, mod, w->modulation, L, D};
  if (!ms.ptok && (rc = WAN_PROF(WAN_K_MISC, s, launch_mod_combine(w->modulation, e0, mod, B, D, s)))) return rc;
  if (is_fp8(dt)) return block_forward_fp8(d, B, x, ctx, ctx_lens, w, rope, ws, lay, ms, s);

  // ---- self-attention branch: x += m2 * Wo . Attn(RoPE(RMSNorm(q,k)), v)
  // bf16 tensor-core path: the QKV GEMM epilogue accumulates each row's sum of
  // squares of q and k, writes gamma * RoPE(y); the attention applies q's RMS
  // factor in its logit scale and a row pass applies k's. Otherwise: plain
  // GEMM, then an RMSNorm + RoPE pass over q and k.
  float *stats = reinterpret_cast<float *>(ws + lay.off[WAN_WS_STATS]);
  GemmArgs gqkv = {};
  gqkv.M = BL; gqkv.N = 3 * D; gqkv.K = D; gqkv.A = act; gqkv.lda = D;
  gqkv.Bseg[0] = w->wq; gqkv.Bseg[1] = w->wk; gqkv.Bseg[2] = w->wv;
  gqkv.bias[0] = w->bq; gqkv.bias[1] = w->bk; gqkv.bias[2] = w->bv;
  gqkv.segN = D; gqkv.nseg = 3; gqkv.C = qkv; gqkv.ldc = 3 * D;
  gqkv.epi = EPI_QKNORM;
  gqkv.gamma[0] = w->gq; gqkv.gamma[1] = w->gk; gqkv.gamma[2] = nullptr;
  const int parts = D >= 256 ? D / 256 : 1;          // partial sums per row (one per 256-column tile)
  const int sstride = 4 * parts;                      // q | k | cross q | cross k partials of a row
  gqkv.ss = stats; gqkv.ss_stride = sstride; gqkv.ss_col[0] = 0; gqkv.ss_col[1] = 1; gqkv.ss_col[2] = -1;
  gqkv.rope = rope; gqkv.rope_mask = 3; gqkv.F = d.F; gqkv.H = d.H; gqkv.W = d.W; gqkv.head_dim = hd;
  AttnArgs aself = {};
  aself.B = B; aself.heads = d.heads; aself.Lq = L; aself.Lk = L; aself.d = hd;
  aself.q = qkv; aself.ldq = 3 * D; aself.k = qkv + D * es; aself.ldk = 3 * D; aself.v = qkv + 2 * D * es; aself.ldv = 3 * D;
  aself.o = o; aself.ldo = D; aself.k_lens = nullptr; aself.scale = 1.0f / sqrtf((float)hd);
  const bool fused = dt == WAN_BF16;
  if (fused && !(gemm_tc_supported(gqkv) && attention_tc_supported(aself)))
    return set_error(WAN_EUNSUPPORTED, "bf16 block: the QKV GEMM or the self-attention is outside the "
                                       "tensor-core kernels' rules (dim %% 256 == 0, head_dim 128)");

  if ((rc = WAN_PROF(WAN_K_LAYERNORM, s, launch_layernorm_mod(x, act, dt, BL, D, ln_of(ms, 0, 1), nullptr, nullptr, d.eps, s)))) return rc;
  if (fused) {
    if ((rc = run_gemm(gqkv, dt, s))) return rc;
    if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, s, launch_scale_rows(qkv + D * es, BL, 3 * D, D, stats + parts, sstride, parts, d.eps, s)))) return rc;
    aself.q_ss = stats; aself.q_ss_stride = sstride; aself.q_ss_parts = parts; aself.q_ss_n = (float)D; aself.q_ss_eps = d.eps;
  } else {
    gqkv.epi = EPI_STORE;
    if ((rc = run_gemm(gqkv, dt, s))) return rc;
    if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, s, launch_rmsnorm_rope(qkv, dt, BL, 3 * D, D, hd, w->gq, d.eps, rope, rope_max_pos, d.F, d.H, d.W, s)))) return rc;
    if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, s, launch_rmsnorm_rope(qkv + D * es, dt, BL, 3 * D, D, hd, w->gk, d.eps, rope, rope_max_pos, d.F, d.H, d.W, s)))) return rc;
  }
  if ((rc = run_attention(aself, dt, s, WAN_K_ATTN_SELF))) return rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = D; g.A = o; g.lda = D;
    g.Bseg[0] = w->wo; g.bias[0] = w->bo; g.segN = D; g.nseg = 1;
    g.epi = EPI_RESID; g.X = x; g.ldx = D;
    gate_of(ms, g, 2);
    if ((rc = run_gemm(g, dt, s))) return rc;
  }

  // ---- cross-attention branch (ungated): x += Wco . Attn(q(norm3 x), k(ctx), v(ctx))
  if ((rc = WAN_PROF(WAN_K_LAYERNORM, s, launch_layernorm_mod(x, act, dt, BL, D, LnMod{}, w->g3, w->b3, d.eps, s)))) return rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = D; g.A = act; g.lda = D;
    g.Bseg[0] = w->cwq; g.bias[0] = w->cbq; g.segN = D; g.nseg = 1;
    g.C = qc; g.ldc = D;
    g.epi = fused ? EPI_QKNORM : EPI_STORE;
    g.gamma[0] = w->cgq; g.ss = stats; g.ss_stride = sstride; g.ss_col[0] = 2; g.ss_col[1] = g.ss_col[2] = -1;
    if ((rc = run_gemm(g, dt, s))) return rc;
  }
  if (!fused && (rc = WAN_PROF(WAN_K_QKNORM_ROPE, s, launch_rmsnorm_rope(qc, dt, BL, D, D, hd, w->cgq, d.eps, nullptr, 0, 1, 1, 1, s)))) return rc;
  if (T > 0) {
    GemmArgs g = {};
    g.M = B * T; g.N = 2 * D; g.K = D; g.A = ctx; g.lda = D;
    g.Bseg[0] = w->cwk; g.Bseg[1] = w->cwv; g.bias[0] = w->cbk; g.bias[1] = w->cbv;
    g.segN = D; g.nseg = 2; g.C = kvc; g.ldc = 2 * D;
    g.epi = fused ? EPI_QKNORM : EPI_STORE;
    g.gamma[0] = w->cgk; g.gamma[1] = nullptr; g.ss = stats; g.ss_stride = sstride;
    g.ss_col[0] = 3; g.ss_col[1] = -1; g.ss_col[2] = -1;
    if ((rc = run_gemm(g, dt, s))) return rc;
    if (fused) {
      if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, s, launch_scale_rows(kvc, B * T, 2 * D, D, stats + 3 * parts, sstride, parts, d.eps, s)))) return rc;
    } else if ((rc = WAN_PROF(WAN_K_QKNORM_ROPE, s, launch_rmsnorm_rope(kvc, dt, B * T, 2 * D, D, hd, w->cgk, d.eps, nullptr, 0, 1, 1, 1, s)))) {
      return rc;
    }
  }
  {
    AttnArgs a = {};
    a.B = B; a.heads = d.heads; a.Lq = L; a.Lk = T; a.d = hd;
    a.q = qc; a.ldq = D; a.k = kvc; a.ldk = 2 * D; a.v = kvc + D * es; a.ldv = 2 * D;
    a.o = oc; a.ldo = D; a.k_lens = ctx_lens; a.scale = 1.0f / sqrtf((float)hd);
    if (fused) {
      a.q_ss = stats + 2 * parts; a.q_ss_stride = sstride; a.q_ss_parts = parts;
      a.q_ss_n = (float)D; a.q_ss_eps = d.eps;
    }
    if ((rc = run_attention(a, dt, s, WAN_K_ATTN_CROSS))) return rc;
  }
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = D; g.A = oc; g.lda = D;
    g.Bseg[0] = w->cwo; g.bias[0] = w->cbo; g.segN = D; g.nseg = 1;
    g.epi = EPI_RESID; g.X = x; g.ldx = D; g.gate = nullptr; g.rows_per_gate = L;
    if ((rc = run_gemm(g, dt, s))) return rc;
  }

  // ---- FFN branch: x += m5 * W2 . gelu_tanh(W1 . (LN(x)(1 + m4) + m3))
  if ((rc = WAN_PROF(WAN_K_LAYERNORM, s, launch_layernorm_mod(x, act, dt, BL, D, ln_of(ms, 3, 4), nullptr, nullptr, d.eps, s)))) return rc;
  {
    GemmArgs g = {};
    g.M = BL; g.N = Fh; g.K = D; g.A = act; g.lda = D;
    g.Bseg[0] = w->w1; g.bias[0] = w->b1; g.segN = Fh; g.nseg = 1;
    g.epi = EPI_GELU; g.C = hbuf; g.ldc = Fh;
    if ((rc = run_gemm(g, dt, s))) return rc;
  }
  {
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = Fh; g.A = hbuf; g.lda = Fh;
    g.Bseg[0] = w->w2; g.bias[0] = w->b2; g.segN = D; g.nseg = 1;
    g.epi = EPI_RESID; g.X = x; g.ldx = D;
    gate_of(ms, g, 5);
    if ((rc = run_gemm(g, dt, s))) return rc;
  }
  return WAN_OK;
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
    return set_error(WAN_ETIMEOUT, "a kernel gave up a bounded wait (code %d)", v);
  }
  return WAN_OK;
}

}  // extern "C"

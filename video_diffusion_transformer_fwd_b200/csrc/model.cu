// Whole-model forward on latents: patch embedding, time and text embeddings,
// the block stack, head and unpatchify ("Wan2.2 code walkthrough"
// (newtid.com): WanModel structure, forward and time-projection snippets;
// "diffusers WanPipeline walkthrough" (huan-yin.github.io): "3D Patchify",
// "Unpatchify"). The GEMMs run through the same tensor-core / CUDA-core
// kernels as the block; the small layout kernels live here.
#include "common.cuh"

#include <math.h>

namespace wan {
namespace {

// latent [B, C, F, H, W] (fp32) -> tokens [B * L, C * 4], token (f, h, w) of
// the (F, H/2, W/2) grid, feature c * 4 + kh * 2 + kw (the Conv3d weight's
// flattened order, kt = 0)
template <typename T>
__global__ void patchify_kernel(const float *__restrict__ lat, T *__restrict__ out, int B, int C, int F,
                                int H, int W) {
  const int Hp = H / 2, Wp = W / 2, L = F * Hp * Wp, nf = C * 4;
  const size_t total = (size_t)B * L * nf;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int feat = (int)(i % nf);
    const size_t row = i / nf;
    const int b = (int)(row / L), tok = (int)(row % L);
    const int c = feat >> 2, kh = (feat >> 1) & 1, kw = feat & 1;
    const int f = tok / (Hp * Wp), hp = (tok / Wp) % Hp, wp = tok % Wp;
    const float v = lat[(((size_t)b * C + c) * F + f) * (size_t)H * W + (size_t)(2 * hp + kh) * W + 2 * wp + kw];
    ElemIO<T>::store(out + i, v);
  }
}

// head output [B * L, C * 4], feature (kh * 2 + kw) * C + c -> [B, C, F, H, W]
template <typename T>
__global__ void unpatchify_kernel(const T *__restrict__ y, float *__restrict__ out, int B, int C, int F, int H,
                                  int W) {
  const int Hp = H / 2, Wp = W / 2;
  const size_t total = (size_t)B * C * F * H * W;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int x = (int)(i % W);
    const int yy = (int)((i / W) % H);
    const int f = (int)((i / ((size_t)W * H)) % F);
    const int c = (int)((i / ((size_t)W * H * F)) % C);
    const int b = (int)(i / ((size_t)W * H * F * C));
    const int hp = yy >> 1, kh = yy & 1, wp = x >> 1, kw = x & 1;
    const size_t row = (size_t)b * F * Hp * Wp + ((size_t)f * Hp + hp) * Wp + wp;
    out[i] = ElemIO<T>::load(y + row * (4 * C) + (kh * 2 + kw) * C + c);
  }
}

// s[b] = [cos(t_b w_j), sin(t_b w_j)], w_j = 10000^(-j / half), j < half (fp64 angles)
__global__ void sinusoid_kernel(const float *__restrict__ t, float *__restrict__ s, int B, int fd) {
  const int half = fd / 2;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * half) return;
  const int b = i / half, j = i % half;
  const double a = (double)t[b] * pow(10000.0, -(double)j / half);
  s[(size_t)b * fd + j] = (float)cos(a);
  s[(size_t)b * fd + half + j] = (float)sin(a);
}

__global__ void silu_kernel(const float *__restrict__ x, float *__restrict__ y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = x[i] / (1.0f + expf(-x[i]));
}

int grid_for(size_t n) {
  size_t g = (n + 255) / 256;
  if (g > 148 * 32) g = 148 * 32;
  return g < 1 ? 1 : (int)g;
}

enum { MW_X, MW_PATCH, MW_CTX, MW_TXT, MW_SIN, MW_H1, MW_E, MW_SE, MW_E0, MW_HOUT, MW_BLOCK, MW_COUNT };

struct ModelLayout {
  size_t off[MW_COUNT];
  size_t total;
  size_t block_bytes;
};

size_t a256(size_t v) { return (v + 255) & ~(size_t)255; }

wan_dims token_dims(const wan_model_dims &m) {
  wan_dims d;
  d.F = m.F; d.H = m.H / 2; d.W = m.W / 2;
  d.dim = m.dim; d.heads = m.heads; d.ffn_dim = m.ffn_dim; d.text_len = m.text_len;
  d.eps = m.eps; d.dtype = m.dtype; d.e0_per_token = m.t_per_token;
  return d;
}

int check_model(const wan_model_dims *m, int B) {
  if (!m) return set_error(WAN_EINVAL, "model dims is NULL");
  if (m->C_in < 1 || m->C_out < 1) return set_error(WAN_EINVAL, "channels %d / %d", m->C_in, m->C_out);
  if (m->H < 2 || m->W < 2 || m->H % 2 || m->W % 2) return set_error(WAN_EINVAL, "latent H, W must be even (%d x %d)", m->H, m->W);
  if (m->freq_dim < 8 || m->freq_dim % 8) return set_error(WAN_EINVAL, "freq_dim %d must be a positive multiple of 8", m->freq_dim);
  if (m->text_len > 0 && (m->text_dim < 64 || m->text_dim % 64))
    return set_error(WAN_EINVAL, "text_dim %d must be a positive multiple of 64", m->text_dim);
  if ((m->C_in * 4) % 8) return set_error(WAN_EUNSUPPORTED, "C_in * 4 must be a multiple of 8");
  if (m->t_per_token != 0 && m->t_per_token != 1) return set_error(WAN_EINVAL, "t_per_token must be 0 or 1");
  const wan_dims d = token_dims(*m);
  if (wan_block_workspace_bytes(&d, B) == 0 && B > 0) return WAN_EINVAL;   // message set by the block check
  return WAN_OK;
}

ModelLayout model_layout(const wan_model_dims &m, int B) {
  ModelLayout l;
  const size_t es = dtype_size(m.dtype);
  const size_t L = (size_t)m.F * (m.H / 2) * (m.W / 2), BL = (size_t)B * L, D = m.dim;
  const size_t BT = (size_t)B * m.text_len;
  const size_t NT = m.t_per_token ? BL : (size_t)B;     // timesteps
  const wan_dims d = token_dims(m);
  l.block_bytes = wan_block_workspace_bytes(&d, B);
  const size_t sz[MW_COUNT] = {
      BL * D * 4,                      // X (fp32 token stream)
      BL * m.C_in * 4 * es,            // PATCH
      BT * D * es,                     // CTX
      BT * D * es,                     // TXT (text MLP hidden)
      NT * m.freq_dim * 4,             // SIN
      NT * D * 4,                      // H1
      NT * D * 4,                      // E
      NT * D * 4,                      // SE
      NT * 6 * D * 4,                  // E0
      BL * m.C_out * 4 * es,           // HOUT
      l.block_bytes,                   // BLOCK (its ACT buffer also holds the head's LN output)
  };
  size_t o = 0;
  for (int i = 0; i < MW_COUNT; ++i) {
    l.off[i] = o;
    o += a256(sz[i]);
  }
  l.total = o;
  return l;
}

// Kernel choice for the model's own GEMMs, by shape and dtype, never as a
// silent fallback: a few rows (the time MLP at M = B) stream the weight once
// in the small-M kernel; fp32 runs the exact CUDA-core GEMM; bf16 runs the
// tensor-core GEMM, except the patch embedding when 4 * C_in is not a
// multiple of 64 (the I2V input's 36 channels: K = 144), which is documented
// to run on the CUDA-core GEMM (`small_k_on_cuda_cores`). Any other bf16 shape
// outside the tensor-core rules is refused.
int gemm_any(const GemmArgs &g, int dtype, cudaStream_t s, bool small_k_on_cuda_cores = false) {
  if (gemm_smallm_supported(g)) return WAN_PROF(WAN_K_MODEL, s, gemm_smallm(g, dtype, s));
  if (dtype == WAN_F32) return WAN_PROF(WAN_K_GEMM_SIMT, s, gemm_simt(g, dtype, s));
  if (gemm_tc_supported(g)) return WAN_PROF(WAN_K_GEMM_TC, s, gemm_tc(g, s));
  if (small_k_on_cuda_cores && g.K % 64) return WAN_PROF(WAN_K_GEMM_SIMT, s, gemm_simt(g, dtype, s));
  return set_error(WAN_EUNSUPPORTED, "model bf16 GEMM M=%d N=%d K=%d outside the tensor-core kernel's rules "
                                     "(K %% 64 == 0, N %% 32 == 0)", g.M, g.N, g.K);
}

}  // namespace
}  // namespace wan

using namespace wan;

extern "C" {

size_t wan_model_workspace_bytes(const wan_model_dims *dims, int B) {
  if (B < 0 || check_model(dims, B) != WAN_OK) return 0;
  return model_layout(*dims, B).total;
}

int wan_model_forward(const wan_model_dims *dims, int B, const float *latent, const float *t,
                      const void *text, const int *ctx_lens, const wan_model_weights *w,
                      const wan_block_weights *blocks, int num_blocks, const float *rope,
                      int rope_max_pos, float *out, void *workspace, size_t ws_bytes,
                      wan_stream_t stream) {
  int rc = check_model(dims, B);
  if (rc) return rc;
  if (B < 0) return set_error(WAN_EINVAL, "B=%d < 0", B);
  if (B == 0) return WAN_OK;
  if (!w || (num_blocks > 0 && !blocks) || num_blocks < 0) return set_error(WAN_EINVAL, "weights");
  const wan_model_dims &m = *dims;
  const void *ptrs[] = {latent, t, out, workspace, rope, w->patch_w, w->patch_b, w->time_w1, w->time_b1,
                        w->time_w2, w->time_b2, w->proj_w, w->proj_b, w->head_mod, w->head_w, w->head_b};
  for (size_t i = 0; i < sizeof(ptrs) / sizeof(ptrs[0]); ++i) {
    if (!ptrs[i]) return set_error(WAN_EINVAL, "model pointer argument #%zu is NULL", i);
    if (!aligned16(ptrs[i])) return set_error(WAN_EALIGN, "model pointer argument #%zu not 16-byte aligned", i);
  }
  if (m.text_len > 0) {
    const void *tp[] = {text, w->text_w1, w->text_b1, w->text_w2, w->text_b2};
    for (const void *p : tp) {
      if (!p) return set_error(WAN_EINVAL, "text input or text weights NULL");
      if (!aligned16(p)) return set_error(WAN_EALIGN, "text pointer not 16-byte aligned");
    }
  }
  const ModelLayout lay = model_layout(m, B);
  if (ws_bytes < lay.total) return set_error(WAN_EINVAL, "workspace %zu bytes < %zu needed", ws_bytes, lay.total);

  cudaStream_t s = (cudaStream_t)stream;
  const int dt = (m.dtype == WAN_FP8 || m.dtype == WAN_FP8_ATTN) ? WAN_BF16 : m.dtype;    // embeddings and head stay bf16 in FP8 mode
  const size_t es = dtype_size(dt);
  const int L = m.F * (m.H / 2) * (m.W / 2), BL = B * L, D = m.dim, T = m.text_len;
  char *ws = static_cast<char *>(workspace);
  float *X = reinterpret_cast<float *>(ws + lay.off[MW_X]);
  void *patch = ws + lay.off[MW_PATCH];
  void *ctx = ws + lay.off[MW_CTX];
  void *txt = ws + lay.off[MW_TXT];
  float *sin_ = reinterpret_cast<float *>(ws + lay.off[MW_SIN]);
  float *h1 = reinterpret_cast<float *>(ws + lay.off[MW_H1]);
  float *e = reinterpret_cast<float *>(ws + lay.off[MW_E]);
  float *se = reinterpret_cast<float *>(ws + lay.off[MW_SE]);
  float *e0 = reinterpret_cast<float *>(ws + lay.off[MW_E0]);
  void *hout = ws + lay.off[MW_HOUT];
  char *bws = ws + lay.off[MW_BLOCK];
  const wan_dims tok = token_dims(m);
  void *act = bws + wan_block_workspace_offset(&tok, B, WAN_WS_ACT);

  // patch embedding: x = patches W^T + b, stored as the fp32 token stream
  {
    const size_t n = (size_t)BL * m.C_in * 4;
    if (dt == WAN_BF16)
      WAN_PROF(WAN_K_MODEL, s, (patchify_kernel<__nv_bfloat16><<<grid_for(n), 256, 0, s>>>(
          latent, (__nv_bfloat16 *)patch, B, m.C_in, m.F, m.H, m.W), 0));
    else
      WAN_PROF(WAN_K_MODEL, s, (patchify_kernel<float><<<grid_for(n), 256, 0, s>>>(
          latent, (float *)patch, B, m.C_in, m.F, m.H, m.W), 0));
    WAN_CHECK_LAUNCH("patchify");
    GemmArgs g = {};
    g.M = BL; g.N = D; g.K = m.C_in * 4; g.A = patch; g.lda = m.C_in * 4;
    g.Bseg[0] = w->patch_w; g.bias[0] = w->patch_b; g.segN = D; g.nseg = 1;
    g.epi = EPI_RESID; g.X = X; g.ldx = D; g.gate = nullptr; g.rows_per_gate = L;
    g.x_store = 1;
    if ((rc = gemm_any(g, dt, s, /*small_k_on_cuda_cores=*/true))) return rc;
  }
  // time embedding (fp32): e = W2 SiLU(W1 sinusoid(t) + b1) + b2; e0 = Wp SiLU(e) + bp,
  // for B timesteps or, per token, B * L
  const int NT = m.t_per_token ? BL : B;
  {
    const int half = m.freq_dim / 2;
    WAN_PROF(WAN_K_MODEL, s, (sinusoid_kernel<<<(NT * half + 255) / 256, 256, 0, s>>>(t, sin_, NT, m.freq_dim), 0));
    WAN_CHECK_LAUNCH("sinusoid");
    GemmArgs g = {};
    g.M = NT; g.N = D; g.K = m.freq_dim; g.A = sin_; g.lda = m.freq_dim;
    g.Bseg[0] = w->time_w1; g.bias[0] = w->time_b1; g.segN = D; g.nseg = 1; g.epi = EPI_SILU; g.C = h1; g.ldc = D;
    if ((rc = gemm_any(g, WAN_F32, s))) return rc;
    g.K = D; g.A = h1; g.lda = D; g.Bseg[0] = w->time_w2; g.bias[0] = w->time_b2; g.epi = EPI_STORE; g.C = e;
    if ((rc = gemm_any(g, WAN_F32, s))) return rc;
    WAN_PROF(WAN_K_MODEL, s, (silu_kernel<<<(NT * D + 255) / 256, 256, 0, s>>>(e, se, NT * D), 0));
    WAN_CHECK_LAUNCH("silu");
    g.A = se; g.N = 6 * D; g.segN = 6 * D; g.Bseg[0] = w->proj_w; g.bias[0] = w->proj_b; g.C = e0; g.ldc = 6 * D;
    if ((rc = gemm_any(g, WAN_F32, s))) return rc;
  }
  // text embedding: ctx = W2 GELU_tanh(W1 text + b1) + b2
  if (T > 0) {
    GemmArgs g = {};
    g.M = B * T; g.N = D; g.K = m.text_dim; g.A = text; g.lda = m.text_dim;
    g.Bseg[0] = w->text_w1; g.bias[0] = w->text_b1; g.segN = D; g.nseg = 1; g.epi = EPI_GELU; g.C = txt; g.ldc = D;
    if ((rc = gemm_any(g, dt, s))) return rc;
    g.K = D; g.A = txt; g.lda = D; g.Bseg[0] = w->text_w2; g.bias[0] = w->text_b2; g.epi = EPI_STORE; g.C = ctx;
    if ((rc = gemm_any(g, dt, s))) return rc;
  }
  // the block stack
  for (int i = 0; i < num_blocks; ++i)
    if ((rc = wan_block_forward(&tok, B, X, T > 0 ? ctx : nullptr, ctx_lens, e0, &blocks[i], rope,
                                rope_max_pos, bws, lay.block_bytes, stream)))
      return rc;
  // head: LN(x) (1 + m1) + m0 with (m0, m1) = head_mod + e (read in place), then Linear(dim -> C_out * 4)
  {
    const LnMod hm{e, m.t_per_token ? 1 : L, (size_t)D, 0, 0, w->head_mod, 0, D};
    if ((rc = WAN_PROF(WAN_K_LAYERNORM, s, launch_layernorm_mod(X, act, dt, BL, D, hm, nullptr, nullptr, m.eps, s))))
      return rc;
    GemmArgs g = {};
    g.M = BL; g.N = m.C_out * 4; g.K = D; g.A = act; g.lda = D;
    g.Bseg[0] = w->head_w; g.bias[0] = w->head_b; g.segN = g.N; g.nseg = 1; g.epi = EPI_STORE;
    g.C = hout; g.ldc = g.N;
    if ((rc = gemm_any(g, dt, s))) return rc;
  }
  // unpatchify
  {
    const size_t n = (size_t)B * m.C_out * m.F * m.H * m.W;
    if (dt == WAN_BF16)
      WAN_PROF(WAN_K_MODEL, s, (unpatchify_kernel<__nv_bfloat16><<<grid_for(n), 256, 0, s>>>(
          (const __nv_bfloat16 *)hout, out, B, m.C_out, m.F, m.H, m.W), 0));
    else
      WAN_PROF(WAN_K_MODEL, s, (unpatchify_kernel<float><<<grid_for(n), 256, 0, s>>>(
          (const float *)hout, out, B, m.C_out, m.F, m.H, m.W), 0));
    WAN_CHECK_LAUNCH("unpatchify");
  }
  (void)es;
  return WAN_OK;
}

}  // extern "C"

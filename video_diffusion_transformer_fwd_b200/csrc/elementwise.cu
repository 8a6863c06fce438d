// Bandwidth-bound kernels of the block and the step: AdaLN-modulated
// LayerNorm, q/k RMSNorm + 3D RoPE, the RoPE table and the CFG-Euler update.
//
// Sources: "Wan2.2 code walkthrough" (newtid.com) -- WanAttentionBlock
// core-logic snippet (fp32 LayerNorm, modulation chunks), 3D RoPE snippet
// (t/h/w split of the complex pairs, interleaved pairs), sampling-loop
// snippet (classifier-free guidance); "Wan paper deep dive"
// (charles2530.github.io), "Video DiT and Flow Matching" (Euler in sigma).
#include "common.cuh"

#include <math.h>

namespace wan {

// ----------------------------------------------------------------------------
// m[b][c][:] = modulation[c][:] + e0[b][c][:]   (e = (modulation + e0).chunk(6))
// ----------------------------------------------------------------------------
__global__ void mod_combine_kernel(const float *__restrict__ modulation,
                                   const float *__restrict__ e0, float *__restrict__ mod,
                                   int B, int D) {
  const int n = 6 * D;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < B * n; i += gridDim.x * blockDim.x)
    mod[i] = modulation[i % n] + e0[i];
}

int launch_mod_combine(const float *modulation, const float *e0, float *mod, int B, int D,
                       cudaStream_t s) {
  const int total = B * 6 * D;
  const int blocks = (total + 255) / 256;
  mod_combine_kernel<<<blocks, 256, 0, s>>>(modulation, e0, mod, B, D);
  WAN_CHECK_LAUNCH("mod_combine");
  return WAN_OK;
}

// ----------------------------------------------------------------------------
// LayerNorm over D (population variance, eps inside the square root), then
// either the AdaLN modulation (1 + scale) * u + shift with chunks taken from
// m[b] (norm1 / norm2), or an affine g * u + beta (norm3). One CTA per row;
// the row stays in registers between the two passes (exact two-pass stats).
// ----------------------------------------------------------------------------
constexpr int LN_THREADS = 256;
constexpr int LN_MAXV = 8;          // float4 per thread: D <= 8192

template <typename OutT>
__global__ void __launch_bounds__(LN_THREADS)
layernorm_mod_kernel(const float *__restrict__ x, OutT *__restrict__ out, int D, int rows_per_b,
                     const float *__restrict__ mod, int shift_chunk, int scale_chunk,
                     const float *__restrict__ g, const float *__restrict__ beta, float eps) {
  __shared__ float red[32];
  const int row = blockIdx.x;
  const float *xr = x + (size_t)row * D;
  const int nv = D >> 2;
  float4 v[LN_MAXV];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < LN_MAXV; ++i) {
    const int c = threadIdx.x + i * LN_THREADS;
    if (c < nv) {
      v[i] = load4(xr + 4 * c);
      s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
    }
  }
  const float mean = block_sum(s, red) / (float)D;
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < LN_MAXV; ++i) {
    const int c = threadIdx.x + i * LN_THREADS;
    if (c < nv) {
      const float a = v[i].x - mean, b = v[i].y - mean, cc = v[i].z - mean, d = v[i].w - mean;
      ss += (a * a + b * b) + (cc * cc + d * d);
    }
  }
  const float var = block_sum(ss, red) / (float)D;
  const float rstd = 1.0f / sqrtf(var + eps);
  const float *mshift = nullptr, *mscale = nullptr;
  if (g == nullptr) {
    const int b = row / rows_per_b;
    mshift = mod + ((size_t)b * 6 + shift_chunk) * D;
    mscale = mod + ((size_t)b * 6 + scale_chunk) * D;
  }
  OutT *orow = out + (size_t)row * D;
#pragma unroll
  for (int i = 0; i < LN_MAXV; ++i) {
    const int c = threadIdx.x + i * LN_THREADS;
    if (c < nv) {
      float4 u = make_float4((v[i].x - mean) * rstd, (v[i].y - mean) * rstd,
                             (v[i].z - mean) * rstd, (v[i].w - mean) * rstd);
      float4 a, b;
      if (g == nullptr) {
        const float4 sc = load4(mscale + 4 * c), sh = load4(mshift + 4 * c);
        a = make_float4(1.f + sc.x, 1.f + sc.y, 1.f + sc.z, 1.f + sc.w);
        b = sh;
      } else {
        a = load4(g + 4 * c);
        b = load4(beta + 4 * c);
      }
      u.x = fmaf(u.x, a.x, b.x);
      u.y = fmaf(u.y, a.y, b.y);
      u.z = fmaf(u.z, a.z, b.z);
      u.w = fmaf(u.w, a.w, b.w);
      store4(orow + 4 * c, u);
    }
  }
}

int launch_layernorm_mod(const float *x, void *out, int dtype, int rows, int D, int rows_per_b,
                         const float *mod, int shift_chunk, int scale_chunk,
                         const float *g, const float *beta, float eps, cudaStream_t s) {
  if (D % 4 || D > 4 * LN_MAXV * LN_THREADS) return set_error(WAN_EUNSUPPORTED, "layernorm: D=%d", D);
  if (rows == 0) return WAN_OK;
  if (dtype == WAN_BF16)
    layernorm_mod_kernel<__nv_bfloat16><<<rows, LN_THREADS, 0, s>>>(
        x, (__nv_bfloat16 *)out, D, rows_per_b, mod, shift_chunk, scale_chunk, g, beta, eps);
  else
    layernorm_mod_kernel<float><<<rows, LN_THREADS, 0, s>>>(
        x, (float *)out, D, rows_per_b, mod, shift_chunk, scale_chunk, g, beta, eps);
  WAN_CHECK_LAUNCH("layernorm_mod");
  return WAN_OK;
}

// ----------------------------------------------------------------------------
// 3D RoPE helpers. Pair j of a head (0 <= j < d/2) belongs to the t axis for
// j < pt, to h for pt <= j < pt + ph, to w otherwise (pt = c - 2(c/3),
// ph = pw = c/3, c = d/2). Token r of a sequence sits at t = r/(H W),
// h = (r/W) % H, w = r % W. table[pos][j] = (cos, sin)(pos * omega_j).
// ----------------------------------------------------------------------------
__device__ __forceinline__ float2 rope_cs(const float *__restrict__ rope, int half, int j,
                                          int pt, int ph, int tpos, int hpos, int wpos) {
  const int pos = j < pt ? tpos : (j < pt + ph ? hpos : wpos);
  return *reinterpret_cast<const float2 *>(rope + ((size_t)pos * half + j) * 2);
}

// In place on one row of q or k: optional RMSNorm over D with gain, then
// optional RoPE. One CTA per row, float4 chunks (two complex pairs each).
template <typename T, bool NORM, bool ROPE>
__global__ void __launch_bounds__(LN_THREADS)
rmsnorm_rope_kernel(T *__restrict__ p, int ld, int D, int head_dim,
                    const float *__restrict__ gain, float eps, const float *__restrict__ rope,
                    int L, int H, int W) {
  __shared__ float red[32];
  const int row = blockIdx.x;
  T *pr = p + (size_t)row * ld;
  const int nv = D >> 2;
  float4 v[LN_MAXV];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < LN_MAXV; ++i) {
    const int c = threadIdx.x + i * LN_THREADS;
    if (c < nv) {
      v[i] = load4(pr + 4 * c);
      ss += (v[i].x * v[i].x + v[i].y * v[i].y) + (v[i].z * v[i].z + v[i].w * v[i].w);
    }
  }
  float r = 1.f;
  if (NORM) r = 1.0f / sqrtf(block_sum(ss, red) / (float)D + eps);
  int tpos = 0, hpos = 0, wpos = 0, half = head_dim >> 1, c3 = half / 3, pt = half - 2 * c3;
  if (ROPE) {
    const int tok = row % L;
    tpos = tok / (H * W);
    hpos = (tok / W) % H;
    wpos = tok % W;
  }
#pragma unroll
  for (int i = 0; i < LN_MAXV; ++i) {
    const int c = threadIdx.x + i * LN_THREADS;
    if (c < nv) {
      float4 u = v[i];
      if (NORM) {
        const float4 g = load4(gain + 4 * c);
        u = make_float4(u.x * r * g.x, u.y * r * g.y, u.z * r * g.z, u.w * r * g.w);
      }
      if (ROPE) {
        const int j0 = ((4 * c) % head_dim) >> 1;        // first pair of this chunk
        const float2 a = rope_cs(rope, half, j0, pt, c3, tpos, hpos, wpos);
        const float2 b = rope_cs(rope, half, j0 + 1, pt, c3, tpos, hpos, wpos);
        u = make_float4(u.x * a.x - u.y * a.y, u.x * a.y + u.y * a.x,
                        u.z * b.x - u.w * b.y, u.z * b.y + u.w * b.x);
      }
      store4(pr + 4 * c, u);
    }
  }
}

template <bool NORM, bool ROPE>
static int launch_rr(void *p, int dtype, int rows, int ld, int D, int head_dim, const float *gain,
                     float eps, const float *rope, int L, int H, int W, cudaStream_t s) {
  if (dtype == WAN_BF16)
    rmsnorm_rope_kernel<__nv_bfloat16, NORM, ROPE><<<rows, LN_THREADS, 0, s>>>(
        (__nv_bfloat16 *)p, ld, D, head_dim, gain, eps, rope, L, H, W);
  else
    rmsnorm_rope_kernel<float, NORM, ROPE><<<rows, LN_THREADS, 0, s>>>(
        (float *)p, ld, D, head_dim, gain, eps, rope, L, H, W);
  WAN_CHECK_LAUNCH("rmsnorm_rope");
  return WAN_OK;
}

int launch_rmsnorm_rope(void *p, int dtype, int rows, int ld, int D, int head_dim,
                        const float *gain, float eps, const float *rope, int rope_max_pos,
                        int F, int H, int W, cudaStream_t s) {
  (void)rope_max_pos;
  if (D % 4 || D > 4 * LN_MAXV * LN_THREADS || head_dim % 4)
    return set_error(WAN_EUNSUPPORTED, "rmsnorm_rope: D=%d head_dim=%d", D, head_dim);
  if (rows == 0) return WAN_OK;
  if (rope) return launch_rr<true, true>(p, dtype, rows, ld, D, head_dim, gain, eps, rope, F * H * W, H, W, s);
  return launch_rr<true, false>(p, dtype, rows, ld, D, head_dim, gain, eps, nullptr, 1, 1, 1, s);
}

int launch_rope_only(void *p, int dtype, int rows, int ld, int D, int head_dim,
                     const float *rope, int rope_max_pos, int F, int H, int W, cudaStream_t s) {
  (void)rope_max_pos;
  if (D % 4 || D > 4 * LN_MAXV * LN_THREADS || head_dim % 4)
    return set_error(WAN_EUNSUPPORTED, "rope: D=%d head_dim=%d", D, head_dim);
  if (rows == 0) return WAN_OK;
  return launch_rr<false, true>(p, dtype, rows, ld, D, head_dim, nullptr, 0.f, rope, F * H * W, H, W, s);
}

// ----------------------------------------------------------------------------
// k rows of the tensor-core path: k[r] *= 1 / sqrt(ss[r] / D + eps) in place
// (the QKV epilogue wrote gamma * RoPE(y) and the row's sum of squares of y).
// One warp per row, 16-byte vectors.
// ----------------------------------------------------------------------------
__global__ void scale_rows_kernel(__nv_bfloat16 *__restrict__ p, int rows, int ld, int D,
                                  const float *__restrict__ ss, int ss_stride, int parts, float inv_d,
                                  float eps) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float part = lane < parts ? ss[(size_t)row * ss_stride + lane] : 0.f;
  const float r = rsqrtf(warp_sum(part) * inv_d + eps);
  uint4 *pr = reinterpret_cast<uint4 *>(p + (size_t)row * ld);
  for (int c = lane; c < D / 8; c += 32) {
    uint4 u = pr[c];
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
      float2 f = __bfloat1622float2(h);
      h = __floats2bfloat162_rn(f.x * r, f.y * r);
      w[e] = *reinterpret_cast<uint32_t *>(&h);
    }
    pr[c] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

int launch_scale_rows(void *p, int rows, int ld, int D, const float *ss, int ss_stride, int parts,
                      float eps, cudaStream_t s) {
  if (rows == 0) return WAN_OK;
  if (D % 8 || ld % 8 || parts < 1 || parts > 32) return set_error(WAN_EUNSUPPORTED, "scale_rows: D=%d", D);
  const int warps = 8;
  scale_rows_kernel<<<(rows + warps - 1) / warps, warps * 32, 0, s>>>(
      static_cast<__nv_bfloat16 *>(p), rows, ld, D, ss, ss_stride, parts, 1.0f / (float)D, eps);
  WAN_CHECK_LAUNCH("scale_rows");
  return WAN_OK;
}

// ----------------------------------------------------------------------------
// RoPE table: one thread per (pos, pair). Angle in fp64, stored as fp32.
// ----------------------------------------------------------------------------
__global__ void rope_table_kernel(int half, int max_pos, double theta, float *__restrict__ table) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= half * max_pos) return;
  const int pos = i / half, j = i % half;
  const int c3 = half / 3, pt = half - 2 * c3;
  int jl, pairs;
  if (j < pt) { jl = j; pairs = pt; }
  else if (j < pt + c3) { jl = j - pt; pairs = c3; }
  else { jl = j - pt - c3; pairs = c3; }
  const double omega = pow(theta, -(2.0 * jl) / (2.0 * pairs));
  const double ang = (double)pos * omega;
  table[2 * (size_t)i] = (float)cos(ang);
  table[2 * (size_t)i + 1] = (float)sin(ang);
}

int launch_rope_table(int head_dim, int max_pos, double theta, float *table, cudaStream_t s) {
  const int half = head_dim / 2;
  const int total = half * max_pos;
  rope_table_kernel<<<(total + 255) / 256, 256, 0, s>>>(half, max_pos, theta, table);
  WAN_CHECK_LAUNCH("rope_table");
  return WAN_OK;
}

// ----------------------------------------------------------------------------
// CFG + Euler: x += dt * (vu + s (vc - vu))   (vu == NULL: x += dt * vc)
// ----------------------------------------------------------------------------
template <typename VT, bool CFG>
__global__ void euler_cfg_kernel(float *__restrict__ x, const VT *__restrict__ vc,
                                 const VT *__restrict__ vu, size_t n, float scale, float dt) {
  const size_t nv = n >> 2;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nv; i += stride) {
    float4 xv = load4(x + 4 * i);
    const float4 c = load4(vc + 4 * i);
    float4 v = c;
    if (CFG) {
      const float4 u = load4(vu + 4 * i);
      v = make_float4(fmaf(scale, c.x - u.x, u.x), fmaf(scale, c.y - u.y, u.y),
                      fmaf(scale, c.z - u.z, u.z), fmaf(scale, c.w - u.w, u.w));
    }
    xv.x = fmaf(dt, v.x, xv.x);
    xv.y = fmaf(dt, v.y, xv.y);
    xv.z = fmaf(dt, v.z, xv.z);
    xv.w = fmaf(dt, v.w, xv.w);
    store4(x + 4 * i, xv);
  }
  // ragged tail (n % 4 elements)
  const size_t t = 4 * nv + blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (blockIdx.x * (size_t)blockDim.x + threadIdx.x < (n & 3)) {
    const float c = ElemIO<VT>::load(vc + t);
    float v = c;
    if (CFG) {
      const float u = ElemIO<VT>::load(vu + t);
      v = fmaf(scale, c - u, u);
    }
    x[t] = fmaf(dt, v, x[t]);
  }
}

template <typename VT>
static void euler_launch(float *x, const void *vc, const void *vu, size_t n, float scale, float dt,
                         cudaStream_t s) {
  const size_t nv = (n >> 2) > 0 ? (n >> 2) : 1;
  int blocks = (int)((nv + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (vu)
    euler_cfg_kernel<VT, true><<<blocks, 256, 0, s>>>(x, (const VT *)vc, (const VT *)vu, n, scale, dt);
  else
    euler_cfg_kernel<VT, false><<<blocks, 256, 0, s>>>(x, (const VT *)vc, nullptr, n, scale, dt);
}

int launch_euler_cfg(float *x, const void *vc, const void *vu, int vdt, size_t n, float scale,
                     float dt, cudaStream_t s) {
  if (n == 0) return WAN_OK;
  if (vdt == WAN_BF16) euler_launch<__nv_bfloat16>(x, vc, vu, n, scale, dt, s);
  else euler_launch<float>(x, vc, vu, n, scale, dt, s);
  WAN_CHECK_LAUNCH("euler_cfg");
  return WAN_OK;
}

}  // namespace wan

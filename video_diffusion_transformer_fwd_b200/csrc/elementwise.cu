// Bandwidth-bound kernels of the block and the step: AdaLN-modulated
// LayerNorm, q/k RMSNorm + 3D RoPE, the RoPE table and the CFG-Euler update.
//
// Sources: "Wan2.2 code walkthrough" (newtid.com) -- WanAttentionBlock
// core-logic snippet (fp32 LayerNorm, modulation chunks), 3D RoPE snippet
// (t/h/w split of the complex pairs, interleaved pairs), sampling-loop
// snippet (classifier-free guidance); "Wan paper deep dive"
// (charles2530.github.io), "Video DiT and Flow Matching" (Euler in sigma).
#include "common.cuh"

#include <cuda_fp8.h>
#include <math.h>

namespace wan {

int sm_count();   // SMs of the current device (tma_host.cu)

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
// e4m3 quantization ("Wan paper deep dive" (charles2530.github.io),
// inference-optimisation table, "FP8 GEMM"): a row's (or tensor's) scale is
// amax / 448 and an element's code is the e4m3 value nearest to
// x * (448 / amax), ties to even, clamped to +-448; both factors and the
// product are rounded to fp32 as formed. An all-zero row gets scale 0.
// ----------------------------------------------------------------------------
constexpr float E4M3_MAX = 448.f;

// four values -> four e4m3 bytes, the first in the lowest byte
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

__device__ __forceinline__ float e4m3_inv_scale(float amax) {
  return amax > 0.f ? __fdiv_rn(E4M3_MAX, amax) : 0.f;
}

__device__ __forceinline__ float absmax4(float4 v) {
  return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

__device__ __forceinline__ float block_max(float v, float *red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = (lane < nw) ? red[lane] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, o));
  return t;
}

__device__ __forceinline__ uint32_t quant4(float4 v, float inv) {
  return e4m3x4(__fmul_rn(v.x, inv), __fmul_rn(v.y, inv), __fmul_rn(v.z, inv), __fmul_rn(v.w, inv));
}

// One CTA per row of src (row stride ld elements): codes [rows, cols], scale [rows].
template <typename T>
__global__ void __launch_bounds__(256) quant_rows_kernel(const T *__restrict__ src, size_t ld, int cols,
                                                         uint8_t *__restrict__ q, float *__restrict__ scale) {
  __shared__ float red[32];
  const size_t row = blockIdx.x;
  const T *sr = src + row * ld;
  float amax = 0.f;
  for (int c = threadIdx.x * 4; c < cols; c += 4 * blockDim.x) amax = fmaxf(amax, absmax4(load4(sr + c)));
  amax = block_max(amax, red);
  const float inv = e4m3_inv_scale(amax);
  uint32_t *qr = reinterpret_cast<uint32_t *>(q + row * cols);
  for (int c = threadIdx.x * 4; c < cols; c += 4 * blockDim.x) qr[c >> 2] = quant4(load4(sr + c), inv);
  if (threadIdx.x == 0) scale[row] = __fdiv_rn(amax, E4M3_MAX);
}

// The same with the row held in registers (one read of the row from DRAM):
// bf16 rows of up to 8 * CH * 256 elements, cols % 8 == 0, 16-byte loads.
template <int CH>
__global__ void __launch_bounds__(256) quant_rows_reg_kernel(const __nv_bfloat16 *__restrict__ src, size_t ld,
                                                             int cols, uint8_t *__restrict__ q,
                                                             float *__restrict__ scale) {
  __shared__ float red[32];
  const size_t row = blockIdx.x;
  const __nv_bfloat16 *sr = src + row * ld;
  uint4 raw[CH];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < CH; ++i) {
    const int c = (threadIdx.x + i * 256) * 8;
    raw[i] = c < cols ? *reinterpret_cast<const uint4 *>(sr + c) : make_uint4(0, 0, 0, 0);
    const uint32_t w4[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w4[e] << 16)), fabsf(__uint_as_float(w4[e] & 0xFFFF0000u))));
  }
  amax = block_max(amax, red);
  const float inv = e4m3_inv_scale(amax);
  uint8_t *qr = q + row * cols;
#pragma unroll
  for (int i = 0; i < CH; ++i) {
    const int c = (threadIdx.x + i * 256) * 8;
    if (c < cols) {
      const uint32_t w4[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
      float f[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w4[e] << 16);
        f[2 * e + 1] = __uint_as_float(w4[e] & 0xFFFF0000u);
      }
      uint2 o;
      o.x = quant4(make_float4(f[0], f[1], f[2], f[3]), inv);
      o.y = quant4(make_float4(f[4], f[5], f[6], f[7]), inv);
      *reinterpret_cast<uint2 *>(qr + c) = o;
    }
  }
  if (threadIdx.x == 0) scale[row] = __fdiv_rn(amax, E4M3_MAX);
}

// Per-tensor: amax into the scale word (as ordered bits of a non-negative
// float), then the codes, then the word becomes amax / 448.
template <typename T>
__global__ void __launch_bounds__(256) amax_kernel(const T *__restrict__ src, size_t n4, unsigned *amax_bits) {
  __shared__ float red[32];
  float amax = 0.f;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x)
    amax = fmaxf(amax, absmax4(load4(src + 4 * i)));
  amax = block_max(amax, red);
  if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(amax));
}

template <typename T>
__global__ void __launch_bounds__(256) quant_tensor_kernel(const T *__restrict__ src, size_t n4,
                                                           const unsigned *__restrict__ amax_bits,
                                                           uint8_t *__restrict__ q) {
  const float inv = e4m3_inv_scale(__uint_as_float(*amax_bits));
  uint32_t *q4 = reinterpret_cast<uint32_t *>(q);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x)
    q4[i] = quant4(load4(src + 4 * i), inv);
}

__global__ void amax_to_scale_kernel(float *scale) { scale[0] = __fdiv_rn(scale[0], E4M3_MAX); }

int launch_quant_rows(const void *src, int dtype, size_t ld, int rows, int cols, uint8_t *q, float *scale,
                      cudaStream_t s) {
  if (cols % 4 || ld % 4) return set_error(WAN_EUNSUPPORTED, "quantize: cols and row stride must be multiples of 4");
  if (rows == 0 || cols == 0) return WAN_OK;
  const bool reg = dtype == WAN_BF16 && cols % 8 == 0 && ld % 8 == 0 &&
                   (reinterpret_cast<uintptr_t>(src) & 15u) == 0 && cols <= 8 * 8 * 256;
  if (reg) {
    const int ch = (cols + 2047) / 2048;         // 16-byte chunks per thread
    if (ch <= 1)
      quant_rows_reg_kernel<1><<<rows, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(src), ld, cols, q, scale);
    else if (ch <= 3)
      quant_rows_reg_kernel<3><<<rows, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(src), ld, cols, q, scale);
    else
      quant_rows_reg_kernel<8><<<rows, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(src), ld, cols, q, scale);
  } else if (dtype == WAN_F32)
    quant_rows_kernel<float><<<rows, 256, 0, s>>>(static_cast<const float *>(src), ld, cols, q, scale);
  else
    quant_rows_kernel<__nv_bfloat16><<<rows, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(src), ld, cols, q, scale);
  WAN_CHECK_LAUNCH("quant_rows");
  return WAN_OK;
}

int launch_quant_tensor(const void *src, int dtype, size_t n, uint8_t *q, float *scale, cudaStream_t s) {
  if (n % 4) return set_error(WAN_EUNSUPPORTED, "quantize: element count must be a multiple of 4");
  WAN_TRY_CUDA(cudaMemsetAsync(scale, 0, sizeof(float), s), "quantize: clear amax");
  if (n == 0) return WAN_OK;
  const size_t n4 = n / 4;
  size_t g = (n4 + 255) / 256;
  if (g > 148 * 8) g = 148 * 8;
  unsigned *bits = reinterpret_cast<unsigned *>(scale);
  if (dtype == WAN_F32) {
    amax_kernel<float><<<(int)g, 256, 0, s>>>(static_cast<const float *>(src), n4, bits);
    quant_tensor_kernel<float><<<(int)g, 256, 0, s>>>(static_cast<const float *>(src), n4, bits, q);
  } else {
    amax_kernel<__nv_bfloat16><<<(int)g, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(src), n4, bits);
    quant_tensor_kernel<__nv_bfloat16><<<(int)g, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(src), n4, bits, q);
  }
  amax_to_scale_kernel<<<1, 1, 0, s>>>(scale);
  WAN_CHECK_LAUNCH("quant_tensor");
  return WAN_OK;
}

// ----------------------------------------------------------------------------
// LayerNorm over D (population variance, eps inside the square root), then
// either the AdaLN modulation (1 + scale) * u + shift with chunks taken from
// m[b] (norm1 / norm2), or an affine g * u + beta (norm3). A CTA of 256
// threads normalises one row at a time with the row in registers (exact
// two-pass statistics: the mean, then the sum of squared deviations), and
// walks rows blockIdx.x, blockIdx.x + gridDim.x, ... (two CTAs per SM): the
// next row's loads are issued before the current row is reduced and stored,
// so HBM reads stay in flight through the reductions. Each block reduction
// takes one barrier (partials double-buffered by reduction parity).
// ----------------------------------------------------------------------------
constexpr int LN_THREADS = 256;
constexpr int LN_MAXV = 8;          // float4 per thread: D <= 8192
constexpr int LN_CTAS_PER_SM = 2;   // two rows in flight per CTA (the next one prefetched)

// Sum (MAX = false) or maximum over the CTA; `red` is this reduction's slot of
// 32 floats, alternating between two slots from one reduction to the next.
template <bool MAX>
__device__ __forceinline__ float block_reduce_1sync(float v, float *red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  constexpr int NW = LN_THREADS / 32;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = MAX ? fmaxf(v, w) : v + w;
  }
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = (lane < NW) ? red[lane] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, t, o);
    t = MAX ? fmaxf(t, w) : t + w;
  }
  return t;
}

template <int VPT>
__device__ __forceinline__ void ln_load_row(float4 (&v)[VPT], const float *__restrict__ xr, int nv) {
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = threadIdx.x + i * LN_THREADS;
    if (c < nv) v[i] = load4(xr + 4 * c);
  }
}

// With OutT = uint8_t the modulated row is quantized to e4m3 with its own
// scale (written to row_scale), the input of an FP8 GEMM. VPT = float4
// chunks per thread (ceil(D / 1024)).
template <typename OutT, int VPT>
__global__ void __launch_bounds__(LN_THREADS, LN_CTAS_PER_SM)
layernorm_mod_kernel(const float *__restrict__ x, OutT *__restrict__ out, int rows, int D, const LnMod md,
                     const float *__restrict__ g, const float *__restrict__ beta, float eps,
                     float *__restrict__ row_scale, int *dbg) {
  const OutT *out_hi = out + (size_t)rows * D;
  __shared__ float red[2][32];
  const int nv = D >> 2;
  int row = blockIdx.x;
  if (row >= rows) return;
  int k = 0;                               // reductions so far (selects the partials slot)
  float4 v[VPT], nxt[VPT];
  ln_load_row<VPT>(v, x + (size_t)row * D, nv);
  for (; row < rows; row += gridDim.x) {
    const int nrow = row + gridDim.x;      // uniform across the CTA
    if (nrow < rows) ln_load_row<VPT>(nxt, x + (size_t)nrow * D, nv);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = threadIdx.x + i * LN_THREADS;
      if (c < nv) s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
    }
    const float mean = block_reduce_1sync<false>(s, red[k++ & 1]) / (float)D;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = threadIdx.x + i * LN_THREADS;
      if (c < nv) {
        const float a = v[i].x - mean, b = v[i].y - mean, cc = v[i].z - mean, d = v[i].w - mean;
        ss += (a * a + b * b) + (cc * cc + d * d);
      }
    }
    const float var = block_reduce_1sync<false>(ss, red[k++ & 1]) / (float)D;
    const float rstd = 1.0f / sqrtf(var + eps);
    const float *mshift = nullptr, *mscale = nullptr, *bshift = nullptr, *bscale = nullptr;
    if (md.mod) {
      const float *mrow = md.mod + (size_t)(row / md.rows_div) * md.row_stride;
      mshift = mrow + md.shift_off;
      mscale = mrow + md.scale_off;
      if (md.bias) {
        bshift = md.bias + md.bias_shift_off;
        bscale = md.bias + md.bias_scale_off;
      }
    }
    OutT *orow = out + (size_t)row * D;
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = threadIdx.x + i * LN_THREADS;
      if (c < nv) {
        float4 u = make_float4((v[i].x - mean) * rstd, (v[i].y - mean) * rstd,
                               (v[i].z - mean) * rstd, (v[i].w - mean) * rstd);
        float4 a, b;
        if (md.mod) {
          float4 sc = load4(mscale + 4 * c), sh = load4(mshift + 4 * c);
          if (bshift) {
            const float4 bs = load4(bscale + 4 * c), bh = load4(bshift + 4 * c);
            sc = make_float4(sc.x + bs.x, sc.y + bs.y, sc.z + bs.z, sc.w + bs.w);
            sh = make_float4(sh.x + bh.x, sh.y + bh.y, sh.z + bh.z, sh.w + bh.w);
          }
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
        if constexpr (sizeof(OutT) == 1) {
          v[i] = u;
          amax = fmaxf(amax, absmax4(u));
        } else {
          if (WAN_DBG_OK(orow + 4 * c, 4 * sizeof(OutT), out, out_hi, dbg, WAN_DBG_CODE_BASE + 4))
            store4(orow + 4 * c, u);
        }
      }
    }
    if constexpr (sizeof(OutT) == 1) {
      amax = block_reduce_1sync<true>(amax, red[k++ & 1]);
      const float inv = e4m3_inv_scale(amax);
      uint32_t *qr = reinterpret_cast<uint32_t *>(orow);
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int c = threadIdx.x + i * LN_THREADS;
        if (c < nv && WAN_DBG_OK(qr + c, 4, out, out_hi, dbg, WAN_DBG_CODE_BASE + 5)) qr[c] = quant4(v[i], inv);
      }
      if (threadIdx.x == 0) row_scale[row] = __fdiv_rn(amax, E4M3_MAX);
    }
#pragma unroll
    for (int i = 0; i < VPT; ++i) v[i] = nxt[i];
  }
}

template <typename OutT, int VPT>
static void ln_launch(const float *x, OutT *out, int rows, int D, const LnMod &m, const float *g,
                      const float *beta, float eps, float *row_scale, cudaStream_t s) {
  const int grid = rows < LN_CTAS_PER_SM * sm_count() ? rows : LN_CTAS_PER_SM * sm_count();
  layernorm_mod_kernel<OutT, VPT><<<grid, LN_THREADS, 0, s>>>(x, out, rows, D, m, g, beta, eps, row_scale,
                                                               dbg_word());
}

template <typename OutT>
static void ln_dispatch(const float *x, OutT *out, int rows, int D, const LnMod &m, const float *g,
                        const float *beta, float eps, float *row_scale, cudaStream_t s) {
  switch ((D / 4 + LN_THREADS - 1) / LN_THREADS) {
    case 1: ln_launch<OutT, 1>(x, out, rows, D, m, g, beta, eps, row_scale, s); break;
    case 2: ln_launch<OutT, 2>(x, out, rows, D, m, g, beta, eps, row_scale, s); break;
    case 3: ln_launch<OutT, 3>(x, out, rows, D, m, g, beta, eps, row_scale, s); break;
    case 4: ln_launch<OutT, 4>(x, out, rows, D, m, g, beta, eps, row_scale, s); break;
    case 5: ln_launch<OutT, 5>(x, out, rows, D, m, g, beta, eps, row_scale, s); break;
    case 6: ln_launch<OutT, 6>(x, out, rows, D, m, g, beta, eps, row_scale, s); break;
    default: ln_launch<OutT, LN_MAXV>(x, out, rows, D, m, g, beta, eps, row_scale, s); break;
  }
}

int launch_layernorm_mod(const float *x, void *out, int dtype, int rows, int D, const LnMod &m,
                         const float *g, const float *beta, float eps, cudaStream_t s) {
  if (D % 4 || D > 4 * LN_MAXV * LN_THREADS) return set_error(WAN_EUNSUPPORTED, "layernorm: D=%d", D);
  if (rows == 0) return WAN_OK;
  if (dtype == WAN_BF16)
    ln_dispatch<__nv_bfloat16>(x, (__nv_bfloat16 *)out, rows, D, m, g, beta, eps, nullptr, s);
  else
    ln_dispatch<float>(x, (float *)out, rows, D, m, g, beta, eps, nullptr, s);
  WAN_CHECK_LAUNCH("layernorm_mod");
  return WAN_OK;
}

int launch_layernorm_mod_fp8(const float *x, uint8_t *q, float *row_scale, int rows, int D, const LnMod &m,
                             const float *g, const float *beta, float eps, cudaStream_t s) {
  if (D % 4 || D > 4 * LN_MAXV * LN_THREADS) return set_error(WAN_EUNSUPPORTED, "layernorm: D=%d", D);
  if (rows == 0) return WAN_OK;
  ln_dispatch<uint8_t>(x, q, rows, D, m, g, beta, eps, row_scale, s);
  WAN_CHECK_LAUNCH("layernorm_mod_fp8");
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
                    int L, int H, int W, int tok0, int rows, int *dbg) {
  __shared__ float red[32];
  const int row = blockIdx.x;
  T *pr = p + (size_t)row * ld;
  const T *p_hi = p + (size_t)(rows - 1) * ld + D;
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
    const int tok = tok0 + row % L;
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
      if (WAN_DBG_OK(pr + 4 * c, 4 * sizeof(T), p, p_hi, dbg, WAN_DBG_CODE_BASE + 6)) store4(pr + 4 * c, u);
    }
  }
}

template <bool NORM, bool ROPE>
static int launch_rr(void *p, int dtype, int rows, int ld, int D, int head_dim, const float *gain,
                     float eps, const float *rope, int L, int H, int W, int tok0, cudaStream_t s) {
  if (dtype == WAN_BF16)
    rmsnorm_rope_kernel<__nv_bfloat16, NORM, ROPE><<<rows, LN_THREADS, 0, s>>>(
        (__nv_bfloat16 *)p, ld, D, head_dim, gain, eps, rope, L, H, W, tok0, rows, dbg_word());
  else
    rmsnorm_rope_kernel<float, NORM, ROPE><<<rows, LN_THREADS, 0, s>>>(
        (float *)p, ld, D, head_dim, gain, eps, rope, L, H, W, tok0, rows, dbg_word());
  WAN_CHECK_LAUNCH("rmsnorm_rope");
  return WAN_OK;
}

int launch_rmsnorm_rope(void *p, int dtype, int rows, int ld, int D, int head_dim,
                        const float *gain, float eps, const float *rope, int rope_max_pos,
                        int F, int H, int W, cudaStream_t s, int rows_per_seq, int tok0) {
  (void)rope_max_pos;
  if (D % 4 || D > 4 * LN_MAXV * LN_THREADS || head_dim % 4)
    return set_error(WAN_EUNSUPPORTED, "rmsnorm_rope: D=%d head_dim=%d", D, head_dim);
  if (rows == 0) return WAN_OK;
  const int L = rows_per_seq > 0 ? rows_per_seq : F * H * W;
  if (rope) return launch_rr<true, true>(p, dtype, rows, ld, D, head_dim, gain, eps, rope, L, H, W, tok0, s);
  return launch_rr<true, false>(p, dtype, rows, ld, D, head_dim, gain, eps, nullptr, 1, 1, 1, 0, s);
}

int launch_rope_only(void *p, int dtype, int rows, int ld, int D, int head_dim,
                     const float *rope, int rope_max_pos, int F, int H, int W, cudaStream_t s) {
  (void)rope_max_pos;
  if (D % 4 || D > 4 * LN_MAXV * LN_THREADS || head_dim % 4)
    return set_error(WAN_EUNSUPPORTED, "rope: D=%d head_dim=%d", D, head_dim);
  if (rows == 0) return WAN_OK;
  return launch_rr<false, true>(p, dtype, rows, ld, D, head_dim, nullptr, 0.f, rope, F * H * W, H, W, 0, s);
}

// ----------------------------------------------------------------------------
// Chunk permutation around the all-to-all of the head-parallel attention:
// src holds prod(dims) chunks of chunk_bytes in row-major order of `dims`;
// dst chunk (j_0, ..., j_{nd-1}) (row-major over dims[perm[k]]) is src chunk
// i with i[perm[k]] = j_k. One 16-byte vector per thread, grid-stride.
// ----------------------------------------------------------------------------
struct PermuteArgs {
  int nd;
  long long dst_ext[5];       // extent of dst axis k (= dims[perm[k]])
  long long src_stride[5];    // src chunk stride of the src axis that dst axis k runs over
};

__global__ void permute_chunks_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, PermuteArgs a,
                                      long long vpc, long long total, int *dbg) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long chunk = i / vpc, v = i - chunk * vpc;
    long long rem = chunk, off = 0;
    for (int k = a.nd - 1; k >= 0; --k) {
      const long long j = rem % a.dst_ext[k];
      rem /= a.dst_ext[k];
      off += j * a.src_stride[k];
    }
    if (WAN_DBG_OK(dst + i, 16, dst, dst + total, dbg, WAN_DBG_CODE_BASE + 7)) dst[i] = src[off * vpc + v];
  }
}

int launch_permute_chunks(const void *src, void *dst, int nd, const int *dims, const int *perm,
                          size_t chunk_bytes, cudaStream_t s) {
  PermuteArgs a = {};
  a.nd = nd;
  long long stride[5], nchunks = 1;
  for (int k = nd - 1; k >= 0; --k) {
    stride[k] = nchunks;
    nchunks *= dims[k];
  }
  for (int k = 0; k < nd; ++k) {
    a.dst_ext[k] = dims[perm[k]];
    a.src_stride[k] = stride[perm[k]];
  }
  const long long vpc = (long long)(chunk_bytes / 16), total = nchunks * vpc;
  if (total == 0) return WAN_OK;
  const long long want = (total + 255) / 256;
  const int blocks = (int)(want < 148LL * 16 ? want : 148LL * 16);
  permute_chunks_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), a,
                                               vpc, total, dbg_word());
  WAN_CHECK_LAUNCH("permute_chunks");
  return WAN_OK;
}

// ----------------------------------------------------------------------------
// k rows of the tensor-core path: k[r] *= 1 / sqrt(ss[r] / D + eps) in place
// (the QKV epilogue wrote gamma * RoPE(y) and the row's sum of squares of y).
// One warp per row, 16-byte vectors.
// ----------------------------------------------------------------------------
__global__ void scale_rows_kernel(__nv_bfloat16 *__restrict__ p, int rows, int ld, int D,
                                  const float *__restrict__ ss, int ss_stride, int parts, float inv_d,
                                  float eps, int *dbg) {
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
    if (WAN_DBG_OK(pr + c, 16, p, p + (size_t)(rows - 1) * ld + D, dbg, WAN_DBG_CODE_BASE + 8))
      pr[c] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

int launch_scale_rows(void *p, int rows, int ld, int D, const float *ss, int ss_stride, int parts,
                      float eps, cudaStream_t s) {
  if (rows == 0) return WAN_OK;
  if (D % 8 || ld % 8 || parts < 1 || parts > 32) return set_error(WAN_EUNSUPPORTED, "scale_rows: D=%d", D);
  const int warps = 8;
  scale_rows_kernel<<<(rows + warps - 1) / warps, warps * 32, 0, s>>>(
      static_cast<__nv_bfloat16 *>(p), rows, ld, D, ss, ss_stride, parts, 1.0f / (float)D, eps, dbg_word());
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
                                 const VT *__restrict__ vu, size_t n, float scale, float dt, int *dbg) {
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
    if (WAN_DBG_OK(x + 4 * i, 16, x, x + n, dbg, WAN_DBG_CODE_BASE + 9)) store4(x + 4 * i, xv);
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
    if (WAN_DBG_OK(x + t, 4, x, x + n, dbg, WAN_DBG_CODE_BASE + 9)) x[t] = fmaf(dt, v, x[t]);
  }
}

template <typename VT>
static void euler_launch(float *x, const void *vc, const void *vu, size_t n, float scale, float dt,
                         cudaStream_t s) {
  const size_t nv = (n >> 2) > 0 ? (n >> 2) : 1;
  int blocks = (int)((nv + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (vu)
    euler_cfg_kernel<VT, true><<<blocks, 256, 0, s>>>(x, (const VT *)vc, (const VT *)vu, n, scale, dt, dbg_word());
  else
    euler_cfg_kernel<VT, false><<<blocks, 256, 0, s>>>(x, (const VT *)vc, nullptr, n, scale, dt, dbg_word());
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

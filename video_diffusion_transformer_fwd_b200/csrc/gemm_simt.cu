// CUDA-core GEMM with fused epilogues: the exact-fp32 path of the block
// (every product and sum an fp32 FMA; no TF32), also usable on bf16 operands.
// C = A B^T (+ bias) as in nn.Linear (W stored [out, in]).
#include "common.cuh"

namespace wan {

namespace {
constexpr int BM = 128, BN = 128, BK = 8, THREADS = 256;

template <typename T>
__device__ __forceinline__ const T *seg_ptr(const GemmArgs &g, int n, int &nn, int &seg) {
  seg = n / g.segN;
  nn = n - seg * g.segN;
  return static_cast<const T *>(g.Bseg[seg]);
}

template <typename T, int EPI>
__global__ void __launch_bounds__(THREADS) gemm_simt_kernel(const GemmArgs g) {
  __shared__ __align__(16) float As[BK][BM + 4];
  __shared__ __align__(16) float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const T *A = static_cast<const T *>(g.A);

  // loader mapping: 128 rows x 8 k = 1024 elements = 256 threads x 4
  const int lrow = tid >> 1, lk = (tid & 1) * 4;
  const int am = m0 + lrow;
  const int bn = n0 + lrow;
  const T *arow = (am < g.M) ? A + (size_t)am * g.lda : nullptr;
  const T *brow = nullptr;
  if (bn < g.N) {
    int nn, seg;
    const T *Bp = seg_ptr<T>(g, bn, nn, seg);
    brow = Bp + (size_t)nn * g.K;
  }

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < g.K; k0 += BK) {
    float4 av = arow ? load4(arow + k0 + lk) : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 bv = brow ? load4(brow + k0 + lk) : make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();
    As[lk + 0][lrow] = av.x; As[lk + 1][lrow] = av.y; As[lk + 2][lrow] = av.z; As[lk + 3][lrow] = av.w;
    Bs[lk + 0][lrow] = bv.x; Bs[lk + 1][lrow] = bv.y; Bs[lk + 2][lrow] = bv.z; Bs[lk + 3][lrow] = bv.w;
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[8], b[8];
      const float4 a0 = *reinterpret_cast<const float4 *>(&As[kk][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4 *>(&As[kk][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[kk][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[kk][tx * 8 + 4]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w; a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w; b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
  }

  // epilogue: 8 consecutive columns per thread (N % 8 == 0, never straddles a segment
  // because segN % 8 == 0)
  const int nb = n0 + tx * 8;
  if (nb >= g.N) return;
  float bias[8];
  {
    const int seg = nb / g.segN, nn = nb - seg * g.segN;
    const T *bp = static_cast<const T *>(g.bias[seg]);
#pragma unroll
    for (int j = 0; j < 8; ++j) bias[j] = bp ? ElemIO<T>::load(bp + nn + j) : 0.f;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + ty * 8 + i;
    if (m >= g.M) break;
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[j] = acc[i][j] + bias[j];
      if (EPI == EPI_GELU) v[j] = gelu_tanh(v[j]);
      if (EPI == EPI_SILU) v[j] = v[j] / (1.0f + expf(-v[j]));
    }
    if (EPI == EPI_RESID) {
      float *xr = g.X + (size_t)m * g.ldx + nb;
      const float *gr = g.gate ? g.gate + (size_t)(m / g.rows_per_gate) * g.gate_stride + nb : nullptr;
#pragma unroll
      for (int j = 0; j < 8; j += 4) {
        float4 xv = g.x_store ? make_float4(0.f, 0.f, 0.f, 0.f) : load4(xr + j);
        float4 gv = gr ? load4(gr + j) : make_float4(1.f, 1.f, 1.f, 1.f);
        if (gr && g.gate_bias) {
          const float4 gb = load4(g.gate_bias + nb + j);
          gv = make_float4(gv.x + gb.x, gv.y + gb.y, gv.z + gb.z, gv.w + gb.w);
        }
        xv.x = fmaf(gv.x, v[j + 0], xv.x);
        xv.y = fmaf(gv.y, v[j + 1], xv.y);
        xv.z = fmaf(gv.z, v[j + 2], xv.z);
        xv.w = fmaf(gv.w, v[j + 3], xv.w);
        if (WAN_DBG_OK(xr + j, 16, g.X, g.X + (size_t)(g.M - 1) * g.ldx + g.N, g.dbg, WAN_DBG_CODE_BASE + 10))
          store4(xr + j, xv);
      }
    } else {
      T *cr = static_cast<T *>(g.C) + (size_t)m * g.ldc + nb;
      const T *c_hi = static_cast<const T *>(g.C) + (size_t)(g.M - 1) * g.ldc + g.N;
      if (WAN_DBG_OK(cr, 8 * sizeof(T), g.C, c_hi, g.dbg, WAN_DBG_CODE_BASE + 11)) {
        store4(cr, make_float4(v[0], v[1], v[2], v[3]));
        store4(cr + 4, make_float4(v[4], v[5], v[6], v[7]));
      }
    }
  }
}

template <typename T>
int launch_t(const GemmArgs &g, cudaStream_t s) {
  dim3 grid((g.N + BN - 1) / BN, (g.M + BM - 1) / BM);
  switch (g.epi) {
    case EPI_STORE: gemm_simt_kernel<T, EPI_STORE><<<grid, THREADS, 0, s>>>(g); break;
    case EPI_GELU: gemm_simt_kernel<T, EPI_GELU><<<grid, THREADS, 0, s>>>(g); break;
    case EPI_SILU: gemm_simt_kernel<T, EPI_SILU><<<grid, THREADS, 0, s>>>(g); break;
    default: gemm_simt_kernel<T, EPI_RESID><<<grid, THREADS, 0, s>>>(g); break;
  }
  WAN_CHECK_LAUNCH("gemm_simt");
  return WAN_OK;
}
}  // namespace

int gemm_simt(const GemmArgs &g, int dtype, cudaStream_t s) {
  if (g.epi == EPI_QKNORM) return set_error(WAN_EUNSUPPORTED, "gemm_simt: q/k-norm epilogue is tensor-core only");
  if (g.K % BK || g.N % 8 || g.segN % 8 || g.lda % 4)
    return set_error(WAN_EUNSUPPORTED, "gemm_simt: M=%d N=%d K=%d", g.M, g.N, g.K);
  if (g.M == 0 || g.N == 0) return WAN_OK;
  if ((g.M + BM - 1) / BM > 65535) return set_error(WAN_EINVAL, "gemm_simt: M too large");
  GemmArgs gd = g;
  if (!gd.dbg) gd.dbg = dbg_word();
  return dtype == WAN_BF16 ? launch_t<__nv_bfloat16>(gd, s) : launch_t<float>(gd, s);
}

}  // namespace wan

// GEMM for a handful of rows (M <= 8): y = A W^T + b (optionally SiLU), the
// shape of the time-embedding MLP and its 6 x dim projection (one row per
// sequence). The weight matrix is streamed once from HBM with 16-byte loads;
// the few A rows stay in L1/L2. Exact fp32 FMA arithmetic.
#include "common.cuh"

namespace wan {

namespace {
constexpr int MAXM = 8;        // rows of A
constexpr int NCOL = 4;        // output columns per warp
constexpr int WARPS = 8;

template <typename T, int EPI>
__global__ void __launch_bounds__(WARPS * 32) gemm_smallm_kernel(const GemmArgs g) {
  const int lane = threadIdx.x & 31;
  const int n0 = (blockIdx.x * WARPS + (threadIdx.x >> 5)) * NCOL;
  if (n0 >= g.N) return;
  const T *A = static_cast<const T *>(g.A);
  const T *Wm = static_cast<const T *>(g.Bseg[0]);
  float acc[MAXM][NCOL];
#pragma unroll
  for (int m = 0; m < MAXM; ++m)
#pragma unroll
    for (int c = 0; c < NCOL; ++c) acc[m][c] = 0.f;
  for (int k = lane * 4; k < g.K; k += 128) {
    float4 w[NCOL];
#pragma unroll
    for (int c = 0; c < NCOL; ++c)
      w[c] = (n0 + c < g.N) ? load4(Wm + (size_t)(n0 + c) * g.K + k) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
      if (m < g.M) {
        const float4 a = load4(A + (size_t)m * g.lda + k);
#pragma unroll
        for (int c = 0; c < NCOL; ++c) {
          acc[m][c] = fmaf(a.x, w[c].x, acc[m][c]);
          acc[m][c] = fmaf(a.y, w[c].y, acc[m][c]);
          acc[m][c] = fmaf(a.z, w[c].z, acc[m][c]);
          acc[m][c] = fmaf(a.w, w[c].w, acc[m][c]);
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MAXM; ++m)
#pragma unroll
    for (int c = 0; c < NCOL; ++c) acc[m][c] = warp_sum(acc[m][c]);
  // lane m * NCOL + c writes y[m, n0 + c]
  const T *bp = static_cast<const T *>(g.bias[0]);
#pragma unroll
  for (int m = 0; m < MAXM; ++m)
#pragma unroll
    for (int c = 0; c < NCOL; ++c) {
      if (lane == m * NCOL + c && m < g.M && n0 + c < g.N) {
        float v = acc[m][c] + (bp ? ElemIO<T>::load(bp + n0 + c) : 0.f);
        if (EPI == EPI_SILU) v = v / (1.0f + expf(-v));
        ElemIO<T>::store(static_cast<T *>(g.C) + (size_t)m * g.ldc + n0 + c, v);
      }
    }
}

template <typename T>
int launch_t(const GemmArgs &g, cudaStream_t s) {
  const int cols_per_cta = WARPS * NCOL;
  const int grid = (g.N + cols_per_cta - 1) / cols_per_cta;
  if (g.epi == EPI_SILU)
    gemm_smallm_kernel<T, EPI_SILU><<<grid, WARPS * 32, 0, s>>>(g);
  else
    gemm_smallm_kernel<T, EPI_STORE><<<grid, WARPS * 32, 0, s>>>(g);
  WAN_CHECK_LAUNCH("gemm_smallm");
  return WAN_OK;
}
}  // namespace

bool gemm_smallm_supported(const GemmArgs &g) {
  return g.M >= 1 && g.M <= MAXM && g.nseg == 1 && g.segN == g.N && g.K % 4 == 0 && g.lda % 4 == 0 &&
         (g.epi == EPI_STORE || g.epi == EPI_SILU) && aligned16(g.A) && aligned16(g.Bseg[0]);
}

int gemm_smallm(const GemmArgs &g, int dtype, cudaStream_t s) {
  if (!gemm_smallm_supported(g)) return set_error(WAN_EUNSUPPORTED, "gemm_smallm: M=%d N=%d K=%d", g.M, g.N, g.K);
  if (g.N == 0) return WAN_OK;
  return dtype == WAN_BF16 ? launch_t<__nv_bfloat16>(g, s) : launch_t<float>(g, s);
}

}  // namespace wan

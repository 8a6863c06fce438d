// Shared helpers of libwan (host + device). Internal header.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/wan.h"

namespace wan {

// ---------------------------------------------------------------- errors
int set_error(int code, const char *fmt, ...);
int cuda_error(cudaError_t e, const char *what);
// Device address of the library's watchdog word on the current device
// (set to a nonzero code by a kernel that gave up a bounded wait).
int *watchdog_ptr();

#define WAN_TRY_CUDA(call, what)                                        \
  do {                                                                  \
    cudaError_t e_ = (call);                                            \
    if (e_ != cudaSuccess) return ::wan::cuda_error(e_, what);          \
  } while (0)

#define WAN_CHECK_LAUNCH(what)                                          \
  do {                                                                  \
    cudaError_t e_ = cudaGetLastError();                                \
    if (e_ != cudaSuccess) return ::wan::cuda_error(e_, what);          \
  } while (0)

// ---------------------------------------------------------------- debug bounds checks
// In a build with -DWAN_DEBUG_BOUNDS (build_lib.build(debug=True)) a kernel
// checks, before each plain global store, that the bytes it writes lie inside
// the extent [lo, hi) that the call's sizes give the buffer; on a violation
// it records `code` in the device status word (the first one is kept), skips
// the store, and wan_device_status returns WAN_EBOUNDS. In other builds the
// check is the constant true and dbg_word() is NULL. (TMA stores and
// reductions are clipped by their tensor maps and are not checked.)
#ifdef WAN_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
__device__ __forceinline__ bool dbg_in(const void *p, size_t n, const void *lo, const void *hi, int *word,
                                       int code) {
  const char *c = static_cast<const char *>(p);
  if (c >= static_cast<const char *>(lo) && c + n <= static_cast<const char *>(hi)) return true;
  if (word) atomicCAS(word, 0, code);
  return false;
}
#define WAN_DBG_OK(p, n, lo, hi, word, code) ::wan::dbg_in((p), (n), (lo), (hi), (word), (code))
#else
constexpr bool kDebugBounds = false;
#define WAN_DBG_OK(p, n, lo, hi, word, code) true
#endif
// Status word the debug checks record into (NULL in other builds).
inline int *dbg_word() { return kDebugBounds ? watchdog_ptr() : nullptr; }
constexpr int WAN_DBG_CODE_BASE = 0x40000000;   // codes >= this are bounds violations (wait codes are < 0x10000)

// ---------------------------------------------------------------- element access
template <typename T> struct ElemIO;
template <> struct ElemIO<float> {
  static __device__ __forceinline__ float load(const float *p) { return *p; }
  static __device__ __forceinline__ void store(float *p, float v) { *p = v; }
};
template <> struct ElemIO<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
};

// load 4 consecutive elements (16-byte aligned for float, 8-byte for bf16)
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
  uint2 u = *reinterpret_cast<const uint2 *>(p);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162 *>(&u.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&u.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ void store4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t *>(&a);
  u.y = *reinterpret_cast<uint32_t *>(&b);
  *reinterpret_cast<uint2 *>(p) = u;
}

// GELU, tanh form: 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3)))
__device__ __forceinline__ float gelu_tanh(float z) {
  const float k0 = 0.7978845608028654f;   // sqrt(2/pi)
  const float k1 = 0.044715f;
  return 0.5f * z * (1.0f + tanhf(k0 * (z + k1 * z * z * z)));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum; `red` is shared scratch of >= 32 floats. All threads get it.
__device__ __forceinline__ float block_sum(float v, float *red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = (lane < nw) ? red[lane] : 0.f;
  return warp_sum(t);
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t dtype_size(int dt) { return dt == WAN_F32 ? 4 : 2; }   // WAN_FP8: bf16 intermediates

// ---------------------------------------------------------------- internal kernels API

enum Epilogue { EPI_STORE = 0, EPI_GELU = 1, EPI_RESID = 2, EPI_QKNORM = 3, EPI_SILU = 4 };

// C = A B^T (+ bias) with a fused epilogue. A [M,K] row-major (lda),
// B given as up to 3 row-major segments [segN, K] (ldb = K) stacked along N,
// so one call can multiply by [Wq; Wk; Wv]. bias per segment [segN] (or NULL).
//   EPI_STORE: C[m,n] = acc + bias
//   EPI_GELU:  C[m,n] = gelu_tanh(acc + bias)
//   EPI_SILU:  C[m,n] = silu(acc + bias)          (CUDA-core GEMM only)
//   EPI_RESID: X[m,n] += g * (acc + bias), g = gate[(m / rows_per_gate) *
//              gate_stride + n] or 1 when gate == NULL  (X float32, ldx)
//   EPI_QKNORM (tensor-core path): per segment s, y = acc + bias; when
//              ss_col[s] >= 0, the sum of y^2 over each 256-column tile t of the
//              segment is written to ss[m * ss_stride + ss_col[s] * (segN / 256) + t]
//              (the consumer adds the segN / 256 partials of a row),
//              and C = gamma[s] * y, rotated by the 3D RoPE of token
//              tok0 + m % rows_per_seq when
//              bit s of rope_mask is set; otherwise C = y. The row's RMS factor
//              is applied later (attention logit scale for q, a row pass for k).
struct GemmArgs {
  int M, N, K;
  const void *A; int lda;
  const void *Bseg[3]; const void *bias[3]; int segN; int nseg;
  int epi;
  void *C; int ldc;
  float *X; int ldx;
  const float *gate; int gate_stride; int rows_per_gate;
  const float *gate_bias;  // optional [N]: g = gate[...] + gate_bias[n] (per-token modulation)
  int x_store;            // EPI_RESID: x = g * y (overwrite) instead of x += g * y
  int fp8;                // A and B are e4m3 codes: y = (A B^T) a_scale[m] b_scale[seg] + bias
  const float *a_scale;   // [M] (device)
  const float *b_scale[3];  // one device float per weight segment
  const float *gamma[3]; float *ss; int ss_stride; int ss_col[3];
  const float *rope; int rope_mask; int F, H, W; int head_dim;
  // rows of A per sequence (0: F*H*W) and the grid index of a sequence's
  // first row: row m is token tok0 + m % rows_per_seq of the (F, H, W) grid
  int rows_per_seq, tok0;
  int *dbg;               // debug bounds checks: status word (dbg_word())
};

int gemm_simt(const GemmArgs &g, int dtype, cudaStream_t s);
int gemm_tc(const GemmArgs &g, cudaStream_t s);           // bf16 tcgen05 path
bool gemm_tc_supported(const GemmArgs &g);
// M <= 8 rows, one weight segment, STORE or SILU epilogue (gemv.cu)
int gemm_smallm(const GemmArgs &g, int dtype, cudaStream_t s);
bool gemm_smallm_supported(const GemmArgs &g);

// Attention over rows of strided matrices. Sequence b, row r of q is at
// q + (b*Lq + r)*ldq + head*d (likewise k, v with Lk, o with Lq).
struct AttnArgs {
  int B, heads, Lq, Lk, d;
  const void *q; int ldq;
  const void *k; int ldk;
  const void *v; int ldv;
  void *o; int ldo;
  const int *k_lens;      // device [B] or NULL
  float scale;
  // optional per-query-row RMS factor folded into the logit scale:
  // scale_row = scale / sqrt(sum_{t < q_ss_parts} q_ss[row * q_ss_stride + t] / q_ss_n + q_ss_eps)
  const float *q_ss; int q_ss_stride; int q_ss_parts; float q_ss_n; float q_ss_eps;
  int *dbg;               // debug bounds checks: status word (dbg_word())
};
int attention_simt(const AttnArgs &a, int dtype, cudaStream_t s);
// 8-bit attention (attn8.cu): bf16 q, k, v, o with head_dim 128; quantizes
// into the workspace, then int8 Q K^T and e4m3 P V on the tensor cores
size_t attention_8bit_ws_bytes(int B, int heads, int Lq, int Lk);
bool attention_8bit_supported(const AttnArgs &a);
int attention_8bit(const AttnArgs &a, void *workspace, cudaStream_t s);
int attention_tc(const AttnArgs &a, cudaStream_t s);      // bf16, d = 128
bool attention_tc_supported(const AttnArgs &a);

// Elementwise / row kernels (elementwise.cu)
int launch_mod_combine(const float *modulation, const float *e0, float *mod, int B, int D,
                       cudaStream_t s);
// out[r] = LN(x[r]) * (1 + mod[b][scale_chunk]) + mod[b][shift_chunk]     (affine == NULL)
// out[r] = LN(x[r]) * g + beta                                            (affine gain g)
// Where a LayerNorm row finds its modulation: shift = mod[(row / rows_div) *
// row_stride + shift_off + c] (+ bias[bias_shift_off + c] when bias is set),
// likewise scale. mod == nullptr: the affine g, beta instead.
struct LnMod {
  const float *mod; int rows_div; size_t row_stride; int shift_off, scale_off;
  const float *bias; int bias_shift_off, bias_scale_off;
};
// chunks of a combined [B, 6, D] modulation, L rows per sequence
inline LnMod ln_mod_seq(const float *mod, int L, int D, int shift_chunk, int scale_chunk) {
  return LnMod{mod, L, (size_t)6 * D, shift_chunk * D, scale_chunk * D, nullptr, 0, 0};
}
// chunks of a per-token e0 [rows, 6, D] plus the block's modulation [6, D]
inline LnMod ln_mod_tok(const float *e0, const float *modulation, int D, int shift_chunk, int scale_chunk) {
  return LnMod{e0, 1, (size_t)6 * D, shift_chunk * D, scale_chunk * D, modulation, shift_chunk * D, scale_chunk * D};
}
int launch_layernorm_mod(const float *x, void *out, int dtype, int rows, int D, const LnMod &m,
                         const float *g, const float *beta, float eps, cudaStream_t s);
// the same with the output quantized per row to e4m3 codes q and scales row_scale
int launch_layernorm_mod_fp8(const float *x, uint8_t *q, float *row_scale, int rows, int D, const LnMod &m,
                             const float *g, const float *beta, float eps, cudaStream_t s);
// e4m3 quantization per row (src rows ld elements apart) or per tensor (n elements)
int launch_quant_rows(const void *src, int dtype, size_t ld, int rows, int cols, uint8_t *q, float *scale,
                      cudaStream_t s);
int launch_quant_tensor(const void *src, int dtype, size_t n, uint8_t *q, float *scale, cudaStream_t s);
// In place on rows of a strided matrix: v = RMSNorm_D(v) * gain, then the 3D
// RoPE of token tok0 + r % rows_per_seq of the (F, H, W) grid when rope != NULL
// (rows_per_seq 0: F*H*W).
int launch_rmsnorm_rope(void *p, int dtype, int rows, int ld, int D, int head_dim,
                        const float *gain, float eps, const float *rope, int rope_max_pos,
                        int F, int H, int W, cudaStream_t s, int rows_per_seq = 0, int tok0 = 0);
// In place 3D RoPE only (no norm), rows of a [rows, heads*d] strided matrix.
int launch_rope_only(void *p, int dtype, int rows, int ld, int D, int head_dim,
                     const float *rope, int rope_max_pos, int F, int H, int W, cudaStream_t s);
// In place: row r of a strided bf16 matrix (D columns) *= 1/sqrt(S/D + eps),
// S = sum of the `parts` partial sums at ss[r * ss_stride + 0 .. parts-1].
int launch_scale_rows(void *p, int rows, int ld, int D, const float *ss, int ss_stride, int parts,
                      float eps, cudaStream_t s);
int launch_rope_table(int head_dim, int max_pos, double theta, float *table, cudaStream_t s);
// dst = src with its chunk axes permuted: src is [dims[0]] ... [dims[nd-1]]
// chunks of chunk_bytes, dst axis k runs over src axis perm[k].
int launch_permute_chunks(const void *src, void *dst, int nd, const int *dims, const int *perm,
                          size_t chunk_bytes, cudaStream_t s);
int launch_euler_cfg(float *x, const void *vc, const void *vu, int vdt, size_t n, float scale,
                     float dt, cudaStream_t s);

// Brackets one kernel launch with profiling events when profiling is on.
struct ProfScope {
  int idx;
  cudaStream_t stream;
  ProfScope(int cls, cudaStream_t s);
  ~ProfScope();
};
#define WAN_PROF(cls, s, expr) ([&]() { ::wan::ProfScope ps_((cls), (s)); return (expr); }())

}  // namespace wan

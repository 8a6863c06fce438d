// CUDA-core online-softmax attention (exact fp32 arithmetic on fp32 or bf16
// inputs): the fp32 path of the block and of wan_attention, any head_dim in
// {32, 64, 128}. Non-causal, all keys of the sequence ("Wan2.2 code
// walkthrough" (newtid.com), self-attention snippet: global window, key
// lengths), softmax scale passed in.
#include "common.cuh"

#include <math.h>

namespace wan {

namespace {
constexpr int QROWS = 32;       // query rows per CTA
constexpr int KTILE = 32;       // keys per shared-memory tile
constexpr int THREADS = 128;    // 4 threads per query row

// Thread part p (0..3) of a row owns dims 16c + 4p + e, c < d/16, e < 4, so
// the four threads of a row read 64 contiguous bytes of a key in shared memory.
template <typename T, int D>
__global__ void __launch_bounds__(THREADS) attn_simt_kernel(const AttnArgs a) {
  constexpr int NC = D / 16;                 // float4 chunks per thread
  __shared__ __align__(16) float Ks[KTILE][D];
  __shared__ __align__(16) float Vs[KTILE][D];
  const int tid = threadIdx.x;
  const int rloc = tid >> 2, part = tid & 3;
  const int b = blockIdx.z, h = blockIdx.y;
  const int r = blockIdx.x * QROWS + rloc;
  const bool active = r < a.Lq;
  const int kl = a.k_lens ? min(max(a.k_lens[b], 0), a.Lk) : a.Lk;

  const T *Q = static_cast<const T *>(a.q);
  const T *K = static_cast<const T *>(a.k);
  const T *V = static_cast<const T *>(a.v);

  float4 q[NC], o[NC];
  const T *qrow = Q + (size_t)(b * a.Lq + (active ? r : 0)) * a.ldq + h * D;
  // optional per-row RMS factor of q (q left un-normalised by its producer)
  float qs = 1.0f;
  if (a.q_ss && active) {
    float sum = 0.f;
    for (int t = 0; t < a.q_ss_parts; ++t) sum += a.q_ss[(size_t)(b * a.Lq + r) * a.q_ss_stride + t];
    qs = 1.0f / sqrtf(sum / a.q_ss_n + a.q_ss_eps);
  }
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    q[c] = active ? load4(qrow + 16 * c + 4 * part) : make_float4(0.f, 0.f, 0.f, 0.f);
    q[c].x *= qs; q[c].y *= qs; q[c].z *= qs; q[c].w *= qs;
    o[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float m = -INFINITY, l = 0.f;

  for (int j0 = 0; j0 < kl; j0 += KTILE) {
    __syncthreads();
    // cooperative tile load: KTILE x D floats of K and of V
    for (int e = tid; e < KTILE * D / 4; e += THREADS) {
      const int jj = e / (D / 4), cc = (e % (D / 4)) * 4;
      const int j = j0 + jj;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (j < kl) {
        const size_t row = (size_t)(b * a.Lk + j);
        kv = load4(K + row * a.ldk + h * D + cc);
        vv = load4(V + row * a.ldv + h * D + cc);
      }
      *reinterpret_cast<float4 *>(&Ks[jj][cc]) = kv;
      *reinterpret_cast<float4 *>(&Vs[jj][cc]) = vv;
    }
    __syncthreads();
    float s[KTILE];
    float tmax = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < KTILE; ++jj) {
      float p = 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const float4 kv = *reinterpret_cast<const float4 *>(&Ks[jj][16 * c + 4 * part]);
        p = fmaf(q[c].x, kv.x, p);
        p = fmaf(q[c].y, kv.y, p);
        p = fmaf(q[c].z, kv.z, p);
        p = fmaf(q[c].w, kv.w, p);
      }
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      p += __shfl_xor_sync(0xffffffffu, p, 2);
      s[jj] = (j0 + jj < kl) ? p * a.scale : -INFINITY;
      tmax = fmaxf(tmax, s[jj]);
    }
    const float mnew = fmaxf(m, tmax);
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - mnew);
    l *= alpha;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      o[c].x *= alpha; o[c].y *= alpha; o[c].z *= alpha; o[c].w *= alpha;
    }
#pragma unroll
    for (int jj = 0; jj < KTILE; ++jj) {
      const float p = (s[jj] == -INFINITY) ? 0.f : expf(s[jj] - mnew);
      l += p;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const float4 vv = *reinterpret_cast<const float4 *>(&Vs[jj][16 * c + 4 * part]);
        o[c].x = fmaf(p, vv.x, o[c].x);
        o[c].y = fmaf(p, vv.y, o[c].y);
        o[c].z = fmaf(p, vv.z, o[c].z);
        o[c].w = fmaf(p, vv.w, o[c].w);
      }
    }
    m = mnew;
  }
  if (!active) return;
  const float inv = (l > 0.f) ? 1.0f / l : 0.f;
  T *orow = static_cast<T *>(a.o) + (size_t)(b * a.Lq + r) * a.ldo + h * D;
  const T *o_hi = static_cast<const T *>(a.o) + (size_t)(a.B * a.Lq - 1) * a.ldo + (size_t)a.heads * D;
#pragma unroll
  for (int c = 0; c < NC; ++c)
    if (WAN_DBG_OK(orow + 16 * c + 4 * part, 4 * sizeof(T), a.o, o_hi, a.dbg, WAN_DBG_CODE_BASE + 12))
      store4(orow + 16 * c + 4 * part, make_float4(o[c].x * inv, o[c].y * inv, o[c].z * inv, o[c].w * inv));
}

template <typename T>
int launch_t(const AttnArgs &a, cudaStream_t s) {
  dim3 grid((a.Lq + QROWS - 1) / QROWS, a.heads, a.B);
  switch (a.d) {
    case 32: attn_simt_kernel<T, 32><<<grid, THREADS, 0, s>>>(a); break;
    case 64: attn_simt_kernel<T, 64><<<grid, THREADS, 0, s>>>(a); break;
    case 128: attn_simt_kernel<T, 128><<<grid, THREADS, 0, s>>>(a); break;
    default: return set_error(WAN_EUNSUPPORTED, "attention_simt: head_dim %d", a.d);
  }
  WAN_CHECK_LAUNCH("attention_simt");
  return WAN_OK;
}
}  // namespace

int attention_simt(const AttnArgs &a, int dtype, cudaStream_t s) {
  if (a.d != 32 && a.d != 64 && a.d != 128)
    return set_error(WAN_EUNSUPPORTED, "attention_simt: head_dim %d", a.d);
  if (a.B == 0 || a.Lq == 0 || a.heads == 0) return WAN_OK;
  if (a.heads > 65535 || a.B > 65535) return set_error(WAN_EINVAL, "attention: grid too large");
  AttnArgs ad = a;
  if (!ad.dbg) ad.dbg = dbg_word();
  return dtype == WAN_BF16 ? launch_t<__nv_bfloat16>(ad, s) : launch_t<float>(ad, s);
}

}  // namespace wan

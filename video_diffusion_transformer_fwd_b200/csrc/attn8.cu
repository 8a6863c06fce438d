// 8-bit flash attention for sm_100a ("Wan paper deep dive"
// (charles2530.github.io), inference-optimisation table, "8-bit
// FlashAttention": int8 for S = Q K^T, FP8 for O = P V, fp32 accumulation
// across key blocks). head_dim 128, non-causal.
//
// Quantization (bf16 inputs, decisions in fp32):
//   q  int8 per (token, head): scale amax/127 over the head's 128 values;
//   k  int8 per (sequence, head): scale amax/127 over all Lk keys;
//   v  e4m3 per (sequence, head, channel): scale amax/448 over all Lk keys,
//      written transposed (V^T rows = channels, 128 keys per 128-byte run)
//      so both MMA operands of P V are K-major;
//   codes: int8 = round-half-even of x * (127 / amax) clamped to +-127;
//   e4m3 = nearest (ties to even) of x * (448 / amax), saturating.
// Kernel (same pipeline as the bf16 attention: 8 softmax warps over 2 query
// tiles, an MMA warp, a TMA warp, S_0 | S_1 | O_0 | O_1 in TMEM):
//   S = Q8 K8^T on kind::i8 into s32 TMEM columns; a softmax thread turns its
//   row's s32 into floats by adding the bits of 1.5 * 2^23 (|S| < 2^22, so the
//   float is exactly 1.5 * 2^23 + S) and folds that offset into the FMA that
//   applies the logit scale c = scale log2(e) s_q s_k (times q's RMS factor
//   when given). A row keeps a frame m, its running max (log2 units) rounded
//   up to a multiple of 8, raised only when a tile's max exceeds it (O and l
//   are then rescaled by an exact power of two); P = exp2(S c - m + 8) lies
//   in (0, 2^8], is written back as e4m3 (4 per TMEM column), and
//   O += P V^T runs on kind::f8f6f4 with P from TMEM. Because the frame only
//   moves in steps of 8, rescales are rare and the e4m3 rounding of P is the
//   same as with the frame recomputed after every tile. The epilogue applies
//   1 / l and the channel scales of v.
#include "common.cuh"
#include "sm100.cuh"

#include <cuda_fp8.h>

namespace wan {

namespace {
using namespace sm100;

constexpr int D = 128;                     // head_dim
constexpr int TQ = 128;
constexpr int TK = 128;
constexpr int NSLOT = 8;                   // K / V^T ring slots
constexpr int TILE = 128 * 128;            // 16 KB: one 8-bit Q, K or V^T tile (one 128-byte swizzled box)
constexpr int THREADS = 320;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_S = idesc_i8(TQ, TK);
constexpr uint32_t IDESC_O = idesc_e4m3(TQ, D);
constexpr int SMEM_BYTES = 1024 + 2 * TILE + NSLOT * TILE + 256;
constexpr uint32_t MAGIC = 0x4B400000u;    // bits of 12582912.0f = 1.5 * 2^23
constexpr float MAGIC_F = 12582912.0f;
constexpr float I8_MAX = 127.f, E4M3_MAX = 448.f;

struct Fa8Params {
  int B, heads, Lq, Lk;
  const int *k_lens;
  float c;                      // scale * log2(e)
  const float *sq;              // [B * Lq, heads]
  const float *sk;              // [B * heads]
  const float *sv;              // [B * heads, 128]
  __nv_bfloat16 *o; int ldo;
  const float *q_ss; int q_ss_stride; int q_ss_parts; float q_ss_inv_n; float q_ss_eps;
  int *watchdog;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}
// four floats -> four e4m3 bytes, the first in the lowest byte
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}
__device__ __forceinline__ uint32_t i8x4(float a, float b, float c, float d, float inv) {
  auto q = [inv](float x) {
    const int v = __float2int_rn(__fmul_rn(x, inv));
    return (uint32_t)(min(max(v, -127), 127) & 0xFF);
  };
  return q(a) | (q(b) << 8) | (q(c) << 16) | (q(d) << 24);
}
// 2^d for an integer-valued d <= 0 (0 below the normal range), exactly
__device__ __forceinline__ float exp2_int(float d) {
  return d >= -126.f ? __int_as_float((127 + (int)d) << 23) : 0.f;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float4 ld_bf16x4(const __nv_bfloat16 *p) {
  const uint2 u = *reinterpret_cast<const uint2 *>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
}

// ---------------------------------------------------------------- quantization passes
// q: one warp per (row, head); lane holds 4 of the 128 values.
__global__ void __launch_bounds__(256) quant_q_kernel(const __nv_bfloat16 *__restrict__ q, int ldq, int rows,
                                                      int heads, int8_t *__restrict__ q8, float *__restrict__ sq) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (gw >= rows * heads) return;
  const int row = gw / heads, h = gw - row * heads;
  const float4 x = ld_bf16x4(q + (size_t)row * ldq + h * D + lane * 4);
  const float amax = warp_max(fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
  const float inv = amax > 0.f ? __fdiv_rn(I8_MAX, amax) : 0.f;
  *reinterpret_cast<uint32_t *>(q8 + (size_t)row * heads * D + h * D + lane * 4) = i8x4(x.x, x.y, x.z, x.w, inv);
  if (lane == 0) sq[(size_t)row * heads + h] = __fdiv_rn(amax, I8_MAX);
}

// k amax per (sequence, head): 32 rows x 128 values per CTA -> atomicMax on
// the ordered bits of a non-negative float.
__global__ void __launch_bounds__(256) amax_k_kernel(const __nv_bfloat16 *__restrict__ k, int ldk, int Lk, int heads,
                                                     unsigned *__restrict__ kbits) {
  __shared__ float red[8];
  const int b = blockIdx.z, h = blockIdx.y, r0 = blockIdx.x * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float m = 0.f;
  for (int r = r0 + warp; r < min(r0 + 32, Lk); r += 8) {
    const float4 x = ld_bf16x4(k + ((size_t)b * Lk + r) * ldk + h * D + lane * 4);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
  }
  m = warp_max(m);
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = red[0];
    for (int w = 1; w < 8; ++w) t = fmaxf(t, red[w]);
    atomicMax(kbits + b * heads + h, __float_as_uint(t));
  }
}

__global__ void __launch_bounds__(256) quant_k_kernel(const __nv_bfloat16 *__restrict__ k, int ldk, int Lk, int B,
                                                      int heads, const unsigned *__restrict__ kbits,
                                                      int8_t *__restrict__ k8) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (gw >= B * Lk * heads) return;
  const int row = gw / heads, h = gw - row * heads, b = row / Lk;
  const float amax = __uint_as_float(kbits[b * heads + h]);
  const float inv = amax > 0.f ? __fdiv_rn(I8_MAX, amax) : 0.f;
  const float4 x = ld_bf16x4(k + (size_t)row * ldk + h * D + lane * 4);
  *reinterpret_cast<uint32_t *>(k8 + (size_t)row * heads * D + h * D + lane * 4) = i8x4(x.x, x.y, x.z, x.w, inv);
}

// v amax per (sequence, channel): 256 rows per CTA, one thread per channel of a head.
__global__ void __launch_bounds__(128) amax_v_kernel(const __nv_bfloat16 *__restrict__ v, int ldv, int Lk, int heads,
                                                     unsigned *__restrict__ vbits) {
  const int b = blockIdx.z, h = blockIdx.y, r0 = blockIdx.x * 256, c = threadIdx.x;
  float m = 0.f;
  const __nv_bfloat16 *col = v + (size_t)b * Lk * ldv + h * D + c;
  for (int r = r0; r < min(r0 + 256, Lk); ++r) m = fmaxf(m, fabsf(__bfloat162float(col[(size_t)r * ldv])));
  atomicMax(vbits + ((size_t)b * heads + h) * D + c, __float_as_uint(m));
}

// V^T tile (128 channels x 128 keys of one head) in e4m3; keys >= Lk are 0.
__global__ void __launch_bounds__(256) quant_vt_kernel(const __nv_bfloat16 *__restrict__ v, int ldv, int Lk, int Lkp,
                                                       int heads, const unsigned *__restrict__ vbits,
                                                       uint8_t *__restrict__ vt) {
  __shared__ uint32_t tile[128 * 33];      // [channel][key / 4], padded against bank conflicts
  const int b = blockIdx.z, h = blockIdx.y, j0 = blockIdx.x * TK;
  const int d = threadIdx.x & 127, jg = threadIdx.x >> 7;
  const float amax = __uint_as_float(vbits[((size_t)b * heads + h) * D + d]);
  const float inv = amax > 0.f ? __fdiv_rn(E4M3_MAX, amax) : 0.f;
  const __nv_bfloat16 *col = v + (size_t)b * Lk * ldv + h * D + d;
  for (int it = 0; it < 16; ++it) {
    const int jj = (it * 2 + jg) * 4;
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = j0 + jj + e;
      x[e] = j < Lk ? __fmul_rn(__bfloat162float(col[(size_t)j * ldv]), inv) : 0.f;
    }
    tile[d * 33 + (jj >> 2)] = e4m3x4(x[0], x[1], x[2], x[3]);
  }
  __syncthreads();
  uint8_t *dst = vt + ((size_t)b * heads + h) * D * (size_t)Lkp + j0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = threadIdx.x + 256 * i;
    const int dd = idx >> 3, part = idx & 7;
    const uint32_t *src = tile + dd * 33 + part * 4;
    *reinterpret_cast<uint4 *>(dst + (size_t)dd * Lkp + part * 16) = make_uint4(src[0], src[1], src[2], src[3]);
  }
}

__global__ void amax_to_scale_kernel(float *s, int n, float qmax) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) s[i] = __fdiv_rn(s[i], qmax);
}

// ---------------------------------------------------------------- the attention kernel
__global__ void __launch_bounds__(THREADS, 1)
attn8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
             const __grid_constant__ CUtensorMap tmV, const Fa8Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sKV = smem + 2 * TILE;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sKV + NSLOT * TILE);
  uint64_t *q_full = bars;
  uint64_t *kv_full = bars + 1;
  uint64_t *kv_empty = bars + 1 + NSLOT;
  uint64_t *s_full = bars + 1 + 2 * NSLOT;
  uint64_t *p_ready = s_full + 2;
  uint64_t *pv_done = p_ready + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(pv_done + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  const int q0 = blockIdx.x * 2 * TQ;
  int kl = p.Lk;
  if (p.k_lens) kl = min(max(p.k_lens[b], 0), p.Lk);
  const int nkt = (kl + TK - 1) / TK;

  if (threadIdx.x == 0) *abort_flag = (p.watchdog && *reinterpret_cast<volatile int *>(p.watchdog)) ? 1 : 0;
  __syncthreads();
  if (*abort_flag) return;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(smem_u32(&kv_full[s]), 1);
      mbar_init(smem_u32(&kv_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&p_ready[i]), 4);
      mbar_init(smem_u32(&pv_done[i]), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int vrow = (b * p.heads + h) * D;      // first V^T row of this (sequence, head)

  if (warp >= 8) {
    if (warp == 9) {
      // ------------------------------------------------ TMA producer
      if (lane == 0 && nkt > 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        const uint32_t qb = smem_u32(q_full);
        mbar_arrive_expect_tx(qb, 2 * TILE);
        for (int i = 0; i < 2; ++i) tma_load_3d(smem_u32(sQ + i * TILE), &tmQ, h * D, q0 + i * TQ, b, qb);
        int slot = 0;
        uint32_t phase = 0;
        int fills[NSLOT] = {0, 0, 0, 0, 0, 0, 0, 0};
        bool ok = true;
        for (int j = 0; j < nkt && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv) {
            if (!mbar_wait(smem_u32(&kv_empty[slot]), phase ^ 1, abort_flag, p.watchdog, 0x301)) { ok = false; break; }
            const uint32_t fb = smem_u32(&kv_full[slot]);
            mbar_arrive_expect_tx(fb, TILE);
            if (kv == 0)
              tma_load_3d(smem_u32(sKV + slot * TILE), &tmK, h * D, j * TK, b, fb);
            else
              tma_load_2d(smem_u32(sKV + slot * TILE), &tmV, j * TK, vrow, fb);
            ++fills[slot];
            if (++slot == NSLOT) { slot = 0; phase ^= 1; }
          }
        }
        int never = 0;
        mbar_wait(qb, 0, &never, p.watchdog, 0x302);
        for (int s = 0; s < NSLOT; ++s)
          if (fills[s] > 0) mbar_wait(smem_u32(&kv_full[s]), (fills[s] - 1) & 1, &never, p.watchdog, 0x303);
      }
    } else if (warp == 8) {
      // ------------------------------------------------ MMA issuer (order as in the bf16 kernel)
      if (lane == 0 && nkt > 0) {
        bool ok = mbar_wait(smem_u32(q_full), 0, abort_flag, p.watchdog, 0x311);
        int slot = 0;
        uint32_t phase = 0;
        auto next = [&]() { if (++slot == NSLOT) { slot = 0; phase ^= 1; } };
        auto issue_s = [&](int i, uint32_t kbase) {
          const uint64_t qd = desc_kmajor_sw128(smem_u32(sQ + i * TILE));
          const uint64_t kd = desc_kmajor_sw128(kbase);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)              // 32 bytes of head_dim per MMA
            mma_ss_i8(tmem + i * TK, qd + 2 * kk, kd + 2 * kk, IDESC_S, kk > 0);
          tc_commit(smem_u32(&s_full[i]));
        };
        auto issue_pv = [&](int i, uint32_t vbase, int j) {
          const uint64_t vd = desc_kmajor_sw128(vbase);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)              // 32 keys (8 TMEM columns of P) per MMA
            mma_ts_f8(tmem + 2 * TK + i * D, tmem + i * TK + kk * 8, vd + 2 * kk, IDESC_O, (j > 0 || kk > 0));
          tc_commit(smem_u32(&pv_done[i]));
        };
        int kslot = slot;
        if (ok && mbar_wait(smem_u32(&kv_full[slot]), phase, abort_flag, p.watchdog, 0x312)) {
          tc_fence_after();
          const uint32_t kbase = smem_u32(sKV + slot * TILE);
          issue_s(0, kbase);
          issue_s(1, kbase);
          tc_commit(smem_u32(&kv_empty[kslot]));
          next();
        } else {
          ok = false;
        }
        for (int j = 0; j < nkt && ok; ++j) {
          if (!mbar_wait(smem_u32(&kv_full[slot]), phase, abort_flag, p.watchdog, 0x314)) break;   // V_j
          const int vslot = slot;
          const uint32_t vbase = smem_u32(sKV + slot * TILE);
          next();
          const bool more = j + 1 < nkt;
          uint32_t kbase = 0;
          kslot = slot;
          if (!mbar_wait(smem_u32(&p_ready[0]), j & 1, abort_flag, p.watchdog, 0x315)) break;
          tc_fence_after();
          issue_pv(0, vbase, j);
          if (more) {
            if (!mbar_wait(smem_u32(&kv_full[slot]), phase, abort_flag, p.watchdog, 0x316)) break;   // K_{j+1}
            tc_fence_after();
            kbase = smem_u32(sKV + slot * TILE);
            next();
            issue_s(0, kbase);
          }
          if (!mbar_wait(smem_u32(&p_ready[1]), j & 1, abort_flag, p.watchdog, 0x317)) break;
          tc_fence_after();
          issue_pv(1, vbase, j);
          tc_commit(smem_u32(&kv_empty[vslot]));
          if (more) {
            issue_s(1, kbase);
            tc_commit(smem_u32(&kv_empty[kslot]));
          }
        }
      }
    }
  } else {
    // ------------------------------------------------ softmax (warps 0..7)
    const int i = warp >> 2;
    const int qw = warp & 3;
    const int row = q0 + i * TQ + qw * 32 + lane;
    const uint32_t lane_off = (uint32_t)(qw * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + i * TK;
    const uint32_t o_addr = tmem + lane_off + 2 * TK + i * D;
    float m = -INFINITY, l = 0.f;
    float crow = 0.f;                            // logit scale of this row (log2 units per unit of S)
    if (row < p.Lq) {
      crow = p.c * p.sq[((size_t)b * p.Lq + row) * p.heads + h] * p.sk[b * p.heads + h];
      if (p.q_ss) {
        const float *qs = p.q_ss + (size_t)(b * p.Lq + row) * p.q_ss_stride;
        float sum = 0.f;
        for (int t = 0; t < p.q_ss_parts; ++t) sum += qs[t];
        crow *= rsqrtf(sum * p.q_ss_inv_n + p.q_ss_eps);
      }
    }
    // an all-zero q row (scale 0) attends uniformly; a positive c keeps the
    // masked keys at -inf instead of 0 * inf
    if (!(crow > 0.f)) crow = 1e-30f;
    bool ok = true;
    for (int j = 0; j < nkt; ++j) {
      if (!mbar_wait(smem_u32(&s_full[i]), j & 1, abort_flag, p.watchdog, 0x321)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));
      tmem_ld_wait();
      // s32 -> float 1.5 * 2^23 + S (exact for |S| < 2^22)
#pragma unroll
      for (int k = 0; k < 128; ++k) s[k] += MAGIC;
      const int kvalid = kl - j * TK;
      if (kvalid < TK) {
#pragma unroll
        for (int k = 0; k < 128; ++k)
          if (k >= kvalid) s[k] = 0xff800000u;     // -inf
      }
      float mx[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mx[a] = fmax3(__uint_as_float(s[a]), __uint_as_float(s[8 + a]), __uint_as_float(s[16 + a]));
#pragma unroll
      for (int k = 24; k < 120; k += 16) {
#pragma unroll
        for (int a = 0; a < 8; ++a) mx[a] = fmax3(mx[a], __uint_as_float(s[k + a]), __uint_as_float(s[k + 8 + a]));
      }
#pragma unroll
      for (int a = 0; a < 8; ++a) mx[a] = fmaxf(mx[a], __uint_as_float(s[120 + a]));
      const float traw = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
      const float tmax = (traw - MAGIC_F) * crow;
      const bool need = (tmax > m) || (m == -INFINITY);
      const float mnew = need ? 8.f * ceilf(tmax * 0.125f) : m;
      const float alpha = (need && j > 0) ? exp2_int(m - mnew) : 1.0f;
      m = mnew;
      // x = (S_f - 1.5 * 2^23) c - m + 8 as one FMA per element
      const float nb = -fmaf(MAGIC_F, crow, m - 8.f);
      const float2 c2 = make_float2(crow, crow);
      const float2 nb2 = make_float2(nb, nb);
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int k = c * 64 + 4 * e;
          const float2 x0 = ffma2(make_float2(__uint_as_float(s[k]), __uint_as_float(s[k + 1])), c2, nb2);
          const float2 x1 = ffma2(make_float2(__uint_as_float(s[k + 2]), __uint_as_float(s[k + 3])), c2, nb2);
          const float2 p0 = make_float2(ex2(x0.x), ex2(x0.y));
          const float2 p1 = make_float2(ex2(x1.x), ex2(x1.y));
          acc0 = fadd2(acc0, p0);
          acc1 = fadd2(acc1, p1);
          pk[e] = e4m3x4(p0.x, p0.y, p1.x, p1.y);
        }
        tmem_st16(s_addr + c * 16, pk);
      }
      const float2 acc = fadd2(acc0, acc1);
      l = l * alpha + (acc.x + acc.y);
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        if (!mbar_wait(smem_u32(&pv_done[i]), (j - 1) & 1, abort_flag, p.watchdog, 0x322)) ok = false;
        __syncwarp();
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[16];
          tmem_ld16(o_addr + c * 16, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st16(o_addr + c * 16, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&p_ready[i]));
      if (!ok) break;
    }
    // epilogue: O / l times the channel scales of v -> bf16
    if (ok && nkt > 0) {
      ok = mbar_wait(smem_u32(&pv_done[i]), (nkt - 1) & 1, abort_flag, p.watchdog, 0x323);
      tc_fence_after();
    }
    const float inv = (l > 0.f) ? 1.0f / l : 0.f;
    const float *svh = p.sv + ((size_t)b * p.heads + h) * D;
    __nv_bfloat16 *orow = p.o + (size_t)(b * p.Lq + (row < p.Lq ? row : 0)) * p.ldo + h * D;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t o[32];
      if (nkt > 0) {
        tmem_ld32(o_addr + c * 32, o);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (row < p.Lq && ok) {
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(o[e]) * inv * svh[c * 32 + e];
        uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_uint4(pack_bf16(f[8 * e + 0], f[8 * e + 1]), pack_bf16(f[8 * e + 2], f[8 * e + 3]),
                              pack_bf16(f[8 * e + 4], f[8 * e + 5]), pack_bf16(f[8 * e + 6], f[8 * e + 7]));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tmem, TMEM_COLS);
}

struct Ws8 {
  int8_t *q8, *k8;
  uint8_t *vt;
  float *sq, *sk, *sv;
  size_t total;
};

size_t al256(size_t v) { return (v + 255) & ~(size_t)255; }

Ws8 ws8_layout(void *base, int B, int heads, int Lq, int Lk) {
  Ws8 w = {};
  const size_t Lkp = (size_t)((Lk + TK - 1) / TK) * TK;
  const size_t sz[6] = {(size_t)B * Lq * heads * D, (size_t)B * Lk * heads * D, (size_t)B * heads * D * (Lkp ? Lkp : TK),
                        (size_t)B * Lq * heads * 4, (size_t)B * heads * 4, (size_t)B * heads * D * 4};
  size_t off[6], o = 0;
  for (int i = 0; i < 6; ++i) {
    off[i] = o;
    o += al256(sz[i]);
  }
  w.total = o;
  if (!base) return w;
  char *c = static_cast<char *>(base);
  w.q8 = reinterpret_cast<int8_t *>(c + off[0]);
  w.k8 = reinterpret_cast<int8_t *>(c + off[1]);
  w.vt = reinterpret_cast<uint8_t *>(c + off[2]);
  w.sq = reinterpret_cast<float *>(c + off[3]);
  w.sk = reinterpret_cast<float *>(c + off[4]);
  w.sv = reinterpret_cast<float *>(c + off[5]);
  return w;
}
}  // namespace

size_t attention_8bit_ws_bytes(int B, int heads, int Lq, int Lk) {
  return ws8_layout(nullptr, B, heads, Lq, Lk).total;
}

bool attention_8bit_supported(const AttnArgs &a) {
  if (a.d != D || a.B < 1 || a.Lq < 1 || a.Lk < 1) return false;
  if (a.ldq % 8 || a.ldk % 8 || a.ldv % 8 || a.ldo % 8) return false;
  if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.o)) return false;
  if ((a.heads * D) % 16) return false;
  if (a.heads > 65535 || a.B > 65535) return false;
  return true;
}

int attention_8bit(const AttnArgs &a, void *workspace, cudaStream_t s) {
  if (!attention_8bit_supported(a)) return set_error(WAN_EUNSUPPORTED, "attention_8bit");
  const Ws8 w = ws8_layout(workspace, a.B, a.heads, a.Lq, a.Lk);
  const int Lkp = ((a.Lk + TK - 1) / TK) * TK;
  const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(a.q);
  const __nv_bfloat16 *k = static_cast<const __nv_bfloat16 *>(a.k);
  const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(a.v);
  unsigned *kbits = reinterpret_cast<unsigned *>(w.sk);
  unsigned *vbits = reinterpret_cast<unsigned *>(w.sv);
  // quantization passes
  {
    const size_t warps_q = (size_t)a.B * a.Lq * a.heads;
    quant_q_kernel<<<(unsigned)((warps_q * 32 + 255) / 256), 256, 0, s>>>(q, a.ldq, a.B * a.Lq, a.heads, w.q8, w.sq);
    WAN_TRY_CUDA(cudaMemsetAsync(w.sk, 0, (size_t)a.B * a.heads * 4, s), "attention_8bit: clear k amax");
    WAN_TRY_CUDA(cudaMemsetAsync(w.sv, 0, (size_t)a.B * a.heads * D * 4, s), "attention_8bit: clear v amax");
    amax_k_kernel<<<dim3((a.Lk + 31) / 32, a.heads, a.B), 256, 0, s>>>(k, a.ldk, a.Lk, a.heads, kbits);
    amax_v_kernel<<<dim3((a.Lk + 255) / 256, a.heads, a.B), 128, 0, s>>>(v, a.ldv, a.Lk, a.heads, vbits);
    const size_t warps_k = (size_t)a.B * a.Lk * a.heads;
    quant_k_kernel<<<(unsigned)((warps_k * 32 + 255) / 256), 256, 0, s>>>(k, a.ldk, a.Lk, a.B, a.heads, kbits, w.k8);
    quant_vt_kernel<<<dim3(Lkp / TK, a.heads, a.B), 256, 0, s>>>(v, a.ldv, a.Lk, Lkp, a.heads, vbits, w.vt);
    amax_to_scale_kernel<<<(a.B * a.heads + 255) / 256, 256, 0, s>>>(w.sk, a.B * a.heads, I8_MAX);
    amax_to_scale_kernel<<<(a.B * a.heads * D + 255) / 256, 256, 0, s>>>(w.sv, a.B * a.heads * D, E4M3_MAX);
    WAN_CHECK_LAUNCH("attention_8bit quantization");
  }
  CUtensorMap tq, tk, tv;
  const uint64_t inner = (uint64_t)a.heads * D;
  int rc = encode_tmap_3d_u8(&tq, w.q8, inner, a.Lq, a.B, inner, (uint64_t)a.Lq * inner, 128, TQ);
  if (rc) return rc;
  if ((rc = encode_tmap_3d_u8(&tk, w.k8, inner, a.Lk, a.B, inner, (uint64_t)a.Lk * inner, 128, TK))) return rc;
  if ((rc = encode_tmap_2d_u8(&tv, w.vt, Lkp, (uint64_t)a.B * a.heads * D, Lkp, 128, 128))) return rc;
  static bool attr_set = false;
  if (!attr_set) {
    WAN_TRY_CUDA(cudaFuncSetAttribute(attn8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
                 "attention_8bit smem attribute");
    attr_set = true;
  }
  Fa8Params p = {};
  p.B = a.B; p.heads = a.heads; p.Lq = a.Lq; p.Lk = a.Lk; p.k_lens = a.k_lens;
  p.c = a.scale * 1.4426950408889634f;
  p.sq = w.sq; p.sk = w.sk; p.sv = w.sv;
  p.q_ss = a.q_ss; p.q_ss_stride = a.q_ss_stride; p.q_ss_parts = a.q_ss_parts;
  p.q_ss_inv_n = a.q_ss_n > 0.f ? 1.0f / a.q_ss_n : 0.f; p.q_ss_eps = a.q_ss_eps;
  p.o = static_cast<__nv_bfloat16 *>(a.o); p.ldo = a.ldo;
  p.watchdog = watchdog_ptr();
  dim3 grid((a.Lq + 2 * TQ - 1) / (2 * TQ), a.heads, a.B);
  attn8_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(tq, tk, tv, p);
  WAN_CHECK_LAUNCH("attention_8bit");
  return WAN_OK;
}

}  // namespace wan

// Tensor-core GEMM for sm_100a: C = A B^T (+ bias) with fused epilogues,
// bf16 operands, fp32 accumulation in TMEM.
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles, K in steps of 64:
//   warp 0      TMA producer: A tile 128x64 and B tile 256x64 per stage into
//               a 4-stage ring (128-byte swizzle), completion on mbarriers;
//   warp 1      MMA issuer: one thread issues tcgen05.mma (M=128, N=256,
//               K=16) x 4 per stage into one of two TMEM accumulators
//               (2 x 256 fp32 columns), commits free the stage / publish
//               the accumulator;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31 = tile rows), bias, GELU or gated
//               residual, stores to global; the second accumulator lets the
//               next tile's MMAs run under this epilogue.
// Tiles are walked in groups of 16 M-tiles so a wave of CTAs shares A and B
// panels in L2. Every wait is bounded (sm100::mbar_wait).
#include "common.cuh"
#include "sm100.cuh"

namespace wan {

namespace {
using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;                   // 16 KB
constexpr int B_BYTES = BN * BK * 2;                   // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr int GROUP_M = 16;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_bf16(BM, BN, 0);
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;

struct TcParams {
  int M, N, K, segN;
  int num_m, num_n, num_tiles, num_k;
  const void *bias[3];
  void *C; int ldc;
  float *X; int ldx;
  const float *gate; int gate_stride; int rows_per_gate;
  int *watchdog;
};

__device__ __forceinline__ void tile_coords(int t, const TcParams &p, int &mb, int &nb) {
  const int group = GROUP_M * p.num_n;
  const int g = t / group;
  const int first_m = g * GROUP_M;
  const int gm = min(p.num_m - first_m, GROUP_M);
  const int r = t - g * group;
  mb = first_m + r % gm;
  nb = r / gm;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t lo16) {
  return __uint_as_float(lo16 << 16);
}

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
               const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
               const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * A_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
  uint64_t *full = bars, *empty = bars + STAGES, *tfull = bars + 2 * STAGES, *tempty = bars + 2 * STAGES + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 4);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // A CTA that starts after another one gave up a wait skips its work, so a
  // failed launch ends within a few waits instead of one per CTA.
  if (threadIdx.x == 0) *abort_flag = (p.watchdog && *reinterpret_cast<volatile int *>(p.watchdog)) ? 1 : 0;
  __syncthreads();
  if (*abort_flag) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmB2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int fills[STAGES] = {0, 0, 0, 0};
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        const int n0 = nb * BN;
        const int seg = n0 / p.segN;
        const CUtensorMap *bm = seg == 0 ? &tmB0 : (seg == 1 ? &tmB1 : &tmB2);
        const int nn0 = n0 - seg * p.segN;
        for (int kb = 0; kb < p.num_k; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, p.watchdog, 0x101)) { ok = false; break; }
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          tma_load_2d(smem_u32(sA + stage * A_BYTES), &tmA, kb * BK, mb * BM, fb);
          tma_load_2d(smem_u32(sB + stage * B_BYTES), bm, kb * BK, nn0, fb);
          ++fills[stage];
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // drain: every issued copy has landed before the CTA may exit
      int never = 0;
      for (int s = 0; s < STAGES; ++s)
        if (fills[s] > 0) mbar_wait(smem_u32(&full[s]), (fills[s] - 1) & 1, &never, p.watchdog, 0x102);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int i = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++i) {
        const int buf = i & 1;
        const uint32_t acc_phase = (i >> 1) & 1;
        if (!mbar_wait(smem_u32(&tempty[buf]), acc_phase ^ 1, abort_flag, p.watchdog, 0x111)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * BN;
        for (int kb = 0; kb < p.num_k; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, p.watchdog, 0x112)) { ok = false; break; }
          tc_fence_after();
          const uint64_t a0 = desc_kmajor_sw128(smem_u32(sA + stage * A_BYTES));
          const uint64_t b0 = desc_kmajor_sw128(smem_u32(sB + stage * B_BYTES));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss(d, a0 + 2 * kk, b0 + 2 * kk, IDESC, (kb | kk) != 0);
          tc_commit(smem_u32(&empty[stage]));
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (ok) tc_commit(smem_u32(&tfull[buf]));
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    int i = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++i) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int buf = i & 1;
      const uint32_t acc_phase = (i >> 1) & 1;
      if (!mbar_wait(smem_u32(&tfull[buf]), acc_phase, abort_flag, p.watchdog, 0x121)) break;
      tc_fence_after();
      const int m = mb * BM + row;
      const int n0 = nb * BN;
      const int seg = n0 / p.segN;
      const __nv_bfloat16 *bias = static_cast<const __nv_bfloat16 *>(p.bias[seg]);
      const int nn0 = n0 - seg * p.segN;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN + c * 32, r);
        tmem_ld_wait();
        if (c == BN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&tempty[buf]));
        }
        const int n = n0 + c * 32;
        if (m >= p.M || n >= p.N) continue;
        float v[32];
        const uint4 *bp = reinterpret_cast<const uint4 *>(bias + nn0 + c * 32);
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          const uint4 bb = bias ? bp[j4] : make_uint4(0, 0, 0, 0);
          const uint32_t w[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            v[j4 * 8 + 2 * e] = __uint_as_float(r[j4 * 8 + 2 * e]) + bf16_bits_to_float(w[e] & 0xFFFFu);
            v[j4 * 8 + 2 * e + 1] = __uint_as_float(r[j4 * 8 + 2 * e + 1]) + bf16_bits_to_float(w[e] >> 16);
          }
        }
        if (EPI == EPI_RESID) {
          float *xr = p.X + (size_t)m * p.ldx + n;
          const float *gr = p.gate ? p.gate + (size_t)(m / p.rows_per_gate) * p.gate_stride + n : nullptr;
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            float4 xv = *reinterpret_cast<const float4 *>(xr + j);
            const float4 gv = gr ? *reinterpret_cast<const float4 *>(gr + j) : make_float4(1.f, 1.f, 1.f, 1.f);
            xv.x = fmaf(gv.x, v[j + 0], xv.x);
            xv.y = fmaf(gv.y, v[j + 1], xv.y);
            xv.z = fmaf(gv.z, v[j + 2], xv.z);
            xv.w = fmaf(gv.w, v[j + 3], xv.w);
            *reinterpret_cast<float4 *>(xr + j) = xv;
          }
        } else {
          __nv_bfloat16 *cr = static_cast<__nv_bfloat16 *>(p.C) + (size_t)m * p.ldc + n;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            float a[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) a[e] = (EPI == EPI_GELU) ? gelu_tanh(v[j + e]) : v[j + e];
            __nv_bfloat162 h0 = __floats2bfloat162_rn(a[0], a[1]);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(a[2], a[3]);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(a[4], a[5]);
            __nv_bfloat162 h3 = __floats2bfloat162_rn(a[6], a[7]);
            uint4 u;
            u.x = *reinterpret_cast<uint32_t *>(&h0);
            u.y = *reinterpret_cast<uint32_t *>(&h1);
            u.z = *reinterpret_cast<uint32_t *>(&h2);
            u.w = *reinterpret_cast<uint32_t *>(&h3);
            *reinterpret_cast<uint4 *>(cr + j) = u;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

template <int EPI>
int launch(const CUtensorMap &ta, const CUtensorMap *tb, const TcParams &p, cudaStream_t s) {
  static bool attr_set = false;     // per process; the attribute is per function
  if (!attr_set) {
    WAN_TRY_CUDA(cudaFuncSetAttribute(gemm_tc_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
                 "gemm_tc smem attribute");
    attr_set = true;
  }
  const int grid = p.num_tiles < sm_count() ? p.num_tiles : sm_count();
  gemm_tc_kernel<EPI><<<grid, THREADS, SMEM_BYTES, s>>>(ta, tb[0], tb[1], tb[2], p);
  WAN_CHECK_LAUNCH("gemm_tc");
  return WAN_OK;
}
}  // namespace

bool gemm_tc_supported(const GemmArgs &g) {
  if (g.M < 1 || g.N < 32 || g.K < BK || g.K % BK || g.N % 32) return false;
  if (g.nseg < 1 || g.nseg > 3 || g.segN * g.nseg != g.N) return false;
  if (g.nseg > 1 && g.segN % BN) return false;
  if (g.lda % 8) return false;
  if (g.epi != EPI_RESID && g.ldc % 8) return false;
  if (g.epi == EPI_RESID && (g.ldx % 4 || (g.gate && g.gate_stride % 4))) return false;
  for (int i = 0; i < g.nseg; ++i)
    if (!aligned16(g.Bseg[i]) || (g.bias[i] && !aligned16(g.bias[i]))) return false;
  return aligned16(g.A);
}

int gemm_tc(const GemmArgs &g, cudaStream_t s) {
  if (!gemm_tc_supported(g)) return set_error(WAN_EUNSUPPORTED, "gemm_tc: M=%d N=%d K=%d", g.M, g.N, g.K);
  CUtensorMap ta, tb[3];
  int rc = encode_tmap_2d_bf16(&ta, g.A, g.K, g.M, (uint64_t)g.lda * 2, BK, BM);
  if (rc) return rc;
  for (int i = 0; i < 3; ++i) {
    const int si = i < g.nseg ? i : 0;
    if ((rc = encode_tmap_2d_bf16(&tb[i], g.Bseg[si], g.K, g.segN, (uint64_t)g.K * 2, BK, BN))) return rc;
  }
  TcParams p = {};
  p.M = g.M; p.N = g.N; p.K = g.K; p.segN = g.segN;
  p.num_m = (g.M + BM - 1) / BM;
  p.num_n = (g.N + BN - 1) / BN;
  p.num_tiles = p.num_m * p.num_n;
  p.num_k = g.K / BK;
  for (int i = 0; i < 3; ++i) p.bias[i] = i < g.nseg ? g.bias[i] : nullptr;
  p.C = g.C; p.ldc = g.ldc; p.X = g.X; p.ldx = g.ldx;
  p.gate = g.gate; p.gate_stride = g.gate_stride; p.rows_per_gate = g.rows_per_gate > 0 ? g.rows_per_gate : 1;
  p.watchdog = watchdog_ptr();
  switch (g.epi) {
    case EPI_STORE: return launch<EPI_STORE>(ta, tb, p, s);
    case EPI_GELU: return launch<EPI_GELU>(ta, tb, p, s);
    default: return launch<EPI_RESID>(ta, tb, p, s);
  }
}

}  // namespace wan

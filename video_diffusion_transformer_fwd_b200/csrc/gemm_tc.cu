// Tensor-core GEMM for sm_100a: C = A B^T (+ bias) with fused epilogues,
// bf16 operands, fp32 accumulation in TMEM. The FP8 variant takes e4m3
// operands with one scale per row of A (per token) and one per weight tensor
// ("Wan paper deep dive" (charles2530.github.io), inference-optimisation
// table, "FP8 GEMM"): a stage holds 128 e4m3 per row instead of 64 bf16 (the
// same 128 bytes), and the epilogue multiplies the accumulator by
// a_scale[m] * b_scale before the bias.
//
// Persistent kernel on CTA pairs (clusters of 2, one CTA per SM) with
// tcgen05.mma.cta_group::2 (M = 256 split 128/128 across the two CTAs' TMEM,
// N = 256 per instruction, K = 16), K in steps of 64, in two tile widths:
//   wide   256 x 512 output tiles (two N = 256 products per K step sharing
//          the A stage): per CTA a stage holds 128 rows of A and 256 rows
//          of B (48 KB), 4 stages; one 512-column TMEM accumulator; 8
//          epilogue warps. A is read once per 512 output columns, so the
//          operand traffic from L2 per flop is 3/4 of the narrow tile's.
//   narrow 256 x 256 tiles, 32 KB stages, 6 stages, two 256-column TMEM
//          accumulators (the epilogue of one tile overlaps the next
//          tile's products), 4 epilogue warps; used when K < 4096 (there
//          the wide tile's epilogue, which cannot overlap, costs more than
//          its saving in operand traffic) or a weight segment is not a
//          multiple of 512 columns.
// Warp roles:
//   warp 0      TMA producer in both CTAs: this CTA's 128 rows of A and its
//               half of B per stage (128-byte swizzle); bytes of both CTAs
//               are counted on the leader CTA's "full" barrier;
//   warp 1      MMA issuer (leader CTA only); commits free the stage in both
//               CTAs and publish the accumulator to both CTAs' epilogues;
//   warps 2..   epilogue in both CTAs: tcgen05.ld of this CTA's 128 rows
//               (warp w reads TMEM lanes 32*(w%4)..+31; in the wide tile
//               warps 2-5 take columns 0-255 and warps 6-9 columns 256-511),
//               bias, GELU or gated residual, stores to global (the residual
//               add x += g*y goes through a swizzled smem tile and a TMA
//               reduce-add into x, or a TMA store when x is written rather
//               than accumulated); then a release arrive on the leader's
//               "accumulator empty" barrier.
// Tiles are walked in groups of 8 M-tiles (2048 rows) so a wave of pairs
// shares A and B panels in L2. Every wait is bounded (sm100::mbar_wait).
#include "common.cuh"
#include "sm100.cuh"

namespace wan {

namespace {
using namespace sm100;

constexpr int BM = 128;                  // rows per CTA (256 per pair)
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;     // 16 KB
constexpr int GROUP_M = 8;               // pair tiles (256 rows) per raster group
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_bf16(2 * BM, 256, 0);
constexpr uint32_t IDESC8 = idesc_e4m3(2 * BM, 256);
constexpr int BK8 = 128;                 // e4m3 elements per stage row (128 bytes)
constexpr int STG_BYTES = 32 * 32 * 4;  // one warp's 32 x 32 fp32 staging tile (128-byte swizzle)
constexpr bool USE_WIDE = true;          // 256 x 512 tiles wherever the shape allows

// Tile geometry of the two variants.
template <bool WIDE>
struct Geo {
  static constexpr int BN = WIDE ? 512 : 256;              // output columns per pair tile
  static constexpr int STAGES = WIDE ? 4 : 6;
  static constexpr int B_BYTES = (BN / 2) * BK * 2;        // this CTA's half of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_WARPS = WIDE ? 8 : 4;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int NACC = WIDE ? 1 : 2;                // TMEM accumulators (BN columns each)
  static constexpr int NSTG = WIDE ? 1 : 2;                // residual staging tiles per epilogue warp
  static constexpr int EPI_SMEM = EPI_WARPS * NSTG * STG_BYTES;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_SMEM + 256;
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static_assert(NACC * BN <= (int)TMEM_COLS, "TMEM columns");
};

struct TcParams {
  int M, N, K, segN;
  int num_m, num_n, num_tiles, num_k;
  const void *bias[3];
  void *C; int ldc;
  float *X; int ldx;
  const float *gate; int gate_stride; int rows_per_gate; int x_store;
  const float *gate_bias;
  const float *a_scale; const float *b_scale[3];      // FP8: per row of A, per weight segment
  // q/k RMSNorm + RoPE epilogue (EPI_QKNORM)
  const float *gamma[3]; float *ss; int ss_stride; int ss_col[3];
  const float *rope; int rope_mask; int rope_vec; int L, H, W; int head_dim; int tok0;   // L: rows per sequence
  int *watchdog;
  const void *ss_hi; int *dbg;            // debug bounds checks: end of ss
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

// GELU (tanh form) for a bf16 output: tanh from the hardware approximation
// (tanh.approx.f32, relative error about 2^-11), below the bf16 rounding of
// the result (2^-9).
__device__ __forceinline__ float gelu_tanh_bf16out(float z) {
  const float k0 = 0.7978845608028654f, k1 = 0.044715f;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(k0 * fmaf(k1 * z, z * z, z)));
  return 0.5f * z * (1.0f + t);
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t lo16) {
  return __uint_as_float(lo16 << 16);
}

template <int EPI, bool F8, bool WIDE>
__global__ void __launch_bounds__(Geo<WIDE>::THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
               const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
               const __grid_constant__ CUtensorMap tmX, const TcParams p) {
  using G = Geo<WIDE>;
  constexpr int BN = G::BN, STAGES = G::STAGES, B_BYTES = G::B_BYTES, STAGE_BYTES = G::STAGE_BYTES;
  constexpr int NACC = G::NACC, NSTG = G::NSTG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * A_BYTES;
  uint8_t *sE = smem + STAGES * STAGE_BYTES;      // epilogue staging (residual epilogue)
  uint64_t *bars = reinterpret_cast<uint64_t *>(sE + G::EPI_SMEM);
  uint64_t *full = bars, *empty = bars + STAGES, *tfull = bars + 2 * STAGES, *tempty = bars + 2 * STAGES + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 4);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile uint32_t *skip = reinterpret_cast<volatile uint32_t *>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  // The leader decides for both CTAs whether to skip (a wait of an earlier
  // CTA already gave up), so the pair always takes the same path. The first
  // cluster barrier guarantees the peer is running before its shared memory
  // is written.
  cluster_sync_all();
  if (leader && threadIdx.x == 0) {
    const uint32_t v = (p.watchdog && *reinterpret_cast<volatile int *>(p.watchdog)) ? 1u : 0u;
    *skip = v;
    st_shared_cluster_u32(mapa_shared(smem_u32((const void *)skip), 1), v);
  }
  cluster_sync_all();
  if (*skip) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 2 * G::EPI_WARPS);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmB2);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();               // barrier inits of both CTAs visible before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int fills[STAGES];
#pragma unroll
      for (int st = 0; st < STAGES; ++st) fills[st] = 0;
      bool ok = true;
      for (int t = pair; t < p.num_tiles && ok; t += npairs) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        const int n0 = nb * BN;
        const int seg = n0 / p.segN;
        const CUtensorMap *bm = seg == 0 ? &tmB0 : (seg == 1 ? &tmB1 : &tmB2);
        const int a_row = mb * 2 * BM + (int)rank * BM;
        const int b_row = n0 - seg * p.segN + (int)rank * 128;   // this CTA's 128 rows of each N = 256 half
        for (int kb = 0; kb < p.num_k; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, p.watchdog, 0x101)) { ok = false; break; }
          const uint32_t fb_local = smem_u32(&full[stage]);
          if (leader) mbar_arrive_expect_tx(fb_local, 2 * STAGE_BYTES);
          const uint32_t fb = mapa_shared(fb_local, 0);
          const int kx = kb * (F8 ? BK8 : BK);
          tma_load_2d_pair(smem_u32(sA + stage * A_BYTES), &tmA, kx, a_row, fb);
          tma_load_2d_pair(smem_u32(sB + stage * B_BYTES), bm, kx, b_row, fb);
          if (WIDE)      // the second N = 256 half of the tile: B rows 256 further
            tma_load_2d_pair(smem_u32(sB + stage * B_BYTES + B_BYTES / 2), bm, kx, b_row + 256, fb);
          ++fills[stage];
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // drain (leader): every issued copy of the pair has landed before exit.
      // The peer's copies complete on the leader's barrier, so the leader's
      // drain also covers them; the final cluster barrier orders the rest.
      if (leader) {
        int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if (fills[s] > 0) mbar_wait(smem_u32(&full[s]), (fills[s] - 1) & 1, &never, p.watchdog, 0x102);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int i = 0;
      bool ok = true;
      for (int t = pair; t < p.num_tiles && ok; t += npairs, ++i) {
        const int buf = i % NACC;
        const uint32_t acc_phase = (i / NACC) & 1;
        if (!mbar_wait(smem_u32(&tempty[buf]), acc_phase ^ 1, abort_flag, p.watchdog, 0x111)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * BN;
        for (int kb = 0; kb < p.num_k; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, p.watchdog, 0x112)) { ok = false; break; }
          tc_fence_after();
          const uint64_t a0 = desc_kmajor_sw128(smem_u32(sA + stage * A_BYTES));
          const uint64_t b0 = desc_kmajor_sw128(smem_u32(sB + stage * B_BYTES));
          // 4 MMAs of 32 bytes of K per stage (16 bf16 or 32 e4m3 each):
          // the descriptor start address advances 32 bytes (2 in 16-byte units)
#pragma unroll
          for (int h = 0; h < BN / 256; ++h) {
            // N = 256 half h: B rows of this half at + h * B_BYTES / 2, accumulator columns + 256 h
            const uint64_t bh = b0 + (uint64_t)((h * (B_BYTES / 2)) >> 4);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              if (F8)
                mma_ss_pair_f8(d + 256 * h, a0 + 2 * kk, bh + 2 * kk, IDESC8, (kb | kk) != 0);
              else
                mma_ss_pair(d + 256 * h, a0 + 2 * kk, bh + 2 * kk, IDESC, (kb | kk) != 0);
            }
          }
          const uint32_t eb = smem_u32(&empty[stage]);
          tc_commit_pair(eb);
          tc_commit_pair(mapa_shared(eb, 1));
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (ok) {
          const uint32_t fb = smem_u32(&tfull[buf]);
          tc_commit_pair(fb);
          tc_commit_pair(mapa_shared(fb, 1));
        }
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2.., both CTAs)
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int ew = warp - 2;                 // epilogue warp index
    const int hcol = WIDE ? (ew >> 2) * 256 : 0;   // first tile column of this warp's 256
    const int row = q * 32 + lane;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[NACC - 1]), 0);
    int stg_count = 0;
    int i = 0;
    for (int t = pair; t < p.num_tiles; t += npairs, ++i) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int buf = i % NACC;
      const uint32_t acc_phase = (i / NACC) & 1;
      const int m = mb * 2 * BM + (int)rank * BM + row;
      const int n0 = nb * BN + hcol;          // this warp's first column
      const int seg = (nb * BN) / p.segN;
      const __nv_bfloat16 *bias = static_cast<const __nv_bfloat16 *>(p.bias[seg]);
      const int nn0 = n0 - seg * p.segN;
      float rs = 1.f;                        // FP8: dequantization factor of this row
      if (F8) rs = (m < p.M ? p.a_scale[m] : 0.f) * *p.b_scale[seg];
      // q/k RMSNorm + RoPE epilogue: per-row sum of squares of y, gamma, rotation
      float sq = 0.f;
      int ss_col = -1, tpos = 0, hpos = 0, wpos = 0;
      bool do_rope = false;
      const float *gam = nullptr;
      if (EPI == EPI_QKNORM) {
        ss_col = p.ss_col[seg];
        gam = p.gamma[seg];
        do_rope = (p.rope_mask >> seg) & 1;
        const int tok = p.tok0 + (m < p.M ? m : 0) % p.L;
        tpos = tok / (p.H * p.W);
        hpos = (tok / p.W) % p.H;
        wpos = tok % p.W;
      }
      // Per-column operands, read while the tile's products still run and
      // spread over the warp: lane l holds columns 8 l .. 8 l + 7 of the warp's
      // 256 (the bias as 8 bf16; gamma, or the gate row when all 32 rows of
      // the warp share one, as 8 floats); each chunk takes them by shuffles.
      const int m0w = mb * 2 * BM + (int)rank * BM + q * 32;       // the warp's first row (warp-uniform)
      const bool lane_cols = n0 + 8 * lane + 8 <= p.N;
      uint4 bias8 = make_uint4(0u, 0u, 0u, 0u);
      float4 col_lo = make_float4(1.f, 1.f, 1.f, 1.f), col_hi = col_lo;
      if (bias && lane_cols) bias8 = *reinterpret_cast<const uint4 *>(bias + nn0 + 8 * lane);
      if (EPI == EPI_QKNORM && gam && lane_cols) {
        col_lo = *reinterpret_cast<const float4 *>(gam + nn0 + 8 * lane);
        col_hi = *reinterpret_cast<const float4 *>(gam + nn0 + 8 * lane + 4);
      }
      bool gate_shared = false;
      if (EPI == EPI_RESID && p.gate && !p.gate_bias && p.rows_per_gate > 1 && m0w < p.M &&
          m0w / p.rows_per_gate == min(m0w + 31, p.M - 1) / p.rows_per_gate) {
        gate_shared = true;
        if (lane_cols) {
          const float *gp = p.gate + (size_t)(m0w / p.rows_per_gate) * p.gate_stride + n0 + 8 * lane;
          col_lo = *reinterpret_cast<const float4 *>(gp);
          col_hi = *reinterpret_cast<const float4 *>(gp + 4);
        }
      }
      // the RoPE-table lines of this row go to L1 meanwhile
      if (n0 < p.N) {
        if (EPI == EPI_QKNORM && do_rope && p.head_dim == 128) {
          // one table row is 64 pairs (512 bytes): t pairs [0, 22), h [22, 43), w [43, 64)
          const char *rt = reinterpret_cast<const char *>(p.rope + (size_t)tpos * 128);
          const char *rh = reinterpret_cast<const char *>(p.rope + (size_t)hpos * 128);
          const char *rw = reinterpret_cast<const char *>(p.rope + (size_t)wpos * 128);
          prefetch_l1(rt); prefetch_l1(rt + 128); prefetch_l1(rt + 168);
          prefetch_l1(rh + 176); prefetch_l1(rh + 296); prefetch_l1(rh + 336);
          prefetch_l1(rw + 344); prefetch_l1(rw + 464); prefetch_l1(rw + 504);
        }
      }
      if (!mbar_wait(smem_u32(&tfull[buf]), acc_phase, abort_flag, p.watchdog, 0x121)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + buf * BN + hcol + c * 32, r);
        tmem_ld_wait();
        if (c == 7) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
        }
        const int n = n0 + c * 32;
        // warp-uniform: rows of the warp beyond M are clipped by the tensor map
        if (m0w >= p.M || n >= p.N) continue;
        float v[32];
        // column j of the chunk is column 32 c + j of the warp: lane 4 c + j / 8 holds it
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          const uint32_t w[4] = {__shfl_sync(0xffffffffu, bias8.x, 4 * c + j4),
                                 __shfl_sync(0xffffffffu, bias8.y, 4 * c + j4),
                                 __shfl_sync(0xffffffffu, bias8.z, 4 * c + j4),
                                 __shfl_sync(0xffffffffu, bias8.w, 4 * c + j4)};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (F8) {
              v[j4 * 8 + 2 * e] = fmaf(__uint_as_float(r[j4 * 8 + 2 * e]), rs, bf16_bits_to_float(w[e] & 0xFFFFu));
              v[j4 * 8 + 2 * e + 1] = fmaf(__uint_as_float(r[j4 * 8 + 2 * e + 1]), rs, bf16_bits_to_float(w[e] >> 16));
            } else {
              v[j4 * 8 + 2 * e] = __uint_as_float(r[j4 * 8 + 2 * e]) + bf16_bits_to_float(w[e] & 0xFFFFu);
              v[j4 * 8 + 2 * e + 1] = __uint_as_float(r[j4 * 8 + 2 * e + 1]) + bf16_bits_to_float(w[e] >> 16);
            }
          }
        }
        if (EPI == EPI_RESID) {
          // x[m, n..n+31] += g * v through a swizzled shared-memory tile and a
          // TMA reduce-add (the read-modify-write of x happens in L2; rows
          // beyond M are clipped by the tensor map)
          const float *gr = (p.gate && m < p.M)
                                ? p.gate + (size_t)(m / p.rows_per_gate) * p.gate_stride + n : nullptr;
          uint8_t *buf = sE + (ew * NSTG + stg_count % NSTG) * STG_BYTES;
          if (lane == 0) bulk_wait_group_read<NSTG - 1>();   // this buffer's previous reduce has read it
          __syncwarp();
#pragma unroll
          for (int j16 = 0; j16 < 8; ++j16) {
            float4 gv = make_float4(1.f, 1.f, 1.f, 1.f);
            if (gate_shared) {
              // columns 4 j16 .. + 3 of the chunk: lane 4 c + j16 / 2, half j16 % 2
              const int sl = 4 * c + (j16 >> 1);
              const float4 &src = (j16 & 1) ? col_hi : col_lo;
              gv = make_float4(__shfl_sync(0xffffffffu, src.x, sl), __shfl_sync(0xffffffffu, src.y, sl),
                               __shfl_sync(0xffffffffu, src.z, sl), __shfl_sync(0xffffffffu, src.w, sl));
              if (m >= p.M) gv = make_float4(0.f, 0.f, 0.f, 0.f);
            } else if (p.gate) {
              gv = gr ? *reinterpret_cast<const float4 *>(gr + 4 * j16) : make_float4(0.f, 0.f, 0.f, 0.f);
              if (p.gate_bias) {
                const float4 gb = *reinterpret_cast<const float4 *>(p.gate_bias + n + 4 * j16);
                gv = make_float4(gv.x + gb.x, gv.y + gb.y, gv.z + gb.z, gv.w + gb.w);
              }
            }
            const float4 o = make_float4(gv.x * v[4 * j16 + 0], gv.y * v[4 * j16 + 1],
                                         gv.z * v[4 * j16 + 2], gv.w * v[4 * j16 + 3]);
            *reinterpret_cast<float4 *>(buf + lane * 128 + ((j16 ^ (lane & 7)) << 4)) = o;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (p.x_store)
              tma_store_2d(&tmX, smem_u32(buf), n, m0w);
            else
              tma_reduce_add_2d(&tmX, smem_u32(buf), n, m0w);
            bulk_commit_group();
          }
          ++stg_count;
        } else {
          if (EPI == EPI_QKNORM) {
            const int col = nn0 + c * 32;            // column within the segment
            if (ss_col >= 0) {
#pragma unroll
              for (int j = 0; j < 32; ++j) sq = fmaf(v[j], v[j], sq);
            }
            if (gam) {
#pragma unroll
              for (int j = 0; j < 32; j += 4) {
                const int sl = 4 * c + (j >> 3);
                const float4 &src = (j & 4) ? col_hi : col_lo;
                v[j] *= __shfl_sync(0xffffffffu, src.x, sl);
                v[j + 1] *= __shfl_sync(0xffffffffu, src.y, sl);
                v[j + 2] *= __shfl_sync(0xffffffffu, src.z, sl);
                v[j + 3] *= __shfl_sync(0xffffffffu, src.w, sl);
              }
            }
            if (do_rope) {
              // pair jp of the head rotates with the t, h or w index:
              // [c - 2(c/3), c/3, c/3] pairs, c = head_dim / 2
              const int half = p.head_dim >> 1, c3 = half / 3, pt = half - 2 * c3;
              const int jp0 = (col % p.head_dim) >> 1;
              // two pairs per load: the entries (pos, jp) and (pos, jp + 1) are
              // adjacent (16 bytes, jp even); where the two pairs take
              // different positions (the t/h and h/w borders) they are read
              // one by one
#pragma unroll
              for (int e2 = 0; e2 < 8; ++e2) {
                const int jp = jp0 + 2 * e2;
                const int pa = jp < pt ? tpos : (jp < pt + c3 ? hpos : wpos);
                const int pb = jp + 1 < pt ? tpos : (jp + 1 < pt + c3 ? hpos : wpos);
                const float *ra = p.rope + ((size_t)pa * half + jp) * 2;
                float4 cs;
                if (pa == pb && p.rope_vec) {
                  cs = *reinterpret_cast<const float4 *>(ra);
                } else {
                  const float2 ca = *reinterpret_cast<const float2 *>(ra);
                  const float2 cb = *reinterpret_cast<const float2 *>(p.rope + ((size_t)pb * half + jp + 1) * 2);
                  cs = make_float4(ca.x, ca.y, cb.x, cb.y);
                }
                const float x0 = v[4 * e2], x1 = v[4 * e2 + 1], x2 = v[4 * e2 + 2], x3 = v[4 * e2 + 3];
                v[4 * e2] = x0 * cs.x - x1 * cs.y;
                v[4 * e2 + 1] = x0 * cs.y + x1 * cs.x;
                v[4 * e2 + 2] = x2 * cs.z - x3 * cs.w;
                v[4 * e2 + 3] = x2 * cs.w + x3 * cs.z;
              }
            }
          }
          // bf16 rows of two consecutive 32-column chunks go through a swizzled
          // 32 x 64 shared-memory tile (128-byte rows, 16-byte chunk k of row r
          // at k ^ (r & 7)) and one TMA store of the tile
          const int sub = c & 1;
          uint8_t *sbuf = sE + (ew * NSTG + stg_count % NSTG) * STG_BYTES;
          if (sub == 0) {
            if (lane == 0) bulk_wait_group_read<NSTG - 1>();   // this tile's previous store has read it
            __syncwarp();
          }
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            float a[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) a[e] = (EPI == EPI_GELU) ? gelu_tanh_bf16out(v[j + e]) : v[j + e];
            __nv_bfloat162 h0 = __floats2bfloat162_rn(a[0], a[1]);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(a[2], a[3]);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(a[4], a[5]);
            __nv_bfloat162 h3 = __floats2bfloat162_rn(a[6], a[7]);
            uint4 u;
            u.x = *reinterpret_cast<uint32_t *>(&h0);
            u.y = *reinterpret_cast<uint32_t *>(&h1);
            u.z = *reinterpret_cast<uint32_t *>(&h2);
            u.w = *reinterpret_cast<uint32_t *>(&h3);
            const int k = sub * 4 + (j >> 3);
            *reinterpret_cast<uint4 *>(sbuf + lane * 128 + ((k ^ (lane & 7)) << 4)) = u;
          }
          if (sub == 1) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmX, smem_u32(sbuf), n - 32, m0w);
              bulk_commit_group();
            }
            ++stg_count;
          }
        }
      }
      // one partial sum per (row, 256-column tile of the segment): no atomics
      if (EPI == EPI_QKNORM && ss_col >= 0 && m < p.M && n0 < p.N)
      {
        float *sp = p.ss + (size_t)m * p.ss_stride + ss_col * (p.segN / 256) + nn0 / 256;
        if (WAN_DBG_OK(sp, 4, p.ss, p.ss_hi, p.dbg, WAN_DBG_CODE_BASE + 2)) *sp = sq;
      }
    }
  }

  if (warp >= 2 && lane == 0) bulk_wait_group_all();   // this warp's TMA stores / reduces are done

  tc_fence_before();
  cluster_sync_all();               // the peer's smem and TMEM stay live until the leader is done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

template <int EPI, bool F8, bool WIDE>
int launch(const CUtensorMap &ta, const CUtensorMap *tb, const CUtensorMap &tx, const TcParams &p,
           cudaStream_t s) {
  using G = Geo<WIDE>;
  static int max_pairs = 0;         // per process; the attribute is per function
  if (!max_pairs) {
    WAN_TRY_CUDA(cudaFuncSetAttribute(gemm_tc_kernel<EPI, F8, WIDE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      G::SMEM_BYTES), "gemm_tc smem attribute");
    cudaLaunchConfig_t qc = {};
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2; qa[0].val.clusterDim.y = 1; qa[0].val.clusterDim.z = 1;
    qc.gridDim = dim3(2 * 74, 1, 1);
    qc.blockDim = dim3(G::THREADS, 1, 1);
    qc.dynamicSmemBytes = G::SMEM_BYTES;
    qc.attrs = qa;
    qc.numAttrs = 1;
    int clusters = 0;
    WAN_TRY_CUDA(cudaOccupancyMaxActiveClusters(&clusters, gemm_tc_kernel<EPI, F8, WIDE>, &qc), "gemm_tc occupancy");
    max_pairs = clusters > 0 ? clusters : sm_count() / 2;
  }
  const int pairs = p.num_tiles < max_pairs ? p.num_tiles : max_pairs;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2; attr[0].val.clusterDim.y = 1; attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(G::THREADS, 1, 1);
  cfg.dynamicSmemBytes = G::SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  WAN_TRY_CUDA(cudaLaunchKernelEx(&cfg, gemm_tc_kernel<EPI, F8, WIDE>, ta, tb[0], tb[1], tb[2], tx, p),
               "gemm_tc launch");
  return WAN_OK;
}

template <bool F8, bool WIDE>
int launch_epi(int epi, const CUtensorMap &ta, const CUtensorMap *tb, const CUtensorMap &tx, const TcParams &p,
               cudaStream_t s) {
  switch (epi) {
    case EPI_STORE: return launch<EPI_STORE, F8, WIDE>(ta, tb, tx, p, s);
    case EPI_GELU: return launch<EPI_GELU, F8, WIDE>(ta, tb, tx, p, s);
    case EPI_QKNORM: return launch<EPI_QKNORM, F8, WIDE>(ta, tb, tx, p, s);
    default: return launch<EPI_RESID, F8, WIDE>(ta, tb, tx, p, s);
  }
}
}  // namespace

bool gemm_tc_supported(const GemmArgs &g) {
  if (g.epi == EPI_SILU) return false;
  const int bk = g.fp8 ? BK8 : BK;
  if (g.M < 1 || g.N < 32 || g.K < bk || g.K % bk || g.N % 32) return false;
  if (g.fp8) {
    if (!g.a_scale || g.lda % 16) return false;
    for (int i = 0; i < g.nseg; ++i)
      if (!g.b_scale[i]) return false;
  }
  if (g.nseg < 1 || g.nseg > 3 || g.segN * g.nseg != g.N) return false;
  if (g.nseg > 1 && g.segN % 256) return false;
  if (g.lda % 8) return false;
  if (g.epi != EPI_RESID && (g.ldc % 8 || g.N % 64 || !aligned16(g.C))) return false;   // staged 64-column TMA stores
  if (g.epi == EPI_RESID && (g.ldx % 4 || !aligned16(g.X) || (g.gate && g.gate_stride % 4))) return false;
  if (g.gate_bias && !aligned16(g.gate_bias)) return false;
  if (g.epi == EPI_QKNORM) {
    for (int i = 0; i < g.nseg; ++i) {
      if (g.ss_col[i] >= 0 && !g.ss) return false;
      if (g.gamma[i] && !aligned16(g.gamma[i])) return false;
    }
    if (g.rope && (g.head_dim % 32 || g.segN % g.head_dim)) return false;
    if (g.segN % 256) return false;            // whole 256-column tiles per segment (partial sums)
  }
  for (int i = 0; i < g.nseg; ++i)
    if (!aligned16(g.Bseg[i]) || (g.bias[i] && !aligned16(g.bias[i]))) return false;
  return aligned16(g.A);
}

int gemm_tc(const GemmArgs &g, cudaStream_t s) {
  if (!gemm_tc_supported(g)) return set_error(WAN_EUNSUPPORTED, "gemm_tc: M=%d N=%d K=%d", g.M, g.N, g.K);
  CUtensorMap ta, tb[3];
  int rc = g.fp8 ? encode_tmap_2d_u8(&ta, g.A, g.K, g.M, (uint64_t)g.lda, BK8, BM)
                 : encode_tmap_2d_bf16(&ta, g.A, g.K, g.M, (uint64_t)g.lda * 2, BK, BM);
  if (rc) return rc;
  for (int i = 0; i < 3; ++i) {
    const int si = i < g.nseg ? i : 0;
    rc = g.fp8 ? encode_tmap_2d_u8(&tb[i], g.Bseg[si], g.K, g.segN, (uint64_t)g.K, BK8, 128)
               : encode_tmap_2d_bf16(&tb[i], g.Bseg[si], g.K, g.segN, (uint64_t)g.K * 2, BK, 128);
    if (rc) return rc;
  }
  TcParams p = {};
  p.M = g.M; p.N = g.N; p.K = g.K; p.segN = g.segN;
  // the wide tile when no 512-column tile straddles two weight segments and K
  // is long enough for its epilogue (which does not overlap the next tile's
  // products) to be a small share of a tile: measured on the workload's
  // blocks, wide is 7% faster at K = 5120, even at K = 3072, and 9-10%
  // slower at K = 1536
  const bool wide = USE_WIDE && g.K >= 4096 && (g.nseg == 1 || g.segN % 512 == 0);
  const int bn = wide ? 512 : 256;
  p.num_m = (g.M + 2 * BM - 1) / (2 * BM);
  p.num_n = (g.N + bn - 1) / bn;
  p.num_tiles = p.num_m * p.num_n;
  p.num_k = g.K / (g.fp8 ? BK8 : BK);
  p.a_scale = g.a_scale;
  for (int i = 0; i < 3; ++i) p.b_scale[i] = g.fp8 ? g.b_scale[i < g.nseg ? i : 0] : nullptr;
  for (int i = 0; i < 3; ++i) p.bias[i] = i < g.nseg ? g.bias[i] : nullptr;
  p.C = g.C; p.ldc = g.ldc; p.X = g.X; p.ldx = g.ldx;
  p.gate = g.gate; p.gate_stride = g.gate_stride; p.rows_per_gate = g.rows_per_gate > 0 ? g.rows_per_gate : 1;
  p.x_store = g.x_store;
  p.gate_bias = g.gate_bias;
  for (int i = 0; i < 3; ++i) {
    p.gamma[i] = i < g.nseg ? g.gamma[i] : nullptr;
    p.ss_col[i] = i < g.nseg ? g.ss_col[i] : -1;
  }
  p.ss = g.ss; p.ss_stride = g.ss_stride;
  p.rope = g.rope; p.rope_mask = g.rope ? g.rope_mask : 0;
  p.L = g.rows_per_seq > 0 ? g.rows_per_seq : (g.F * g.H * g.W > 0 ? g.F * g.H * g.W : 1);
  p.H = g.H > 0 ? g.H : 1; p.W = g.W > 0 ? g.W : 1;
  p.tok0 = g.tok0;
  p.head_dim = g.head_dim > 0 ? g.head_dim : 128;
  p.rope_vec = aligned16(g.rope) && p.head_dim % 4 == 0;   // 16-byte loads of two table entries
  p.watchdog = watchdog_ptr();
  p.dbg = g.dbg ? g.dbg : dbg_word();
  if (g.ss) p.ss_hi = g.ss + (size_t)g.M * g.ss_stride;
  // the epilogue's store target: x (fp32, 32 x 32 boxes) for the residual, else C (bf16, 64 x 32 boxes)
  CUtensorMap tx = ta;
  if (g.epi == EPI_RESID) {
    if ((rc = encode_tmap_2d_f32(&tx, g.X, g.N, g.M, (uint64_t)g.ldx * 4, 32, 32))) return rc;
  } else if ((rc = encode_tmap_2d_bf16(&tx, g.C, g.N, g.M, (uint64_t)g.ldc * 2, 64, 32))) {
    return rc;
  }
  if (g.fp8) return wide ? launch_epi<true, true>(g.epi, ta, tb, tx, p, s) : launch_epi<true, false>(g.epi, ta, tb, tx, p, s);
  return wide ? launch_epi<false, true>(g.epi, ta, tb, tx, p, s) : launch_epi<false, false>(g.epi, ta, tb, tx, p, s);
}

}  // namespace wan

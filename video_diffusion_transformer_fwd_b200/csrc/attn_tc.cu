// Flash attention forward for sm_100a: bf16 q, k, v with head_dim 128,
// non-causal, online softmax in fp32, tensor-core products accumulated in TMEM.
// ("Wan2.2 code walkthrough" (newtid.com), self-attention snippet: global
// window, key lengths; softmax(q k^T * scale) v.)
//
// One CTA = 2 query tiles of 128 rows of one (sequence, head):
//   warps 0..3 / 4..7  softmax of query tile 0 / 1: thread = one query row;
//               loads its row of S (128 keys, fp32) from TMEM and releases
//               the S columns at once, keeps a running max m (log2 domain)
//               and sum l, and writes P = exp2(S c - m) as bf16 into a
//               shared-memory tile in the MMA's swizzled K-major layout; it
//               rescales its O row in TMEM only when m grows by more than 8
//               (P stays <= 2^8 otherwise, the final O / l is unchanged);
//   warp 8      MMA issuer: S_i(j+1) = Q_i K_{j+1}^T as soon as both the K
//               tile and the S_i columns are free (while the softmax of tile
//               j still runs), then O_i += P_i(j) V_j (A = P, B = V MN-major,
//               both from shared memory);
//   warp 9      TMA producer: Q tiles once, then K tiles into a 2-slot ring
//               (K_{j+2} as soon as S(j) is done) and V tiles into one slot
//               (V_{j+1} once PV(j) is done), 32 KB each (128-byte swizzle).
// TMEM: S_0 | S_1 | O_0 | O_1, 128 fp32 columns each (512 total).
// At the end each softmax thread writes its row of O / l (bf16) into its
// tile's P buffer, in the same swizzled layout, and one thread per tile
// stores the tile with two TMA stores.
// Every wait is bounded (sm100::mbar_wait); keys at or beyond the sequence's
// key length are masked; rows of a tile beyond Lq are computed but clipped by
// the output's tensor map.
#include "common.cuh"
#include "sm100.cuh"

namespace wan {

namespace {
using namespace sm100;

constexpr int D = 128;                 // head_dim
constexpr int TQ = 128;                // query rows per tile
constexpr int TK = 128;                // keys per tile
constexpr int NSLOT = 3;               // K slots 0, 1 and the V slot
constexpr int TILE_BYTES = 128 * D * 2;  // 32 KB: one Q, K, V or P tile (two 64-column boxes)
constexpr int BOX_BYTES = TILE_BYTES / 2;
constexpr int THREADS = 320;                // 8 softmax warps + MMA warp + TMA warp
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_S = idesc_bf16(TQ, TK, 0);
constexpr uint32_t IDESC_O = idesc_bf16(TQ, D, 1);
constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units
constexpr int SMEM_BYTES = 1024 + 4 * TILE_BYTES + NSLOT * TILE_BYTES + 256;   // Q_0, Q_1, P_0, P_1, ring

struct FaParams {
  int B, heads, Lq, Lk;
  const int *k_lens;
  float c;                    // scale * log2(e)
  __nv_bfloat16 *o; int ldo;
  const float *q_ss; int q_ss_stride; int q_ss_parts; float q_ss_inv_n; float q_ss_eps;   // optional per-row RMS factor of q
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

// Two fp32 lanes per instruction (Blackwell packed f32x2 arithmetic).
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

// 3D tiled store from shared memory (x inner, y row, z batch); rows and
// columns beyond the tensor are clipped
__device__ __forceinline__ void tma_store_3d(const void *tmap, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(tmap)), "r"(src), "r"(x), "r"(y), "r"(z) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__global__ void __launch_bounds__(THREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
               const FaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;                               // 2 tiles
  uint8_t *sP = smem + 2 * TILE_BYTES;              // 2 tiles
  uint8_t *sKV = smem + 4 * TILE_BYTES;             // NSLOT tiles
  uint64_t *bars = reinterpret_cast<uint64_t *>(sKV + NSLOT * TILE_BYTES);
  uint64_t *q_full = bars;
  uint64_t *kv_full = bars + 1;                     // [0], [1]: K slots; [2]: V slot
  uint64_t *kv_empty = bars + 1 + NSLOT;
  uint64_t *s_full = bars + 1 + 2 * NSLOT;          // S_i computed
  uint64_t *s_free = s_full + 2;                    // S_i read by its softmax
  uint64_t *p_full = s_free + 2;                    // P_i written to shared memory
  uint64_t *pv_done = p_full + 2;                   // O_i += P_i V done (P_i free, O_i stable)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(pv_done + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  const int q0 = blockIdx.x * 2 * TQ;
  int kl = p.Lk;
  if (p.k_lens) kl = min(max(p.k_lens[b], 0), p.Lk);
  const int nkt = (kl + TK - 1) / TK;

  // A CTA that starts after another one gave up a wait skips its work, so a
  // failed launch ends within a few waits instead of one per CTA.
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
      mbar_init(smem_u32(&s_free[i]), 4);
      mbar_init(smem_u32(&p_full[i]), 4);
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
  // K_j sits in slot j % 2 (its (j / 2)-th fill); V_j in slot 2 (its j-th fill)
  auto kslot = [](int j) { return j & 1; };
  auto kphase = [](int j) { return (uint32_t)((j >> 1) & 1); };
  constexpr int VSLOT = 2;

  if (warp >= 8) {
    if (warp == 9) {
      // ------------------------------------------------ TMA producer
      if (lane == 0 && nkt > 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        const uint32_t qb = smem_u32(q_full);
        mbar_arrive_expect_tx(qb, 2 * TILE_BYTES);
        for (int i = 0; i < 2; ++i)
          for (int half = 0; half < 2; ++half)
            tma_load_3d(smem_u32(sQ + i * TILE_BYTES + half * BOX_BYTES), &tmQ, h * D + half * 64,
                        q0 + i * TQ, b, qb);
        int fills[NSLOT] = {0, 0, 0};
        auto load = [&](int slot, uint32_t empty_phase, const CUtensorMap *tm, int j) {
          if (!mbar_wait(smem_u32(&kv_empty[slot]), empty_phase, abort_flag, p.watchdog, 0x201)) return false;
          const uint32_t fb = smem_u32(&kv_full[slot]);
          mbar_arrive_expect_tx(fb, TILE_BYTES);
          for (int half = 0; half < 2; ++half)
            tma_load_3d(smem_u32(sKV + slot * TILE_BYTES + half * BOX_BYTES), tm, h * D + half * 64, j * TK, b, fb);
          ++fills[slot];
          return true;
        };
        // K_0, K_1, V_0, then K_{j+2} (frees after S(j)) before V_{j+1} (frees after PV(j))
        bool ok = load(kslot(0), kphase(0) ^ 1, &tmK, 0);
        if (ok && nkt > 1) ok = load(kslot(1), kphase(1) ^ 1, &tmK, 1);
        if (ok) ok = load(VSLOT, 1, &tmV, 0);
        for (int j = 0; j < nkt && ok; ++j) {
          if (j + 2 < nkt) ok = load(kslot(j + 2), kphase(j + 2) ^ 1, &tmK, j + 2);
          if (ok && j + 1 < nkt) ok = load(VSLOT, ((j + 1) & 1) ^ 1, &tmV, j + 1);
        }
        int never = 0;
        mbar_wait(qb, 0, &never, p.watchdog, 0x202);
        for (int s = 0; s < NSLOT; ++s)
          if (fills[s] > 0) mbar_wait(smem_u32(&kv_full[s]), (fills[s] - 1) & 1, &never, p.watchdog, 0x203);
      }
    } else if (warp == 8) {
      // ------------------------------------------------ MMA issuer
      if (lane == 0 && nkt > 0) {
        // Per key tile j: S_0(j+1), S_1(j+1) as soon as K_{j+1} has landed
        // and each S_i(j) has been read; then PV_0(j), PV_1(j) once V_j has
        // landed and each P_i(j) is written. The tensor pipe computes the next
        // scores while the softmax still works on the current ones.
        bool ok = mbar_wait(smem_u32(q_full), 0, abort_flag, p.watchdog, 0x211);
        auto issue_s = [&](int i, uint32_t kbase) {
          const uint32_t qbase = smem_u32(sQ + i * TILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * BOX_BYTES + (kk & 3) * 32;
            mma_ss(tmem + i * TK, desc_kmajor_sw128(qbase + off), desc_kmajor_sw128(kbase + off), IDESC_S, kk > 0);
          }
          tc_commit(smem_u32(&s_full[i]));
        };
        auto issue_pv = [&](int i, uint32_t vbase, int j) {
          const uint32_t pbase = smem_u32(sP + i * TILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < TK / 16; ++kk) {
            const uint32_t off = (kk >> 2) * BOX_BYTES + (kk & 3) * 32;
            mma_ss(tmem + 2 * TK + i * D, desc_kmajor_sw128(pbase + off),
                   desc_mnmajor_sw128(vbase + kk * 16 * 128, BOX_BYTES, 1024), IDESC_O, (j > 0 || kk > 0));
          }
          tc_commit(smem_u32(&pv_done[i]));
        };
        // prologue: S_0(0), S_1(0)
        if (ok && mbar_wait(smem_u32(&kv_full[kslot(0)]), kphase(0), abort_flag, p.watchdog, 0x212)) {
          tc_fence_after();
          const uint32_t kbase = smem_u32(sKV + kslot(0) * TILE_BYTES);
          issue_s(0, kbase);
          issue_s(1, kbase);
          tc_commit(smem_u32(&kv_empty[kslot(0)]));
        } else {
          ok = false;
        }
        for (int j = 0; j < nkt && ok; ++j) {
          if (j + 1 < nkt) {
            const int ks = kslot(j + 1);
            if (!mbar_wait(smem_u32(&kv_full[ks]), kphase(j + 1), abort_flag, p.watchdog, 0x213)) break;
            const uint32_t kbase = smem_u32(sKV + ks * TILE_BYTES);
            if (!mbar_wait(smem_u32(&s_free[0]), j & 1, abort_flag, p.watchdog, 0x214)) break;
            tc_fence_after();
            issue_s(0, kbase);
            if (!mbar_wait(smem_u32(&s_free[1]), j & 1, abort_flag, p.watchdog, 0x215)) break;
            tc_fence_after();
            issue_s(1, kbase);
            tc_commit(smem_u32(&kv_empty[ks]));
          }
          if (!mbar_wait(smem_u32(&kv_full[VSLOT]), j & 1, abort_flag, p.watchdog, 0x216)) break;
          const uint32_t vbase = smem_u32(sKV + VSLOT * TILE_BYTES);
          if (!mbar_wait(smem_u32(&p_full[0]), j & 1, abort_flag, p.watchdog, 0x217)) break;
          tc_fence_after();
          issue_pv(0, vbase, j);
          if (!mbar_wait(smem_u32(&p_full[1]), j & 1, abort_flag, p.watchdog, 0x218)) break;
          tc_fence_after();
          issue_pv(1, vbase, j);
          tc_commit(smem_u32(&kv_empty[VSLOT]));
        }
      }
    }
  } else {
    // ------------------------------------------------ softmax (warps 0..7)
    const int i = warp >> 2;                       // query tile
    const int qw = warp & 3;                       // TMEM lane quarter
    const int r = qw * 32 + lane;                  // row in the tile
    const int row = q0 + i * TQ + r;               // query row in the sequence
    const uint32_t lane_off = (uint32_t)(qw * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + i * TK;
    const uint32_t o_addr = tmem + lane_off + 2 * TK + i * D;
    // this row of P_i in the 128-byte swizzled K-major layout: box (64 keys),
    // row r at r * 128 bytes, 16-byte chunk c at (c ^ (r & 7)) * 16
    const uint32_t p_row = smem_u32(sP + i * TILE_BYTES) + r * 128;
    float m = -INFINITY, l = 0.f;
    // logit scale of this row: scale * log2(e), times q's RMS factor when the
    // QKV epilogue left q un-normalised (q_ss holds the row's sum of squares)
    float crow = p.c;
    if (p.q_ss && row < p.Lq) {
      const float *qs = p.q_ss + (size_t)(b * p.Lq + row) * p.q_ss_stride;
      float sum = 0.f;
      for (int t = 0; t < p.q_ss_parts; ++t) sum += qs[t];
      crow *= rsqrtf(sum * p.q_ss_inv_n + p.q_ss_eps);
    }
    bool ok = true;
    for (int j = 0; j < nkt; ++j) {
      if (!mbar_wait(smem_u32(&s_full[i]), j & 1, abort_flag, p.watchdog, 0x221)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));
      tmem_ld_wait();
      // S_i is in registers: its TMEM columns may take S_i(j+1)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s_free[i]));
      const int kvalid = kl - j * TK;              // keys of this tile that are valid
      const bool full_tile = kvalid >= TK;         // uniform across the CTA
      if (!full_tile) {
#pragma unroll
        for (int k = 0; k < 128; ++k)
          if (k >= kvalid) s[k] = 0xff800000u;     // -inf
      }
      // row max of the raw scores (the scale c is positive), 3-input max tree
      float mx[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mx[a] = fmaxf(__uint_as_float(s[a]), __uint_as_float(s[8 + a]));
#pragma unroll
      for (int k = 16; k < 128; k += 16) {
#pragma unroll
        for (int a = 0; a < 8; ++a) mx[a] = fmax3(mx[a], __uint_as_float(s[k + a]), __uint_as_float(s[k + 8 + a]));
      }
      const float tmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * crow;
      // running max; l and O are rescaled only when m grows by more than the
      // threshold (or on the first tile)
      const bool need = (tmax > m + RESCALE_THRESHOLD) || (m == -INFINITY);
      const float mnew = need ? tmax : m;
      const float alpha = (need && j > 0) ? ex2(m - mnew) : 1.0f;
      m = mnew;
      // P = exp2(s c - m) as bf16 pairs, packed into s[0..63]
      const float2 c2 = make_float2(crow, crow);
      const float2 nm2 = make_float2(-m, -m);
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        const float2 x = ffma2(make_float2(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1])), c2, nm2);
        const float2 pp = make_float2(ex2(x.x), ex2(x.y));
        acc = fadd2(acc, pp);
        s[e] = pack_bf16(pp.x, pp.y);
      }
      l = l * alpha + (acc.x + acc.y);
      // P_i and O_i are still in use by PV_i(j-1) until it completes
      if (j > 0) {
        if (!mbar_wait(smem_u32(&pv_done[i]), (j - 1) & 1, abort_flag, p.watchdog, 0x222)) ok = false;
        tc_fence_after();
      }
      // O rescale (TMEM accesses are warp-collective: a warp rescales when
      // any of its rows must)
      if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[16];
          tmem_ld16(o_addr + c * 16, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st16(o_addr + c * 16, o);
        }
        tmem_st_wait();
      }
      // P row -> shared memory: keys 8c .. 8c + 7 form 16-byte chunk c
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t addr = p_row + (c >> 3) * BOX_BYTES + ((((uint32_t)c & 7u) ^ ((uint32_t)r & 7u)) << 4);
        st_shared_v4(addr, s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&p_full[i]));
      if (!ok) break;
    }
    // epilogue: O / l -> bf16
    if (ok && nkt > 0) {
      ok = mbar_wait(smem_u32(&pv_done[i]), (nkt - 1) & 1, abort_flag, p.watchdog, 0x223);
      tc_fence_after();
    }
    // O / l as bf16 into the P_i tile (free once PV_i of the last key tile is
    // done; the same swizzled layout, two boxes of 64 columns), then one
    // thread of the tile writes it with two TMA stores (rows beyond Lq are
    // clipped by the tensor map)
    const float inv = (l > 0.f) ? 1.0f / l : 0.f;
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
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t k = (uint32_t)(c * 4 + e);                     // 16-byte chunk of the row
        const uint32_t addr = p_row + (k >> 3) * BOX_BYTES + (((k & 7u) ^ ((uint32_t)r & 7u)) << 4);
        st_shared_v4(addr, pack_bf16(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv),
                     pack_bf16(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv),
                     pack_bf16(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv),
                     pack_bf16(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv));
      }
    }
    fence_proxy_async_smem();
    asm volatile("bar.sync %0, 128;" ::"r"(1 + i) : "memory");      // the tile's 4 warps
    if (qw == 0 && lane == 0 && ok) {
      for (int half = 0; half < 2; ++half)
        tma_store_3d(&tmO, smem_u32(sP + i * TILE_BYTES + half * BOX_BYTES), h * D + half * 64, q0 + i * TQ, b);
      bulk_commit_group();
      bulk_wait_group_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tmem, TMEM_COLS);
}
}  // namespace

bool attention_tc_supported(const AttnArgs &a) {
  if (a.d != D || a.B < 1 || a.Lq < 1 || a.Lk < 0) return false;
  if (a.ldq % 8 || a.ldk % 8 || a.ldv % 8 || a.ldo % 8) return false;
  if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.o)) return false;
  if (a.heads > 65535 || a.B > 65535) return false;
  return true;
}

int attention_tc(const AttnArgs &a, cudaStream_t s) {
  if (!attention_tc_supported(a)) return set_error(WAN_EUNSUPPORTED, "attention_tc");
  const int Lk = a.Lk > 0 ? a.Lk : 1;
  CUtensorMap tq, tk, tv;
  const uint64_t inner = (uint64_t)a.heads * D;
  int rc = encode_tmap_3d_bf16(&tq, a.q, inner, a.Lq, a.B, (uint64_t)a.ldq * 2, (uint64_t)a.Lq * a.ldq * 2, 64, TQ);
  if (rc) return rc;
  if ((rc = encode_tmap_3d_bf16(&tk, a.k, inner, Lk, a.B, (uint64_t)a.ldk * 2, (uint64_t)a.Lk * a.ldk * 2 + (a.Lk ? 0 : 16), 64, TK))) return rc;
  if ((rc = encode_tmap_3d_bf16(&tv, a.v, inner, Lk, a.B, (uint64_t)a.ldv * 2, (uint64_t)a.Lk * a.ldv * 2 + (a.Lk ? 0 : 16), 64, TK))) return rc;
  CUtensorMap to;
  if ((rc = encode_tmap_3d_bf16(&to, a.o, inner, a.Lq, a.B, (uint64_t)a.ldo * 2, (uint64_t)a.Lq * a.ldo * 2, 64, TQ))) return rc;
  static bool attr_set = false;
  if (!attr_set) {
    WAN_TRY_CUDA(cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES),
                 "attention_tc smem attribute");
    attr_set = true;
  }
  FaParams p = {};
  p.B = a.B; p.heads = a.heads; p.Lq = a.Lq; p.Lk = a.Lk; p.k_lens = a.k_lens;
  p.c = a.scale * 1.4426950408889634f;
  p.q_ss = a.q_ss; p.q_ss_stride = a.q_ss_stride; p.q_ss_parts = a.q_ss_parts;
  p.q_ss_inv_n = a.q_ss_n > 0.f ? 1.0f / a.q_ss_n : 0.f; p.q_ss_eps = a.q_ss_eps;
  p.o = static_cast<__nv_bfloat16 *>(a.o); p.ldo = a.ldo;
  p.watchdog = watchdog_ptr();
  dim3 grid((a.Lq + 2 * TQ - 1) / (2 * TQ), a.heads, a.B);
  attn_tc_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(tq, tk, tv, to, p);
  WAN_CHECK_LAUNCH("attention_tc");
  return WAN_OK;
}

}  // namespace wan

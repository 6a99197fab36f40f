// prefill.cu -- causal attention of a whole sequence over itself in the *expanded* form
// ("Module 05 -- MLA", section 5: prefill, where every token is a query and the pass is
// compute-heavy, may prefer the naive algebra): keys and values are first expanded per
// head from the latents (k_j = U_h^K c_j, v_j = U_h^V c_j, mla_expand_kv), then
//   out[t, h] = sum_{j <= t} softmax_j(scale * q[t, h] . k[j, h]) v[j, h]
// with 256-dimensional heads.  The absorbed form of the same prefill runs through the
// decode path (mla_absorb_q, mla_attend_dense with q_len = L, mla_up_proj); measuring the
// two side by side is the comparison that section asks for.
//
// One CTA per (block of 128 queries, head, sequence); 7 warps:
//   warp 0      TMA producer: 64-key tiles of K and V (4 boxes of 64 dims each) into a
//               3-stage ring;
//   warp 1      score MMAs S[q, keys] = Q * K_tile^T with Q read from TMEM (M = 128
//               queries, N = 64 keys, K = 256), double-buffered S;
//   warps 2-5   softmax, one query row per thread (the row is one TMEM lane, so its max
//               and sum need no shuffles), lazy rescale of O in TMEM, P (bf16) to shared
//               memory; at the end the normalised output;
//   warp 6      value MMAs O[q, d] += P * V_tile (M = 128, N = 256, K = 64 keys).
// TMEM: Q as the A operand (128 columns), two S buffers (64 each), O (256).
#include <math.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"

namespace mla {
namespace prefill {

constexpr int kQBlock = 128;                       // queries per CTA (MMA M)
constexpr int kKTile = 64;                         // keys per tile (score N, value K)
constexpr int kStages = 3;                         // K/V ring
constexpr int kBoxBytes = kKTile * 64 * 2;         // 64 keys x 64 dims: 8 KB
constexpr int kKBytes = 4 * kBoxBytes;             // 32 KB
constexpr int kStageBytes = 2 * kKBytes;           // K then V: 64 KB
constexpr int kPBytes = kQBlock * kKTile * 2;      // 16 KB
constexpr int kThreads = 224;
constexpr float kTau = 8.0f;                       // lazy rescale threshold (log2 units)

constexpr int kOffKV = 0;
constexpr int kOffP = kOffKV + kStages * kStageBytes;
constexpr int kOffBar = kOffP + kPBytes;
constexpr int kBarFull = 0, kBarEmpty = kStages, kBarSFull = 2 * kStages, kBarSEmpty = kBarSFull + 2,
              kBarPFull = kBarSEmpty + 2, kBarPEmpty = kBarPFull + 1, kBarQ = kBarPEmpty + 1, kBarO = kBarQ + 1,
              kBarDrain = kBarO + 1, kNumBars = kBarDrain + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemQ = 0;      // 128 columns: 256 bf16 of Q per lane
constexpr uint32_t kTmemS = 128;    // 2 x 64 columns
constexpr uint32_t kTmemO = 256;    // 256 columns

struct Params {
  const uint16_t *q;  // [B, L, H, D]
  uint16_t *out;      // [B, L, H, D]
  float *lse;         // [B, L, H] or null
  int B, L;
  float scale_log2;
  int32_t *status;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bar = reinterpret_cast<uint64_t *>(base + kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(base + kOffMisc + 4);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nqb = (p.L + kQBlock - 1) / kQBlock;
  const int qb = nqb - 1 - (int)blockIdx.x;  // the longest causal ranges start first
  const int h = blockIdx.y, b = blockIdx.z;
  const int q0 = qb * kQBlock;
  const int n_kt = min((p.L + kKTile - 1) / kKTile, (q0 + kQBlock - 1) / kKTile + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar[kBarFull + s], 1);
      mbar_init(&bar[kBarEmpty + s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[kBarSFull + i], 1);
      mbar_init(&bar[kBarSEmpty + i], 4);
    }
    mbar_init(&bar[kBarPFull], 4);
    mbar_init(&bar[kBarPEmpty], 1);
    mbar_init(&bar[kBarQ], 4);
    mbar_init(&bar[kBarO], 1);
    mbar_init(&bar[kBarDrain], 2);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  grid_dep_launch();
  grid_dep_wait();  // q, k, v come from the kernels before
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long tok0 = (long long)b * p.L;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      uint32_t issued = 0;
      for (int kt = 0; kt < n_kt; ++kt) {
        const int s = kt % kStages;
        if (!mbar_wait(&bar[kBarEmpty + s], ((kt / kStages) & 1) ^ 1, abort_flag, p.status)) break;
        mbar_arrive_expect_tx(&bar[kBarFull + s], kStageBytes);
        uint8_t *dst = base + kOffKV + s * kStageBytes;
        const int tok = (int)(tok0 + kt * kKTile);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tma_load_3d(dst + c * kBoxBytes, &tm_k, &bar[kBarFull + s], c * 64, h, tok);
          tma_load_3d(dst + kKBytes + c * kBoxBytes, &tm_v, &bar[kBarFull + s], c * 64, h, tok);
        }
        issued = kt + 1;
      }
      // every issued copy lands before the CTA may exit (also after an abort)
      if (!drain_ring(&bar[kBarFull], kStages, issued)) report_status(p.status, kStatusTimeout);
    }
  } else if (warp == 1) {
    // S[q, keys] = Q (TMEM) * K_tile^T; K_tile K-major: K step of 16 dims = 32 bytes in a
    // 128-byte swizzle row, steps 4k..4k+3 in box k
    constexpr uint32_t idesc = idesc_bf16_f32(kQBlock, kKTile, false, false);
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bar[kBarQ], 0, abort_flag, p.status));
    for (int kt = 0; kt < n_kt && ok; ++kt) {
      const int s = kt % kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar[kBarFull + s], (kt / kStages) & 1, abort_flag, p.status));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar[kBarSEmpty + (kt & 1)], ((kt >> 1) & 1) ^ 1, abort_flag,
                                                     p.status));
      if (!ok) break;
      tc_fence_after();
      const uint32_t kbase = smem_u32(base + kOffKV + s * kStageBytes);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
          const uint64_t bd = sw128_desc(kbase + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
          umma_bf16_tmem_a(tmem + kTmemS + (kt & 1) * kKTile, tmem + kTmemQ + kk * 8, bd, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bar[kBarSFull + (kt & 1)]);
      }
      __syncwarp();
    }
  } else if (warp == 6) {
    // O[q, d] += P[q, keys] * V_tile: P K-major (one 128-byte row per query), V MN-major
    // (dims along the 128-byte rows, 64-dim atoms 8 KB apart, 8-key groups 1 KB apart)
    constexpr uint32_t idesc = idesc_bf16_f32(kQBlock, 256, false, true);
    const uint32_t pbase = smem_u32(base + kOffP);
    bool ok = true;
    for (int kt = 0; kt < n_kt; ++kt) {
      const int s = kt % kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar[kBarPFull], kt & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      const uint32_t vbase = smem_u32(base + kOffKV + s * kStageBytes + kKBytes);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kKTile / 16; ++kk) {
          const uint64_t ad = sw128_desc(pbase + kk * 32, 16, 1024);
          const uint64_t bd = sw128_desc(vbase + kk * 2048, kBoxBytes, 1024);
          umma_bf16(tmem + kTmemO, ad, bd, idesc, (kt > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bar[kBarPEmpty]);
        umma_commit(&bar[kBarEmpty + s]);
        if (kt == n_kt - 1) umma_commit(&bar[kBarO]);
      }
      __syncwarp();
    }
  } else {
    // ---- softmax warps 2-5: thread owns query row m (TMEM lane m)
    const int quad = warp & 3;
    const int m = quad * 32 + lane;
    const int t = q0 + m;  // query position in the sequence
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
    // Q row -> TMEM (the A operand of the score MMAs): 128 columns of bf16 pairs
    {
      const uint4 *src = reinterpret_cast<const uint4 *>(p.q + ((tok0 + t) * kHeads + h) * kHeadDim);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 x = (t < p.L) ? src[c * 8 + u] : make_uint4(0u, 0u, 0u, 0u);
          r[4 * u] = x.x;
          r[4 * u + 1] = x.y;
          r[4 * u + 2] = x.z;
          r[4 * u + 3] = x.w;
        }
        tmem_st32(t_lane + kTmemQ + c * 32, r);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kBarQ]);
    }
    const uint32_t prow = smem_u32(base + kOffP) + (uint32_t)m * 128;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int kt = 0; kt < n_kt && ok; ++kt) {
      ok = mbar_wait(&bar[kBarSFull + (kt & 1)], (kt >> 1) & 1, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float s[kKTile];
      {
        uint32_t r[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          tmem_ld32(t_lane + kTmemS + (kt & 1) * kKTile + half * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int key = kt * kKTile + half * 32 + j;
            s[half * 32 + j] = (key <= t) ? __uint_as_float(r[j]) * p.scale_log2 : -INFINITY;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kBarSEmpty + (kt & 1)]);
      float mt = -INFINITY;
#pragma unroll
      for (int j = 0; j < kKTile; ++j) mt = fmaxf(mt, s[j]);
      const bool raise = mt > m_run + kTau || (m_run == -INFINITY && mt != -INFINITY);
      // the P buffer (and O) are free once the value product of the previous tile is done
      ok = __all_sync(0xffffffffu, mbar_wait(&bar[kBarPEmpty], (kt & 1) ^ 1, abort_flag, p.status));
      if (!ok) break;
      float alpha = 1.f;
      if (raise) {
        alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - mt);
        l_run *= alpha;
        m_run = mt;
      }
      if (kt > 0 && __any_sync(0xffffffffu, raise)) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t r[32];
          tmem_ld32(t_lane + kTmemO + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
          tmem_st32(t_lane + kTmemO + c * 32, r);
        }
        tmem_st_wait();
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = s[u * 8 + 2 * e], x1 = s[u * 8 + 2 * e + 1];
          const float p0 = (x0 == -INFINITY) ? 0.f : fast_exp2(x0 - m_run);
          const float p1 = (x1 == -INFINITY) ? 0.f : fast_exp2(x1 - m_run);
          w[e] = pack_bf16x2(p0, p1);
          l_run += bf16lo_to_f32(w[e]) + bf16hi_to_f32(w[e]);
        }
        st_shared_v4(prow + (((uint32_t)u ^ (uint32_t)(m & 7)) << 4), w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kBarPFull]);
    }
    // ---- epilogue: out = O / l
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar[kBarO], 0, abort_flag, p.status));
    tc_fence_after();
    const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
    uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((tok0 + t) * kHeads + h) * kHeadDim);
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t r[32];
      tmem_ld32(t_lane + kTmemO + c * 32, r);
      tmem_ld_wait();
      if (ok && t < p.L) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r[8 * u + 0]) * inv, __uint_as_float(r[8 * u + 1]) * inv);
          v.y = pack_bf16x2(__uint_as_float(r[8 * u + 2]) * inv, __uint_as_float(r[8 * u + 3]) * inv);
          v.z = pack_bf16x2(__uint_as_float(r[8 * u + 4]) * inv, __uint_as_float(r[8 * u + 5]) * inv);
          v.w = pack_bf16x2(__uint_as_float(r[8 * u + 6]) * inv, __uint_as_float(r[8 * u + 7]) * inv);
          dst[c * 4 + u] = v;
        }
      }
    }
    if (ok && t < p.L && p.lse != nullptr)
      p.lse[(tok0 + t) * kHeads + h] = (l_run > 0.f) ? (m_run + log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
  }

  __syncwarp();
  // after an abort, both MMA issuers' MMAs finish before TMEM is released
  if (warp == 6 && *abort_flag) {
    if (lane == 0) umma_commit(&bar[kBarDrain]);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*abort_flag) {
      if (lane == 0) {
        umma_commit(&bar[kBarDrain]);
        if (!mbar_wait_drain(&bar[kBarDrain], 0)) report_status(p.status, kStatusTimeout);
      }
      __syncwarp();
    }
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace prefill

cudaError_t launch_prefill(const CUtensorMap &tm_k, const CUtensorMap &tm_v, const uint16_t *q, uint16_t *out,
                           float *lse, int B, int L, float scale, int32_t *status, cudaStream_t stream) {
  static std::atomic<int> configured_device{-1};
  const cudaError_t e0 = set_smem_limit_once(prefill::prefill_kernel, prefill::kSmemBytes, configured_device);
  if (e0 != cudaSuccess) return e0;
  prefill::Params p{q, out, lse, B, L, scale * 1.4426950408889634f, status};
  const int nqb = (L + prefill::kQBlock - 1) / prefill::kQBlock;
  return launch_chained(prefill::prefill_kernel, dim3(nqb, kHeads, B), dim3(prefill::kThreads), prefill::kSmemBytes,
                        stream, tm_k, tm_v, p);
}

}  // namespace mla

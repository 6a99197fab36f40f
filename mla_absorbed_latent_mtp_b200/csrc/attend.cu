// attend.cu -- split-L latent attention (Module 05, section 3: scores q~.c_j at the
// original scale, softmax over the causally visible positions of section 4, value
// sum kept in latent space) for a contiguous, paged or index-listed latent cache.
//
// Work decomposition.  Every sequence's visible rows are cut into 128-row tiles; the
// tiles of all sequences form one list that G CTA groups split into equal contiguous
// ranges (a range may cross sequence boundaries; each piece is a "segment").  A group
// holds one CTA per query of a verify window (Q CTAs for dense/paged caches, all reading
// the same tiles at the same time, so all but the first read hit L2), or one CTA per
// (sequence, query) list for the indexed mode.  Each segment leaves an unnormalised
// partial (O, running max m, running sum l) in the workspace; the combine kernel merges
// them with their log-sum-exp weights.
//
// Per CTA (320 threads): warp 0 loads (TMA for dense/paged rows and q~, 16-byte async
// copies for indexed rows), warp 1 issues tcgen05 MMAs, warps 2-9 run the softmax and
// the epilogue as two warpgroups of 32 head columns each.  The 64 query rows (heads) of
// one query sit on the MMA N side and the 128 cache rows of a tile on the M side:
//   S^T[tile rows, heads]  = C_tile (128 x 512, K-major)  *  Q~^T          (TMEM, fp32)
//   O^T[latent, heads]    += C_tile^T (512 x 128, MN-major) * P^T          (TMEM, fp32)
// so the latent dimension of O lives in TMEM lanes (4 blocks x 64 columns) and one
// softmax thread owns one cache row of the tile and 32 heads.  A tile stays in shared
// memory from its score GEMM to its value GEMM, so every cache byte is read once.
#include <math.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"

namespace mla {
namespace attend {

constexpr int kTile = 128;                      // cache rows per tile (MMA M of the score GEMM)
constexpr int kRows = 64;                       // query rows per CTA = heads (MMA N)
constexpr int kChunks = kLatent / 64;           // latent split in 128-byte swizzle columns
constexpr int kChunkBytes = kTile * 64 * 2;     // 16 KB: 128 rows x 64 latent
constexpr int kQtChunkBytes = kRows * 64 * 2;   // 8 KB: 64 heads x 64 latent
constexpr int kPBytes = kTile * kRows * 2;      // 16 KB: P^T, 128 rows x 64 heads (bf16)
constexpr int kThreads = 320;  // producer, MMA, 8 softmax warps
constexpr int kSoftmaxWarps = 8;
constexpr float kTau = 8.0f;  // lazy rescale: the running max is raised only when a score
                              // exceeds it by more than 2^8 (probabilities stay <= 256)

constexpr int kOffC = 0;
constexpr int kOffQt = kOffC + kChunks * kChunkBytes;
constexpr int kOffP = kOffQt + kChunks * kQtChunkBytes;
constexpr int kOffRed = kOffP + kPBytes;         // [4][64] floats
constexpr int kOffMUsed = kOffRed + 4 * 64 * 4;  // [64] floats
constexpr int kOffAlpha = kOffMUsed + 64 * 4;    // [64] floats
constexpr int kOffBar = kOffAlpha + 64 * 4;
// barriers
constexpr int kBarCFull = 0, kBarCEmpty = 8, kBarQFull = 16, kBarQEmpty = 17, kBarSFull = 18, kBarSEmpty = 20,
              kBarPFull = 22, kBarPEmpty = 23, kBarOFull = 24, kBarOEmpty = 25, kNumBars = 26;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemUsed = kOffMisc + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;  // slack for 1024-byte alignment of the base
static_assert(kSmemBytes <= 232448, "shared memory budget");

// TMEM columns: two score buffers, then O^T as four 128-lane blocks of 64 columns.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemO = 256;

// ------------------------------------------------------------------ sequences and tiles

// Rows of data of tile-list sequence s: the cache length L_b (dense/paged) or the list
// length K (indexed: one list per (b, i)).
__device__ __forceinline__ int seq_rows(const AttendParams &p, int mode, int s) {
  if (mode == kModeIndexed) return p.K;
  int L = p.seq_lens ? p.seq_lens[s] : p.Lmax;
  const int cap = (mode == kModePaged) ? p.max_pages * kPageTokens : p.Lmax;
  return min(max(L, 0), cap);
}
__device__ __forceinline__ int num_seqs(const AttendParams &p, int mode) {
  return mode == kModeIndexed ? p.B * p.Q : p.B;
}
__device__ __forceinline__ int seq_tiles(const AttendParams &p, int mode, int s) {
  return (seq_rows(p, mode, s) + kTile - 1) / kTile;
}

// Total tiles over all sequences (computed by one warp).
__device__ long long warp_total_tiles(const AttendParams &p, int mode, int lane) {
  long long acc = 0;
  const int ns = num_seqs(p, mode);
  for (int s = lane; s < ns; s += 32) acc += seq_tiles(p, mode, s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

__device__ __forceinline__ long long group_start(long long g, long long T, long long G) { return g * T / G; }

struct Seg {
  int s;      // sequence in the tile list
  int lo, hi; // tile range within the sequence
  int rows;   // data rows of the sequence
};

// Walks the segments of a contiguous range [t, t_end) of the global tile list.
struct SegIter {
  long long t, t_end, base;
  int s;
  __device__ SegIter(long long t0, long long t1) : t(t0), t_end(t1), base(0), s(0) {}
  __device__ bool next(const AttendParams &p, int mode, Seg &sg) {
    if (t >= t_end) return false;
    int nt = seq_tiles(p, mode, s);
    while (base + nt <= t) {
      base += nt;
      ++s;
      nt = seq_tiles(p, mode, s);
    }
    sg.s = s;
    sg.lo = (int)(t - base);
    const long long hi = min(t_end - base, (long long)nt);
    sg.hi = (int)hi;
    sg.rows = seq_rows(p, mode, s);
    t = base + hi;
    return true;
  }
};

// ------------------------------------------------------------------ cache addressing
// Row (in units of R latent values) of logical position j of sequence b.  Shared by the
// attend producers and the debug gather, so the latter checks the former bit for bit.
__device__ __forceinline__ long long dense_row(int b, int j, int Lmax) { return (long long)b * Lmax + j; }

__device__ __forceinline__ long long paged_row(const int32_t *table, int b, int j, int max_pages, int num_pages,
                                               bool &bad) {
  const int page = table[(long long)b * max_pages + j / kPageTokens];
  if (page < 0 || page >= num_pages) {
    bad = true;
    return 0;
  }
  return (long long)page * kPageTokens + (j % kPageTokens);
}

// Indexed: list position k of query i of sequence b; valid entries lie in [0, limit].
__device__ __forceinline__ long long indexed_row(const int32_t *indices, int b, int i, int k, int Q, int K,
                                                 int Lmax, int limit, bool &bad) {
  const int j = indices[((long long)b * Q + i) * K + k];
  if (j < 0 || j > limit || j >= Lmax) {
    bad = true;
    return 0;
  }
  return (long long)b * Lmax + j;
}

__device__ __forceinline__ int query_limit(const AttendParams &p, int b, int i) {
  const int L = p.seq_lens ? p.seq_lens[b] : p.Lmax;
  return L - p.Q + i;  // position of query i; it sees rows 0..limit
}

// ------------------------------------------------------------------ shared state
struct Shared {
  uint8_t *base;
  uint64_t *bar;
  float *red, *m_used, *alpha;
  uint32_t *tmem_slot;
  volatile int *abort_flag;
  __device__ uint8_t *chunk(int c) const { return base + kOffC + c * kChunkBytes; }
  __device__ uint8_t *qt(int c) const { return base + kOffQt + c * kQtChunkBytes; }
  __device__ uint8_t *pbuf() const { return base + kOffP; }
};

__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, const Shared &sh, int32_t *status) {
  const bool ok = mbar_wait(bar, parity, sh.abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// ------------------------------------------------------------------ producer (warp 0)
// Streams, per segment, q~ (64 heads x 512) once and then every tile's 8 latent chunks
// into the 8-slot ring; slot c of tile t is refilled once the value GEMM of tile t-1 has
// consumed chunk c.
template <int kMode>
__device__ void producer_role(const AttendParams &p, const Shared &sh, const CUtensorMap *tm_cache,
                              const CUtensorMap *tm_qt, int iq, long long t0, long long t1, int lane) {
  uint64_t *bar = sh.bar;
  uint32_t tile_k = 0, q_use = 0;
  SegIter it(t0, t1);
  Seg sg;
  while (it.next(p, kMode, sg)) {
    const int b = (kMode == kModeIndexed) ? sg.s / p.Q : sg.s;
    const int qi = (kMode == kModeIndexed) ? sg.s % p.Q : iq;
    const int qrow0 = (b * p.Q + qi) * kRows;
    bool ok;
    if constexpr (kMode == kModeIndexed)
      ok = wait_warp(&bar[kBarQEmpty], (q_use & 1) ^ 1, sh, p.status);  // whole warp runs this role
    else
      ok = mbar_wait(&bar[kBarQEmpty], (q_use & 1) ^ 1, sh.abort_flag, p.status);  // lane 0 only
    if (!ok) return;
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar[kBarQFull], kChunks * kQtChunkBytes);
#pragma unroll
      for (int c = 0; c < kChunks; ++c) tma_load_2d(sh.qt(c), tm_qt, &bar[kBarQFull], c * 64, qrow0);
    }
    ++q_use;
    for (int t = sg.lo; t < sg.hi; ++t, ++tile_k) {
      if constexpr (kMode == kModeIndexed) {
        // four tile rows per lane; rows past the list end are zero-filled
        const int limit = query_limit(p, b, qi);
        const uint16_t *src[4];
        uint32_t nbytes[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int k = t * kTile + lane + 32 * m;
          bool bad = false;
          long long row = 0;
          if (k < p.K) row = indexed_row(p.indices, b, qi, k, p.Q, p.K, p.Lmax, limit, bad);
          if (bad) report_status(p.status, kStatusIndex);
          src[m] = p.cache + row * kLatent;
          nbytes[m] = (k < p.K && !bad) ? 16u : 0u;
        }
        for (int c = 0; c < kChunks; ++c) {
          if (!wait_warp(&bar[kBarCEmpty + c], (tile_k & 1) ^ 1, sh, p.status)) return;
          const uint32_t dst_c = smem_u32(sh.chunk(c));
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int r = lane + 32 * m;
            const uint32_t dst_r = dst_c + r * 128;
#pragma unroll
            for (int pc = 0; pc < 8; ++pc)
              cp_async_16(dst_r + ((pc ^ (r & 7)) << 4), src[m] + c * 64 + pc * 8, nbytes[m]);
          }
          cp_async_arrive_noinc(&bar[kBarCFull + c]);
        }
      } else {
        const int j0 = t * kTile;
        long long row[2] = {0, 0};
        bool load[2];
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          const int jj = j0 + hb * 64;
          load[hb] = jj < sg.rows;
          if (load[hb]) {
            if constexpr (kMode == kModePaged) {
              bool bad = false;
              row[hb] = paged_row(p.page_table, b, jj, p.max_pages, p.num_pages, bad);
              if (bad) report_status(p.status, kStatusIndex);
            } else {
              row[hb] = dense_row(b, jj, p.Lmax);
            }
          }
        }
        const uint32_t bytes = (load[0] ? 8192u : 0u) + (load[1] ? 8192u : 0u);
        for (int c = 0; c < kChunks; ++c) {
          if (!mbar_wait(&bar[kBarCEmpty + c], (tile_k & 1) ^ 1, sh.abort_flag, p.status)) return;
          mbar_arrive_expect_tx(&bar[kBarCFull + c], bytes);
#pragma unroll
          for (int hb = 0; hb < 2; ++hb)
            if (load[hb]) tma_load_2d(sh.chunk(c) + hb * 8192, tm_cache, &bar[kBarCFull + c], c * 64, (int)row[hb]);
        }
      }
    }
  }
}

// ------------------------------------------------------------------ MMA issuer (warp 1)
// Rows past the end of the sequence may hold any bits: zero them in the landed chunk so
// that a masked (zero) probability never meets a NaN or Inf in the value product.
template <int kMode>
__device__ __forceinline__ void prepare_chunk(uint32_t cbase, int n_valid, int lane) {
  if (kMode != kModeIndexed && n_valid < kTile) {
    for (int idx = lane; idx < (kTile - n_valid) * 8; idx += 32)
      st_shared_v4(cbase + (n_valid + idx / 8) * 128 + (idx % 8) * 16, 0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if (kMode == kModeIndexed) fence_proxy_async_smem();  // rows written by 16-byte async copies
  __syncwarp();
}

template <int kMode>
__device__ void mma_role(const AttendParams &p, const Shared &sh, uint32_t tmem, long long t0, long long t1,
                         int lane) {
  uint64_t *bar = sh.bar;
  constexpr uint32_t idesc_s = idesc_bf16_f32(128, kRows, false, false);
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, kRows, true, true);
  uint32_t tile_k = 0, s_use = 0, p_use = 0, q_use = 0, o_use = 0;
  const uint32_t c_base = smem_u32(sh.chunk(0));
  const uint32_t qt_base = smem_u32(sh.qt(0));
  const uint32_t p_base = smem_u32(sh.pbuf());
  SegIter it(t0, t1);
  Seg sg;
  while (it.next(p, kMode, sg)) {
    if (!wait_warp(&bar[kBarQFull], q_use & 1, sh, p.status)) return;
    ++q_use;
    for (int t = sg.lo; t < sg.hi; ++t, ++tile_k) {
      const int n_valid = min(kTile, sg.rows - t * kTile);
      // S^T[tile rows, heads] = C_tile * Q~^T, K = 512 latent in 8 chunks of 4 MMA steps
      const uint32_t sb = s_use & 1;
      if (!wait_warp(&bar[kBarSEmpty + sb], ((s_use >> 1) & 1) ^ 1, sh, p.status)) return;
      tc_fence_after();
      for (int c = 0; c < kChunks; ++c) {
        if (!wait_warp(&bar[kBarCFull + c], tile_k & 1, sh, p.status)) return;
        prepare_chunk<kMode>(c_base + c * kChunkBytes, n_valid, lane);
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = sw128_desc(c_base + c * kChunkBytes + kk * 32, 16, 1024);
            const uint64_t bdesc = sw128_desc(qt_base + c * kQtChunkBytes + kk * 32, 16, 1024);
            umma_bf16(tmem + kTmemS + sb * kRows, a, bdesc, idesc_s, (c | kk) != 0);
          }
        }
        __syncwarp();
      }
      if (lane == 0) {
        umma_commit(&bar[kBarSFull + sb]);
        if (t == sg.hi - 1) umma_commit(&bar[kBarQEmpty]);
      }
      ++s_use;
      // O^T[latent, heads] += C_tile^T * P^T, four 128-lane latent blocks, K = 128 rows
      if (!wait_warp(&bar[kBarPFull], p_use & 1, sh, p.status)) return;
      ++p_use;
      if (t == sg.lo && !wait_warp(&bar[kBarOEmpty], (o_use & 1) ^ 1, sh, p.status)) return;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            // A = C_tile^T: latent (M) along the 128-byte rows, 64-wide atoms in the two
            // chunks 2mb, 2mb+1 (LBO = chunk stride); cache rows (K) in 8-row groups.
            const uint64_t a = sw128_desc(c_base + (2 * mb) * kChunkBytes + kk * 2048, kChunkBytes, 1024);
            // B = P^T: heads (N) along the 128-byte rows, cache rows (K) in 8-row groups.
            const uint64_t bdesc = sw128_desc(p_base + kk * 2048, 8192, 1024);
            umma_bf16(tmem + kTmemO + mb * kRows, a, bdesc, idesc_o, (t > sg.lo || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bar[kBarCEmpty + 2 * mb]);
          umma_commit(&bar[kBarCEmpty + 2 * mb + 1]);
        }
        umma_commit(&bar[kBarPEmpty]);
      }
      __syncwarp();
    }
    if (lane == 0) umma_commit(&bar[kBarOFull]);
    ++o_use;
  }
}

// ------------------------------------------------------------------ softmax + epilogue (warps 2-9)
// Two warpgroups; warpgroup wg owns head columns [32 wg, 32 wg + 32) of S^T and O^T.  Thread
// `row` of a warpgroup owns cache row `row` of the tile.  The running max per column lives
// in shared memory (read with broadcast loads).  With 10 warps, three share an SM
// sub-partition's register file, which caps a thread at 168 registers.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int kMode>
__device__ void softmax_role(const AttendParams &p, const Shared &sh, uint32_t tmem, int g, int iq, long long t0,
                             long long t1, int warp, int lane) {
  uint64_t *bar = sh.bar;
  const int wg = (warp - 2) >> 2;              // warpgroup: head columns [32 wg, 32 wg + 32)
  const int wq = warp & 3;                     // TMEM lane quadrant of this warp
  const int tid = ((warp - 2) & 3) * 32 + lane;  // 0..127 within the warpgroup
  const int row = wq * 32 + lane;              // tile row (TMEM lane) owned by this thread
  const uint32_t bar_id = 1 + wg;
  const int col0 = wg * 32;
  const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
  const uint32_t p_row = smem_u32(sh.pbuf()) + row * 128;
  float *red = sh.red;          // [4 quadrants][64 columns]
  float *m_used = sh.m_used;    // [64]
  float *alpha = sh.alpha;      // [64]
  uint32_t s_use = 0, p_use = 0, o_use = 0;
  const float *mu = m_used + col0;  // running max of this warpgroup's columns (log2 units)
  if (tid < 32) m_used[col0 + tid] = -INFINITY;
  named_bar_sync(bar_id, 128);
  SegIter it(t0, t1);
  Seg sg;
  while (it.next(p, kMode, sg)) {
    const int qi = (kMode == kModeIndexed) ? sg.s % p.Q : iq;
    // positions of this CTA's query that are visible: dense/paged rows 0..L_b-Q+qi, or the list
    const int n_vis = (kMode == kModeIndexed) ? p.K : sg.rows - p.Q + qi + 1;
    float l_part[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) l_part[c] = 0.f;
    for (int t = sg.lo; t < sg.hi; ++t) {
      const uint32_t sb = s_use & 1;
      mbar_wait(&bar[kBarSFull + sb], (s_use >> 1) & 1, sh.abort_flag, p.status);
      tc_fence_after();
      const bool valid = (t * kTile + row) < n_vis;
      float s2[32];
      {
        uint32_t r[32];
        tmem_ld32(t_lane + kTmemS + sb * kRows + col0, r);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) s2[c] = valid ? __uint_as_float(r[c]) * p.scale_log2 : -INFINITY;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kBarSEmpty + sb]);
      ++s_use;
      bool flag = false;
#pragma unroll
      for (int c = 0; c < 32; ++c) flag |= s2[c] > mu[c] + kTau;
      const bool any = named_bar_or(bar_id, 128, flag);
      if (*sh.abort_flag) return;
      if (any) {
        // new running max for this warpgroup's 32 columns
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float mx = warp_max_f32(s2[c]);
          if (lane == c) red[wq * kRows + col0 + c] = mx;
        }
        named_bar_sync(bar_id, 128);
        if (tid < 32) {
          const int c = col0 + tid;
          const float mt = fmaxf(fmaxf(red[c], red[kRows + c]), fmaxf(red[2 * kRows + c], red[3 * kRows + c]));
          const float mo = m_used[c];
          const float mn = fmaxf(mo, mt);
          alpha[c] = (mn == -INFINITY) ? 1.f : fast_exp2(mo - mn);
          m_used[c] = mn;
        }
        named_bar_sync(bar_id, 128);
#pragma unroll
        for (int c = 0; c < 32; ++c) l_part[c] *= alpha[col0 + c];
      }
      // the P buffer is free and the previous value product has finished
      mbar_wait(&bar[kBarPEmpty], (p_use & 1) ^ 1, sh.abort_flag, p.status);
      tc_fence_after();
      if (any && t > sg.lo) {
        // running max moved: rescale this warpgroup's O^T columns in TMEM
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
          uint32_t r[32];
          const uint32_t addr = t_lane + kTmemO + mb * kRows + col0;
          tmem_ld32(addr, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha[col0 + j]);
          tmem_st32(addr, r);
        }
        tmem_st_wait();
      }
      // probabilities, rounded to bf16 for the value product; l sums the rounded values
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c0 = pc * 8 + 2 * e;
          const float p0 = (s2[c0] == -INFINITY) ? 0.f : fast_exp2(s2[c0] - mu[c0]);
          const float p1 = (s2[c0 + 1] == -INFINITY) ? 0.f : fast_exp2(s2[c0 + 1] - mu[c0 + 1]);
          w[e] = pack_bf16x2(p0, p1);
          l_part[c0] += bf16lo_to_f32(w[e]);
          l_part[c0 + 1] += bf16hi_to_f32(w[e]);
        }
        st_shared_v4(p_row + (((wg * 4 + pc) ^ (row & 7)) << 4), w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kBarPFull]);
      ++p_use;
    }
    // ---- epilogue: l column sums, partial O, (m, l) -> workspace
    mbar_wait(&bar[kBarOFull], o_use & 1, sh.abort_flag, p.status);
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      float v = l_part[c];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == c) red[wq * kRows + col0 + c] = v;
    }
    named_bar_sync(bar_id, 128);
    if (*sh.abort_flag) return;
    const long long slot =
        (kMode == kModeIndexed) ? (long long)g + sg.s : ((long long)g + sg.s) * p.Q + iq;
    if (tid < 32) {
      const int c = col0 + tid;
      p.part_m[slot * kRows + c] = m_used[c];
      p.part_l[slot * kRows + c] = red[c] + red[kRows + c] + red[2 * kRows + c] + red[3 * kRows + c];
    }
    float *po = p.part_o + slot * kRows * kLatent;
#pragma unroll 1
    for (int mb = 0; mb < 4; ++mb) {
      uint32_t r[32];
      tmem_ld32(t_lane + kTmemO + mb * kRows + col0, r);
      tmem_ld_wait();
      const int lat = mb * 128 + wq * 32 + lane;
#pragma unroll
      for (int j = 0; j < 32; ++j) po[(col0 + j) * kLatent + lat] = __uint_as_float(r[j]);
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar[kBarOEmpty]);
    ++o_use;
    named_bar_sync(bar_id, 128);
    if (tid < 32) m_used[col0 + tid] = -INFINITY;
    named_bar_sync(bar_id, 128);
  }
}

// ------------------------------------------------------------------ kernel
template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tm_cache, const __grid_constant__ CUtensorMap tm_qt,
                  const AttendParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Shared sh;
  sh.base = base;
  sh.bar = reinterpret_cast<uint64_t *>(base + kOffBar);
  sh.red = reinterpret_cast<float *>(base + kOffRed);
  sh.m_used = reinterpret_cast<float *>(base + kOffMUsed);
  sh.alpha = reinterpret_cast<float *>(base + kOffAlpha);
  sh.tmem_slot = reinterpret_cast<uint32_t *>(base + kOffMisc);
  sh.abort_flag = reinterpret_cast<volatile int *>(base + kOffMisc + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = blockIdx.x / p.group_size;
  const int iq = blockIdx.x % p.group_size;

  if (threadIdx.x == 0) {
    for (int c = 0; c < kChunks; ++c) {
      mbar_init(&sh.bar[kBarCFull + c], kMode == kModeIndexed ? 32 : 1);
      mbar_init(&sh.bar[kBarCEmpty + c], 1);
    }
    mbar_init(&sh.bar[kBarQFull], 1);
    mbar_init(&sh.bar[kBarQEmpty], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.bar[kBarSFull + i], 1);
      mbar_init(&sh.bar[kBarSEmpty + i], kSoftmaxWarps);
    }
    mbar_init(&sh.bar[kBarPFull], kSoftmaxWarps);
    mbar_init(&sh.bar[kBarPEmpty], 1);
    mbar_init(&sh.bar[kBarOFull], 1);
    mbar_init(&sh.bar[kBarOEmpty], kSoftmaxWarps);
    *sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(sh.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // tile range of this CTA's group
  const long long T = warp_total_tiles(p, kMode, lane);
  const long long G = p.groups;
  const long long t0 = group_start(g, T, G), t1 = group_start(g + 1, T, G);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sh.tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tm_qt);
      if (kMode != kModeIndexed) prefetch_tensormap(&tm_cache);
    }
    if (kMode == kModeIndexed || lane == 0) producer_role<kMode>(p, sh, &tm_cache, &tm_qt, iq, t0, t1, lane);
  } else if (warp == 1) {
    mma_role<kMode>(p, sh, tmem, t0, t1, lane);
  } else {
    softmax_role<kMode>(p, sh, tmem, g, iq, t0, t1, warp, lane);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*sh.abort_flag) {
      // drain: let every issued MMA finish before TMEM is released, and give in-flight
      // copies time to land before the shared memory is handed to another CTA
      if (lane == 0) {
        umma_commit(&sh.bar[kBarOFull]);
        const long long t_start = clock64();
        while (clock64() - t_start < 2000000) {
        }
      }
      __syncwarp();
    }
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ combine
// One block per (sequence b, query i) and pair of heads; thread t owns latent 4t..4t+3.
// The partial of every CTA group that processed tiles of b is weighted by
// 2^(m_g - M) (M the largest running max) and the weighted sums are normalised.
constexpr int kCombineHeads = 2;
constexpr int kMaxSlotsPerSeq = 1024;

__global__ void __launch_bounds__(128) combine_kernel(const AttendParams p, int mode) {
  const int v = blockIdx.x;  // b * Q + i
  const int b = v / p.Q, i = v % p.Q;
  const int s = (mode == kModeIndexed) ? v : b;
  __shared__ long long sh_info[3];
  __shared__ float sh_w[kCombineHeads][kMaxSlotsPerSeq];
  __shared__ float sh_l[kCombineHeads][kMaxSlotsPerSeq];
  __shared__ float sh_norm[kCombineHeads][2];  // 1/den, lse
  const int tid = threadIdx.x;
  if (tid < 32) {
    const int ns = num_seqs(p, mode);
    long long before = 0, total = 0;
    for (int x = tid; x < ns; x += 32) {
      const int nt = seq_tiles(p, mode, x);
      total += nt;
      if (x < s) before += nt;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      before += __shfl_xor_sync(0xffffffffu, before, o);
      total += __shfl_xor_sync(0xffffffffu, total, o);
    }
    if (tid == 0) {
      sh_info[0] = before;
      sh_info[1] = seq_tiles(p, mode, s);
      sh_info[2] = total;
      if (blockIdx.y == 0 && i == 0 && mode != kModeIndexed && p.seq_lens != nullptr) {
        const int L = p.seq_lens[b];
        const int cap = (mode == kModePaged) ? p.max_pages * kPageTokens : p.Lmax;
        if (L < 0 || L > cap) report_status(p.status, kStatusIndex);
      }
    }
  }
  __syncthreads();
  const long long ts = sh_info[0], nt = sh_info[1], T = sh_info[2], G = p.groups;
  long long g_first = 0, g_last = -1;
  if (nt > 0) {
    g_first = ((ts + 1) * G - 1) / T;
    g_last = ((ts + nt) * G - 1) / T;
  }
  const int nslot = (int)min(g_last - g_first + 1, (long long)kMaxSlotsPerSeq);
  auto slot_of = [&](long long gg) -> long long {
    return (mode == kModeIndexed) ? gg + s : (gg + s) * p.Q + i;
  };
  const int h0 = blockIdx.y * kCombineHeads;
  // weights: running maxima of the non-empty groups, then 2^(m - M) and the normaliser
  for (int x = tid; x < kCombineHeads * nslot; x += 128) {
    const int hh = x / nslot, k = x % nslot;
    const long long gg = g_first + k;
    float m = -INFINITY, l = 0.f;
    if (group_start(gg, T, G) < group_start(gg + 1, T, G)) {
      m = p.part_m[slot_of(gg) * kRows + h0 + hh];
      l = p.part_l[slot_of(gg) * kRows + h0 + hh];
    }
    sh_w[hh][k] = m;
    sh_l[hh][k] = l;
  }
  __syncthreads();
  if (tid < kCombineHeads) {
    const int hh = tid;
    float M = -INFINITY;
    for (int k = 0; k < nslot; ++k) M = fmaxf(M, sh_w[hh][k]);
    float den = 0.f;
    for (int k = 0; k < nslot; ++k) {
      const float m = sh_w[hh][k];
      const float w = (m == -INFINITY) ? 0.f : exp2f(m - M);
      sh_w[hh][k] = w;
      den += w * sh_l[hh][k];
    }
    const bool ok = (M != -INFINITY) && den > 0.f;
    sh_norm[hh][0] = ok ? 1.f / den : 0.f;
    sh_norm[hh][1] = ok ? (M + log2f(den)) * 0.69314718055994530942f : -INFINITY;
  }
  __syncthreads();
  const int lat = tid * 4;
#pragma unroll
  for (int hh = 0; hh < kCombineHeads; ++hh) {
    const int h = h0 + hh;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int k = 0; k < nslot; ++k) {
      const float w = sh_w[hh][k];
      if (w != 0.f) {
        const float4 o = *reinterpret_cast<const float4 *>(p.part_o + (slot_of(g_first + k) * kRows + h) * kLatent + lat);
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
      }
    }
    const float inv = sh_norm[hh][0];
    uint2 outv;
    outv.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    outv.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(p.o_latent + ((long long)v * kRows + h) * kLatent + lat) = outv;
    if (p.lse != nullptr && tid == 0) p.lse[(long long)v * kRows + h] = sh_norm[hh][1];
  }
}

// ------------------------------------------------------------------ debug gather
__global__ void debug_gather_kernel(int mode, const uint16_t *src, const int32_t *page_table,
                                    const int32_t *indices, int Q, int R, int Lmax, int max_pages, int num_pages,
                                    int K, int B, const int32_t *req, int n_req, uint16_t *out, int32_t *status) {
  const int r = blockIdx.x;
  if (r >= n_req) return;
  const int b = req[3 * r], i = req[3 * r + 1], k = req[3 * r + 2];
  bool bad = (b < 0 || b >= B);
  long long row = 0;
  if (!bad) {
    if (mode == kModeDense) {
      bad = (k < 0 || k >= Lmax);
      if (!bad) row = dense_row(b, k, Lmax);
    } else if (mode == kModePaged) {
      bad = (k < 0 || k >= max_pages * kPageTokens);
      if (!bad) row = paged_row(page_table, b, k, max_pages, num_pages, bad);
    } else {
      bad = (i < 0 || i >= Q || k < 0 || k >= K);
      if (!bad) row = indexed_row(indices, b, i, k, Q, K, Lmax, Lmax - 1, bad);
    }
  }
  if (bad && threadIdx.x == 0) report_status(status, kStatusIndex);
  for (int x = threadIdx.x; x < R; x += blockDim.x) out[(long long)r * R + x] = bad ? 0 : src[row * R + x];
}

}  // namespace attend

// ------------------------------------------------------------------ host launchers
size_t attend_slots(int B, int Q, int sms) {
  const size_t g_dense = (size_t)std::max(1, sms / std::max(Q, 1));
  const size_t a = (g_dense + (size_t)B) * (size_t)Q;
  const size_t c = (size_t)sms + (size_t)B * (size_t)Q;
  return a > c ? a : c;
}

size_t attend_workspace_bytes_for(int B, int Q, int sms) {
  const size_t slots = attend_slots(B, Q, sms);
  return slots * kHeads * kLatent * sizeof(float) + 2 * slots * kHeads * sizeof(float);
}

template <int kMode>
static cudaError_t launch_attend_mode(const CUtensorMap &tm_cache, const CUtensorMap &tm_qt, const AttendParams &p,
                                      cudaStream_t stream) {
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(attend::attend_kernel<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         attend::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  const int grid = p.groups * p.group_size;
  attend::attend_kernel<kMode><<<grid, attend::kThreads, attend::kSmemBytes, stream>>>(tm_cache, tm_qt, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 cgrid(p.B * p.Q, kHeads / attend::kCombineHeads);
  attend::combine_kernel<<<cgrid, 128, 0, stream>>>(p, kMode);
  return cudaGetLastError();
}

cudaError_t launch_attend(int mode, const CUtensorMap &tm_cache, const CUtensorMap &tm_qt, const AttendParams &p,
                          cudaStream_t stream) {
  switch (mode) {
    case kModeDense:
      return launch_attend_mode<kModeDense>(tm_cache, tm_qt, p, stream);
    case kModePaged:
      return launch_attend_mode<kModePaged>(tm_cache, tm_qt, p, stream);
    default:
      return launch_attend_mode<kModeIndexed>(tm_cache, tm_qt, p, stream);
  }
}

cudaError_t launch_debug_gather(int mode, const uint16_t *src, const int32_t *page_table, const int32_t *indices,
                                int B, int Q, int R, int Lmax, int max_pages, int num_pages, int K,
                                const int32_t *req, int n_req, uint16_t *out, int32_t *status, cudaStream_t stream) {
  attend::debug_gather_kernel<<<n_req, 128, 0, stream>>>(mode, src, page_table, indices, Q, R, Lmax, max_pages,
                                                         num_pages, K, B, req, n_req, out, status);
  return cudaGetLastError();
}

}  // namespace mla

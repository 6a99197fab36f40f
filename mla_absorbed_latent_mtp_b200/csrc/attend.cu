// attend.cu -- split-L latent attention (Module 05, section 3: scores q~.c_j at the
// original scale, softmax over the causally visible positions of section 4, value
// sum kept in latent space) for a contiguous, paged or index-listed latent cache.
//
// Work decomposition.  Every sequence's visible rows are cut into 64-row tiles; the
// tiles of all sequences form one list that G CTA groups split into equal contiguous
// ranges (a range may cross sequence boundaries; each piece is a "segment").  A group
// holds one CTA per query of a verify window (Q CTAs for dense/paged caches, all reading
// the same tiles at the same time, so all but the first read hit L2), or one CTA per
// (sequence, query) list for the indexed mode.  Each segment leaves an unnormalised
// partial (O, running max m, running sum l) in the workspace; the combine kernel merges
// them with their log-sum-exp weights -- or, for index lists whose CTAs run as one
// thread-block cluster per list, the cluster merges them itself after a cluster barrier.
//
// Per CTA (384 threads): warp 0 loads (one TMA copy per ring slot for dense/paged rows,
// one for q~; 16-byte async copies for indexed rows, shared with warp 11), warp 1 issues
// the score MMAs and warp 10 the value MMAs (tcgen05), warps 2-9 run the softmax and the
// epilogue as two warpgroups of 32 head columns each.  The 64 query rows (heads) of one
// query sit on the MMA N side and the 64 cache rows of a tile on the M side:
//   S^T[tile rows, heads]  = C_tile (64 x 512, K-major)  *  Q~^T           (TMEM, fp32)
//   O^T[latent, heads]    += C_tile^T (512 x 64, MN-major) * P^T           (TMEM, fp32)
// so the latent dimension of O lives in TMEM lanes (4 blocks x 64 columns).  A tile
// stays in shared memory from its score GEMM to its value GEMM, so every cache byte is
// read once.  The ring holds 2.25 tiles: while the softmax works on tile t, the score
// GEMM of tile t+1 runs and tile t+2 streams in; the MMA warp issues each tile's value
// GEMM as soon as its probabilities are ready, which frees its ring slots.
#include <math.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "internal.h"
#include "sm100.cuh"
#include "split.cuh"

namespace mla {
namespace attend {

constexpr int kTile = 64;                       // cache rows per tile (MMA M of the score GEMM)
constexpr int kRows = 64;                       // query rows per CTA = heads (MMA N)
constexpr int kSlotQuarters = kLatent / 128;    // a tile is 4 ring slots of 128 latent values
constexpr int kSlots = 9;                       // ring slots (2.25 tiles)
constexpr int kAtomBytes = kTile * 128;         // 8 KB: 64 rows x 64 latent, 128-byte swizzle
constexpr int kSlotBytes = 2 * kAtomBytes;      // 16 KB: 64 rows x 128 latent
constexpr int kQtChunks = kLatent / 64;
constexpr int kQtChunkBytes = kRows * 64 * 2;   // 8 KB: 64 heads x 64 latent
constexpr int kPBytes = kTile * kRows * 2;      // 8 KB: P^T, 64 rows x 64 heads (bf16)
constexpr int kThreads = 384;  // producer, score MMA, 8 softmax warps, value MMA, second gather warp
constexpr int kSoftmaxWarps = 8;
constexpr float kTau = 8.0f;  // lazy rescale: the running max is raised only when a score
                              // exceeds it by more than 2^8 (probabilities stay <= 256)

constexpr int kOffC = 0;
constexpr int kOffQt = kOffC + kSlots * kSlotBytes;
constexpr int kOffP = kOffQt + kQtChunks * kQtChunkBytes;
constexpr int kOffRed = kOffP + 2 * kPBytes;     // [4][64] floats
constexpr int kOffMUsed = kOffRed + 4 * 64 * 4;  // [64] floats
constexpr int kOffAlpha = kOffMUsed + 64 * 4;    // [64] floats
constexpr int kOffBar = kOffAlpha + 64 * 4;
// barriers
constexpr int kBarCFull = 0, kBarCEmpty = kSlots, kBarQFull = 2 * kSlots, kBarQEmpty = kBarQFull + 1,
              kBarSFull = kBarQEmpty + 1, kBarSEmpty = kBarSFull + 2, kBarPFull = kBarSEmpty + 2,
              kBarPEmpty = kBarPFull + 2, kBarOFull = kBarPEmpty + 2, kBarOEmpty = kBarOFull + 1,
              kBarDrain = kBarOEmpty + 1, kNumBars = kBarDrain + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemUsed = kOffMisc + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;  // slack for 1024-byte alignment of the base
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kPageTokens == kTile, "a paged tile is exactly one page");

// TMEM columns: two score buffers (M = 64 accumulators: lanes 0-15 of each 32-lane
// quadrant hold tile rows 16q..16q+15), then O^T as four 128-lane blocks of 64 columns.
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
using split::group_start;
using split::num_seqs;
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

// Position of every sequence in the tile list (first tile, tile count), for the combine
// (computed by one warp with an exclusive scan in steps of 32 sequences).
__device__ void warp_write_seq_prefix(const AttendParams &p, int mode, int lane) {
  const int ns = num_seqs(p, mode);
  long long base = 0;
  for (int s0 = 0; s0 < ns; s0 += 32) {
    const int s = s0 + lane;
    const int nt = s < ns ? seq_tiles(p, mode, s) : 0;
    long long x = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (s < ns) {
      p.seq_ts[s] = base + x - nt;
      p.seq_nt[s] = nt;
    }
    base += __shfl_sync(0xffffffffu, x, 31);
  }
}

struct Seg {
  int s;       // sequence in the tile list
  int lo, hi;  // tile range within the sequence (clipped to the query's causal window)
  int rows;    // data rows of the sequence
  bool empty;  // no tile of the range is visible to this CTA's query
};

// Walks the segments of a contiguous range [t, t_end) of the global tile list.  For a
// dense or paged cache the range of query iq is clipped to the tiles holding a visible row
// (0 .. L - Q + iq): tiles past the causal window are neither loaded nor multiplied, which
// matters when a window holds many queries (a prefill through this path).  A segment left
// without tiles is returned with `empty` set; its partial is written as empty.
struct SegIter {
  long long t, t_end, base;
  int s, iq;
  __device__ SegIter(long long t0, long long t1, int iq_) : t(t0), t_end(t1), base(0), s(0), iq(iq_) {}
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
    sg.empty = false;
    if (mode != kModeIndexed) {
      const int n_vis = sg.rows - p.Q + iq + 1;
      const int vis_tiles = n_vis > 0 ? (n_vis + kTile - 1) / kTile : 0;
      if (sg.hi > vis_tiles) sg.hi = max(vis_tiles, sg.lo);
      sg.empty = sg.hi <= sg.lo;
    }
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

// Indexed: row of list entry j of sequence b; valid entries lie in [0, limit] and below Lmax.
__device__ __forceinline__ long long indexed_row_of(int b, int j, int Lmax, int limit, bool &bad) {
  if (j < 0 || j > limit || j >= Lmax) {
    bad = true;
    return 0;
  }
  return (long long)b * Lmax + j;
}

// Indexed: list position k of query i of sequence b.
__device__ __forceinline__ long long indexed_row(const int32_t *indices, int b, int i, int k, int Q, int K,
                                                 int Lmax, int limit, bool &bad) {
  return indexed_row_of(b, indices[((long long)b * Q + i) * K + k], Lmax, limit, bad);
}

// An index-list entry of -1 is unused (fixed-width lists shorter than their width).
constexpr int kUnusedEntry = -1;

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
  __device__ uint8_t *slot(int r) const { return base + kOffC + r * kSlotBytes; }
  __device__ uint8_t *qt(int c) const { return base + kOffQt + c * kQtChunkBytes; }
  __device__ uint8_t *pbuf(int i) const { return base + kOffP + i * kPBytes; }
};

__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, const Shared &sh, int32_t *status) {
  const bool ok = mbar_wait(bar, parity, sh.abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// Ring slot k (k = 4 * tile + quarter, counted over the CTA's tiles): position and use.
__device__ __forceinline__ uint32_t ring_pos(uint32_t k) { return k % kSlots; }
__device__ __forceinline__ uint32_t ring_use(uint32_t k) { return k / kSlots; }

// ------------------------------------------------------------------ producer (warp 0)
// Issues the loads; counts the q~ loads and the ring-slot loads it issued (for the drain).
template <int kMode>
// Index lists are gathered by two warps (half 0: warp 0, tile rows 0-31 and the q~ loads;
// half 1: warp 11, tile rows 32-63); dense and paged tiles by lane 0 of warp 0 (half 0).
__device__ void producer_loads(const AttendParams &p, const Shared &sh, const CUtensorMap *tm_cache,
                               const CUtensorMap *tm_qt, int iq, long long t0, long long t1, int lane, int half,
                               uint32_t &q_use, uint32_t &slots_issued) {
  uint64_t *bar = sh.bar;
  uint32_t tile_k = 0;
  SegIter it(t0, t1, iq);
  Seg sg;
  while (it.next(p, kMode, sg)) {
    if (sg.empty) continue;
    const int b = (kMode == kModeIndexed) ? sg.s / p.Q : sg.s;
    const int qi = (kMode == kModeIndexed) ? sg.s % p.Q : iq;
    const int qrow0 = (b * p.Q + qi) * kRows;
    if (half == 0) {
      bool ok;
      if constexpr (kMode == kModeIndexed)
        ok = wait_warp(&bar[kBarQEmpty], (q_use & 1) ^ 1, sh, p.status);  // whole warp runs this role
      else
        ok = mbar_wait(&bar[kBarQEmpty], (q_use & 1) ^ 1, sh.abort_flag, p.status);  // lane 0 only
      if (!ok) return;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar[kBarQFull], kQtChunks * kQtChunkBytes);
        tma_load_3d(sh.qt(0), tm_qt, &bar[kBarQFull], 0, qrow0, 0);  // all 8 chunks in one copy
      }
      ++q_use;
    }
    // indexed: the list entry of this lane's row of the next tile is read while this
    // tile's rows are copied, so the index load latency is off the copy path
    const int32_t *list = p.indices + ((long long)b * p.Q + qi) * p.K;
    const int row_lane = 32 * half + lane;  // the tile row whose list entry this lane holds
    int nxt = 0;
    if constexpr (kMode == kModeIndexed) {
      const int k = sg.lo * kTile + row_lane;
      if (k < p.K) nxt = list[k];
    }
    for (int t = sg.lo; t < sg.hi; ++t, ++tile_k) {
      if constexpr (kMode == kModeIndexed) {
        // rows past the list end are zero-filled
        const int limit = query_limit(p, b, qi);
        const int cur = nxt;
        if (t + 1 < sg.hi) {
          const int k = (t + 1) * kTile + row_lane;
          if (k < p.K) nxt = list[k];
        }
        // cache row (in units of R) of tile row row_lane, -1 when unused
        int rowi;
        {
          const int k = t * kTile + row_lane;
          bool bad = false;
          long long row = 0;
          const bool used = k < p.K && cur != kUnusedEntry;
          if (used) row = indexed_row_of(b, cur, p.Lmax, limit, bad);
          if (bad) report_status(p.status, kStatusIndex);
          rowi = (used && !bad) ? (int)row : -1;
        }
        // Each copy instruction moves two tile rows' 256-byte slice of this slot: lanes
        // 0-15 row 2i, lanes 16-31 row 2i + 1, 16 bytes each, so every instruction reads four
        // whole 128-byte lines (B * Lmax < 2^31 rows, so a row fits an int).  This warp's
        // half of the slot is its 32 rows.
        const int u = lane & 15, at = u >> 3, pc = u & 7;
        for (int qq = 0; qq < kSlotQuarters; ++qq) {
          const uint32_t k = tile_k * kSlotQuarters + qq;
          const uint32_t rp = ring_pos(k);
          if (!wait_warp(&bar[kBarCEmpty + rp], (ring_use(k) & 1) ^ 1, sh, p.status)) return;
          const uint32_t dst_s = smem_u32(sh.slot(rp)) + at * kAtomBytes;
          const uint16_t *src_q = p.cache + qq * 128 + at * 64 + pc * 8;
#pragma unroll
          for (int i = 0; i < kTile / 4; ++i) {
            const int r = 32 * half + 2 * i + (lane >> 4);
            const int ri = __shfl_sync(0xffffffffu, rowi, r & 31);
            cp_async_16(dst_s + r * 128 + ((pc ^ (r & 7)) << 4), src_q + (long long)max(ri, 0) * kLatent,
                        ri >= 0 ? 16u : 0u);
          }
          cp_async_arrive_noinc(&bar[kBarCFull + rp]);
          slots_issued = k + 1;
        }
      } else {
        const int j0 = t * kTile;
        long long row = 0;
        if constexpr (kMode == kModePaged) {
          bool bad = false;
          row = paged_row(p.page_table, b, j0, p.max_pages, p.num_pages, bad);
          if (bad) report_status(p.status, kStatusIndex);
        } else {
          row = dense_row(b, j0, p.Lmax);
        }
        for (int qq = 0; qq < kSlotQuarters; ++qq) {
          const uint32_t k = tile_k * kSlotQuarters + qq;
          const uint32_t rp = ring_pos(k);
          if (!mbar_wait(&bar[kBarCEmpty + rp], (ring_use(k) & 1) ^ 1, sh.abort_flag, p.status)) return;
          mbar_arrive_expect_tx(&bar[kBarCFull + rp], kSlotBytes);
          // one copy per slot: a 3-D box {64 latent, 64 rows, 2 chunks} lands as the slot's two atoms
          tma_load_3d(sh.slot(rp), tm_cache, &bar[kBarCFull + rp], 0, (int)row, 2 * qq);
          slots_issued = k + 1;
        }
      }
    }
  }
}

// The producer role: the loads, then (also after an abort) a wait until every copy it
// issued has landed.
template <int kMode>
__device__ void producer_role(const AttendParams &p, const Shared &sh, const CUtensorMap *tm_cache,
                              const CUtensorMap *tm_qt, int iq, long long t0, long long t1, int lane, int half) {
  uint32_t q_use = 0, slots_issued = 0;
  producer_loads<kMode>(p, sh, tm_cache, tm_qt, iq, t0, t1, lane, half, q_use, slots_issued);
  if constexpr (kMode == kModeIndexed) cp_async_wait_all();  // this lane's row copies
  if (lane == 0) {
    bool ok = drain_ring(&sh.bar[kBarQFull], 1, q_use);
    if constexpr (kMode != kModeIndexed) ok = drain_ring(&sh.bar[kBarCFull], kSlots, slots_issued) && ok;
    if (!ok) report_status(p.status, kStatusTimeout);
  }
}

// ------------------------------------------------------------------ MMA issuer (warp 1)
// Rows past the end of the sequence may hold any bits: zero them in the landed slot so
// that a masked (zero) probability never meets a NaN or Inf in the value product.
template <int kMode>
__device__ __forceinline__ void prepare_slot(uint32_t sbase, int n_valid, int lane) {
  if (kMode != kModeIndexed && n_valid < kTile) {
    const int n_zero = (kTile - n_valid) * 8;  // 16-byte units per atom
    for (int idx = lane; idx < 2 * n_zero; idx += 32) {
      const int at = idx / n_zero, u = idx % n_zero;
      st_shared_v4(sbase + at * kAtomBytes + (n_valid + u / 8) * 128 + (u % 8) * 16, 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  if (kMode == kModeIndexed) fence_proxy_async_smem();  // rows written by 16-byte async copies
  __syncwarp();
}

// Two warps feed the tensor pipe with independent streams, each with plain blocking waits:
// warp 1 issues the score GEMM of every tile, ring slot by ring slot as slots land, and
// warp 10 issues the value GEMM of every tile as soon as its probabilities are ready (which
// releases its ring slots).  MMAs of different threads are unordered, and the two streams
// touch disjoint TMEM columns, so the pipe simply interleaves them.  Loop state and MMA
// operands are warp-uniform; one elected lane issues.
template <int kMode>
__device__ void score_mma_role(const AttendParams &p, const Shared &sh, uint32_t tmem, int iq, long long t0,
                               long long t1, int lane) {
  uint64_t *bar = sh.bar;
  constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kRows, false, false);
  const uint32_t c_base = smem_u32(sh.slot(0));
  const uint32_t qt_base = smem_u32(sh.qt(0));
  uint32_t ns = 0, q_use = 0;
  SegIter it(t0, t1, iq);
  Seg sg;
  while (it.next(p, kMode, sg)) {
    if (sg.empty) continue;
    if (!wait_warp(&bar[kBarQFull], q_use & 1, sh, p.status)) return;
    ++q_use;
    for (int t = sg.lo; t < sg.hi; ++t, ++ns) {
      const int n_valid = min(kTile, sg.rows - t * kTile);
      if (!wait_warp(&bar[kBarSEmpty + (ns & 1)], ((ns >> 1) & 1) ^ 1, sh, p.status)) return;
      const uint32_t d = tmem + kTmemS + (ns & 1) * kRows;
#pragma unroll
      for (uint32_t sq = 0; sq < kSlotQuarters; ++sq) {
        // S^T[tile rows, heads] = C_tile * Q~^T; this slot holds K = 128 latent (8 steps)
        const uint32_t k = ns * kSlotQuarters + sq;
        if (!wait_warp(&bar[kBarCFull + ring_pos(k)], ring_use(k) & 1, sh, p.status)) return;
        const uint32_t sbase = c_base + ring_pos(k) * kSlotBytes;
        prepare_slot<kMode>(sbase, n_valid, lane);
        tc_fence_after();
        const uint64_t a0 = sw128_desc(sbase, 16, 1024);
        const uint64_t b0 = sw128_desc(qt_base + 2 * sq * kQtChunkBytes, 16, 1024);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // K step of 16 latent: 32 bytes inside a 128-byte swizzle row; the second four
            // steps are in the slot's second atom (A) and the next q~ chunk (B)
            const uint32_t ao = ((kk >> 2) * kAtomBytes + (kk & 3) * 32) >> 4;
            const uint32_t bo = ((kk >> 2) * kQtChunkBytes + (kk & 3) * 32) >> 4;
            umma_bf16(d, a0 + ao, b0 + bo, idesc_s, (sq != 0 || kk != 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      }
      if (elect_one()) {
        umma_commit(&bar[kBarSFull + (ns & 1)]);
        if (t == sg.hi - 1) umma_commit(&bar[kBarQEmpty]);
      }
      __syncwarp();
    }
  }
}

template <int kMode>
__device__ void value_mma_role(const AttendParams &p, const Shared &sh, uint32_t tmem, int iq, long long t0,
                               long long t1) {
  uint64_t *bar = sh.bar;
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, kRows, true, true);
  const uint32_t c_base = smem_u32(sh.slot(0));
  const uint32_t p_base = smem_u32(sh.pbuf(0));
  uint32_t no = 0, o_use = 0;
  SegIter it(t0, t1, iq);
  Seg sg;
  while (it.next(p, kMode, sg)) {
    if (sg.empty) continue;
    if (!wait_warp(&bar[kBarOEmpty], (o_use & 1) ^ 1, sh, p.status)) return;
    for (int t = sg.lo; t < sg.hi; ++t, ++no) {
      if (!wait_warp(&bar[kBarPFull + (no & 1)], (no >> 1) & 1, sh, p.status)) return;
      tc_fence_after();
      // O^T[latent, heads] += C_tile^T * P^T, four 128-lane latent blocks, K = 64 rows.
      // A = C_tile^T: latent (M) along the 128-byte rows, 64-wide atoms LBO apart; cache
      // rows (K) in 8-row groups.  B = P^T: heads (N) along the 128-byte rows, rows (K) in
      // 8-row groups.  A K step of 16 rows advances both by 2 KB (128 in descriptor units).
      const uint64_t b0 = sw128_desc(p_base + (no & 1) * kPBytes, kPBytes, 1024);
      uint64_t a0[kSlotQuarters];
      uint32_t rp[kSlotQuarters];
#pragma unroll
      for (int mb = 0; mb < kSlotQuarters; ++mb) {
        rp[mb] = ring_pos(no * kSlotQuarters + mb);
        a0[mb] = sw128_desc(c_base + rp[mb] * kSlotBytes, kAtomBytes, 1024);
      }
      const uint32_t acc0 = (t > sg.lo) ? 1u : 0u;
      if (elect_one()) {
#pragma unroll
        for (int mb = 0; mb < kSlotQuarters; ++mb) {
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_bf16(tmem + kTmemO + mb * kRows, a0[mb] + kk * 128, b0 + kk * 128, idesc_o, kk > 0 ? 1u : acc0);
          umma_commit(&bar[kBarCEmpty + rp[mb]]);
        }
        umma_commit(&bar[kBarPEmpty + (no & 1)]);
        if (t == sg.hi - 1) umma_commit(&bar[kBarOFull]);
      }
      __syncwarp();
    }
    ++o_use;
  }
}

// ------------------------------------------------------------------ softmax + epilogue (warps 2-9)
// Two warpgroups; warpgroup wg owns head columns [32 wg, 32 wg + 32) of S^T and O^T.  Warp
// quadrant wq holds tile rows 16 wq .. 16 wq + 15 (the M = 64 accumulator layout); thread t
// owns rows 16 wq + t/4 and 16 wq + t/4 + 8 and the 8 head columns 8j + 2(t%4) + {0,1}.
// The running max per column lives in shared memory and in registers.
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
  const int r0 = wq * 16 + (lane >> 2);        // tile rows r0 and r0 + 8 owned by this thread
  const int cq = lane & 3;                     // column pair within each 8-column block
  const uint32_t bar_id = 1 + wg;
  const int col0 = wg * 32;
  const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
  const uint32_t p_off = (uint32_t)r0 * 128 + cq * 4;
  float *red = sh.red;          // [4 quadrants][64 columns]
  float *m_used = sh.m_used;    // [64]
  float *alpha = sh.alpha;      // [64]
  uint32_t n = 0, o_use = 0;    // tiles seen by this CTA, segments finished
  if (tid < 32) m_used[col0 + tid] = -INFINITY;
  named_bar_sync(bar_id, 128);
  SegIter it(t0, t1, iq);
  Seg sg;
  while (it.next(p, kMode, sg)) {
    if (sg.empty) {
      // no visible tile: an empty partial (weight zero in the merge)
      if (tid < 32) {
        const long long slot = split::partial_slot(p, kMode, g, sg.s, iq);
        p.part_m[slot * kRows + col0 + tid] = -INFINITY;
        p.part_l[slot * kRows + col0 + tid] = 0.f;
      }
      continue;
    }
    const int qi = (kMode == kModeIndexed) ? sg.s % p.Q : iq;
    // positions of this CTA's query that are visible: dense/paged rows 0..L_b-Q+qi, or the list
    const int n_vis = (kMode == kModeIndexed) ? p.K : sg.rows - p.Q + qi + 1;
    float l_part[8], m_reg[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      l_part[c] = 0.f;
      m_reg[c] = -INFINITY;
    }
    // indexed: the list entries of this thread's two rows of the next tile are read ahead
    // (a -1 entry is unused and its row is masked)
    const int32_t *list = (kMode == kModeIndexed)
                              ? p.indices + ((long long)(sg.s / p.Q) * p.Q + (sg.s % p.Q)) * p.K
                              : nullptr;
    int ent_next[2] = {0, 0};
    if constexpr (kMode == kModeIndexed) {
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int k = sg.lo * kTile + r0 + 8 * h2;
        if (k < p.K) ent_next[h2] = list[k];
      }
    }
    for (int t = sg.lo; t < sg.hi; ++t, ++n) {
      const uint32_t sb = n & 1;
      int ent[2] = {ent_next[0], ent_next[1]};
      if constexpr (kMode == kModeIndexed) {
        if (t + 1 < sg.hi) {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int k = (t + 1) * kTile + r0 + 8 * h2;
            if (k < p.K) ent_next[h2] = list[k];
          }
        }
      }
      mbar_wait(&bar[kBarSFull + sb], (n >> 1) & 1, sh.abort_flag, p.status);
      tc_fence_after();
      bool v0 = (t * kTile + r0) < n_vis, v1 = (t * kTile + r0 + 8) < n_vis;
      if constexpr (kMode == kModeIndexed) {
        v0 = v0 && ent[0] != kUnusedEntry;
        v1 = v1 && ent[1] != kUnusedEntry;
      }
      float s2[16];
      {
        uint32_t r[16];
        tmem_ld16x256_x4(t_lane + kTmemS + sb * kRows + col0, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          s2[4 * j + 0] = v0 ? __uint_as_float(r[4 * j + 0]) * p.scale_log2 : -INFINITY;
          s2[4 * j + 1] = v0 ? __uint_as_float(r[4 * j + 1]) * p.scale_log2 : -INFINITY;
          s2[4 * j + 2] = v1 ? __uint_as_float(r[4 * j + 2]) * p.scale_log2 : -INFINITY;
          s2[4 * j + 3] = v1 ? __uint_as_float(r[4 * j + 3]) * p.scale_log2 : -INFINITY;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kBarSEmpty + sb]);
      // column h = 2j + e of this thread (j: 8-column block, e: pair member)
      bool flag = false;
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          flag |= fmaxf(s2[4 * j + e], s2[4 * j + 2 + e]) > m_reg[2 * j + e] + kTau;
      const bool any = named_bar_or(bar_id, 128, flag);
      if (*sh.abort_flag) return;
      if (any) {
        // new running max for this warpgroup's 32 columns
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float mx = fmaxf(s2[4 * j + e], s2[4 * j + 2 + e]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            if (lane < 4) red[wq * kRows + col0 + 8 * j + 2 * cq + e] = mx;
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
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = col0 + 8 * j + 2 * cq + e;
            l_part[2 * j + e] *= alpha[c];
            m_reg[2 * j + e] = m_used[c];
          }
      }
      // probabilities, rounded to bf16 for the value product; l sums the rounded values.
      // They are computed into registers first: the wait for this P buffer (the value
      // product of tile n-2) then overlaps the exponentials instead of preceding them.
      uint32_t pw[8];
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // h = 0: row r0, h = 1: row r0 + 8
          const float x0 = s2[4 * j + 2 * h], x1 = s2[4 * j + 2 * h + 1];
          const float p0 = (x0 == -INFINITY) ? 0.f : fast_exp2(x0 - m_reg[2 * j]);
          const float p1 = (x1 == -INFINITY) ? 0.f : fast_exp2(x1 - m_reg[2 * j + 1]);
          const uint32_t w = pack_bf16x2(p0, p1);
          l_part[2 * j] += bf16lo_to_f32(w);
          l_part[2 * j + 1] += bf16hi_to_f32(w);
          pw[2 * j + h] = w;
        }
      // this P buffer is free (the value product of tile n-2 has finished)
      mbar_wait(&bar[kBarPEmpty + sb], ((n >> 1) & 1) ^ 1, sh.abort_flag, p.status);
      if (any && t > sg.lo) {
        // running max moved: once the value product of tile n-1 has finished, rescale this
        // warpgroup's O^T columns in TMEM
        mbar_wait(&bar[kBarPEmpty + (sb ^ 1)], ((n - 1) >> 1) & 1, sh.abort_flag, p.status);
        tc_fence_after();
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
      const uint32_t pb = smem_u32(sh.pbuf(sb)) + p_off;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t sw = (uint32_t)(((wg * 4 + j) ^ (r0 & 7)) << 4);
#pragma unroll
        for (int h = 0; h < 2; ++h) st_shared_b32(pb + h * 8 * 128 + sw, pw[2 * j + h]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[kBarPFull + sb]);
    }
    // ---- epilogue: l column sums, partial O, (m, l) -> workspace
    mbar_wait(&bar[kBarOFull], o_use & 1, sh.abort_flag, p.status);
    tc_fence_after();
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = l_part[2 * j + e];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        if (lane < 4) red[wq * kRows + col0 + 8 * j + 2 * cq + e] = v;
      }
    named_bar_sync(bar_id, 128);
    if (*sh.abort_flag) return;
    const long long slot = split::partial_slot(p, kMode, g, sg.s, iq);
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

// ------------------------------------------------------------------ cluster merge (indexed)
// The C CTAs of a cluster split one index list into C segments and write their partials to
// the workspace as usual.  After one cluster barrier (release / acquire at cluster scope:
// the partials are visible to the whole cluster) CTA `rank` merges heads
// [rank * 64 / C, (rank + 1) * 64 / C) of the list from the C partials, which are still in
// L2, and writes o_latent and lse: no combine kernel, and no wait on CTAs outside the
// cluster (its CTAs are co-scheduled).  The merge is the combine kernel's, step for step --
// partials in group order, in chunks of kMergeChunk, each chunk raising the running max M
// and rescaling by 2^(M_old - M), then O / l and lse = (M + log2 l) ln 2 -- so the two
// paths round identically.  Run by the eight softmax warps; every thread of the CTA takes
// part in the cluster barrier (all reach it: every wait before it is bounded).
constexpr int kMaxCluster = 8;
constexpr int kMergeChunk = 3;
constexpr int kMergeChunks = (kMaxCluster + kMergeChunk - 1) / kMergeChunk;
constexpr int kCoef = 16;  // per head: kMergeChunks rescale factors, kMaxCluster weights, 1 / l
static_assert(kMergeChunks + kMaxCluster + 1 <= kCoef, "merge coefficients");

// Phase 1, one thread per head of this rank: the merge coefficients (all C partials' m and l
// are loaded first, then folded chunk by chunk as the combine does).  Loads bypass L1: the
// partials were written by other SMs during this kernel.
template <int CC>
__device__ __forceinline__ void merge_coefficients(const AttendParams &p, float *coef, int v, int h, int t) {
  float mk[kMergeChunks * kMergeChunk], lk[kMergeChunks * kMergeChunk];
#pragma unroll
  for (int k = 0; k < kMergeChunks * kMergeChunk; ++k) {
    mk[k] = -INFINITY;
    lk[k] = 0.f;
  }
#pragma unroll
  for (int k = 0; k < CC; ++k) {
    const long long row = split::partial_slot(p, kModeIndexed, (long long)v * CC + k, v, 0) * kRows + h;
    mk[k] = __ldcg(p.part_m + row);
    lk[k] = __ldcg(p.part_l + row);
  }
  float *cf = coef + t * kCoef;
  float M = -INFINITY, den = 0.f;
#pragma unroll
  for (int c = 0; c < kMergeChunks; ++c) {
    if (c * kMergeChunk >= CC) break;
    float mx = M;
#pragma unroll
    for (int j = 0; j < kMergeChunk; ++j) mx = fmaxf(mx, mk[c * kMergeChunk + j]);
    if (mx == -INFINITY) {
      cf[c] = -1.f;
      continue;
    }
    const float a = exp2f(M - mx);  // 0 when M was -inf
    cf[c] = a;
    den *= a;
#pragma unroll
    for (int j = 0; j < kMergeChunk; ++j) {
      const int k = c * kMergeChunk + j;
      const float w = exp2f(mk[k] - mx);  // 0 for empty partials (m = -inf)
      if (k < kMaxCluster) cf[kMergeChunks + k] = w;
      if (w == 0.f) continue;
      den += w * lk[k];
    }
    M = mx;
  }
  const bool good = (M != -INFINITY) && den > 0.f;
  cf[kMergeChunks + kMaxCluster] = good ? 1.f / den : 0.f;
  if (p.lse != nullptr)
    p.lse[(long long)v * kRows + h] = good ? (M + log2f(den)) * 0.69314718055994530942f : -INFINITY;
}

// Phase 2, 256 threads over this rank's (head, 4 latents) elements: the loads of U elements
// (U * CC float4, 16 or fewer) are issued together before any is used, then each element is
// folded with the coefficients exactly as the combine folds its partials.
template <int CC>
__device__ __forceinline__ void merge_rows(const AttendParams &p, const float *coef, int v, int h0, int nh, int t) {
  constexpr int U = (16 / CC) > 8 ? 8 : (16 / CC);
  constexpr int kStride = 32 * kSoftmaxWarps;
  const float *part[CC];
#pragma unroll
  for (int k = 0; k < CC; ++k)
    part[k] = p.part_o + split::partial_slot(p, kModeIndexed, (long long)v * CC + k, v, 0) * kRows * kLatent;
  const int total = nh * (kLatent / 4);  // a multiple of 128: every warp's elements are all in or all out
  for (int e0 = t; e0 < total; e0 += U * kStride) {
    float4 o[U][CC];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int e = e0 + u * kStride;
      if (e < total) {
        const int off = (h0 + e / (kLatent / 4)) * kLatent + (e % (kLatent / 4)) * 4;
#pragma unroll
        for (int k = 0; k < CC; ++k) o[u][k] = __ldcg(reinterpret_cast<const float4 *>(part[k] + off));
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int e = e0 + u * kStride;
      if (e >= total) continue;
      const int hl = e / (kLatent / 4), lat = (e % (kLatent / 4)) * 4;
      const float *cf = coef + hl * kCoef;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int c = 0; c < kMergeChunks; ++c) {
        if (c * kMergeChunk >= CC) break;
        const float a = cf[c];
        if (a < 0.f) continue;  // every partial of the chunk is empty
        acc.x *= a;
        acc.y *= a;
        acc.z *= a;
        acc.w *= a;
#pragma unroll
        for (int j = 0; j < kMergeChunk; ++j) {
          const int k = c * kMergeChunk + j;
          if (k >= CC) break;
          const float w = cf[kMergeChunks + k];
          if (w == 0.f) continue;  // an empty partial's O is never used
          acc.x += w * o[u][k].x;
          acc.y += w * o[u][k].y;
          acc.z += w * o[u][k].z;
          acc.w += w * o[u][k].w;
        }
      }
      const float inv = cf[kMergeChunks + kMaxCluster];
      uint2 outv;
      outv.x = pack_bf16x2(acc.x * inv, acc.y * inv);
      outv.y = pack_bf16x2(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2 *>(p.o_latent + ((long long)v * kRows + h0 + hl) * kLatent + lat) = outv;
    }
  }
}

template <int CC>
__device__ void cluster_merge_n(const AttendParams &p, const Shared &sh, int t) {
  const int rank = (int)cluster_ctarank();
  const int v = blockIdx.x / CC;  // the list: b * Q + i
  const int h0 = rank * kHeads / CC, nh = (rank + 1) * kHeads / CC - h0;
  // per-head coefficients, staged over the q~ area (free by now): for chunk c the rescale
  // factor a_c (-1: the chunk is skipped, all its partials empty), the weights w_k, 1 / l
  float *coef = reinterpret_cast<float *>(sh.base + kOffQt);
  if (t < nh) merge_coefficients<CC>(p, coef, v, h0 + t, t);
  named_bar_sync(3, 32 * kSoftmaxWarps);
  merge_rows<CC>(p, coef, v, h0, nh, t);
}

__device__ void cluster_merge(const AttendParams &p, const Shared &sh, int warp, int lane) {
  cluster_sync_all();  // every partial of the cluster's list is in the workspace
  if (warp >= 2 && warp < 2 + kSoftmaxWarps && !*sh.abort_flag) {
    const int t = (warp - 2) * 32 + lane;  // 0..255
    switch (p.cluster) {
      case 1: cluster_merge_n<1>(p, sh, t); break;
      case 2: cluster_merge_n<2>(p, sh, t); break;
      case 3: cluster_merge_n<3>(p, sh, t); break;
      case 4: cluster_merge_n<4>(p, sh, t); break;
      case 5: cluster_merge_n<5>(p, sh, t); break;
      case 6: cluster_merge_n<6>(p, sh, t); break;
      case 7: cluster_merge_n<7>(p, sh, t); break;
      default: cluster_merge_n<8>(p, sh, t); break;
    }
  }
}

// ------------------------------------------------------------------ kernel
template <int kMode>
// Bounds for 384 threads: eleven warps put three on some SM sub-partitions, whose 16K
// registers then cap a thread at 168 (the 352-thread bound alone would allow 184).
__global__ void __launch_bounds__(384, 1)
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
    for (int c = 0; c < kSlots; ++c) {
      mbar_init(&sh.bar[kBarCFull + c], kMode == kModeIndexed ? 64 : 1);  // indexed: 2 warps of copies
      mbar_init(&sh.bar[kBarCEmpty + c], 1);
    }
    mbar_init(&sh.bar[kBarQFull], 1);
    mbar_init(&sh.bar[kBarQEmpty], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.bar[kBarSFull + i], 1);
      mbar_init(&sh.bar[kBarSEmpty + i], kSoftmaxWarps);
      mbar_init(&sh.bar[kBarPFull + i], kSoftmaxWarps);
      mbar_init(&sh.bar[kBarPEmpty + i], 1);
    }
    mbar_init(&sh.bar[kBarOFull], 1);
    mbar_init(&sh.bar[kBarOEmpty], kSoftmaxWarps);
    mbar_init(&sh.bar[kBarDrain], 2);
    *sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(sh.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  grid_dep_launch();
  if (kMode == kModeDense && p.group_size == 1 && threadIdx.x == 0) {
    // Decode (one query per sequence), while the previous kernel finishes: bring this
    // CTA's first two tiles into L2, at the place they would be if every sequence held
    // Lmax rows.  (A verify group's CTAs share their tiles; there the extra requests cost
    // more than the early start gains.)  It reads nothing: a wrong
    // guess (shorter sequences) costs a wasted prefetch, and every prefetched row lies in
    // the cache ([B, Lmax] rows).  Data written by an earlier kernel is not at risk: L2 is
    // where those writes land.
    const long long nt = (p.Lmax + kTile - 1) / kTile;
    const long long T_est = (long long)p.B * nt;
    const long long t0 = group_start(g, T_est, p.groups);
    if (t0 < T_est) {
      const long long s = t0 / nt, j = (t0 % nt) * kTile;
      const long long rows = min((long long)2 * kTile, (long long)p.Lmax - j);
      bulk_prefetch_l2(p.cache + (s * p.Lmax + j) * kLatent, (uint32_t)(rows * kLatent * 2));
    }
  }
  grid_dep_wait();  // inputs (q~, lengths, tables, cache) may come from the previous kernel
  // tile range of this CTA's group
  const long long T = warp_total_tiles(p, kMode, lane);
  const long long G = p.groups;
  if (blockIdx.x == 0 && warp == 0) warp_write_seq_prefix(p, kMode, lane);
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
    if (kMode == kModeIndexed || lane == 0) producer_role<kMode>(p, sh, &tm_cache, &tm_qt, iq, t0, t1, lane, 0);
  } else if (warp == 11) {
    if (kMode == kModeIndexed) producer_role<kMode>(p, sh, &tm_cache, &tm_qt, iq, t0, t1, lane, 1);
  } else if (warp == 1) {
    score_mma_role<kMode>(p, sh, tmem, iq, t0, t1, lane);
  } else if (warp == 10) {
    value_mma_role<kMode>(p, sh, tmem, iq, t0, t1);
  } else {
    softmax_role<kMode>(p, sh, tmem, g, iq, t0, t1, warp, lane);
  }

  __syncwarp();
  // After an abort, the MMAs issued by the two MMA warps (lane 0 of each) must finish
  // before TMEM is released: each commits to the drain barrier, warp 1 waits for both.
  // (The producer has already waited for its copies.)
  if (warp == 10 && *sh.abort_flag) {
    if (lane == 0) umma_commit(&sh.bar[kBarDrain]);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*sh.abort_flag) {
      if (lane == 0) {
        umma_commit(&sh.bar[kBarDrain]);
        if (!mbar_wait_drain(&sh.bar[kBarDrain], 0)) report_status(p.status, kStatusTimeout);
      }
      __syncwarp();
    }
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if constexpr (kMode == kModeIndexed) {
    if (p.cluster > 0) cluster_merge(p, sh, warp, lane);
  }
}

// ------------------------------------------------------------------ combine
// One block per (query row v = b * Q + i) and pair of heads; thread t owns latent 4t..4t+3
// of both heads.  The partials of the CTA groups that processed tiles of the row's
// sequence are merged online in chunks of three, all loads of a chunk in flight at once
// (chunks this small keep a thread at 64 registers, so eight blocks fit on an SM and the
// 1,024 blocks of a 32-row step run in one wave):
// with M the largest running max so far, O = sum 2^(m_g - M) O_g and l = sum 2^(m_g - M) l_g,
// then O / l and lse = M + log2 l.  The sequence's place in the tile list comes from the
// table the attend kernel wrote.
constexpr int kCombineHeads = 2;
constexpr int kCombineChunk = 3;
static_assert(kCombineChunk == kMergeChunk, "the cluster merge rounds like the combine");

__global__ void __launch_bounds__(128, 8) combine_kernel(const AttendParams p, int mode) {
  grid_dep_launch();
  grid_dep_wait();  // the partials come from the attend kernel just before
  const int v = blockIdx.x;  // b * Q + i
  const int b = v / p.Q, i = v % p.Q;
  const int s = (mode == kModeIndexed) ? v : b;
  const int tid = threadIdx.x;
  // The sequence's partials are block-uniform and cost 64-bit divisions: one thread finds
  // them (their workspace slots, up to kMaxPartials; beyond that the range is consecutive).
  constexpr int kMaxPartials = 256;
  __shared__ long long sh_slot[kMaxPartials];
  __shared__ split::GroupRange sh_gr;
  if (tid == 0) {
    const split::GroupRange gr = split::seq_group_range(p, mode, s);
    sh_gr = gr;
    if (blockIdx.y == 0 && i == 0 && mode != kModeIndexed && p.seq_lens != nullptr) {
      const int L = p.seq_lens[b];
      const int cap = (mode == kModePaged) ? p.max_pages * kPageTokens : p.Lmax;
      if (L < 0 || L > cap) report_status(p.status, kStatusIndex);
    }
  }
  __syncthreads();
  const split::GroupRange gr = sh_gr;
  const int nslot = gr.count;
  for (int k = tid; k < nslot && k < kMaxPartials; k += blockDim.x)
    sh_slot[k] = split::partial_slot(p, mode, gr.partial_group(k), s, i);
  __syncthreads();
  const int h0 = blockIdx.y * kCombineHeads;
  const int lat = tid * 4;
  float M[kCombineHeads], den[kCombineHeads];
  float4 acc[kCombineHeads];
#pragma unroll
  for (int hh = 0; hh < kCombineHeads; ++hh) {
    M[hh] = -INFINITY;
    den[hh] = 0.f;
    acc[hh] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int k0 = 0; k0 < nslot; k0 += kCombineChunk) {
    float mk[kCombineHeads][kCombineChunk], lk[kCombineHeads][kCombineChunk];
    float4 ok[kCombineHeads][kCombineChunk];
#pragma unroll
    for (int j = 0; j < kCombineChunk; ++j) {
      const int k = k0 + j;
      const bool live = k < nslot;
      const long long slot =
          !live ? 0 : (k < kMaxPartials ? sh_slot[k] : split::partial_slot(p, mode, gr.partial_group(k), s, i));
#pragma unroll
      for (int hh = 0; hh < kCombineHeads; ++hh) {
        const long long row = slot * kRows + h0 + hh;
        mk[hh][j] = live ? p.part_m[row] : -INFINITY;
        lk[hh][j] = live ? p.part_l[row] : 0.f;
        ok[hh][j] = live ? *reinterpret_cast<const float4 *>(p.part_o + row * kLatent + lat)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int hh = 0; hh < kCombineHeads; ++hh) {
      float mx = M[hh];
#pragma unroll
      for (int j = 0; j < kCombineChunk; ++j) mx = fmaxf(mx, mk[hh][j]);
      if (mx == -INFINITY) continue;
      const float a = exp2f(M[hh] - mx);  // 0 when M was -inf
      den[hh] *= a;
      acc[hh].x *= a;
      acc[hh].y *= a;
      acc[hh].z *= a;
      acc[hh].w *= a;
#pragma unroll
      for (int j = 0; j < kCombineChunk; ++j) {
        const float w = exp2f(mk[hh][j] - mx);  // 0 for empty slots (m = -inf)
        if (w == 0.f) continue;                  // an empty partial's O is never summed in
        den[hh] += w * lk[hh][j];
        acc[hh].x += w * ok[hh][j].x;
        acc[hh].y += w * ok[hh][j].y;
        acc[hh].z += w * ok[hh][j].z;
        acc[hh].w += w * ok[hh][j].w;
      }
      M[hh] = mx;
    }
  }
#pragma unroll
  for (int hh = 0; hh < kCombineHeads; ++hh) {
    const int h = h0 + hh;
    const bool good = (M[hh] != -INFINITY) && den[hh] > 0.f;
    const float inv = good ? 1.f / den[hh] : 0.f;
    uint2 outv;
    outv.x = pack_bf16x2(acc[hh].x * inv, acc[hh].y * inv);
    outv.y = pack_bf16x2(acc[hh].z * inv, acc[hh].w * inv);
    *reinterpret_cast<uint2 *>(p.o_latent + ((long long)v * kRows + h) * kLatent + lat) = outv;
    if (p.lse != nullptr && tid == 0)
      p.lse[(long long)v * kRows + h] = good ? (M[hh] + log2f(den[hh])) * 0.69314718055994530942f : -INFINITY;
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

// ------------------------------------------------------------------ bounded-wait check
// The bounded mbarrier wait of every pipeline role, on a barrier that nothing completes:
// it must give up after about `limit` SM cycles, record MLA_ERR_TIMEOUT and return.
__global__ void wait_timeout_kernel(long long limit, int32_t *status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0, &abort_flag, status, limit);
}

}  // namespace attend

cudaError_t launch_wait_timeout(long long limit_cycles, int32_t *status, cudaStream_t stream) {
  attend::wait_timeout_kernel<<<1, 32, 0, stream>>>(limit_cycles, status);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ host launchers
size_t attend_slots(int B, int Q, int sms) {
  const size_t g_dense = (size_t)std::max(1, sms / std::max(Q, 1));
  const size_t a = (g_dense + (size_t)B) * (size_t)Q;
  const size_t c = (size_t)sms + (size_t)B * (size_t)Q;
  return a > c ? a : c;
}

size_t attend_workspace_bytes_for(int B, int Q, int sms) {
  const size_t slots = attend_slots(B, Q, sms);
  // partial O, m and l per slot, then per sequence of the tile list (at most B*Q of them)
  // its first tile (int64) and tile count (int32)
  return slots * kHeads * kLatent * sizeof(float) + 2 * slots * kHeads * sizeof(float) +
         (size_t)B * (size_t)Q * (sizeof(long long) + sizeof(int32_t));
}

template <int kMode>
static cudaError_t launch_attend_mode(const CUtensorMap &tm_cache, const CUtensorMap &tm_qt, const AttendParams &p,
                                      cudaStream_t stream, bool with_combine) {
  static std::atomic<int> configured_device{-1};
  const cudaError_t e0 = set_smem_limit_once(attend::attend_kernel<kMode>, attend::kSmemBytes, configured_device);
  if (e0 != cudaSuccess) return e0;
  const int grid = p.groups * p.group_size;
  if (kMode == kModeIndexed && p.cluster > 0) {
    // one cluster per index list; the cluster merges its partials and writes o_latent / lse
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(attend::kThreads);
    cfg.dynamicSmemBytes = attend::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)p.cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, attend::attend_kernel<kMode>, tm_cache, tm_qt, p);
  }
  cudaError_t e = launch_chained(attend::attend_kernel<kMode>, dim3(grid), dim3(attend::kThreads), attend::kSmemBytes,
                                 stream, tm_cache, tm_qt, p);
  if (e != cudaSuccess || !with_combine) return e;
  dim3 cgrid(p.B * p.Q, kHeads / attend::kCombineHeads);
  return launch_chained(attend::combine_kernel, cgrid, dim3(128), 0, stream, p, (int)kMode);
}

int attend_indexed_cluster_capacity(int csize) {
  if (csize < 1 || csize > attend::kMaxCluster) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  // per (device, cluster size), computed once; the lock makes concurrent first calls safe
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto it = cache.find({dev, csize});
  if (it != cache.end()) return it->second;
  int n = 0;
  if (cudaFuncSetAttribute(attend::attend_kernel<kModeIndexed>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           attend::kSmemBytes) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize);
    cfg.blockDim = dim3(attend::kThreads);
    cfg.dynamicSmemBytes = attend::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, attend::attend_kernel<kModeIndexed>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();  // a failed query is not an error of the caller's: the combine path runs
  cache[{dev, csize}] = n;
  return n;
}

cudaError_t launch_attend(int mode, const CUtensorMap &tm_cache, const CUtensorMap &tm_qt, const AttendParams &p,
                          cudaStream_t stream, bool with_combine) {
  switch (mode) {
    case kModeDense:
      return launch_attend_mode<kModeDense>(tm_cache, tm_qt, p, stream, with_combine);
    case kModePaged:
      return launch_attend_mode<kModePaged>(tm_cache, tm_qt, p, stream, with_combine);
    default:
      return launch_attend_mode<kModeIndexed>(tm_cache, tm_qt, p, stream, with_combine);
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

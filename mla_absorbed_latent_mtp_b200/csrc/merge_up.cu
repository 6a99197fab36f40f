// merge_up.cu -- the split-L merge fused with the value up-projection ("Module 05 -- MLA",
// section 3: the attention output stays in latent space, o_h = sum_j a_j c_j, and is
// expanded once at the end, out_h = U_h^V o_h).
//
// The attend kernel leaves one unnormalised partial (O_g, m_g, l_g) per CTA-group segment
// of a sequence.  Merged with their log-sum-exp weights,
//   o[r] = sum_g 2^(m_g - M) O_g[r] / sum_g 2^(m_g - M) l_g,   M = max_g m_g,
// and projected, out[d] = sum_r W_UV[h][d][r] o[r].  Both are linear in o once the weights
// are known, so the latent dimension can be split: a cluster of 2 CTAs handles one head
// and one tile of up to 32 query rows, CTA k the latent chunk r in [256k, 256k + 256):
//   1. it streams W_UV[h][0..255][chunk] (128 KB) by TMA before waiting for the attend
//      kernel (programmatic dependent launch), so the weights arrive during its tail;
//   2. its eight warps merge the chunk of every query row's partials (fp32) straight into
//      the MMA's B operand (bf16, 128-byte-swizzled K-major rows in shared memory), and
//      optionally store the normalised latent output o and the log-sum-exp;
//   3. one thread issues D[d, rows] = W_UV[h][d][chunk] * o[rows][chunk]^T on tcgen05
//      (two M = 128 blocks of d, N = 32 query rows, K = 256) into TMEM;
//   4. the two partial products are summed over distributed shared memory: each CTA
//      stages its fp32 D, the cluster synchronises, and CTA k adds up d in [128k, 128k + 128)
//      from both and writes those outputs in bf16.
// Clusters of two (rather than four 128-wide chunks) keep the whole grid resident at once:
// clusters of four with two CTAs per SM were limited to 33 active clusters on B200, so the
// 64 clusters of a 32-row step ran in two waves.
// No partial is read twice and no merged o makes a round trip through global memory.
#include <math.h>

#include "internal.h"
#include "sm100.cuh"
#include "split.cuh"

namespace mla {
namespace mergeup {

constexpr int kChunks = 2;                  // cluster size: latent chunks
constexpr int kChunk = kLatent / kChunks;   // 256 latent values per CTA
constexpr int kBoxesPerBlock = kChunk / 64; // W boxes (64 r wide) per 128-row d block
constexpr int kVecs = kChunk / 128;         // float4 of a partial's chunk per lane
constexpr int kNTile = 32;                  // query rows per CTA (MMA N)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kWBoxBytes = 128 * 64 * 2;    // W box: 128 d x 64 r
constexpr int kWBytes = 2 * kBoxesPerBlock * kWBoxBytes;  // 2 d blocks x the chunk: 128 KB
constexpr int kBAtomBytes = kNTile * 128;   // o rows x 64 r
constexpr int kBBytes = kBoxesPerBlock * kBAtomBytes;  // 16 KB
constexpr int kStageBytes = kNTile * kHeadDim * 4;  // fp32 D staged as [row][d]: 32 KB
constexpr int kOffW = 0;
constexpr int kOffB = kOffW + kWBytes;
constexpr int kOffStage = kOffB + kBBytes;
constexpr int kOffRows = kOffStage + kStageBytes;        // RowInfo per query row of the tile
constexpr int kOffBar = kOffRows + kNTile * 64;
constexpr int kOffMisc = kOffBar + 2 * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-byte alignment
constexpr uint32_t kTmemCols = 2 * kNTile;
constexpr int kMaxBatch = 6;                // partials of each of two rows loaded together
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kNTile % (2 * kWarps) == 0, "rows are merged two at a time per warp");
static_assert(kTmemCols == 64, "TMEM allocation is a power of two >= 32");

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The split-L partials of one query row (tile-list sequence s, query i): found once per
// row by one thread.
struct RowInfo {
  split::GroupRange gr;
  int s, i;
  __device__ __forceinline__ long long slot(const AttendParams &p, int mode, int k) const {
    return split::partial_slot(p, mode, gr.partial_group(k), s, i);
  }
};
static_assert(sizeof(RowInfo) <= 64, "row table entry");

__global__ void __launch_bounds__(kThreads, 1)
    merge_up_kernel(const __grid_constant__ CUtensorMap tm_w, const AttendParams p, int mode, uint16_t *out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bar_w = reinterpret_cast<uint64_t *>(base + kOffBar);
  uint64_t *bar_done = bar_w + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(base + kOffMisc + 4);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int kc = (int)cluster_ctarank();  // == blockIdx.x: the latent chunk
  const int h = blockIdx.y;
  const int v0 = blockIdx.z * kNTile;
  const int n = p.B * p.Q;

  if (tid == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_launch();
  if (tid == 0) {
    // the weights never come from an earlier kernel: stream them before the dependency wait
    prefetch_tensormap(&tm_w);
    mbar_arrive_expect_tx(bar_w, kWBytes);
#pragma unroll
    for (int mb = 0; mb < 2; ++mb)
#pragma unroll
      for (int j = 0; j < kBoxesPerBlock; ++j)
        tma_load_3d(base + kOffW + (mb * kBoxesPerBlock + j) * kWBoxBytes, &tm_w, bar_w, kc * kChunk + j * 64,
                    mb * 128, h);
  }
  grid_dep_wait();  // the partials, the tile table and the lengths come from the attend kernel

  // ---- merge.  Every load of a round is issued before any is used, and the rounds are
  // few: (1) one thread per query row finds its range of partials; (2) each warp loads the
  // running maxima and sums of its four rows' partials (lane k: partial k) and forms the
  // merge weights; (3) it loads the 128-wide chunk of every partial of two rows at a time
  // (lane l: latent 4l .. 4l + 3), weighs and sums them.
  RowInfo *rows = reinterpret_cast<RowInfo *>(base + kOffRows);
  if (tid < kNTile) {
    RowInfo ri;
    ri.gr.count = 0;
    ri.s = ri.i = 0;
    const int v = v0 + tid;
    if (v < n) {
      ri.i = v % p.Q;
      ri.s = (mode == kModeIndexed) ? v : v / p.Q;
      ri.gr = split::seq_group_range(p, mode, ri.s);
    }
    rows[tid] = ri;
  }
  __syncthreads();
  const uint32_t b_base = smem_u32(base + kOffB);
  constexpr int kRowsPerWarp = kNTile / kWarps;  // 4
  const RowInfo *ri = rows + warp;  // row j of this warp: ri[kWarps * j]
  float M[kRowsPerWarp], mk[kRowsPerWarp], lk[kRowsPerWarp];
  long long sl[kRowsPerWarp];
  int maxslot = 0;
#pragma unroll
  for (int j = 0; j < kRowsPerWarp; ++j) maxslot = max(maxslot, ri[kWarps * j].gr.count);
  // (2) maxima; the first 32 partials' (m, l) stay in registers for the weights
#pragma unroll
  for (int j = 0; j < kRowsPerWarp; ++j) {
    M[j] = -INFINITY;
    mk[j] = -INFINITY;
    lk[j] = 0.f;
    sl[j] = 0;
  }
  for (int k0 = 0; k0 < maxslot; k0 += 32) {
#pragma unroll
    for (int j = 0; j < kRowsPerWarp; ++j) {
      const int k = k0 + lane;
      if (k < ri[kWarps * j].gr.count) {
        const long long slot = ri[kWarps * j].slot(p, mode, k);
        const float m = p.part_m[slot * kHeads + h];
        M[j] = fmaxf(M[j], m);
        if (k0 == 0) {
          mk[j] = m;
          lk[j] = p.part_l[slot * kHeads + h];
          sl[j] = slot;
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kRowsPerWarp; ++j) M[j] = warp_max(M[j]);
  // (3) weighted sums, two rows at a time, partials in chunks of 32 (weights lane-held);
  // lane l holds latent 128 v + 4 l .. + 3 of the chunk, v < kVecs
#pragma unroll
  for (int jp = 0; jp < kRowsPerWarp; jp += 2) {
    float4 acc[2][kVecs];
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int u = 0; u < kVecs; ++u) acc[e][u] = make_float4(0.f, 0.f, 0.f, 0.f);
    float dsum[2] = {0.f, 0.f};
    const int pair_max = max(ri[kWarps * jp].gr.count, ri[kWarps * (jp + 1)].gr.count);
    for (int k0 = 0; k0 < pair_max; k0 += 32) {
      float w[2];
      long long slot[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = jp + e;
        float m = mk[j], l = lk[j];
        slot[e] = sl[j];
        if (k0 > 0) {  // beyond the first 32 partials: load this chunk's terms
          const int k = k0 + lane;
          m = -INFINITY;
          l = 0.f;
          if (k < ri[kWarps * j].gr.count) {
            slot[e] = ri[kWarps * j].slot(p, mode, k);
            m = p.part_m[slot[e] * kHeads + h];
            l = p.part_l[slot[e] * kHeads + h];
          }
        }
        w[e] = (M[j] == -INFINITY || m == -INFINITY) ? 0.f : exp2f(m - M[j]);
        dsum[e] += w[e] * l;
      }
      const int cnt = min(32, pair_max - k0);
      for (int q0 = 0; q0 < cnt; q0 += kMaxBatch) {
        float4 x[2][kMaxBatch][kVecs];
        float wq[2][kMaxBatch];
#pragma unroll
        for (int q = 0; q < kMaxBatch; ++q)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int src = (q0 + q) & 31;
            wq[e][q] = (q0 + q < cnt) ? __shfl_sync(0xffffffffu, w[e], src) : 0.f;
            const long long so = __shfl_sync(0xffffffffu, slot[e], src);
            const float4 *row = reinterpret_cast<const float4 *>(p.part_o + (so * kHeads + h) * kLatent + kc * kChunk +
                                                                 4 * lane);
#pragma unroll
            for (int u = 0; u < kVecs; ++u)
              x[e][q][u] = (wq[e][q] != 0.f) ? row[32 * u] : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
        for (int q = 0; q < kMaxBatch; ++q)
#pragma unroll
          for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int u = 0; u < kVecs; ++u) {
              acc[e][u].x += wq[e][q] * x[e][q][u].x;
              acc[e][u].y += wq[e][q] * x[e][q][u].y;
              acc[e][u].z += wq[e][q] * x[e][q][u].z;
              acc[e][u].w += wq[e][q] * x[e][q][u].w;
            }
      }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = jp + e;
      const int t = warp + kWarps * j;
      const int v = v0 + t;
      const float den = warp_sum(dsum[e]);
      const bool good = v < n && M[j] != -INFINITY && den > 0.f;
      const float inv = good ? 1.f / den : 0.f;
      if (v < n && p.lse != nullptr && kc == 0 && lane == 0)
        p.lse[(long long)v * kHeads + h] = good ? (M[j] + log2f(den)) * 0.69314718055994530942f : -INFINITY;
#pragma unroll
      for (int u = 0; u < kVecs; ++u) {
        const uint32_t lo = pack_bf16x2(acc[e][u].x * inv, acc[e][u].y * inv);
        const uint32_t hi = pack_bf16x2(acc[e][u].z * inv, acc[e][u].w * inv);
        if (v < n && p.o_latent != nullptr)
          *reinterpret_cast<uint2 *>(p.o_latent + ((long long)v * kHeads + h) * kLatent + kc * kChunk + 128 * u +
                                     4 * lane) = make_uint2(lo, hi);
        // B operand: row t, latent 128 u + 4 lane .. + 3 of the chunk, 128-byte swizzle
        const int atom = 2 * u + (lane >> 4), unit = (lane & 15) >> 1;
        st_shared_v2(b_base + atom * kBAtomBytes + t * 128 + ((unit ^ (t & 7)) << 4) + (lane & 1) * 8, lo, hi);
      }
    }
  }
  fence_proxy_async_smem();  // make the B tile visible to the tensor core
  tc_fence_before();
  __syncthreads();

  // ---- D[d, rows] = W_UV[h][d][chunk] * o[rows][chunk]^T, two M = 128 blocks of d
  if (warp == 0) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar_w, 0, abort_flag, p.status));
    tc_fence_after();
    if (ok && elect_one()) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kNTile, false, false);
      const uint32_t w_base = smem_u32(base + kOffW);
#pragma unroll
      for (int mb = 0; mb < 2; ++mb)
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
          // K step of 16 latent: 32 bytes inside a 128-byte swizzle row; steps 4-7 in the
          // second 64-wide half (next W box, next B atom)
          const uint64_t a =
              sw128_desc(w_base + (mb * kBoxesPerBlock + (kk >> 2)) * kWBoxBytes + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sw128_desc(b_base + (kk >> 2) * kBAtomBytes + (kk & 3) * 32, 16, 1024);
          umma_bf16(tmem + mb * kNTile, a, b, idesc, kk > 0 ? 1u : 0u);
        }
      umma_commit(bar_done);
    }
    __syncwarp();
  }

  // ---- stage D (fp32) as [row][d]: warp w reads lane quadrant w % 4 of block w / 4
  {
    const bool ok = mbar_wait(bar_done, 0, abort_flag, p.status);
    __syncwarp();
    tc_fence_after();
    const int mb = warp >> 2, q = warp & 3;
    uint32_t r[32];
    tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + mb * kNTile, r);
    tmem_ld_wait();
    float *stage = reinterpret_cast<float *>(base + kOffStage);
    const int d = mb * 128 + q * 32 + lane;
#pragma unroll
    for (int t = 0; t < kNTile; ++t) stage[t * kHeadDim + d] = ok ? __uint_as_float(r[t]) : 0.f;
  }
  tc_fence_before();
  cluster_sync_all();

  // ---- sum the chunks' products for this CTA's share of d: kDPerCta values of each of the
  // kNTile rows, kDPerThread per thread
  {
    constexpr int kDPerCta = kHeadDim / kChunks;
    constexpr int kDPerThread = kDPerCta * kNTile / kThreads;
    static_assert(kDPerThread % 8 == 0 && kThreads % kNTile == 0, "reduction mapping");
    const int t = tid / (kThreads / kNTile);
    const int d0 = kc * kDPerCta + (tid % (kThreads / kNTile)) * kDPerThread;
    const uint32_t local = smem_u32(base + kOffStage) + (uint32_t)(t * kHeadDim + d0) * 4;
    float acc[kDPerThread];
#pragma unroll
    for (int x = 0; x < kDPerThread; ++x) acc[x] = 0.f;
#pragma unroll
    for (int rk = 0; rk < kChunks; ++rk) {
      const uint32_t a = map_shared_rank(local, (uint32_t)rk);
#pragma unroll
      for (int x = 0; x < kDPerThread; x += 4) {
        const float4 y = ld_cluster_v4(a + 4 * x);
        acc[x] += y.x;
        acc[x + 1] += y.y;
        acc[x + 2] += y.z;
        acc[x + 3] += y.w;
      }
    }
    const int v = v0 + t;
    if (v < n) {
#pragma unroll
      for (int x = 0; x < kDPerThread; x += 8) {
        uint4 pk;
        pk.x = pack_bf16x2(acc[x], acc[x + 1]);
        pk.y = pack_bf16x2(acc[x + 2], acc[x + 3]);
        pk.z = pack_bf16x2(acc[x + 4], acc[x + 5]);
        pk.w = pack_bf16x2(acc[x + 6], acc[x + 7]);
        *reinterpret_cast<uint4 *>(out + ((long long)v * kHeads + h) * kHeadDim + d0 + x) = pk;
      }
    }
  }
  cluster_sync_all();  // the other CTAs may still be reading this CTA's staged products
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mergeup

cudaError_t launch_merge_up(const CUtensorMap &tm_w, const AttendParams &p, int mode, uint16_t *out,
                            cudaStream_t stream) {
  static std::atomic<int> configured_device{-1};
  const cudaError_t e0 = set_smem_limit_once(mergeup::merge_up_kernel, mergeup::kSmemBytes, configured_device);
  if (e0 != cudaSuccess) return e0;
  const int n = p.B * p.Q;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(mergeup::kChunks, kHeads, (n + mergeup::kNTile - 1) / mergeup::kNTile);
  cfg.blockDim = dim3(mergeup::kThreads);
  cfg.dynamicSmemBytes = mergeup::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = mergeup::kChunks;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, mergeup::merge_up_kernel, tm_w, p, mode, out);
}

}  // namespace mla

// merge_up.cu -- the split-L merge fused with the value up-projection ("Module 05 -- MLA",
// section 3: the attention output stays in latent space, o_h = sum_j a_j c_j, and is
// expanded once at the end, out_h = U_h^V o_h).
//
// The attend kernel leaves one unnormalised partial (O_g, m_g, l_g) per CTA-group segment
// of a sequence.  Merged with their log-sum-exp weights,
//   o[r] = sum_g 2^(m_g - M) O_g[r] / sum_g 2^(m_g - M) l_g,   M = max_g m_g,
// and projected, out[d] = sum_r W_UV[h][d][r] o[r].  Both are linear in o once the weights
// are known, so the latent dimension can be split: a cluster of 4 CTAs handles one head
// and one tile of up to 32 query rows, CTA k the latent chunk r in [128k, 128k + 128):
//   1. it streams W_UV[h][0..255][chunk] (64 KB) by TMA before waiting for the attend
//      kernel (programmatic dependent launch), so the weights arrive during its tail;
//   2. its eight warps merge the chunk of every query row's partials (fp32) straight into
//      the MMA's B operand (bf16, 128-byte-swizzled K-major rows in shared memory), and
//      optionally store the normalised latent output o and the log-sum-exp;
//   3. one thread issues D[d, rows] = W_UV[h][d][chunk] * o[rows][chunk]^T on tcgen05
//      (two M = 128 blocks of d, N = 32 query rows, K = 128) into TMEM;
//   4. the four partial products are summed over distributed shared memory: each CTA
//      stages its fp32 D, the cluster synchronises, and CTA k adds up d in [64k, 64k + 64)
//      from all four and writes those outputs in bf16.
// No partial is read twice and no merged o makes a round trip through global memory.
#include <math.h>

#include "internal.h"
#include "sm100.cuh"
#include "split.cuh"

namespace mla {
namespace mergeup {

constexpr int kChunks = 4;                  // cluster size: latent chunks
constexpr int kChunk = kLatent / kChunks;   // 128 latent values per CTA
constexpr int kNTile = 32;                  // query rows per CTA (MMA N)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kWBoxBytes = 128 * 64 * 2;    // W box: 128 d x 64 r
constexpr int kWBytes = 4 * kWBoxBytes;     // 2 d blocks x 2 r halves: 64 KB
constexpr int kBAtomBytes = kNTile * 128;   // o rows x 64 r
constexpr int kBBytes = 2 * kBAtomBytes;    // 8 KB
constexpr int kStageBytes = kNTile * kHeadDim * 4;  // fp32 D staged as [row][d]: 32 KB
constexpr int kOffW = 0;
constexpr int kOffB = kOffW + kWBytes;
constexpr int kOffStage = kOffB + kBBytes;
constexpr int kOffBar = kOffStage + kStageBytes;
constexpr int kOffMisc = kOffBar + 2 * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-byte alignment
constexpr uint32_t kTmemCols = 2 * kNTile;
constexpr int kMaxBatch = 8;                // partials of one row loaded together
static_assert(kSmemBytes <= 113 * 1024, "two CTAs per SM");
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

// Merges the latent chunk [r0, r0 + 128) of query row v (b = v / Q, i = v % Q) for head h.
// Lane l returns o[r0 + 4l .. r0 + 4l + 3] (normalised; zero when the row saw nothing);
// M and den (log2-domain max and weighted sum) come back for the log-sum-exp.
__device__ __forceinline__ float4 merge_row(const AttendParams &p, int mode, int v, int h, int r0, int lane,
                                            float &M, float &den) {
  const int b = v / p.Q, i = v % p.Q;
  const int s = (mode == kModeIndexed) ? v : b;
  const split::GroupRange gr = split::seq_group_range(p, mode, s);
  const long long G = p.groups;
  M = -INFINITY;
  for (int k = lane; k < gr.nslot; k += 32) {
    const long long g = gr.g_first + k;
    if (split::group_live(g, gr.T, G)) M = fmaxf(M, p.part_m[split::partial_slot(p, mode, g, s, i) * kHeads + h]);
  }
  M = warp_max(M);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float dsum = 0.f;
  if (M != -INFINITY) {
    for (int k0 = 0; k0 < gr.nslot; k0 += 32) {
      // lane j holds the weight of partial k0 + j (0 for an empty group)
      float w = 0.f;
      long long my_slot = 0;
      {
        const int k = k0 + lane;
        const long long g = gr.g_first + k;
        if (k < gr.nslot && split::group_live(g, gr.T, G)) {
          my_slot = split::partial_slot(p, mode, g, s, i);
          w = exp2f(p.part_m[my_slot * kHeads + h] - M);
          dsum += w * p.part_l[my_slot * kHeads + h];
        }
      }
      const int cnt = min(32, gr.nslot - k0);
      for (int j0 = 0; j0 < cnt; j0 += kMaxBatch) {
        float4 x[kMaxBatch];
        float wj[kMaxBatch];
#pragma unroll
        for (int j = 0; j < kMaxBatch; ++j) {
          wj[j] = __shfl_sync(0xffffffffu, w, (j0 + j) & 31);
          const long long sl = __shfl_sync(0xffffffffu, my_slot, (j0 + j) & 31);
          x[j] = (j0 + j < cnt && wj[j] != 0.f)
                     ? *reinterpret_cast<const float4 *>(p.part_o + (sl * kHeads + h) * kLatent + r0 + 4 * lane)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < kMaxBatch; ++j) {
          const float a = (j0 + j < cnt) ? wj[j] : 0.f;
          acc.x += a * x[j].x;
          acc.y += a * x[j].y;
          acc.z += a * x[j].z;
          acc.w += a * x[j].w;
        }
      }
    }
  }
  den = warp_sum(dsum);
  const float inv = (M != -INFINITY && den > 0.f) ? 1.f / den : 0.f;
  return make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

__global__ void __launch_bounds__(kThreads, 2)
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
      for (int j = 0; j < 2; ++j)
        tma_load_3d(base + kOffW + (mb * 2 + j) * kWBoxBytes, &tm_w, bar_w, kc * kChunk + j * 64, mb * 128, h);
  }
  grid_dep_wait();  // the partials, the tile table and the lengths come from the attend kernel

  // ---- merge: warp w takes query rows w, w + 8, w + 16, w + 24 of the tile
  const uint32_t b_base = smem_u32(base + kOffB);
  for (int t = warp; t < kNTile; t += kWarps) {
    const int v = v0 + t;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (v < n) {
      float M, den;
      o = merge_row(p, mode, v, h, kc * kChunk, lane, M, den);
      const uint32_t lo = pack_bf16x2(o.x, o.y), hi = pack_bf16x2(o.z, o.w);
      if (p.o_latent != nullptr)
        *reinterpret_cast<uint2 *>(p.o_latent + ((long long)v * kHeads + h) * kLatent + kc * kChunk + 4 * lane) =
            make_uint2(lo, hi);
      if (p.lse != nullptr && kc == 0 && lane == 0)
        p.lse[(long long)v * kHeads + h] =
            (M != -INFINITY && den > 0.f) ? (M + log2f(den)) * 0.69314718055994530942f : -INFINITY;
    }
    // B operand: row t, latent 4*lane .. 4*lane+3 of the chunk, 128-byte swizzle
    const uint32_t lo = pack_bf16x2(o.x, o.y), hi = pack_bf16x2(o.z, o.w);
    const int atom = lane >> 4, unit = (lane & 15) >> 1;
    st_shared_v2(b_base + atom * kBAtomBytes + t * 128 + ((unit ^ (t & 7)) << 4) + (lane & 1) * 8, lo, hi);
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
          const uint64_t a = sw128_desc(w_base + (mb * 2 + (kk >> 2)) * kWBoxBytes + (kk & 3) * 32, 16, 1024);
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

  // ---- sum the four chunks' products for d in [64 kc, 64 kc + 64): thread -> (row, 8 d)
  {
    const int t = tid >> 3;
    const int d0 = kc * 64 + (tid & 7) * 8;
    const uint32_t local = smem_u32(base + kOffStage) + (uint32_t)(t * kHeadDim + d0) * 4;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int rk = 0; rk < kChunks; ++rk) {
      const uint32_t a = map_shared_rank(local, (uint32_t)rk);
      const float4 x0 = ld_cluster_v4(a), x1 = ld_cluster_v4(a + 16);
      acc[0] += x0.x; acc[1] += x0.y; acc[2] += x0.z; acc[3] += x0.w;
      acc[4] += x1.x; acc[5] += x1.y; acc[6] += x1.z; acc[7] += x1.w;
    }
    const int v = v0 + t;
    if (v < n) {
      uint4 pk;
      pk.x = pack_bf16x2(acc[0], acc[1]);
      pk.y = pack_bf16x2(acc[2], acc[3]);
      pk.z = pack_bf16x2(acc[4], acc[5]);
      pk.w = pack_bf16x2(acc[6], acc[7]);
      *reinterpret_cast<uint4 *>(out + ((long long)v * kHeads + h) * kHeadDim + d0) = pk;
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
  static int configured_device = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device != dev) {
    cudaError_t e = cudaFuncSetAttribute(mergeup::merge_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         mergeup::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
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

// kpool.cu -- k-pool index producer feeding the index-list attention.
//
// "GLM-5.3-Flash engine (c/glm53.c)" (colibri docs), section "Architecture notes", DSA with
// k-pooling: keys are grouped into pools of `pool` consecutive positions; a pool's key is a
// per-channel softmax mixture of its members rather than their average; only complete,
// causally visible pools are selectable; the incomplete tail is appended when asked for
// (a row topk + pool - 1 wide); ties go to the lower index, so selection is deterministic.
// The pages give no indexer projections: the key of a position is its cached latent and the
// indexer query is an input vector w[b, i] of the latent width.
//
// pool_kernel:   pooled[b, p, d] = sum_j softmax_j(c[b, p*pool + j, d]) * c[b, p*pool + j, d]
//                for every complete pool of sequence b (one pass over the cache, online
//                max/sum per channel; thread t owns channels 4t..4t+3).
// select_kernel: one block per (b, i): scores w . pooled[p] of the pools that end at or
//                before the query's position (one warp per pool), then topk / pool rounds
//                of a block-wide argmax (larger score, then lower pool), the chosen pools'
//                positions in ascending order, -1 padding, and the tail.
#include <math.h>

#include <algorithm>

#include "internal.h"
#include "mla.h"
#include "sm100.cuh"

namespace mla {
namespace kpool {

constexpr int kThreads = 128;        // pool kernel: 4 channels per thread
constexpr int kSelectThreads = 1024;  // select kernel: 32 warps
constexpr int kMaxChosen = 1024;     // topk / pool bound (shared-memory list)
constexpr int kChunkRows = 16;       // pool members per step of the pooling
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float bf16_to_f32(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

__global__ void __launch_bounds__(kThreads) pool_kernel(const uint16_t *cache, const int32_t *seq_lens, int Lmax,
                                                        int pool, int max_pools, float *pooled) {
  grid_dep_launch();
  grid_dep_wait();
  const int b = blockIdx.y;
  const int L = seq_lens ? min(max(seq_lens[b], 0), Lmax) : Lmax;
  const int n_pools = L / pool;
  const int ch = threadIdx.x * 4;
  for (int p = blockIdx.x; p < n_pools; p += gridDim.x) {
    const uint16_t *src = cache + ((long long)b * Lmax + (long long)p * pool) * kLatent + ch;
    float m[4], s[4], ws[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      m[c] = -INFINITY;
      s[c] = 0.f;
      ws[c] = 0.f;
    }
    // 16 members at a time: the chunk's max first, so each member costs one exponential
    // and the running sums are rescaled once per chunk
    for (int j0 = 0; j0 < pool; j0 += kChunkRows) {
      const int nr = min(kChunkRows, pool - j0);
      float x[kChunkRows][4];
#pragma unroll
      for (int r = 0; r < kChunkRows; ++r) {
        if (r < nr) {
          const uint2 raw = *reinterpret_cast<const uint2 *>(src + (long long)(j0 + r) * kLatent);
          x[r][0] = bf16_to_f32((uint16_t)(raw.x & 0xFFFFu));
          x[r][1] = bf16_to_f32((uint16_t)(raw.x >> 16));
          x[r][2] = bf16_to_f32((uint16_t)(raw.y & 0xFFFFu));
          x[r][3] = bf16_to_f32((uint16_t)(raw.y >> 16));
        } else {
          x[r][0] = x[r][1] = x[r][2] = x[r][3] = -INFINITY;
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float cm = m[c];
#pragma unroll
        for (int r = 0; r < kChunkRows; ++r) cm = fmaxf(cm, x[r][c]);
        const float cm2 = cm * kLog2e;
        const float a = exp2f(m[c] * kLog2e - cm2);  // 0 on the first chunk
        s[c] *= a;
        ws[c] *= a;
#pragma unroll
        for (int r = 0; r < kChunkRows; ++r) {
          if (r < nr) {
            const float e = exp2f(fmaf(x[r][c], kLog2e, -cm2));
            s[c] += e;
            ws[c] += e * x[r][c];
          }
        }
        m[c] = cm;
      }
    }
    float4 out = make_float4(ws[0] / s[0], ws[1] / s[1], ws[2] / s[2], ws[3] / s[3]);
    *reinterpret_cast<float4 *>(pooled + ((long long)b * max_pools + p) * kLatent + ch) = out;
  }
}

// Better candidate: higher score, then lower pool index.
__device__ __forceinline__ bool better(float s1, int p1, float s2, int p2) {
  return s1 > s2 || (s1 == s2 && p1 < p2);
}

__global__ void __launch_bounds__(kSelectThreads) select_kernel(const float *pooled, const uint16_t *w_query,
                                                                const int32_t *seq_lens, int Q, int Lmax, int pool,
                                                                int topk, int with_tail, int max_pools,
                                                                int32_t *indices, int W) {
  extern __shared__ float sh_score[];  // [max_pools]
  __shared__ float sh_best_s[kSelectThreads / 32];
  __shared__ int sh_best_p[kSelectThreads / 32];
  __shared__ int sh_chosen[kMaxChosen];
  grid_dep_launch();
  grid_dep_wait();
  const int v = blockIdx.x, b = v / Q, i = v % Q;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int L = seq_lens ? min(max(seq_lens[b], 0), Lmax) : Lmax;
  const int pos = L - Q + i;  // the query's position; it sees 0..pos
  const int n_sel = pos >= 0 ? min((pos + 1) / pool, max_pools) : 0;
  // scores of the selectable pools: one warp per pool, lane owns 16 channels
  {
    float w[16];
    const uint16_t *wq = w_query + (long long)v * kLatent + lane * 16;
#pragma unroll
    for (int c = 0; c < 16; ++c) w[c] = bf16_to_f32(wq[c]);
    constexpr int kWarps = kSelectThreads / 32;
    for (int p0 = warp; p0 < n_sel; p0 += 2 * kWarps) {  // two pools per pass, loads in flight together
      float acc[2] = {0.f, 0.f};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int p = p0 + u * kWarps;
        if (p < n_sel) {
          const float4 *row =
              reinterpret_cast<const float4 *>(pooled + ((long long)b * max_pools + p) * kLatent + lane * 16);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const float4 x = row[c4];
            acc[u] += x.x * w[4 * c4] + x.y * w[4 * c4 + 1] + x.z * w[4 * c4 + 2] + x.w * w[4 * c4 + 3];
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
        const int p = p0 + u * kWarps;
        if (lane == 0 && p < n_sel) sh_score[p] = acc[u];
      }
    }
  }
  __syncthreads();
  // topk / pool rounds of argmax; a taken pool's score becomes NaN (never better)
  const int k_sel = min(topk / pool, n_sel);
  for (int r = 0; r < k_sel; ++r) {
    float bs = -INFINITY;
    int bp = 0x7fffffff;
    for (int p = threadIdx.x; p < n_sel; p += kSelectThreads) {
      const float s = sh_score[p];
      if (!isnan(s) && (bp == 0x7fffffff || better(s, p, bs, bp))) {
        bs = s;
        bp = p;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int op = __shfl_xor_sync(0xffffffffu, bp, o);
      if (op != 0x7fffffff && (bp == 0x7fffffff || better(os, op, bs, bp))) {
        bs = os;
        bp = op;
      }
    }
    if (lane == 0) {
      sh_best_s[warp] = bs;
      sh_best_p[warp] = bp;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = sh_best_s[0];
      int p = sh_best_p[0];
      for (int x = 1; x < kSelectThreads / 32; ++x)
        if (sh_best_p[x] != 0x7fffffff && (p == 0x7fffffff || better(sh_best_s[x], sh_best_p[x], s, p))) {
          s = sh_best_s[x];
          p = sh_best_p[x];
        }
      sh_chosen[r] = p;
      sh_score[p] = NAN;
    }
    __syncthreads();
  }
  // ascending pool order (k_sel is small: one thread sorts)
  if (threadIdx.x == 0) {
    for (int x = 1; x < k_sel; ++x) {
      const int key = sh_chosen[x];
      int y = x - 1;
      while (y >= 0 && sh_chosen[y] > key) {
        sh_chosen[y + 1] = sh_chosen[y];
        --y;
      }
      sh_chosen[y + 1] = key;
    }
  }
  __syncthreads();
  int32_t *out = indices + (long long)v * W;
  for (int x = threadIdx.x; x < topk; x += kSelectThreads)
    out[x] = (x < k_sel * pool) ? sh_chosen[x / pool] * pool + (x % pool) : -1;
  if (with_tail) {
    const int start = n_sel * pool;  // first position of the incomplete pool
    for (int x = threadIdx.x; x < pool - 1; x += kSelectThreads)
      out[topk + x] = (start + x <= pos) ? start + x : -1;
  }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace kpool
}  // namespace mla

extern "C" {

mla_status mla_kpool_keys(const uint16_t *cache, const int32_t *seq_lens, int B, int R, int Lmax, int pool,
                          float *pooled, void *stream) {
  using namespace mla;
  if (cache == nullptr || pooled == nullptr || B < 1 || Lmax < 1 || pool < 1) return MLA_ERR_ARG;
  if (R != kLatent) return MLA_ERR_UNSUPPORTED;
  if (B > 65535) return MLA_ERR_UNSUPPORTED;  // one grid row per sequence
  if (!kpool::aligned16(cache) || !kpool::aligned16(pooled)) return MLA_ERR_UNSUPPORTED;
  const int max_pools = Lmax / pool;
  if (max_pools < 1) return MLA_OK;
  const int blocks_x = std::min(max_pools, std::max(1, device_sm_count() * 8 / B + 1));
  return record_cuda_error(launch_chained(kpool::pool_kernel, dim3(blocks_x, B), dim3(kpool::kThreads), 0,
                                          reinterpret_cast<cudaStream_t>(stream), cache, seq_lens, Lmax, pool,
                                          max_pools, pooled));
}

mla_status mla_kpool_select(const float *pooled, const uint16_t *w_query, const int32_t *seq_lens, int B, int Q, int R,
                            int Lmax, int pool, int topk, int with_tail, int32_t *indices, int W, void *stream) {
  using namespace mla;
  if (pooled == nullptr || w_query == nullptr || indices == nullptr || B < 1 || Q < 1 || Lmax < 1 || pool < 1)
    return MLA_ERR_ARG;
  if ((long long)B * Q >= (1LL << 31)) return MLA_ERR_ARG;  // one block per query row
  if (R != kLatent) return MLA_ERR_UNSUPPORTED;
  if (topk < pool || topk % pool != 0 || topk / pool > kpool::kMaxChosen) return MLA_ERR_ARG;
  if (W != topk + (with_tail ? pool - 1 : 0)) return MLA_ERR_ARG;
  if (!kpool::aligned16(pooled)) return MLA_ERR_UNSUPPORTED;
  const int max_pools = Lmax / pool;
  const size_t smem = (size_t)std::max(max_pools, 1) * sizeof(float);
  if (smem > 200 * 1024) return MLA_ERR_UNSUPPORTED;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kpool::select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return record_cuda_error(e);
  }
  return record_cuda_error(launch_chained(kpool::select_kernel, dim3(B * Q), dim3(kpool::kSelectThreads), smem,
                                          reinterpret_cast<cudaStream_t>(stream), pooled, w_query, seq_lens, Q, Lmax,
                                          pool, topk, with_tail, max_pools, indices, W));
}

}  // extern "C"

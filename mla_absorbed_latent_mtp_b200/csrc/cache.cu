// cache.cu -- latent-cache bookkeeping around a speculative verify step.
//
// "Module 08 -- Vision, MTP, and Hybrid Serving State" (jared-hpc.com, GLM-5.3-Flash
// Architecture Mastery, Lecture-08), section 3: the MLA latent cache is indexed by token
// position, so a verify step's q_len rows are appended after each sequence's current
// length and, once the target has accepted a prefix of them, the cache is truncated to
// that prefix.  The state after the rollback must be the state of a run that never
// generated the rejected rows: truncation therefore also zeroes the rows it discards, so
// a cache whose unused rows are zero is left identical, bit for bit, to one that never
// held them.
//
// One CTA per sequence (128 threads, 16 bytes per thread and step, a 1 KiB row in 64
// steps).  A CTA validates its sequence first and touches nothing if any position it
// would write falls outside the cache or on a page-table entry outside the pool.
#include "internal.h"
#include "mla.h"
#include "sm100.cuh"

namespace mla {
namespace cache {

constexpr int kThreads = 128;
constexpr int kRowUnits = kLatent * 2 / 16;  // 16-byte units per latent row

struct Layout {
  int mode;                   // kModeDense or kModePaged
  uint16_t *store;            // dense cache [B, Lmax, R] or pool [num_pages, 64, R]
  const int32_t *page_table;  // paged: [B, max_pages]
  int Lmax, max_pages, num_pages;
};

__device__ __forceinline__ int capacity(const Layout &lay) {
  return lay.mode == kModePaged ? lay.max_pages * kPageTokens : lay.Lmax;
}

// Row index (in latent rows) of position j of sequence b, or -1 if it has no valid slot.
__device__ __forceinline__ long long row_of(const Layout &lay, int b, int j) {
  if (j < 0 || j >= capacity(lay)) return -1;
  if (lay.mode == kModePaged) {
    const int page = lay.page_table[(long long)b * lay.max_pages + j / kPageTokens];
    if (page < 0 || page >= lay.num_pages) return -1;
    return (long long)page * kPageTokens + (j % kPageTokens);
  }
  return (long long)b * lay.Lmax + j;
}

// Positions [lo, hi) of sequence b all have slots (checked by one warp).
__device__ bool range_ok(const Layout &lay, int b, int lo, int hi, int lane) {
  bool ok = lo >= 0 && hi <= capacity(lay);
  if (ok && lay.mode == kModePaged)
    for (int j = lo + lane; j < hi; j += 32) ok = ok && row_of(lay, b, j) >= 0;
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kThreads) append_kernel(const Layout lay, int32_t *seq_lens,
                                                          const uint16_t *rows, int Q, int32_t *status) {
  grid_dep_launch();
  grid_dep_wait();  // the cache and the lengths may still be read or written by the previous kernel
  const int b = blockIdx.x;
  __shared__ int sh_ok;
  const int L = seq_lens[b];
  if (threadIdx.x < 32) {
    const bool ok = L >= 0 && range_ok(lay, b, L, L + Q, threadIdx.x);
    if (threadIdx.x == 0) {
      sh_ok = ok;
      if (!ok) report_status(status, kStatusIndex);
    }
  }
  __syncthreads();
  if (!sh_ok) return;
  const uint4 *src = reinterpret_cast<const uint4 *>(rows + (long long)b * Q * kLatent);
  uint4 *dst = reinterpret_cast<uint4 *>(lay.store);
  for (int x = threadIdx.x; x < Q * kRowUnits; x += kThreads) {
    const int i = x / kRowUnits, u = x % kRowUnits;
    dst[row_of(lay, b, L + i) * kRowUnits + u] = src[x];
  }
  __syncthreads();  // every thread has read L before it moves
  if (threadIdx.x == 0) seq_lens[b] = L + Q;
}

__global__ void __launch_bounds__(kThreads) truncate_kernel(const Layout lay, int32_t *seq_lens,
                                                            const int32_t *keep, int Q, int32_t *status) {
  grid_dep_launch();
  grid_dep_wait();
  const int b = blockIdx.x;
  __shared__ int sh_ok;
  const int L = seq_lens[b];
  const int k = keep[b];
  const int new_len = L - Q + k;
  if (threadIdx.x < 32) {
    const bool ok = k >= 0 && k <= Q && L - Q >= 0 && range_ok(lay, b, new_len, L, threadIdx.x);
    if (threadIdx.x == 0) {
      sh_ok = ok;
      if (!ok) report_status(status, kStatusIndex);
    }
  }
  __syncthreads();
  if (!sh_ok) return;
  uint4 *dst = reinterpret_cast<uint4 *>(lay.store);
  const int n = (L - new_len) * kRowUnits;
  for (int x = threadIdx.x; x < n; x += kThreads) {
    const int i = x / kRowUnits, u = x % kRowUnits;
    dst[row_of(lay, b, new_len + i) * kRowUnits + u] = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();
  if (threadIdx.x == 0) seq_lens[b] = new_len;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mla_status check(const Layout &lay, const int32_t *seq_lens, const void *in, int B, int Q, int R, int page_size) {
  if (lay.store == nullptr || seq_lens == nullptr || in == nullptr || B < 1 || Q < 1) return MLA_ERR_ARG;
  if (R != kLatent) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(lay.store) || !aligned16(in)) return MLA_ERR_UNSUPPORTED;
  if (lay.mode == kModePaged) {
    if (lay.page_table == nullptr || lay.max_pages < 1 || lay.num_pages < 1) return MLA_ERR_ARG;
    if (page_size != kPageTokens) return MLA_ERR_UNSUPPORTED;
    if ((long long)lay.max_pages * kPageTokens >= (1LL << 31)) return MLA_ERR_ARG;
  } else if (lay.Lmax < 1 || (long long)B * lay.Lmax >= (1LL << 40)) {
    return MLA_ERR_ARG;
  }
  return MLA_OK;
}

mla_status append(const Layout &lay, int32_t *seq_lens, const uint16_t *rows, int B, int Q, int R, int page_size,
                  int32_t *status, void *stream) {
  if (mla_status s = check(lay, seq_lens, rows, B, Q, R, page_size); s != MLA_OK) return s;
  return record_cuda_error(launch_chained(append_kernel, dim3(B), dim3(kThreads), 0,
                                          reinterpret_cast<cudaStream_t>(stream), lay, seq_lens, rows, Q, status));
}

mla_status truncate(const Layout &lay, int32_t *seq_lens, const int32_t *keep, int B, int Q, int R, int page_size,
                    int32_t *status, void *stream) {
  if (mla_status s = check(lay, seq_lens, keep, B, Q, R, page_size); s != MLA_OK) return s;
  return record_cuda_error(launch_chained(truncate_kernel, dim3(B), dim3(kThreads), 0,
                                          reinterpret_cast<cudaStream_t>(stream), lay, seq_lens, keep, Q, status));
}

}  // namespace cache
}  // namespace mla

extern "C" {

mla_status mla_cache_append_dense(uint16_t *cache, int32_t *seq_lens, const uint16_t *rows, int B, int Q, int R,
                                  int Lmax, int32_t *status, void *stream) {
  const mla::cache::Layout lay{mla::kModeDense, cache, nullptr, Lmax, 0, 0};
  return mla::cache::append(lay, seq_lens, rows, B, Q, R, 0, status, stream);
}

mla_status mla_cache_append_paged(uint16_t *pool, const int32_t *page_table, int32_t *seq_lens, const uint16_t *rows,
                                  int B, int Q, int R, int page_size, int max_pages, int num_pages, int32_t *status,
                                  void *stream) {
  const mla::cache::Layout lay{mla::kModePaged, pool, page_table, 0, max_pages, num_pages};
  return mla::cache::append(lay, seq_lens, rows, B, Q, R, page_size, status, stream);
}

mla_status mla_cache_truncate_dense(uint16_t *cache, int32_t *seq_lens, const int32_t *keep, int B, int Q, int R,
                                    int Lmax, int32_t *status, void *stream) {
  const mla::cache::Layout lay{mla::kModeDense, cache, nullptr, Lmax, 0, 0};
  return mla::cache::truncate(lay, seq_lens, keep, B, Q, R, 0, status, stream);
}

mla_status mla_cache_truncate_paged(uint16_t *pool, const int32_t *page_table, int32_t *seq_lens, const int32_t *keep,
                                    int B, int Q, int R, int page_size, int max_pages, int num_pages, int32_t *status,
                                    void *stream) {
  const mla::cache::Layout lay{mla::kModePaged, pool, page_table, 0, max_pages, num_pages};
  return mla::cache::truncate(lay, seq_lens, keep, B, Q, R, page_size, status, stream);
}

}  // extern "C"

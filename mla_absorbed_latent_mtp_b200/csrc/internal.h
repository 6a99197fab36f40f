// internal.h -- host-side declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <utility>

namespace mla {

// Address modes of the attend kernel.
enum AttendMode : int { kModeDense = 0, kModePaged = 1, kModeIndexed = 2 };

// Fixed problem geometry of this version (Module 05 section 1).
constexpr int kHeads = 64;
constexpr int kHeadDim = 256;
constexpr int kLatent = 512;
constexpr int kPageTokens = 64;

// Everything the attend and combine kernels need besides the two tensor maps.
struct AttendParams {
  const int32_t *seq_lens;    // [B] or null (dense/indexed: every sequence has Lmax rows)
  const int32_t *page_table;  // paged: [B, max_pages]
  const int32_t *indices;     // indexed: [B, Q, K]
  const uint16_t *cache;      // indexed: raw pointer of the [B, Lmax, R] cache
  int B, Q, Lmax, max_pages, num_pages, K;
  int groups;                 // G: CTA groups that split the tile list
  int group_size;             // CTAs per group: Q (dense/paged, one per query) or 1 (indexed)
  int cluster;                // indexed: CTAs per list, launched as one thread-block cluster that
                              // merges its partials in distributed shared memory and writes
                              // o_latent / lse itself (no combine); 0: partials to the workspace
  float scale_log2;           // softmax scale * log2(e)
  float *part_o;              // [slots, H, R] unnormalised partial outputs
  float *part_m;              // [slots, H] running max (log2 units)
  float *part_l;              // [slots, H] running sum
  long long *seq_ts;          // [num_seqs] tiles of the list before sequence s (written by CTA 0)
  int32_t *seq_nt;            // [num_seqs] tiles of sequence s
  uint16_t *o_latent;         // [B, Q, H, R] result
  float *lse;                 // [B, Q, H] or null
  int32_t *status;
};

// Partial-result slots needed for B sequences of Q queries with `sms` SMs.
size_t attend_slots(int B, int Q, int sms);
size_t attend_workspace_bytes_for(int B, int Q, int sms);

// The attend kernel, then (with_combine, and p.cluster == 0) the split-L combine that
// writes o_latent / lse.
cudaError_t launch_attend(int mode, const CUtensorMap &tm_cache, const CUtensorMap &tm_qt,
                          const AttendParams &p, cudaStream_t stream, bool with_combine = true);
// Clusters of `csize` indexed-mode attend CTAs (one CTA per SM) that can be resident at once
// on the current device (0 when the launch configuration is not possible).
int attend_indexed_cluster_capacity(int csize);
// The split-L merge fused with the W_UV up-projection: out [B*Q, H, D] from the attend
// kernel's partials (o_latent / lse in p written too when non-null).
cudaError_t launch_merge_up(const CUtensorMap &tm_w, const AttendParams &p, int mode, uint16_t *out,
                            cudaStream_t stream);
cudaError_t launch_debug_gather(int mode, const uint16_t *src, const int32_t *page_table,
                                const int32_t *indices, int B, int Q, int R, int Lmax, int max_pages,
                                int num_pages, int K, const int32_t *req, int n_req, uint16_t *out,
                                int32_t *status, cudaStream_t stream);

// Per-head projection GEMM: out[n, h, m] = sum_k A_h[m, k] * X[n, h, k].
// absorb (a_mn_major = true):  A_h[m=r, k=d] = W_UK[h][d][r]  (M = R, K = D)
// up-proj (a_mn_major = false): A_h[m=d, k=r] = W_UV[h][d][r] (M = D, K = R)
// x_bcast: X is [n, K] (one row per token for every head), read with head coordinate 0.
cudaError_t launch_proj(bool a_mn_major, const CUtensorMap &tm_w, const CUtensorMap &tm_x, int n, int H,
                        int M_total, int K_total, int n_tile, uint16_t *out, cudaStream_t stream,
                        bool x_bcast = false);

// Causal self-attention of B sequences of L tokens in the expanded form (64 heads of 256):
// q, out [B, L, H, D]; k, v through tensor maps over [B*L, H, D] (boxes of 64 dims x 64 tokens).
cudaError_t launch_prefill(const CUtensorMap &tm_k, const CUtensorMap &tm_v, const uint16_t *q, uint16_t *out,
                           float *lse, int B, int L, float scale, int32_t *status, cudaStream_t stream);

int device_sm_count();
cudaError_t launch_wait_timeout(long long limit_cycles, int32_t *status, cudaStream_t stream);

// Launch with programmatic stream serialization: the kernel may start while the previous
// kernel in the stream is still running, once that kernel's CTAs have all signalled
// (griddepcontrol.launch_dependents) or exited.  Every kernel of this library launched
// this way executes griddepcontrol.wait before it reads anything an earlier kernel could
// have written; before that it only initialises itself and reads weights.
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                           Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
// Raises a kernel's dynamic shared-memory limit to `bytes` on the current device, once per
// device switch (`configured` remembers the device it was last set on).  Safe from several
// host threads: the attribute call is idempotent, so concurrent first calls may both make it.
template <typename... KArgs>
cudaError_t set_smem_limit_once(void (*kernel)(KArgs...), int bytes, std::atomic<int> &configured) {
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return e;
  if (configured.load(std::memory_order_acquire) == dev) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) configured.store(dev, std::memory_order_release);
  return e;
}
// Records e as the calling thread's last CUDA error; returns MLA_ERR_CUDA (MLA_OK for success).
int32_t record_cuda_error(cudaError_t e);

}  // namespace mla

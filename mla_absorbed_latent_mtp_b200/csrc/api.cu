// api.cu -- the C ABI (include/mla.h): argument validation, TMA tensor-map encoding and
// kernel launches on the caller's stream.  No allocation, no synchronisation.
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>
#include <mutex>

#include "mla.h"
#include "internal.h"

namespace mla {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor map with 128-byte swizzle; dims/strides innermost first, strides in bytes
// for dims 1..rank-1; out-of-range boxes read as zero.
bool make_map(CUtensorMap *map, const void *ptr, int rank, const uint64_t *dims, const uint64_t *strides,
              const uint32_t *box) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t gdim[3], gstride[2];
  cuuint32_t bdim[3], estride[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) gstride[i] = strides[i];
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(ptr), gdim, gstride, bdim,
                  estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count_for(int dev) {
  static std::atomic<int> cache[64];  // 0: not read yet (concurrent first calls both read it)
  if (dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// W_UV[h][d][r] for the fused merge + up-projection: dims {R, D, H}, boxes of 64 r x 128 d.
bool make_w_uv_map(CUtensorMap *map, const uint16_t *w_uv) {
  const uint64_t dims[3] = {(uint64_t)kLatent, (uint64_t)kHeadDim, (uint64_t)kHeads};
  const uint64_t strides[2] = {(uint64_t)kLatent * 2, (uint64_t)kHeadDim * kLatent * 2};
  const uint32_t box[3] = {64, 128, 1};
  return make_map(map, w_uv, 3, dims, strides, box);
}

}  // namespace

static thread_local cudaError_t g_last_error = cudaSuccess;

static mla_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MLA_OK;
  g_last_error = e;
  return MLA_ERR_CUDA;
}

mla_status record_cuda_error(cudaError_t e) { return cuda_status(e); }

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  return sm_count_for(dev);
}

// Shared validation and launch for the three attend modes.  With w_uv / out given, the
// split-L merge runs fused with the up-projection (o_latent optional); without, the combine
// writes o_latent (required).
static mla_status attend_common(int mode, const uint16_t *q_tilde, const uint16_t *cache, const int32_t *page_table,
                                const int32_t *indices, const int32_t *seq_lens, int B, int Q, int H, int R, int Lmax,
                                int page_size, int max_pages, int num_pages, int K, float scale, void *workspace,
                                size_t ws_bytes, uint16_t *o_latent, float *lse, int32_t *status, void *stream,
                                const uint16_t *w_uv = nullptr, int D = 0, uint16_t *out = nullptr) {
  const bool fused = (w_uv != nullptr || out != nullptr);
  if (q_tilde == nullptr || cache == nullptr) return MLA_ERR_ARG;
  if (fused ? (w_uv == nullptr || out == nullptr) : (o_latent == nullptr)) return MLA_ERR_ARG;
  if (fused && D != kHeadDim) return MLA_ERR_UNSUPPORTED;
  if (fused && (!aligned16(w_uv) || !aligned16(out))) return MLA_ERR_UNSUPPORTED;
  if (o_latent != nullptr && !aligned16(o_latent)) return MLA_ERR_UNSUPPORTED;
  if (B < 1 || Q < 1 || !isfinite(scale)) return MLA_ERR_ARG;
  if (H != kHeads || R != kLatent) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(q_tilde) || !aligned16(cache)) return MLA_ERR_UNSUPPORTED;
  if ((long long)B * Q * H >= (1LL << 31)) return MLA_ERR_ARG;
  if (mode == kModePaged) {
    if (page_table == nullptr || seq_lens == nullptr) return MLA_ERR_ARG;
    if (page_size != kPageTokens) return MLA_ERR_UNSUPPORTED;
    if (max_pages < 1 || num_pages < 1) return MLA_ERR_ARG;
    if ((long long)num_pages * kPageTokens >= (1LL << 31)) return MLA_ERR_ARG;
    if ((long long)max_pages * kPageTokens >= (1LL << 31)) return MLA_ERR_ARG;  // positions are int32
  } else {
    if (Lmax < 1 || (long long)B * Lmax >= (1LL << 31)) return MLA_ERR_ARG;
  }
  if (mode == kModeIndexed && (indices == nullptr || K < 1)) return MLA_ERR_ARG;
  int dev = 0;
  if (cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) return cuda_status(e);
  const int sms = sm_count_for(dev);
  const size_t need = attend_workspace_bytes_for(B, Q, sms);
  if (workspace == nullptr || ws_bytes < need || !aligned16(workspace)) return MLA_ERR_WORKSPACE;

  CUtensorMap tm_cache, tm_qt;
  {
    // cache rows seen as {64 latent, rows, R/64 chunks of 64 latent} (strides 1,024 and 128
    // bytes): one box {64, 64, 2} is a ring slot, 64 rows x 128 latent, landing as two
    // 128-byte-swizzled 64 x 64 atoms -- one copy per slot instead of two
    const uint64_t rows = (mode == kModePaged) ? (uint64_t)num_pages * kPageTokens : (uint64_t)B * Lmax;
    const uint64_t dims[3] = {64, rows, (uint64_t)R / 64};
    const uint64_t strides[2] = {(uint64_t)R * 2, 128};
    const uint32_t box[3] = {64, 64, 2};
    if (!make_map(&tm_cache, cache, 3, dims, strides, box)) return cuda_status(cudaErrorInvalidValue);
  }
  {
    // q~ rows (one per head) the same way: one box {64, 64 heads, 8 chunks} is a query's
    // whole q~, eight 64 x 64 atoms
    const uint64_t dims[3] = {64, (uint64_t)B * Q * H, (uint64_t)R / 64};
    const uint64_t strides[2] = {(uint64_t)R * 2, 128};
    const uint32_t box[3] = {64, 64, (uint32_t)R / 64};
    if (!make_map(&tm_qt, q_tilde, 3, dims, strides, box)) return cuda_status(cudaErrorInvalidValue);
  }
  AttendParams p;
  p.seq_lens = seq_lens;
  p.page_table = page_table;
  p.indices = indices;
  p.cache = cache;
  p.B = B;
  p.Q = Q;
  p.Lmax = (mode == kModePaged) ? max_pages * kPageTokens : Lmax;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.K = K;
  if (mode == kModeIndexed) {
    // Every list has the same tile count, so a group count that is a multiple of the number
    // of lists splits each list into equal parts and no CTA straddles two lists (one
    // segment, one epilogue, one q~ load per CTA), at the price of some idle SMs.
    p.group_size = 1;
    const int lists = B * Q;
    const int nt = (K + 63) / 64;
    const int per_list = std::min(sms / lists, nt);
    p.groups = per_list >= 1 ? per_list * lists : sms;
    // When a list's CTAs fit one thread-block cluster and all the clusters can be resident
    // at once, they merge their partials in distributed shared memory (no partial stores,
    // no combine kernel).  The fused up-projection path keeps the workspace partials.
    p.cluster = 0;
    if (!fused && per_list >= 1 && per_list <= 8 && attend_indexed_cluster_capacity(per_list) >= lists)
      p.cluster = per_list;
  } else {
    p.group_size = Q;
    p.groups = std::max(1, sms / Q);
    p.cluster = 0;
  }
  p.scale_log2 = scale * 1.4426950408889634f;
  const size_t slots = attend_slots(B, Q, sms);
  p.part_o = reinterpret_cast<float *>(workspace);
  p.part_m = p.part_o + slots * kHeads * kLatent;
  p.part_l = p.part_m + slots * kHeads;
  p.seq_ts = reinterpret_cast<long long *>(p.part_l + slots * kHeads);
  p.seq_nt = reinterpret_cast<int32_t *>(p.seq_ts + (size_t)B * Q);
  p.o_latent = o_latent;
  p.lse = lse;
  p.status = status;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!fused) return cuda_status(launch_attend(mode, tm_cache, tm_qt, p, st));
  CUtensorMap tm_w;
  if (!make_w_uv_map(&tm_w, w_uv)) return cuda_status(cudaErrorInvalidValue);
  if (cudaError_t e = launch_attend(mode, tm_cache, tm_qt, p, st, false); e != cudaSuccess) return cuda_status(e);
  return cuda_status(launch_merge_up(tm_w, p, mode, out, st));
}

static mla_status proj_common(bool absorb, const uint16_t *x, const uint16_t *w, uint16_t *out, int n, int H, int D,
                              int R, void *stream) {
  if (x == nullptr || w == nullptr || out == nullptr) return MLA_ERR_ARG;
  if (n < 1) return MLA_ERR_ARG;
  if (H != kHeads || D != kHeadDim || R != kLatent) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(w) || !aligned16(out)) return MLA_ERR_UNSUPPORTED;
  if ((long long)n * H >= (1LL << 31)) return MLA_ERR_ARG;
  const int K_total = absorb ? D : R;
  const int M_total = absorb ? R : D;
  const int n_tile = std::min(128, (n + 31) / 32 * 32);
  CUtensorMap tm_w, tm_x;
  {
    // W[h][d][r]: dims {R, D, H}
    const uint64_t dims[3] = {(uint64_t)R, (uint64_t)D, (uint64_t)H};
    const uint64_t strides[2] = {(uint64_t)R * 2, (uint64_t)D * R * 2};
    const uint32_t box_mn[3] = {64, 64, 1};
    const uint32_t box_k[3] = {64, 128, 1};
    if (!make_map(&tm_w, w, 3, dims, strides, absorb ? box_mn : box_k)) return cuda_status(cudaErrorInvalidValue);
  }
  {
    // X[n][h][k]: dims {K, H, n}
    const uint64_t dims[3] = {(uint64_t)K_total, (uint64_t)H, (uint64_t)n};
    const uint64_t strides[2] = {(uint64_t)K_total * 2, (uint64_t)H * K_total * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)n_tile};
    if (!make_map(&tm_x, x, 3, dims, strides, box)) return cuda_status(cudaErrorInvalidValue);
  }
  return cuda_status(launch_proj(absorb, tm_w, tm_x, n, H, M_total, K_total, n_tile, out,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

static mla_status expand_common(const uint16_t *c, const uint16_t *w_uk, const uint16_t *w_uv, uint16_t *k, uint16_t *v,
                                int n, int H, int D, int R, void *stream) {
  if (c == nullptr || w_uk == nullptr || w_uv == nullptr || k == nullptr || v == nullptr) return MLA_ERR_ARG;
  if (n < 1) return MLA_ERR_ARG;
  if (H != kHeads || D != kHeadDim || R != kLatent) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(c) || !aligned16(w_uk) || !aligned16(w_uv) || !aligned16(k) || !aligned16(v))
    return MLA_ERR_UNSUPPORTED;
  if ((long long)n * H >= (1LL << 31)) return MLA_ERR_ARG;
  const int n_tile = std::min(128, (n + 31) / 32 * 32);
  CUtensorMap tm_wk, tm_wv, tm_x;
  {
    const uint64_t dims[3] = {(uint64_t)R, (uint64_t)D, (uint64_t)H};
    const uint64_t strides[2] = {(uint64_t)R * 2, (uint64_t)D * R * 2};
    const uint32_t box[3] = {64, 128, 1};
    if (!make_map(&tm_wk, w_uk, 3, dims, strides, box) || !make_map(&tm_wv, w_uv, 3, dims, strides, box))
      return cuda_status(cudaErrorInvalidValue);
  }
  {
    // c[n][r] seen as X[n][1][r]: one row per token, shared by every head
    const uint64_t dims[3] = {(uint64_t)R, 1, (uint64_t)n};
    const uint64_t strides[2] = {(uint64_t)R * 2, (uint64_t)R * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)n_tile};
    if (!make_map(&tm_x, c, 3, dims, strides, box)) return cuda_status(cudaErrorInvalidValue);
  }
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = launch_proj(false, tm_wk, tm_x, n, H, D, R, n_tile, k, st, true); e != cudaSuccess)
    return cuda_status(e);
  return cuda_status(launch_proj(false, tm_wv, tm_x, n, H, D, R, n_tile, v, st, true));
}

static mla_status prefill_common(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int L, int H, int D,
                                 float scale, uint16_t *out, float *lse, int32_t *status, void *stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return MLA_ERR_ARG;
  if (B < 1 || L < 1 || !isfinite(scale)) return MLA_ERR_ARG;
  if (H != kHeads || D != kHeadDim) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return MLA_ERR_UNSUPPORTED;
  if ((long long)B * L * H >= (1LL << 31)) return MLA_ERR_ARG;
  if ((L + 127) / 128 > 65535 || B > 65535) return MLA_ERR_ARG;  // grid limits
  CUtensorMap tm_k, tm_v;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)H, (uint64_t)B * L};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)H * D * 2};
  const uint32_t box[3] = {64, 1, 64};
  if (!make_map(&tm_k, k, 3, dims, strides, box) || !make_map(&tm_v, v, 3, dims, strides, box))
    return cuda_status(cudaErrorInvalidValue);
  return cuda_status(launch_prefill(tm_k, tm_v, q, out, lse, B, L, scale, status, reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace mla

extern "C" {

mla_status mla_prefill_expanded(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int L, int H, int D,
                                float scale, uint16_t *out, float *lse, int32_t *status, void *stream) {
  return mla::prefill_common(q, k, v, B, L, H, D, scale, out, lse, status, stream);
}

mla_status mla_expand_kv(const uint16_t *c, const uint16_t *w_uk, const uint16_t *w_uv, uint16_t *k, uint16_t *v,
                         int n, int H, int D, int R, void *stream) {
  return mla::expand_common(c, w_uk, w_uv, k, v, n, H, D, R, stream);
}

const char *mla_last_error_string(void) { return cudaGetErrorString(mla::g_last_error); }

const char *mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK:
      return "MLA_OK";
    case MLA_ERR_ARG:
      return "MLA_ERR_ARG";
    case MLA_ERR_UNSUPPORTED:
      return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_CUDA:
      return "MLA_ERR_CUDA";
    case MLA_ERR_WORKSPACE:
      return "MLA_ERR_WORKSPACE";
    case MLA_ERR_INDEX:
      return "MLA_ERR_INDEX";
    case MLA_ERR_TIMEOUT:
      return "MLA_ERR_TIMEOUT";
    default:
      return "MLA_ERR_UNKNOWN";
  }
}

mla_status mla_absorb_q(const uint16_t *q, const uint16_t *w_uk, uint16_t *q_tilde, int n, int H, int D, int R,
                        void *stream) {
  return mla::proj_common(true, q, w_uk, q_tilde, n, H, D, R, stream);
}

mla_status mla_up_proj(const uint16_t *o_latent, const uint16_t *w_uv, uint16_t *out, int n, int H, int D, int R,
                       void *stream) {
  return mla::proj_common(false, o_latent, w_uv, out, n, H, D, R, stream);
}

mla_status mla_attend_dense(const uint16_t *q_tilde, const uint16_t *cache, const int32_t *seq_lens, int B, int Q,
                            int H, int R, int Lmax, float scale, void *workspace, size_t ws_bytes,
                            uint16_t *o_latent, float *lse, int32_t *status, void *stream) {
  return mla::attend_common(mla::kModeDense, q_tilde, cache, nullptr, nullptr, seq_lens, B, Q, H, R, Lmax, 0, 0, 0,
                            0, scale, workspace, ws_bytes, o_latent, lse, status, stream);
}

mla_status mla_attend_paged(const uint16_t *q_tilde, const uint16_t *pool, const int32_t *page_table,
                            const int32_t *seq_lens, int B, int Q, int H, int R, int page_size, int max_pages,
                            int num_pages, float scale, void *workspace, size_t ws_bytes, uint16_t *o_latent,
                            float *lse, int32_t *status, void *stream) {
  return mla::attend_common(mla::kModePaged, q_tilde, pool, page_table, nullptr, seq_lens, B, Q, H, R, 0, page_size,
                            max_pages, num_pages, 0, scale, workspace, ws_bytes, o_latent, lse, status, stream);
}

mla_status mla_attend_indexed(const uint16_t *q_tilde, const uint16_t *cache, const int32_t *indices,
                              const int32_t *seq_lens, int B, int Q, int H, int R, int Lmax, int K, float scale,
                              void *workspace, size_t ws_bytes, uint16_t *o_latent, float *lse, int32_t *status,
                              void *stream) {
  return mla::attend_common(mla::kModeIndexed, q_tilde, cache, nullptr, indices, seq_lens, B, Q, H, R, Lmax, 0, 0, 0,
                            K, scale, workspace, ws_bytes, o_latent, lse, status, stream);
}

mla_status mla_attend_up_dense(const uint16_t *q_tilde, const uint16_t *cache, const int32_t *seq_lens, int B, int Q,
                               int H, int R, int Lmax, float scale, const uint16_t *w_uv, int D, void *workspace,
                               size_t ws_bytes, uint16_t *out, uint16_t *o_latent, float *lse, int32_t *status,
                               void *stream) {
  return mla::attend_common(mla::kModeDense, q_tilde, cache, nullptr, nullptr, seq_lens, B, Q, H, R, Lmax, 0, 0, 0,
                            0, scale, workspace, ws_bytes, o_latent, lse, status, stream, w_uv, D, out);
}

mla_status mla_attend_up_paged(const uint16_t *q_tilde, const uint16_t *pool, const int32_t *page_table,
                               const int32_t *seq_lens, int B, int Q, int H, int R, int page_size, int max_pages,
                               int num_pages, float scale, const uint16_t *w_uv, int D, void *workspace,
                               size_t ws_bytes, uint16_t *out, uint16_t *o_latent, float *lse, int32_t *status,
                               void *stream) {
  return mla::attend_common(mla::kModePaged, q_tilde, pool, page_table, nullptr, seq_lens, B, Q, H, R, 0, page_size,
                            max_pages, num_pages, 0, scale, workspace, ws_bytes, o_latent, lse, status, stream, w_uv,
                            D, out);
}

mla_status mla_attend_up_indexed(const uint16_t *q_tilde, const uint16_t *cache, const int32_t *indices,
                                 const int32_t *seq_lens, int B, int Q, int H, int R, int Lmax, int K, float scale,
                                 const uint16_t *w_uv, int D, void *workspace, size_t ws_bytes, uint16_t *out,
                                 uint16_t *o_latent, float *lse, int32_t *status, void *stream) {
  return mla::attend_common(mla::kModeIndexed, q_tilde, cache, nullptr, indices, seq_lens, B, Q, H, R, Lmax, 0, 0, 0,
                            K, scale, workspace, ws_bytes, o_latent, lse, status, stream, w_uv, D, out);
}

size_t mla_attend_workspace_bytes(int B, int Q, int H, int R) {
  if (B < 1 || Q < 1 || H != mla::kHeads || R != mla::kLatent) return 0;
  return mla::attend_workspace_bytes_for(B, Q, mla::device_sm_count());
}

mla_status mla_debug_gather(int mode, const uint16_t *src, const int32_t *page_table, const int32_t *indices, int B,
                            int Q, int R, int Lmax, int max_pages, int num_pages, int K, const int32_t *req,
                            int n_req, uint16_t *out, int32_t *status, void *stream) {
  if (src == nullptr || req == nullptr || out == nullptr || n_req < 0 || B < 1 || R < 1) return MLA_ERR_ARG;
  if (mode < 0 || mode > 2) return MLA_ERR_ARG;
  if (mode == mla::kModePaged && (page_table == nullptr || max_pages < 1 || num_pages < 1)) return MLA_ERR_ARG;
  if (mode == mla::kModePaged && (long long)max_pages * mla::kPageTokens >= (1LL << 31)) return MLA_ERR_ARG;
  if (mode == mla::kModeIndexed && (indices == nullptr || K < 1 || Q < 1)) return MLA_ERR_ARG;
  if (mode != mla::kModePaged && Lmax < 1) return MLA_ERR_ARG;
  if (n_req == 0) return MLA_OK;
  return mla::cuda_status(mla::launch_debug_gather(mode, src, page_table, indices, B, Q, R, Lmax, max_pages, num_pages,
                                                  K, req, n_req, out, status, reinterpret_cast<cudaStream_t>(stream)));
}

mla_status mla_debug_wait_timeout(long long limit_cycles, int32_t *status, void *stream) {
  if (status == nullptr || limit_cycles < 1 || limit_cycles > 2000000000LL) return MLA_ERR_ARG;
  return mla::cuda_status(mla::launch_wait_timeout(limit_cycles, status, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

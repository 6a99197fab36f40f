// proj.cu -- the two per-head projections around latent attention (Module 05, section 3):
//   absorb:  q~[n, h, r]  = sum_d W_UK[h][d][r] * q[n, h, d]      (q~_h = U_h^K^T q_h)
//   up-proj: out[n, h, d] = sum_r W_UV[h][d][r] * o[n, h, r]      (out_h = U_h^V o_h)
// Both are weight-streaming GEMMs with few token rows, so the weights go on the MMA M
// side (128 rows per CTA) and the tokens on N:
//   D[m, n] = A_h[m, k] * X[n, h, k]^T,   A_h = W_UK[h]^T (MN-major) or W_UV[h] (K-major).
// One CTA per (head, 128-row weight block, token tile): warp 0 streams 64-wide K chunks
// through a TMA ring, warp 1 issues tcgen05 MMAs into TMEM, warps 2-5 convert the
// fp32 accumulator to bf16 and store it.  All K chunks of the weight block are in flight
// at once when shared memory allows (up to 8 stages).
#include <algorithm>

#include "internal.h"
#include "sm100.cuh"

namespace mla {
namespace proj {

constexpr int kThreads = 192;
constexpr int kMaxStages = 8;
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kABytes = kBM * kBK * 2;  // 16 KB per stage
constexpr uint32_t kTmemCols = 128;
constexpr int kSmemLimit = 227 * 1024;

// Shared memory: `stages` A tiles (16 KB), `stages` B tiles (n_tile x 128 B), barriers.
__host__ __device__ constexpr int smem_bytes(int stages, int n_tile) {
  return stages * (kABytes + n_tile * kBK * 2) + (2 * kMaxStages + 1) * 8 + 16 + 1024;
}

struct Params {
  int n, H, M_total, K_total, n_tile, stages;
  int x_bcast;  // 1: X has one row per token shared by every head (X[n][k], the latents c)
  uint16_t *out;
};

template <bool kAMajorMN>
__global__ void __launch_bounds__(kThreads, 1)
    proj_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int kStages = p.stages;
  const int b_bytes = p.n_tile * kBK * 2;
  uint8_t *a_stage0 = base;
  uint8_t *b_stage0 = base + kStages * kABytes;
  uint64_t *full = reinterpret_cast<uint64_t *>(b_stage0 + kStages * b_bytes);
  uint64_t *empty = full + kMaxStages;
  uint64_t *done = empty + kMaxStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.x, mb = blockIdx.y, nt = blockIdx.z;
  grid_dep_launch();
  const int NT = p.n_tile;
  const int nk = p.K_total / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
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

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tm_w);
      prefetch_tensormap(&tm_x);
      auto load_a = [&](int kc, int s) {
        uint8_t *a_dst = a_stage0 + s * kABytes;
        if (kAMajorMN) {
          // W_UK[h][d][r]: box {64 r, 64 d}; two boxes cover the 128 r of this block
          tma_load_3d(a_dst, &tm_w, &full[s], mb * kBM, kc * kBK, h);
          tma_load_3d(a_dst + kABytes / 2, &tm_w, &full[s], mb * kBM + 64, kc * kBK, h);
        } else {
          // W_UV[h][d][r]: box {64 r, 128 d}
          tma_load_3d(a_dst, &tm_w, &full[s], kc * kBK, mb * kBM, h);
        }
      };
      // The weights never come from an earlier kernel: the first ring's worth streams in
      // while the preceding kernel finishes; the token rows are read after it has.
      const int pre = min(kStages, nk);
      for (int kc = 0; kc < pre; ++kc) {
        mbar_arrive_expect_tx(&full[kc], kABytes + NT * kBK * 2);
        load_a(kc, kc);
      }
      grid_dep_wait();
      const int xh = p.x_bcast ? 0 : h;
      for (int kc = 0; kc < pre; ++kc) tma_load_3d(b_stage0 + kc * b_bytes, &tm_x, &full[kc], kc * kBK, xh, nt * NT);
      int issued = pre;
      for (int kc = pre; kc < nk; ++kc) {
        const int s = kc % kStages, use = kc / kStages;
        if (!mbar_wait(&empty[s], (use & 1) ^ 1, abort_flag, nullptr)) break;
        mbar_arrive_expect_tx(&full[s], kABytes + NT * kBK * 2);
        load_a(kc, s);
        tma_load_3d(b_stage0 + s * b_bytes, &tm_x, &full[s], kc * kBK, xh, nt * NT);
        issued = kc + 1;
      }
      // every issued copy lands before the CTA may exit (also after an abort)
      drain_ring(full, (uint32_t)kStages, (uint32_t)issued);
    }
  } else if (warp == 1) {
    const uint32_t idesc = idesc_bf16_f32(kBM, NT, kAMajorMN, false);
    bool ok = true;
    for (int kc = 0; kc < nk && ok; ++kc) {
      const int s = kc % kStages, use = kc / kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&full[s], use & 1, abort_flag, nullptr));
      if (!ok) break;
      tc_fence_after();
      // MN-major A: 64-wide r atoms 8 KB apart (LBO), 8-row d groups 1 KB apart (SBO), K step
      // = 2 KB; K-major A/B: 128-byte rows, 8-row groups 1 KB apart, K step = 32 bytes.
      const uint64_t a0 = kAMajorMN ? sw128_desc(smem_u32(a_stage0 + s * kABytes), kABytes / 2, 1024)
                                    : sw128_desc(smem_u32(a_stage0 + s * kABytes), 16, 1024);
      const uint64_t b0 = sw128_desc(smem_u32(b_stage0 + s * b_bytes), 16, 1024);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_bf16(tmem, a0 + (kAMajorMN ? kk * 128 : kk * 2), b0 + kk * 2, idesc, (kc | kk) != 0);
        umma_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (elect_one()) umma_commit(done);
    __syncwarp();
  } else {
    const bool ok = mbar_wait(done, 0, abort_flag, nullptr);
    tc_fence_after();
    const int wq = warp & 3;
    const int m = mb * kBM + wq * 32 + lane;
    for (int n0 = 0; n0 < NT; n0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(wq * 32) << 16) + n0, r);
      tmem_ld_wait();
      if (ok) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int n = nt * NT + n0 + j;
          if (n < p.n) {
            const uint32_t v = pack_bf16x2(__uint_as_float(r[j]), 0.f);
            p.out[((long long)n * p.H + h) * p.M_total + m] = (uint16_t)(v & 0xFFFFu);
          }
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace proj

template <bool kAMajorMN>
static cudaError_t launch_proj_t(const CUtensorMap &tm_w, const CUtensorMap &tm_x, const proj::Params &p,
                                 cudaStream_t stream) {
  static std::atomic<int> configured_device{-1};
  const cudaError_t e0 = set_smem_limit_once(proj::proj_kernel<kAMajorMN>, proj::kSmemLimit, configured_device);
  if (e0 != cudaSuccess) return e0;
  dim3 grid(p.H, p.M_total / proj::kBM, (p.n + p.n_tile - 1) / p.n_tile);
  return launch_chained(proj::proj_kernel<kAMajorMN>, grid, dim3(proj::kThreads), proj::smem_bytes(p.stages, p.n_tile),
                        stream, tm_w, tm_x, p);
}

cudaError_t launch_proj(bool a_mn_major, const CUtensorMap &tm_w, const CUtensorMap &tm_x, int n, int H,
                        int M_total, int K_total, int n_tile, uint16_t *out, cudaStream_t stream, bool x_bcast) {
  // keep every K chunk of the weight block in flight when it fits
  int stages = std::min(proj::kMaxStages, K_total / proj::kBK);
  while (stages > 2 && proj::smem_bytes(stages, n_tile) > proj::kSmemLimit) --stages;
  proj::Params p{n, H, M_total, K_total, n_tile, stages, x_bcast ? 1 : 0, out};
  return a_mn_major ? launch_proj_t<true>(tm_w, tm_x, p, stream) : launch_proj_t<false>(tm_w, tm_x, p, stream);
}

}  // namespace mla

// Calibration covariance H = alpha * A^T A + beta * H  [wmrh §二; aimodeling:
// H ≈ H_X ⊗ H_G with H_X = XᵀX/n over activations and H_G = GᵀG/n over output
// gradients from one backward pass, gptget-en Methodology].
//
// bf16 path: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32 in TMEM). A CTA owns a
// 256x256 tile of H (two M=128 accumulators = all 512 TMEM columns) and
// streams the n rows of A through a 3-stage TMA ring, 64 rows per stage. Both
// MMA operands are the same row slab of A read feature-contiguous
// ("MN-major"), so A is consumed in place without a transpose. Only tiles on
// or above the diagonal are computed; each value ends in (i,j) and in its
// mirror (j,i), so both triangles are bitwise equal. Tiles are visited in
// 12x12 super-tiles so that the CTAs resident at one time touch a small set
// of feature columns and share each A slab through L2.
//
// The tensor core's fp32 accumulation loses part of an ulp per step in one
// direction (measured: a sum of 131072 squares comes out 6.6e-4 low when
// accumulated in TMEM alone). The accumulator therefore restarts every
// CHUNK rows of A: eight epilogue warps fold each chunk's sum into H with
// round-to-nearest fp32 adds (through the mirror (j,i), whose addresses are
// consecutive across a warp's lanes) while the MMA waits, and the last fold
// writes both triangles. A chunk of 16384 rows keeps the drift near 5e-5
// (the measured loss is about 0.9 ulp per MMA step of 16 rows).
//
// fp32 path: plain FFMA tiles (used for fp32 calibration data).
#include <cooperative_groups.h>

#include "kernels.cuh"

namespace cg = cooperative_groups;

namespace kronq {
namespace {

constexpr int CT = 256;               // tile edge
constexpr int CBK = 64;               // rows of A per stage
constexpr int CSTAGES = 3;
constexpr int CBOX = 64 * CBK * 2;    // one TMA box: 64 rows x 64 features bf16
constexpr int CSTAGE_BYTES = 8 * CBOX;  // 4 boxes for the row panel, 4 for the column panel
constexpr int CTHREADS = 320;         // TMA warp, MMA warp, 8 epilogue warps
constexpr int SUPER = 12;
constexpr int CHUNK = 16384;          // rows of A per TMEM accumulation
constexpr int CHUNK_K = CHUNK / CBK;  // stages per chunk

struct CovCtl {
  uint64_t full[CSTAGES];
  uint64_t empty[CSTAGES];
  uint64_t chunk_done;  // MMAs of a chunk finished (commit)
  uint64_t folded;      // the epilogue warps have read the accumulator (256)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr int CSMEM = CSTAGES * CSTAGE_BYTES + 1024 + sizeof(CovCtl) + 64;

// Upper-triangle tile t of an nt x nt grid, super-tile raster.
__device__ void cov_tile(int64_t t, int nt, int &bi, int &bj) {
  const int ns = (nt + SUPER - 1) / SUPER;
  for (int si = 0; si < ns; ++si) {
    for (int sj = si; sj < ns; ++sj) {
      const int r0 = si * SUPER, r1 = min(nt, r0 + SUPER);
      const int c0 = sj * SUPER, c1 = min(nt, c0 + SUPER);
      int64_t cnt;
      if (si < sj) {
        cnt = int64_t(r1 - r0) * (c1 - c0);
      } else {
        const int w = r1 - r0;
        cnt = int64_t(w) * (w + 1) / 2;
      }
      if (t < cnt) {
        if (si < sj) {
          bi = r0 + static_cast<int>(t / (c1 - c0));
          bj = c0 + static_cast<int>(t % (c1 - c0));
        } else {
          const int w = r1 - r0;
          int i = 0;
          while (t >= w - i) {
            t -= w - i;
            ++i;
          }
          bi = r0 + i;
          bj = r0 + i + static_cast<int>(t);
        }
        return;
      }
      t -= cnt;
    }
  }
  bi = bj = 0;
}

__global__ void __launch_bounds__(CTHREADS, 1)
    cov_bf16_kernel(const __grid_constant__ CUtensorMap tmX, int64_t n,
                    int64_t d, float alpha, float beta, float *__restrict__ H,
                    int32_t *info) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  CovCtl *ctl = reinterpret_cast<CovCtl *>(smem + CSTAGES * CSTAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = static_cast<int>((d + CT - 1) / CT);
  const int64_t tiles = int64_t(nt) * (nt + 1) / 2;
  const int64_t rounds = (tiles + gridDim.x - 1) / gridDim.x;
  const int nk = static_cast<int>((n + CBK - 1) / CBK);
  const int nchunks = nk > 0 ? (nk + CHUNK_K - 1) / CHUNK_K : 0;
  cg::grid_group grid = cg::this_grid();

  if (threadIdx.x == 0) {
    for (int s = 0; s < CSTAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->chunk_done, 1);
    mbar_init(&ctl->folded, 256);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = ctl->tmem_base;
  volatile int *abort = &ctl->abort;

  // Pipeline positions run on across the CTA's tiles: g counts stages
  // (ring slot g % CSTAGES, phase g / CSTAGES), cgl counts accumulator
  // chunks (the chunk_done / folded phases).
  int64_t g_tma = 0, g_mma = 0;
  int64_t cgl_mma = 0, cgl_epi = 0;
  int64_t issued = 0;
  for (int64_t r = 0; r < rounds; ++r) {
    const int64_t t = blockIdx.x + r * gridDim.x;
    if (t < tiles && !*abort) {
      int bi, bj;
      cov_tile(t, nt, bi, bj);
      const int64_t i0 = int64_t(bi) * CT, j0 = int64_t(bj) * CT;
      if (warp == 0 && lane == 0) {
        for (int it = 0; it < nk; ++it, ++g_tma) {
          const int s = static_cast<int>(g_tma % CSTAGES);
          if (g_tma >= CSTAGES &&
              !mbar_wait(&ctl->empty[s], ((g_tma / CSTAGES) - 1) & 1, abort))
            break;
          uint8_t *st = smem + s * CSTAGE_BYTES;
          const int32_t k0 = static_cast<int32_t>(int64_t(it) * CBK);
          mbar_expect_tx(&ctl->full[s], CSTAGE_BYTES);
          for (int c = 0; c < 4; ++c)
            tma_load_2d(st + c * CBOX, &tmX, &ctl->full[s],
                        static_cast<int32_t>(i0 + 64 * c), k0);
          for (int c = 0; c < 4; ++c)
            tma_load_2d(st + (4 + c) * CBOX, &tmX, &ctl->full[s],
                        static_cast<int32_t>(j0 + 64 * c), k0);
          issued = g_tma + 1;
        }
      } else if (warp == 1 && lane == 0) {
        // bf16 operands, both MN-major, 128 x 256 per instruction
        const uint32_t idesc = idesc_make(1, 1, 1, 128, 256);
        for (int it = 0; it < nk; ++it, ++g_mma) {
          const int s = static_cast<int>(g_mma % CSTAGES);
          const int first = it % CHUNK_K == 0;
          // a new chunk overwrites the accumulator once the last one is folded
          if (first) {
            if (cgl_mma > 0 && !mbar_wait(&ctl->folded, (cgl_mma - 1) & 1, abort)) break;
            ++cgl_mma;
          }
          if (!mbar_wait(&ctl->full[s], (g_mma / CSTAGES) & 1, abort)) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * CSTAGE_BYTES);
          const uint32_t b0 = a0 + 4 * CBOX;
#pragma unroll
          for (int kk = 0; kk < CBK / 16; ++kk) {
            const uint64_t db = sdesc_sw128(b0 + kk * 2048, CBOX, 1024);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t da = sdesc_sw128(a0 + h * 2 * CBOX + kk * 2048, CBOX, 1024);
              umma_bf16(tbase + 256 * h, da, db, idesc, (!first || kk != 0) ? 1u : 0u);
            }
          }
          umma_commit(&ctl->empty[s]);
          if (it % CHUNK_K == CHUNK_K - 1 || it == nk - 1) umma_commit(&ctl->chunk_done);
          // the fold of this chunk reads the running sums (rows j of the
          // mirror block): bring them back into L2, which the streamed rows of
          // A evicted
          const int ci = it / CHUNK_K;
          const bool fold_reads = ci > 0 || beta != 0.f;
          if (fold_reads && (it % CHUNK_K == CHUNK_K - 8 || (it == nk - 8 && nk >= 8))) {
            const int64_t cols = kq_min<int64_t>(CT, d - i0);
            const uint32_t bytes = static_cast<uint32_t>(cols * 4) & ~15u;
            for (int64_t j = j0; j < kq_min<int64_t>(j0 + CT, d) && bytes > 0; ++j)
              prefetch_l2_bulk(H + j * d + i0, bytes);
          }
        }
      } else if (warp >= 2) {
        // ---- epilogue warps: warp w folds accumulator (w-2)/4, TMEM lanes
        // 32*(w%4) .. +31 (tile rows), all 256 columns of its half
        const int h = (warp - 2) >> 2, q = warp & 3;
        const int64_t i = i0 + 128 * h + 32 * q + lane;
        const bool diag = (bi == bj);
        for (int ci = 0; ci < nchunks; ++ci, ++cgl_epi) {
          const bool ok = mbar_wait(&ctl->chunk_done, cgl_epi & 1, abort);
          if (!__all_sync(0xffffffffu, ok)) break;
          tc_fence_after();
          const bool last = ci == nchunks - 1;
          for (int c = 0; c < CT / 32; ++c) {
            float v[32];
            tmem_ld32(tbase + (static_cast<uint32_t>(32 * q) << 16) + 256 * h + 32 * c, v);
            const int64_t jc = j0 + 32 * c;
            if (jc >= d) continue;
            // running sum (or the old H) at the mirror: all 32 loads before
            // any store (their addresses are d apart, which the compiler
            // cannot separate from the stores)
            const bool need = ci > 0 || beta != 0.f;  // uniform across the CTA
            const float bw = ci > 0 ? 1.f : beta;
            float prev[32];
            if (need) {  // unconditional loads at clamped (in-bounds) addresses
              const int64_t ic = kq_min<int64_t>(i, d - 1);
#pragma unroll
              for (int tt = 0; tt < 32; ++tt)
                prev[tt] = __ldcg(H + kq_min<int64_t>(jc + tt, d - 1) * d + ic);
            } else {
#pragma unroll
              for (int tt = 0; tt < 32; ++tt) prev[tt] = 0.f;
            }
#pragma unroll
            for (int tt = 0; tt < 32; ++tt) {
              const int64_t j = jc + tt;
              if (!((i < d) && (j < d) && (!diag || j >= i))) continue;
              const float o = fmaf(bw, prev[tt], alpha * v[tt]);
              H[j * d + i] = o;
              if (last && j != i) H[i * d + j] = o;
            }
          }
          tc_fence_before();
          mbar_arrive(&ctl->folded);
        }
      }
    }
    __syncwarp();
    // every CTA of the grid starts the next round together, so that the
    // tiles of a round stream the same rows of A at the same time and share
    // them through L2 (all CTAs take the same number of barriers, also after
    // a timeout)
    tc_fence_before();
    grid.sync();
    tc_fence_after();
  }

  tc_fence_before();
  __syncthreads();
  if (*abort) {
    if (threadIdx.x == 0) report(info, KRONQ_ERR_TIMEOUT);
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = globaltimer();
      for (int s = 0; s < CSTAGES && s < issued; ++s) {
        const int64_t last = ((issued - 1 - s) / CSTAGES) * CSTAGES + s;
        while (!mbar_try_wait(&ctl->full[s], (last / CSTAGES) & 1) &&
               globaltimer() - t0 < kWaitLimitNs) {
        }
      }
    }
    if (warp == 1 && lane == 0) {
      umma_commit(&ctl->drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&ctl->drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---- fp32 path: 64x64 output tiles, 16 rows of A per step, 4x4 per thread.
constexpr int FT = 64, FK = 16;
__global__ void __launch_bounds__(256)
    cov_f32_kernel(const float *__restrict__ A, int64_t n, int64_t d,
                   int64_t lda, float alpha, float beta, float *__restrict__ H) {
  __shared__ float As[FK][FT];
  __shared__ float Bs[FK][FT];
  const int nt = static_cast<int>((d + FT - 1) / FT);
  int64_t t = blockIdx.x;
  int bi = 0;
  while (t >= nt - bi) {
    t -= nt - bi;
    ++bi;
  }
  const int bj = bi + static_cast<int>(t);
  const int64_t i0 = int64_t(bi) * FT, j0 = int64_t(bj) * FT;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < n; k0 += FK) {
    for (int e = threadIdx.x; e < FK * FT; e += 256) {
      const int kr = e / FT, cc = e % FT;
      const int64_t k = k0 + kr;
      As[kr][cc] = (k < n && i0 + cc < d) ? A[k * lda + i0 + cc] : 0.f;
      Bs[kr][cc] = (k < n && j0 + cc < d) ? A[k * lda + j0 + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kr = 0; kr < FK; ++kr) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = As[kr][ty + 16 * u];
        b[u] = Bs[kr][tx + 16 * u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], b[w], acc[u][w]);
    }
    __syncthreads();
  }
  const bool diag = bi == bj;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int64_t i = i0 + ty + 16 * u, j = j0 + tx + 16 * w;
      if (i >= d || j >= d || (diag && j < i)) continue;
      float o = alpha * acc[u][w];
      if (beta != 0.f) o += beta * H[i * d + j];
      H[i * d + j] = o;
      if (j != i) H[j * d + i] = o;
    }
  }
}

__global__ void scale_kernel(float *H, int64_t n, float beta) {
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n;
       e += int64_t(gridDim.x) * blockDim.x)
    H[e] = beta == 0.f ? 0.f : beta * H[e];
}

}  // namespace

kronq_status scale_matrix(cudaStream_t st, float *H, int64_t n_elems, float beta) {
  if (n_elems <= 0) return KRONQ_OK;
  const int64_t blocks = kq_min<int64_t>(ceil_div(n_elems, 256), 148 * 16);
  scale_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(H, n_elems, beta);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

kronq_status cov_bf16(cudaStream_t st, const __nv_bfloat16 *A, int64_t n,
                      int64_t d, int64_t lda, float alpha, float beta,
                      float *H, int32_t *info) {
  if (n == 0) return scale_matrix(st, H, d * d, beta);
  CUtensorMap tm;
  KQ_TRY(make_tmap_2d(&tm, A, true, d, n, lda, 64, CBK));
  const int64_t nt = ceil_div(d, CT);
  const int64_t tiles = nt * (nt + 1) / 2;
  KQ_TRY(smem_attr(cov_bf16_kernel, CSMEM));
  // persistent: one CTA per SM (the 196 KB ring allows one), all resident
  // (cooperative launch), taking the tiles in rounds
  int dev = 0, sms = 0, per_sm = 0;
  KQ_CUDA(cudaGetDevice(&dev));
  KQ_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  KQ_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, cov_bf16_kernel, CTHREADS,
                                                        CSMEM));
  if (per_sm < 1) return KRONQ_ERR_UNSUPPORTED;
  const unsigned grid = static_cast<unsigned>(kq_min<int64_t>(tiles, int64_t(sms) * per_sm));
  void *args[] = {const_cast<CUtensorMap *>(&tm), &n, &d, &alpha, &beta, &H, &info};
  KQ_CUDA(cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(cov_bf16_kernel), grid,
                                      CTHREADS, args, CSMEM, st));
  count_launch();
  return KRONQ_OK;
}

kronq_status cov_f32(cudaStream_t st, const float *A, int64_t n, int64_t d,
                     int64_t lda, float alpha, float beta, float *H) {
  if (n == 0) return scale_matrix(st, H, d * d, beta);
  const int64_t nt = ceil_div(d, FT);
  const int64_t tiles = nt * (nt + 1) / 2;
  cov_f32_kernel<<<static_cast<unsigned>(tiles), 256, 0, st>>>(A, n, d, lda,
                                                               alpha, beta, H);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

}  // namespace kronq

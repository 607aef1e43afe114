// fp32-accurate GEMM on the sm_100a tensor cores: C = beta*C + alpha*A*B^T
// with every fp32 operand split into TF32 hi + lo parts and three tcgen05
// MMAs (hi*hi + hi*lo + lo*hi) per k-step into an fp32 TMEM accumulator.
//
// Used by the blocked Cholesky/inverse, the OBS trailing updates and the
// layer loss. One CTA computes a 128x128 tile:
//   warp 0      TMA producer (one elected lane), 3-stage ring of 32-wide k-slabs
//   warp 1      TMEM owner and MMA issuer (one elected lane)
//   warps 2..5  write the TF32 low part of each landed fp32 slab next to it in
//               shared memory (the raw slab itself serves as the high part),
//               then run the epilogue (TMEM -> registers -> C).
#include "kernels.cuh"

namespace kronq {
namespace {

constexpr int BM = 128, BN = 128, BK = 32, STAGES = 3;
constexpr int TILE_BYTES = BM * BK * 4;        // one 128 x 32 fp32 slab
constexpr int STAGE_BYTES = 4 * TILE_BYTES;    // A_hi, A_lo, B_hi, B_lo
constexpr int NTHREADS = 192;
constexpr int GROUP_M = 16;                    // tile raster: 16 rows per band

struct Ctl {
  uint64_t full[STAGES];   // TMA landed (expect_tx)
  uint64_t conv[STAGES];   // hi/lo split written (128 arrivals)
  uint64_t empty[STAGES];  // MMAs that read the stage finished (commit)
  uint64_t done;           // all MMAs finished (commit)
  uint64_t drain;          // teardown drain after an abort
  uint32_t tmem_base;
  int abort;
};
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + sizeof(Ctl) + 64;

// The tf32 MMA reads an fp32 operand by dropping its 13 low mantissa bits
// (truncation, measured on sm_100a), so the raw slab already is the hi part;
// only lo = x - trunc(x) (exact in fp32) has to be written.
__device__ __forceinline__ float4 tf32_lo(float4 x) {
  const uint32_t mask = 0xffffe000u;
  return make_float4(x.x - __uint_as_float(__float_as_uint(x.x) & mask),
                     x.y - __uint_as_float(__float_as_uint(x.y) & mask),
                     x.z - __uint_as_float(__float_as_uint(x.z) & mask),
                     x.w - __uint_as_float(__float_as_uint(x.w) & mask));
}

__global__ void __launch_bounds__(NTHREADS, 1)
    gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, int64_t M,
                       int64_t N, int64_t K, float *__restrict__ C, int64_t ldc,
                       float alpha, float beta, uint32_t kflags, int a_mn,
                       int b_mn, int upper_only, int tiles_m, int tiles_n,
                       int vec_ok, int32_t *info) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl *ctl = reinterpret_cast<Ctl *>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- tile coordinates
  int64_t bi, bj;
  {
    int64_t t = blockIdx.x;
    if (upper_only) {
      bi = 0;
      while (t >= tiles_n - bi) {
        t -= tiles_n - bi;
        ++bi;
      }
      bj = bi + t;
    } else {
      const int64_t band = t / (int64_t(GROUP_M) * tiles_n);
      const int64_t rows = kq_min<int64_t>(GROUP_M, tiles_m - band * GROUP_M);
      const int64_t r = t - band * GROUP_M * tiles_n;
      bi = band * GROUP_M + r % rows;
      bj = r / rows;
    }
  }
  const int64_t m0 = bi * BM, n0 = bj * BN;
  int64_t kb = 0, ke = K;
  if (kflags & KR_A_UPPER) kb = kq_max<int64_t>(kb, m0);
  if (kflags & KR_B_UPPER) kb = kq_max<int64_t>(kb, n0);
  if (kflags & KR_A_LOWER) ke = kq_min<int64_t>(ke, m0 + BM);
  if (kflags & KR_B_LOWER) ke = kq_min<int64_t>(ke, n0 + BN);
  kb = (kb / BK) * BK;
  const int nk = ke > kb ? static_cast<int>((ke - kb + BK - 1) / BK) : 0;

  // ---- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->conv[s], 128);
      mbar_init(&ctl->empty[s], 1);
    }
    mbar_init(&ctl->done, 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = ctl->tmem_base;
  volatile int *abort = &ctl->abort;

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      for (int it = 0; it < nk; ++it) {
        const int s = it % STAGES;
        if (it >= STAGES &&
            !mbar_wait(&ctl->empty[s], ((it / STAGES) - 1) & 1, abort))
          break;
        uint8_t *st = smem + s * STAGE_BYTES;
        const int32_t k0 = static_cast<int32_t>(kb + int64_t(it) * BK);
        mbar_expect_tx(&ctl->full[s], 2 * TILE_BYTES);
        if (!a_mn) {
          tma_load_2d(st, &tmA, &ctl->full[s], k0, static_cast<int32_t>(m0));
        } else {
          for (int c = 0; c < 4; ++c)
            tma_load_2d(st + c * (TILE_BYTES / 4), &tmA, &ctl->full[s],
                        static_cast<int32_t>(m0 + 32 * c), k0);
        }
        uint8_t *sb = st + 2 * TILE_BYTES;
        if (!b_mn) {
          tma_load_2d(sb, &tmB, &ctl->full[s], k0, static_cast<int32_t>(n0));
        } else {
          for (int c = 0; c < 4; ++c)
            tma_load_2d(sb + c * (TILE_BYTES / 4), &tmB, &ctl->full[s],
                        static_cast<int32_t>(n0 + 32 * c), k0);
        }
        issued = it + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_make(2, a_mn, b_mn, BM, BN);
      const uint32_t lbo_a = a_mn ? TILE_BYTES / 4 : 16;
      const uint32_t lbo_b = b_mn ? TILE_BYTES / 4 : 16;
      // K-major: 8-row groups of 128 B rows (16-byte swizzle granules);
      // MN-major tf32: 4-row groups, 32-byte granules (layout type 1)
      const uint32_t sbo_a = a_mn ? 512 : 1024, sbo_b = b_mn ? 512 : 1024;
      const uint32_t lay_a = a_mn ? 1 : 2, lay_b = b_mn ? 1 : 2;
      int it = 0;
      for (; it < nk; ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(&ctl->conv[s], (it / STAGES) & 1, abort)) break;
        tc_fence_after();
        const uint32_t a_hi = smem_u32(smem + s * STAGE_BYTES);
        const uint32_t a_lo = a_hi + TILE_BYTES;
        const uint32_t b_hi = a_hi + 2 * TILE_BYTES;
        const uint32_t b_lo = a_hi + 3 * TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 8; ++kk) {
          const uint32_t ao = a_mn ? kk * 1024 : kk * 32;
          const uint32_t bo = b_mn ? kk * 1024 : kk * 32;
          const uint64_t dah = sdesc(a_hi + ao, lbo_a, sbo_a, lay_a);
          const uint64_t dal = sdesc(a_lo + ao, lbo_a, sbo_a, lay_a);
          const uint64_t dbh = sdesc(b_hi + bo, lbo_b, sbo_b, lay_b);
          const uint64_t dbl = sdesc(b_lo + bo, lbo_b, sbo_b, lay_b);
          umma_tf32(tbase, dal, dbh, idesc, (it | kk) != 0);
          umma_tf32(tbase, dah, dbl, idesc, 1);
          umma_tf32(tbase, dah, dbh, idesc, 1);
        }
        umma_commit(&ctl->empty[s]);
      }
      if (nk > 0)
        umma_commit(&ctl->done);
      else
        mbar_arrive(&ctl->done);
    }
  } else {
    // ---- hi/lo split of every landed slab
    const int ct = threadIdx.x - 64;
    for (int it = 0; it < nk; ++it) {
      const int s = it % STAGES;
      if (!mbar_wait(&ctl->full[s], (it / STAGES) & 1, abort)) break;
      float4 *st = reinterpret_cast<float4 *>(smem + s * STAGE_BYTES);
      constexpr int Q = TILE_BYTES / 16;
#pragma unroll 4
      for (int i = ct; i < Q; i += 128) {
        st[Q + i] = tf32_lo(st[i]);
        st[3 * Q + i] = tf32_lo(st[2 * Q + i]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&ctl->conv[s]);
    }
    // ---- epilogue: TMEM lanes 32q..32q+31 hold tile rows 32q..32q+31
    const bool ok = mbar_wait(&ctl->done, 0, abort);
    const bool have = __all_sync(0xffffffffu, ok) && nk > 0;
    tc_fence_after();
    const int q = warp & 3;
    const int64_t row = m0 + 32 * q + lane;
    for (int c = 0; c < BN / 32; ++c) {
      float v[32];
      if (have) {
        tmem_ld32(tbase + (static_cast<uint32_t>(32 * q) << 16) + 32 * c, v);
      } else {
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = 0.f;
      }
      if (row >= M) continue;
      const int64_t col0 = n0 + 32 * c;
      float *crow = C + row * ldc + col0;
      if (vec_ok && col0 + 32 <= N) {
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          float4 o = make_float4(alpha * v[t], alpha * v[t + 1],
                                 alpha * v[t + 2], alpha * v[t + 3]);
          if (beta != 0.f) {
            const float4 old = *reinterpret_cast<const float4 *>(crow + t);
            o.x += beta * old.x;
            o.y += beta * old.y;
            o.z += beta * old.z;
            o.w += beta * old.w;
          }
          *reinterpret_cast<float4 *>(crow + t) = o;
        }
      } else {
        for (int t = 0; t < 32 && col0 + t < N; ++t) {
          float o = alpha * v[t];
          if (beta != 0.f) o += beta * crow[t];
          crow[t] = o;
        }
      }
    }
  }

  // ---- teardown: after an abort make sure no copy or MMA is still in flight
  tc_fence_before();
  __syncthreads();
  if (ctl->abort) {
    if (threadIdx.x == 0) report(info, KRONQ_ERR_TIMEOUT);
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = globaltimer();
      for (int s = 0; s < STAGES && s < issued; ++s) {
        const int last = ((issued - 1 - s) / STAGES) * STAGES + s;
        while (!mbar_try_wait(&ctl->full[s], (last / STAGES) & 1) &&
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
    tmem_dealloc(tbase, 128);
  }
}

}  // namespace

kronq_status gemm_tf32x3(cudaStream_t st, const GemmArgs &g, int32_t *info) {
  if (g.M < 0 || g.N < 0 || g.K < 0) return KRONQ_ERR_INVALID_ARG;
  if (g.M == 0 || g.N == 0) return KRONQ_OK;
  if (g.upper_tiles_only && g.M != g.N) return KRONQ_ERR_INVALID_ARG;
  CUtensorMap ta, tb;
  // A: K-major -> rows M of K; MN-major -> rows K of M
  if (g.K > 0) {
    KQ_TRY(make_tmap_2d(&ta, g.A, false, g.a_mn ? g.M : g.K,
                        g.a_mn ? g.K : g.M, g.lda, 32, g.a_mn ? 32 : 128, g.a_mn));
    KQ_TRY(make_tmap_2d(&tb, g.B, false, g.b_mn ? g.N : g.K,
                        g.b_mn ? g.K : g.N, g.ldb, 32, g.b_mn ? 32 : 128, g.b_mn));
  } else {
    memset(&ta, 0, sizeof(ta));
    memset(&tb, 0, sizeof(tb));
  }
  const int64_t tm = ceil_div(g.M, BM), tn = ceil_div(g.N, BN);
  const int64_t tiles = g.upper_tiles_only ? tn * (tn + 1) / 2 : tm * tn;
  if (tiles > 0x7fffffff) return KRONQ_ERR_UNSUPPORTED;
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(gemm_tf32x3_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    attr_done = true;
  }
  const int vec_ok = (reinterpret_cast<uintptr_t>(g.C) % 16 == 0) && (g.ldc % 4 == 0);
  gemm_tf32x3_kernel<<<static_cast<unsigned>(tiles), NTHREADS, SMEM_BYTES, st>>>(
      ta, tb, g.M, g.N, g.K, g.C, g.ldc, g.alpha, g.beta, g.kflags,
      g.a_mn ? 1 : 0, g.b_mn ? 1 : 0, g.upper_tiles_only ? 1 : 0,
      static_cast<int>(tm), static_cast<int>(tn), vec_ok, info);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

}  // namespace kronq

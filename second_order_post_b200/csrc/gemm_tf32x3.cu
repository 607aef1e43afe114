// fp32-accurate GEMM on the sm_100a tensor cores: C = beta*C + alpha*A*B^T
// with every fp32 operand split into TF32 hi + lo parts and three tcgen05
// MMAs (hi*hi + hi*lo + lo*hi) per k-step into an fp32 TMEM accumulator.
//
// Used by the blocked Cholesky/inverse, the OBS trailing updates and the
// layer loss. One CTA computes a 128 x BN tile (BN = 256 for wide outputs,
// 128 otherwise):
//   warp 0      TMA producer (one elected lane), ring of BK-wide k-slabs
//   warp 1      TMEM owner and MMA issuer (one elected lane)
//   warps 2..5  write the TF32 low part of each landed fp32 slab next to it in
//               shared memory (the raw slab itself serves as the high part),
//               then run the epilogue (TMEM -> registers -> C).
// The split warps load a whole slab into registers before they store any low
// part (the two share one array, so interleaved loads and stores would run
// one round trip at a time). Low parts precomputed in global memory instead
// would double the L2 -> SM traffic, which costs more than the split.
#include "kernels.cuh"

namespace kronq {
namespace {

constexpr int BM = 128;
constexpr int NTHREADS = 192;
constexpr int GROUP_M = 16;                    // tile raster: 16 rows per band

template <int STAGES>
struct Ctl {
  uint64_t full[STAGES];   // TMA landed (expect_tx)
  uint64_t conv[STAGES];   // hi/lo split written (128 arrivals)
  uint64_t empty[STAGES];  // MMAs that read the stage finished (commit)
  uint64_t done;           // all MMAs finished (commit)
  uint64_t drain;          // teardown drain after an abort
  uint32_t tmem_base;
  int abort;
};

// Tile configuration: BN output columns, BK-wide k-slabs, STAGES-deep ring.
// K-major slabs are rows of BK fp32 (128 or 64 bytes, swizzled to match);
// MN-major slabs are 32-wide MN chunks of BK k-rows (32-byte granules).
template <int BN_, int BK_, int STAGES_>
struct Cfg {
  static constexpr int BN = BN_, BK = BK_, STAGES = STAGES_;
  static constexpr int TA = BM * BK * 4;           // one A slab (bytes)
  static constexpr int TB = BN * BK * 4;           // one B slab
  static constexpr int STAGE = 2 * TA + 2 * TB;    // A_hi, A_lo, B_hi, B_lo
  static constexpr int SMEM = STAGES * STAGE + 1024 + sizeof(Ctl<STAGES>) + 64;
  static constexpr uint32_t K_LAYOUT = BK * 4 == 128 ? 2 : 4;  // SW128 / SW64
  static constexpr int K_TMAP = BK * 4 == 128 ? TMAP_SW128 : TMAP_SW64;
  static constexpr uint32_t K_SBO = 8 * BK * 4;    // 8-row group
  static constexpr uint32_t MN_CHUNK = BK * 128;   // one 32-wide MN chunk
  static_assert(BK * 4 == 128 || BK * 4 == 64, "k-slab rows of 64 or 128 bytes");
  static_assert(BN == 128 || BN == 256, "tile width");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};
using Narrow = Cfg<128, 32, 3>;
using Wide = Cfg<256, 16, 4>;

// First column tile on or right of the diagonal for row tile bi.
template <class C>
__host__ __device__ constexpr int64_t upper_first(int64_t bi) {
  return bi * BM / C::BN;
}

struct GemmP {
  int64_t M, N, K;
  float *C;
  int64_t ldc;
  float alpha, beta;
  uint32_t kflags;
  int a_mn, b_mn, upper_only, tiles_m, tiles_n, vec_ok;
  int32_t *info;
};

template <class C>
__global__ void __launch_bounds__(NTHREADS, 1)
    gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, const GemmP p) {
  constexpr int BN = C::BN, BK = C::BK, STAGES = C::STAGES;
  constexpr int TA = C::TA, TB = C::TB;
  const int64_t M = p.M, N = p.N, K = p.K;
  const int a_mn = p.a_mn, b_mn = p.b_mn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl<STAGES> *ctl = reinterpret_cast<Ctl<STAGES> *>(smem + STAGES * C::STAGE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = p.tiles_n, tiles_m = p.tiles_m;
  const uint32_t kflags = p.kflags;

  // ---- tile coordinates
  int64_t bi, bj;
  {
    int64_t t = blockIdx.x;
    if (p.upper_only) {
      bi = 0;
      while (t >= tiles_n - upper_first<C>(bi)) {
        t -= tiles_n - upper_first<C>(bi);
        ++bi;
      }
      bj = upper_first<C>(bi) + t;
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
    tmem_alloc(&ctl->tmem_base, BN);
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
        uint8_t *st = smem + s * C::STAGE;
        const int32_t k0 = static_cast<int32_t>(kb + int64_t(it) * BK);
        mbar_expect_tx(&ctl->full[s], TA + TB);
        if (!a_mn) {
          tma_load_2d(st, &tmA, &ctl->full[s], k0, static_cast<int32_t>(m0));
        } else {
          for (int c = 0; c < BM / 32; ++c)
            tma_load_2d(st + c * C::MN_CHUNK, &tmA, &ctl->full[s],
                        static_cast<int32_t>(m0 + 32 * c), k0);
        }
        uint8_t *sb = st + 2 * TA;
        if (!b_mn) {
          tma_load_2d(sb, &tmB, &ctl->full[s], k0, static_cast<int32_t>(n0));
        } else {
          for (int c = 0; c < BN / 32; ++c)
            tma_load_2d(sb + c * C::MN_CHUNK, &tmB, &ctl->full[s],
                        static_cast<int32_t>(n0 + 32 * c), k0);
        }
        issued = it + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_make(2, a_mn, b_mn, BM, BN);
      // K-major: 8-row groups of BK-float rows (16-byte swizzle granules);
      // MN-major tf32: 4-row groups, 32-byte granules (layout type 1)
      const uint32_t lbo_a = a_mn ? C::MN_CHUNK : 16;
      const uint32_t lbo_b = b_mn ? C::MN_CHUNK : 16;
      const uint32_t sbo_a = a_mn ? 512 : C::K_SBO, sbo_b = b_mn ? 512 : C::K_SBO;
      const uint32_t lay_a = a_mn ? 1 : C::K_LAYOUT, lay_b = b_mn ? 1 : C::K_LAYOUT;
      int it = 0;
      for (; it < nk; ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(&ctl->conv[s], (it / STAGES) & 1, abort)) break;
        tc_fence_after();
        const uint32_t a_hi = smem_u32(smem + s * C::STAGE);
        const uint32_t a_lo = a_hi + TA;
        const uint32_t b_hi = a_hi + 2 * TA;
        const uint32_t b_lo = b_hi + TB;
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
      float4 *sa = reinterpret_cast<float4 *>(smem + s * C::STAGE);
      float4 *sb = sa + 2 * (TA / 16);
      // all loads first: the slabs and their low parts share one array
      float4 ra[TA / 16 / 128], rb[TB / 16 / 128];
#pragma unroll
      for (int j = 0; j < TA / 16 / 128; ++j) ra[j] = sa[ct + 128 * j];
#pragma unroll
      for (int j = 0; j < TB / 16 / 128; ++j) rb[j] = sb[ct + 128 * j];
#pragma unroll
      for (int j = 0; j < TA / 16 / 128; ++j) sa[TA / 16 + ct + 128 * j] = tf32_lo(ra[j]);
#pragma unroll
      for (int j = 0; j < TB / 16 / 128; ++j) sb[TB / 16 + ct + 128 * j] = tf32_lo(rb[j]);
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
      const int64_t col0 = n0 + 32 * c;
      if (col0 >= N) break;
      float v[32];
      if (have) {
        tmem_ld32(tbase + (static_cast<uint32_t>(32 * q) << 16) + 32 * c, v);
      } else {
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = 0.f;
      }
      if (row >= M) continue;
      float *crow = p.C + row * p.ldc + col0;
      if (p.vec_ok && col0 + 32 <= N) {
#pragma unroll
        for (int t = 0; t < 32; t += 4) {
          float4 o = make_float4(p.alpha * v[t], p.alpha * v[t + 1],
                                 p.alpha * v[t + 2], p.alpha * v[t + 3]);
          if (p.beta != 0.f) {
            const float4 old = *reinterpret_cast<const float4 *>(crow + t);
            o.x += p.beta * old.x;
            o.y += p.beta * old.y;
            o.z += p.beta * old.z;
            o.w += p.beta * old.w;
          }
          *reinterpret_cast<float4 *>(crow + t) = o;
        }
      } else {
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          if (col0 + t < N) {
            float o = p.alpha * v[t];
            if (p.beta != 0.f) o += p.beta * crow[t];
            crow[t] = o;
          }
        }
      }
    }
  }

  // ---- teardown: after an abort make sure no copy or MMA is still in flight
  tc_fence_before();
  __syncthreads();
  if (ctl->abort) {
    if (threadIdx.x == 0) report(p.info, KRONQ_ERR_TIMEOUT);
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
    tmem_dealloc(tbase, BN);
  }
}

template <class C>
kronq_status launch(cudaStream_t st, const GemmArgs &g, int32_t *info) {
  CUtensorMap ta, tb;
  // A: K-major -> rows M of K; MN-major -> rows K of M (32-wide chunks)
  if (g.K > 0) {
    KQ_TRY(g.a_mn ? make_tmap_2d(&ta, g.A, false, g.M, g.K, g.lda, 32, C::BK, TMAP_SW128_32B)
                  : make_tmap_2d(&ta, g.A, false, g.K, g.M, g.lda, C::BK, BM, C::K_TMAP));
    KQ_TRY(g.b_mn ? make_tmap_2d(&tb, g.B, false, g.N, g.K, g.ldb, 32, C::BK, TMAP_SW128_32B)
                  : make_tmap_2d(&tb, g.B, false, g.K, g.N, g.ldb, C::BK, C::BN, C::K_TMAP));
  } else {
    memset(&ta, 0, sizeof(ta));
    memset(&tb, 0, sizeof(tb));
  }
  const int64_t tm = ceil_div(g.M, BM), tn = ceil_div(g.N, C::BN);
  int64_t tiles = tm * tn;
  if (g.upper_tiles_only) {
    tiles = 0;
    for (int64_t bi = 0; bi < tm; ++bi) tiles += tn - upper_first<C>(bi);
  }
  if (tiles > 0x7fffffff) return KRONQ_ERR_UNSUPPORTED;
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(gemm_tf32x3_kernel<C>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    attr_done = true;
  }
  GemmP p;
  p.M = g.M; p.N = g.N; p.K = g.K;
  p.C = g.C; p.ldc = g.ldc;
  p.alpha = g.alpha; p.beta = g.beta;
  p.kflags = g.kflags;
  p.a_mn = g.a_mn ? 1 : 0;
  p.b_mn = g.b_mn ? 1 : 0;
  p.upper_only = g.upper_tiles_only ? 1 : 0;
  p.tiles_m = static_cast<int>(tm);
  p.tiles_n = static_cast<int>(tn);
  p.vec_ok = (reinterpret_cast<uintptr_t>(g.C) % 16 == 0) && (g.ldc % 4 == 0);
  p.info = info;
  gemm_tf32x3_kernel<C><<<static_cast<unsigned>(tiles), NTHREADS, C::SMEM, st>>>(
      ta, tb, p);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

}  // namespace

kronq_status gemm_tf32x3(cudaStream_t st, const GemmArgs &g, int32_t *info) {
  if (g.M < 0 || g.N < 0 || g.K < 0) return KRONQ_ERR_INVALID_ARG;
  if (g.M == 0 || g.N == 0) return KRONQ_OK;
  if (g.upper_tiles_only && g.M != g.N) return KRONQ_ERR_INVALID_ARG;
  // wide tiles when they fill the GPU at least once and waste at most an
  // eighth of the last column tile's width
  const int64_t wide_tiles = ceil_div(g.M, BM) * ceil_div(g.N, Wide::BN);
  const int64_t pad = ceil_div(g.N, Wide::BN) * Wide::BN - g.N;
  if (wide_tiles >= 148 && pad * 8 <= ceil_div(g.N, Wide::BN) * Wide::BN)
    return launch<Wide>(st, g, info);
  return launch<Narrow>(st, g, info);
}

}  // namespace kronq

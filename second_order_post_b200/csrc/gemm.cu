// fp32-accurate GEMM on the sm_100a tensor cores: C = beta*C + alpha*A*B^T,
// each fp32 operand split into a high and a low part and three tcgen05 MMAs
// (hi*hi + hi*lo + lo*hi) per k-step into an fp32 TMEM accumulator. Used by
// the blocked Cholesky/inverse, the OBS trailing updates and the layer loss.
//
// Two splits share one kernel template:
//   TF32   the raw fp32 slab is the high part (the MMA drops its 13 low
//          mantissa bits); split warps write the low part next to each landed
//          slab. Works on K- and MN-major operands in place; per product it
//          keeps all but 1.5 * 2^-20 |a b|.
//   FP16   a split pass writes each operand as two K-major fp16 planes,
//          x * s = hi + lo (+ rest), with s a power of two per operand row
//          that puts the row's largest magnitude in [2^14, 2^15); the kernel
//          only loads and multiplies, and the epilogue divides the scales out.
//          Per product it keeps all but about 3 * 2^-22 |a b|. An fp16 MMA
//          costs well under half the energy of a TF32 one, and under the
//          1 kW cap the GEMM is power-bound, so this path runs about twice as
//          fast; it needs scratch for the planes and a split launch or two,
//          so the large products take it and the small ones stay on TF32.
// One CTA computes a 128 x BN tile (BN = 256 for wide outputs, 128 otherwise):
//   warp 0      TMA producer (one elected lane), ring of BK-wide k-slabs
//   warp 1      TMEM owner and MMA issuer (one elected lane)
//   warps 2..5  (TF32) the split of each landed slab: a whole slab is loaded
//               into registers before any low part is stored, since both
//               share one array; then the epilogue (TMEM -> registers -> C).
#include <cuda_fp16.h>

#include "kernels.cuh"

namespace kronq {
namespace {

constexpr int BM = 128;
constexpr int NTHREADS = 192;
constexpr int GROUP_M = 16;                    // tile raster: 16 rows per band
constexpr int KCHUNK = 8192;                   // k per main-accumulator chunk

template <int STAGES>
struct Ctl {
  uint64_t full[STAGES];   // TMA landed (expect_tx)
  uint64_t conv[STAGES];   // hi/lo split written (128 arrivals)
  uint64_t empty[STAGES];  // MMAs that read the stage finished (commit)
  uint64_t done;           // all MMAs finished (commit)
  uint64_t chunk_done;     // hi*hi MMAs of a k-chunk finished (commit)
  uint64_t folded;         // epilogue warps read the main accumulator (128)
  uint64_t drain;          // teardown drain after an abort
  uint32_t tmem_base;
  int abort;
};

// Tile configuration: BN output columns, BK-wide k-slabs, STAGES-deep ring,
// fp16 pieces (F16) or fp32 slabs. K-major slabs are rows of BK elements
// (128 or 64 bytes, swizzled to match); MN-major slabs (TF32 only) are 32-wide
// MN chunks of BK k-rows (32-byte granules).
template <int BN_, int BK_, int STAGES_, bool F16_>
struct Cfg {
  static constexpr int BN = BN_, BK = BK_, STAGES = STAGES_;
  static constexpr bool F16 = F16_;
  static constexpr int ES = F16 ? 2 : 4;           // bytes per element in smem
  static constexpr int TA = BM * BK * ES;          // one A slab (bytes)
  static constexpr int TB = BN * BK * ES;          // one B slab
  static constexpr int STAGE = 2 * TA + 2 * TB;    // A_hi, A_lo, B_hi, B_lo
  static constexpr int SMEM = STAGES * STAGE + 1024 + sizeof(Ctl<STAGES>) + 64;
  static constexpr uint32_t K_LAYOUT = BK * ES == 128 ? 2 : 4;  // SW128 / SW64
  static constexpr int K_TMAP = BK * ES == 128 ? TMAP_SW128 : TMAP_SW64;
  static constexpr uint32_t K_SBO = 8 * BK * ES;   // 8-row group
  static constexpr uint32_t MN_CHUNK = BK * 128;   // one 32-wide MN chunk
  static constexpr int KSTEP = F16 ? 16 : 8;       // K of one MMA (32 bytes)
  static constexpr int CH = KCHUNK / BK;           // stages per k-chunk
  static_assert(BK * ES == 128 || BK * ES == 64, "k-slab rows of 64 or 128 bytes");
  static_assert(BN == 128 || BN == 256, "tile width");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};
using Narrow = Cfg<128, 32, 3, false>;
using Wide = Cfg<256, 16, 4, false>;
using WideH = Cfg<256, 32, 4, true>;

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
  const float *inv_sa, *inv_sb;  // F16: 1 / row scale of A and of B
  int32_t *info;
};

template <class C>
__global__ void __launch_bounds__(NTHREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmAl,
                const __grid_constant__ CUtensorMap tmBl, const GemmP p) {
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
    mbar_init(&ctl->chunk_done, 1);
    mbar_init(&ctl->folded, 128);
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (C::F16) {
      prefetch_tmap(&tmAl);
      prefetch_tmap(&tmBl);
    }
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, 2 * BN);
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
        mbar_expect_tx(&ctl->full[s], C::F16 ? 2 * (TA + TB) : TA + TB);
        if (C::F16) {  // four K-major fp16 planes
          tma_load_2d(st, &tmA, &ctl->full[s], k0, static_cast<int32_t>(m0));
          tma_load_2d(st + TA, &tmAl, &ctl->full[s], k0, static_cast<int32_t>(m0));
          tma_load_2d(st + 2 * TA, &tmB, &ctl->full[s], k0, static_cast<int32_t>(n0));
          tma_load_2d(st + 2 * TA + TB, &tmBl, &ctl->full[s], k0,
                      static_cast<int32_t>(n0));
          issued = it + 1;
          continue;
        }
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
      const uint32_t idesc = idesc_make(C::F16 ? 0 : 2, a_mn, b_mn, BM, BN);
      // K-major: 8-row groups of BK-float rows (16-byte swizzle granules);
      // MN-major tf32: 4-row groups, 32-byte granules (layout type 1)
      const uint32_t lbo_a = a_mn ? C::MN_CHUNK : 16;
      const uint32_t lbo_b = b_mn ? C::MN_CHUNK : 16;
      const uint32_t sbo_a = a_mn ? 512 : C::K_SBO, sbo_b = b_mn ? 512 : C::K_SBO;
      const uint32_t lay_a = a_mn ? 1 : C::K_LAYOUT, lay_b = b_mn ? 1 : C::K_LAYOUT;
      // hi*hi into the main accumulator (columns [0, BN)), restarted every
      // k-chunk after the epilogue warps folded it into C; the two cross
      // terms into a second accumulator (columns [BN, 2 BN)) that runs over
      // all of K (its one-way rounding drift is relative to a value ~2^-11
      // the size of the main one)
      for (int it = 0; it < nk; ++it) {
        const int s = it % STAGES;
        const int ci = it / C::CH, first = it % C::CH == 0;
        if (first && ci > 0 && !mbar_wait(&ctl->folded, (ci - 1) & 1, abort)) break;
        if (!mbar_wait(C::F16 ? &ctl->full[s] : &ctl->conv[s], (it / STAGES) & 1, abort))
          break;
        tc_fence_after();
        const uint32_t a_hi = smem_u32(smem + s * C::STAGE);
        const uint32_t a_lo = a_hi + TA;
        const uint32_t b_hi = a_hi + 2 * TA;
        const uint32_t b_lo = b_hi + TB;
#pragma unroll
        for (int kk = 0; kk < BK / C::KSTEP; ++kk) {
          const uint32_t ao = a_mn ? kk * 1024 : kk * 32;
          const uint32_t bo = b_mn ? kk * 1024 : kk * 32;
          const uint64_t dah = sdesc(a_hi + ao, lbo_a, sbo_a, lay_a);
          const uint64_t dal = sdesc(a_lo + ao, lbo_a, sbo_a, lay_a);
          const uint64_t dbh = sdesc(b_hi + bo, lbo_b, sbo_b, lay_b);
          const uint64_t dbl = sdesc(b_lo + bo, lbo_b, sbo_b, lay_b);
          const uint32_t cross = (it | kk) != 0, main = !(first && kk == 0);
          if (C::F16) {
            umma_bf16(tbase + BN, dal, dbh, idesc, cross);
            umma_bf16(tbase + BN, dah, dbl, idesc, 1);
            umma_bf16(tbase, dah, dbh, idesc, main);
          } else {
            umma_tf32(tbase + BN, dal, dbh, idesc, cross);
            umma_tf32(tbase + BN, dah, dbl, idesc, 1);
            umma_tf32(tbase, dah, dbh, idesc, main);
          }
        }
        umma_commit(&ctl->empty[s]);
        if (it % C::CH == C::CH - 1 && it != nk - 1) umma_commit(&ctl->chunk_done);
      }
      if (nk > 0)
        umma_commit(&ctl->done);
      else
        mbar_arrive(&ctl->done);
    }
  } else {
    const int ct = threadIdx.x - 64;
    const int q = warp & 3;
    const int64_t row = m0 + 32 * q + lane;
    int folds = 0;
    // C (+)= the main accumulator (and, at the end, the cross terms): the first
    // write applies beta to the old C, later ones add to what is there
    auto fold = [&](bool final) -> bool {
      const bool ok = mbar_wait(final ? &ctl->done : &ctl->chunk_done,
                                final ? 0u : static_cast<uint32_t>(folds & 1), abort);
      if (!__all_sync(0xffffffffu, ok)) return false;
      tc_fence_after();
      for (int c = 0; c < BN / 32; ++c) {
        const int64_t col0 = n0 + 32 * c;
        if (col0 >= N) break;
        float v[32];
        if (nk > 0) {
          const uint32_t ta = tbase + (static_cast<uint32_t>(32 * q) << 16) + 32 * c;
          tmem_ld32(ta, v);
          if (final) {
            float u[32];
            tmem_ld32(ta + BN, u);
#pragma unroll
            for (int t = 0; t < 32; ++t) v[t] += u[t];
          }
        } else {
#pragma unroll
          for (int t = 0; t < 32; ++t) v[t] = 0.f;
        }
        if (row >= M) continue;
        if (C::F16) {  // divide the operand row scales out
          const float ra = p.alpha * p.inv_sa[row];
#pragma unroll
          for (int t = 0; t < 32; ++t)
            v[t] *= ra * (col0 + t < N ? p.inv_sb[col0 + t] : 0.f);
        } else {
#pragma unroll
          for (int t = 0; t < 32; ++t) v[t] *= p.alpha;
        }
        float *crow = p.C + row * p.ldc + col0;
        const bool fresh = folds == 0, keep = !fresh || p.beta != 0.f;
        const float bw = fresh ? p.beta : 1.f;
        if (p.vec_ok && col0 + 32 <= N) {
          float4 old[8];  // all loads before any store
          if (keep) {
#pragma unroll
            for (int t = 0; t < 8; ++t) old[t] = __ldcg(reinterpret_cast<const float4 *>(crow) + t);
          } else {
#pragma unroll
            for (int t = 0; t < 8; ++t) old[t] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const float4 o = make_float4(fmaf(bw, old[t].x, v[4 * t]),
                                         fmaf(bw, old[t].y, v[4 * t + 1]),
                                         fmaf(bw, old[t].z, v[4 * t + 2]),
                                         fmaf(bw, old[t].w, v[4 * t + 3]));
            reinterpret_cast<float4 *>(crow)[t] = o;
          }
        } else {
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            if (col0 + t < N) {
              float o = v[t];
              if (keep) o += bw * crow[t];
              crow[t] = o;
            }
          }
        }
      }
      tc_fence_before();
      if (!final) mbar_arrive(&ctl->folded);
      ++folds;
      return true;
    };
    bool alive = true;
    if (!C::F16) {
      // ---- hi/lo split of every landed slab, folding each finished chunk
      for (int it = 0; it < nk; ++it) {
        if (it > 0 && it % C::CH == 0 && !fold(false)) {
          alive = false;
          break;
        }
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
    } else {
      const int nchunks = nk > 0 ? (nk + C::CH - 1) / C::CH : 0;
      for (int c = 0; c + 1 < nchunks && alive; ++c) alive = fold(false);
    }
    if (alive) fold(true);
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
    tmem_dealloc(tbase, 2 * BN);
  }
}

// fp16 planes of one operand for the F16 path: x[r][k] * s_r ~ hi + lo
struct Planes {
  const __half *hi, *lo;  // [rows][ldp], K-major
  int64_t ldp;
  const float *inv;       // [rows] 1 / s_r
};

template <class C>
kronq_status launch(cudaStream_t st, const GemmArgs &g, int32_t *info,
                    const Planes *pa = nullptr, const Planes *pb = nullptr) {
  CUtensorMap ta, tb, tal, tbl;
  memset(&ta, 0, sizeof(ta));
  memset(&tb, 0, sizeof(tb));
  memset(&tal, 0, sizeof(tal));
  memset(&tbl, 0, sizeof(tbl));
  if (g.K > 0 && C::F16) {
    // 16-bit elements (the map's element type only sets size and fill)
    KQ_TRY(make_tmap_2d(&ta, pa->hi, true, g.K, g.M, pa->ldp, C::BK, BM, C::K_TMAP));
    KQ_TRY(make_tmap_2d(&tal, pa->lo, true, g.K, g.M, pa->ldp, C::BK, BM, C::K_TMAP));
    KQ_TRY(make_tmap_2d(&tb, pb->hi, true, g.K, g.N, pb->ldp, C::BK, C::BN, C::K_TMAP));
    KQ_TRY(make_tmap_2d(&tbl, pb->lo, true, g.K, g.N, pb->ldp, C::BK, C::BN, C::K_TMAP));
  } else if (g.K > 0) {
    // A: K-major -> rows M of K; MN-major -> rows K of M (32-wide chunks)
    KQ_TRY(g.a_mn ? make_tmap_2d(&ta, g.A, false, g.M, g.K, g.lda, 32, C::BK, TMAP_SW128_32B)
                  : make_tmap_2d(&ta, g.A, false, g.K, g.M, g.lda, C::BK, BM, C::K_TMAP));
    KQ_TRY(g.b_mn ? make_tmap_2d(&tb, g.B, false, g.N, g.K, g.ldb, 32, C::BK, TMAP_SW128_32B)
                  : make_tmap_2d(&tb, g.B, false, g.K, g.N, g.ldb, C::BK, C::BN, C::K_TMAP));
  }
  const int64_t tm = ceil_div(g.M, BM), tn = ceil_div(g.N, C::BN);
  int64_t tiles = tm * tn;
  if (g.upper_tiles_only) {
    tiles = 0;
    for (int64_t bi = 0; bi < tm; ++bi) tiles += tn - upper_first<C>(bi);
  }
  if (tiles > 0x7fffffff) return KRONQ_ERR_UNSUPPORTED;
  KQ_TRY(smem_attr(gemm_kernel<C>, C::SMEM));
  GemmP p;
  p.M = g.M; p.N = g.N; p.K = g.K;
  p.C = g.C; p.ldc = g.ldc;
  p.alpha = g.alpha; p.beta = g.beta;
  p.kflags = g.kflags;
  p.a_mn = C::F16 ? 0 : (g.a_mn ? 1 : 0);
  p.b_mn = C::F16 ? 0 : (g.b_mn ? 1 : 0);
  p.upper_only = g.upper_tiles_only ? 1 : 0;
  p.tiles_m = static_cast<int>(tm);
  p.tiles_n = static_cast<int>(tn);
  p.vec_ok = (reinterpret_cast<uintptr_t>(g.C) % 16 == 0) && (g.ldc % 4 == 0);
  p.inv_sa = pa ? pa->inv : nullptr;
  p.inv_sb = pb ? pb->inv : nullptr;
  p.info = info;
  gemm_kernel<C><<<static_cast<unsigned>(tiles), NTHREADS, C::SMEM, st>>>(ta, tb, tal, tbl, p);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

// ---------------------------------------------------------------- F16 split
// Power of two that puts magnitude m in [2^14, 2^15) (1 for m = 0, inf, nan).
__device__ __forceinline__ float row_scale(float m) {
  if (!(m > 0.f) || !isfinite(m)) return 1.f;
  int e;
  frexpf(m, &e);                      // m = f 2^e, f in [0.5, 1)
  return ldexpf(1.f, kq_min(15 - e, 125));
}

__device__ __forceinline__ void split2(float v, __half &h, __half &l) {
  h = __float2half_rn(v);
  l = __float2half_rn(v - __half2float(h));
}

__device__ __forceinline__ float block_max(float m, float *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (warp == 0) {
    m = lane < static_cast<int>(blockDim.x >> 5) ? red[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[32] = m;
  }
  __syncthreads();
  m = red[32];
  __syncthreads();
  return m;
}

// K-major source X[rows][K]: one CTA per row (grid-stride): the row's largest
// magnitude, then its scaled hi/lo planes.
__global__ void __launch_bounds__(256)
    split_rows_kernel(const float *__restrict__ X, int64_t ldx, int64_t rows, int64_t K,
                      __half *__restrict__ hi, __half *__restrict__ lo, int64_t ldp,
                      float *__restrict__ inv, int vec) {
  __shared__ float red[33];
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const float *xr = X + r * ldx;
    __half *hr = hi + r * ldp, *lr = lo + r * ldp;
    float m = 0.f;
    if (vec) {
      for (int64_t c = 4 * threadIdx.x; c < K; c += 4 * blockDim.x) {
        const float4 v = *reinterpret_cast<const float4 *>(xr + c);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
    } else {
      for (int64_t c = threadIdx.x; c < K; c += blockDim.x) m = fmaxf(m, fabsf(xr[c]));
    }
    const float s = row_scale(block_max(m, red));
    if (threadIdx.x == 0) inv[r] = 1.f / s;
    if (vec) {
      for (int64_t c = 4 * threadIdx.x; c < K; c += 4 * blockDim.x) {
        const float4 v = *reinterpret_cast<const float4 *>(xr + c);
        __align__(8) __half h[4], l[4];
        split2(v.x * s, h[0], l[0]);
        split2(v.y * s, h[1], l[1]);
        split2(v.z * s, h[2], l[2]);
        split2(v.w * s, h[3], l[3]);
        *reinterpret_cast<uint2 *>(hr + c) = *reinterpret_cast<const uint2 *>(h);
        *reinterpret_cast<uint2 *>(lr + c) = *reinterpret_cast<const uint2 *>(l);
      }
    } else {
      for (int64_t c = threadIdx.x; c < K; c += blockDim.x) split2(xr[c] * s, hr[c], lr[c]);
    }
  }
}

// MN-major source X[K][cols] (operand row j = column j): column maxima as
// float bit patterns (non-negative floats order like unsigned integers).
__global__ void colmax_kernel(const float *__restrict__ X, int64_t ldx, int64_t K,
                              int64_t cols, int64_t kchunk, unsigned *__restrict__ maxbits) {
  const int64_t j = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (j >= cols) return;
  const int64_t k1 = kq_min<int64_t>(K, (blockIdx.y + 1) * kchunk);
  float m = 0.f;
  for (int64_t k = blockIdx.y * kchunk; k < k1; ++k) m = fmaxf(m, fabsf(X[k * ldx + j]));
  atomicMax(maxbits + j, __float_as_uint(m));
}

// ... then 32 x 32 tiles transposed through shared memory into the planes.
__global__ void __launch_bounds__(256)
    split_cols_kernel(const float *__restrict__ X, int64_t ldx, int64_t K, int64_t cols,
                      const unsigned *__restrict__ maxbits, __half *__restrict__ hi,
                      __half *__restrict__ lo, int64_t ldp, float *__restrict__ inv) {
  __shared__ float tile[32][33];
  __shared__ float sc[32];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t j0 = blockIdx.x * 32, k0 = blockIdx.y * 32;
  if (ty == 0) {
    const int64_t j = j0 + tx;
    const float s = j < cols ? row_scale(__uint_as_float(maxbits[j])) : 1.f;
    sc[tx] = s;
    if (blockIdx.y == 0 && j < cols) inv[j] = 1.f / s;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t k = k0 + ty + 8 * i, j = j0 + tx;
    tile[ty + 8 * i][tx] = (k < K && j < cols) ? X[k * ldx + j] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t j = j0 + ty + 8 * i, k = k0 + tx;
    if (j < cols && k < K)
      split2(tile[tx][ty + 8 * i] * sc[ty + 8 * i], hi[j * ldp + k], lo[j * ldp + k]);
  }
}

constexpr int64_t kF16MinWork = int64_t(1) << 33;  // M*N*K below which TF32 stays

size_t al256(size_t b) { return (b + 255) / 256 * 256; }
int64_t plane_pitch(int64_t K) { return (K + 7) / 8 * 8; }
size_t planes_bytes(int64_t rows, int64_t K) {
  return 2 * al256(static_cast<size_t>(rows) * plane_pitch(K) * 2) +
         al256(static_cast<size_t>(rows) * 4) + al256(static_cast<size_t>(rows) * 4);
}

// Splits one operand (rows of length K, K-major or stored transposed) into
// planes carved from `w`.
kronq_status split_operand(cudaStream_t st, const float *X, int64_t ld, bool mn,
                           int64_t rows, int64_t K, uint8_t *w, Planes *out) {
  const int64_t ldp = plane_pitch(K);
  __half *hi = reinterpret_cast<__half *>(w);
  w += al256(static_cast<size_t>(rows) * ldp * 2);
  __half *lo = reinterpret_cast<__half *>(w);
  w += al256(static_cast<size_t>(rows) * ldp * 2);
  float *inv = reinterpret_cast<float *>(w);
  w += al256(static_cast<size_t>(rows) * 4);
  unsigned *maxbits = reinterpret_cast<unsigned *>(w);
  if (!mn) {
    const int vec = reinterpret_cast<uintptr_t>(X) % 16 == 0 && ld % 4 == 0 && K % 4 == 0;
    split_rows_kernel<<<static_cast<unsigned>(kq_min<int64_t>(rows, 148 * 16)), 256, 0, st>>>(
        X, ld, rows, K, hi, lo, ldp, inv, vec);
    KQ_CHECK_LAUNCH();
  } else {
    KQ_CUDA(cudaMemsetAsync(maxbits, 0, static_cast<size_t>(rows) * 4, st));
    const int64_t kchunk = 256;
    dim3 gm(static_cast<unsigned>(ceil_div(rows, 256)),
            static_cast<unsigned>(ceil_div(K, kchunk)));
    colmax_kernel<<<gm, 256, 0, st>>>(X, ld, K, rows, kchunk, maxbits);
    KQ_CHECK_LAUNCH();
    dim3 gs(static_cast<unsigned>(ceil_div(rows, 32)), static_cast<unsigned>(ceil_div(K, 32)));
    split_cols_kernel<<<gs, 256, 0, st>>>(X, ld, K, rows, maxbits, hi, lo, ldp, inv);
    KQ_CHECK_LAUNCH();
  }
  out->hi = hi;
  out->lo = lo;
  out->ldp = ldp;
  out->inv = inv;
  return KRONQ_OK;
}

bool wide_ok(const GemmArgs &g) {
  // wide tiles when they fill the GPU at least once and waste at most an
  // eighth of the last column tile's width
  const int64_t wide_tiles = ceil_div(g.M, BM) * ceil_div(g.N, Wide::BN);
  const int64_t pad = ceil_div(g.N, Wide::BN) * Wide::BN - g.N;
  return wide_tiles >= 148 && pad * 8 <= ceil_div(g.N, Wide::BN) * Wide::BN;
}

bool same_operand(const GemmArgs &g) {
  return g.A == g.B && g.a_mn == g.b_mn && g.lda == g.ldb && g.M == g.N;
}

// ------------------------------------------------------------- small products
// The small products at the bottom of the Cholesky recursion (128 .. 256 on a
// side) sit one after another on its critical path, where a tensor-core
// launch costs its pipeline fill and TMEM set-up for a few k-steps of work.
// These run on the CUDA cores instead: plain fp32 FMA (exact products), one
// 32 x 32 tile of C per CTA, the tile's A and B panels staged in shared
// memory KC columns of k at a time with every load of a stage in flight at
// once. The zero blocks of triangular operands are skipped like the tensor
// kernel does, at this tile's granularity.
constexpr int ST = 32;                 // tile edge
constexpr int SKC = 128;               // k per shared-memory stage
constexpr int STHREADS = 256;          // 16 x 16 threads, 2 x 2 outputs each
constexpr int64_t kSmallMaxWork = int64_t(1) << 24;  // M*N*K at most (256^3)

__global__ void __launch_bounds__(STHREADS)
    small_gemm_kernel(GemmArgs g, int tiles_n) {
  __shared__ __align__(16) float As[SKC][ST + 2];  // As[k][i]
  __shared__ __align__(16) float Bs[SKC][ST + 2];  // Bs[k][j]
  const int bm = blockIdx.x / tiles_n, bn = blockIdx.x % tiles_n;
  if (g.upper_tiles_only && bm > bn) return;
  const int64_t m0 = int64_t(bm) * ST, n0 = int64_t(bn) * ST;
  int64_t kb = 0, ke = g.K;
  if (g.kflags & KR_A_UPPER) kb = kq_max(kb, m0);
  if (g.kflags & KR_B_UPPER) kb = kq_max(kb, n0);
  if (g.kflags & KR_B_LOWER) ke = kq_min(ke, n0 + ST);
  const int t = threadIdx.x, tx = t % 16, ty = t / 16;
  float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  for (int64_t k0 = kb; k0 < ke; k0 += SKC) {
    const int kc = static_cast<int>(kq_min<int64_t>(SKC, ke - k0));
    // stage: element e of the 32 x SKC panel; K-major operands are read along
    // k (consecutive threads, consecutive k), MN-major ones along i / j
    float va[ST * SKC / STHREADS], vb[ST * SKC / STHREADS];
#pragma unroll
    for (int u = 0; u < ST * SKC / STHREADS; ++u) {
      const int e = t + u * STHREADS;
      int i, kk;
      if (g.a_mn) { kk = e / ST; i = e % ST; } else { i = e / SKC; kk = e % SKC; }
      const int64_t gi = m0 + i, gk = k0 + kk;
      va[u] = (gi < g.M && kk < kc)
                  ? (g.a_mn ? g.A[gk * g.lda + gi] : g.A[gi * g.lda + gk])
                  : 0.f;
      int j, kj;
      if (g.b_mn) { kj = e / ST; j = e % ST; } else { j = e / SKC; kj = e % SKC; }
      const int64_t gj = n0 + j, gkb = k0 + kj;
      vb[u] = (gj < g.N && kj < kc)
                  ? (g.b_mn ? g.B[gkb * g.ldb + gj] : g.B[gj * g.ldb + gkb])
                  : 0.f;
    }
    __syncthreads();  // the previous stage's readers are done
#pragma unroll
    for (int u = 0; u < ST * SKC / STHREADS; ++u) {
      const int e = t + u * STHREADS;
      if (g.a_mn) As[e / ST][e % ST] = va[u]; else As[e % SKC][e / SKC] = va[u];
      if (g.b_mn) Bs[e / ST][e % ST] = vb[u]; else Bs[e % SKC][e / SKC] = vb[u];
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kc; ++kk) {
      const float2 a = *reinterpret_cast<const float2 *>(&As[kk][2 * ty]);
      const float2 b = *reinterpret_cast<const float2 *>(&Bs[kk][2 * tx]);
      acc[0][0] = fmaf(a.x, b.x, acc[0][0]);
      acc[0][1] = fmaf(a.x, b.y, acc[0][1]);
      acc[1][0] = fmaf(a.y, b.x, acc[1][0]);
      acc[1][1] = fmaf(a.y, b.y, acc[1][1]);
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int64_t i = m0 + 2 * ty + r;
    if (i >= g.M) continue;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int64_t j = n0 + 2 * tx + c;
      if (j >= g.N) continue;
      float *cp = g.C + i * g.ldc + j;
      const float v = g.alpha * acc[r][c];
      *cp = g.beta != 0.f ? fmaf(g.beta, *cp, v) : v;
    }
  }
}

bool small_ok(const GemmArgs &g) { return g.M * g.N * g.K <= kSmallMaxWork; }

kronq_status launch_small(cudaStream_t st, const GemmArgs &g) {
  const int64_t tm = ceil_div(g.M, ST), tn = ceil_div(g.N, ST);
  if (tm * tn > 0x7fffffff) return KRONQ_ERR_UNSUPPORTED;
  small_gemm_kernel<<<static_cast<unsigned>(tm * tn), STHREADS, 0, st>>>(
      g, static_cast<int>(tn));
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

}  // namespace

kronq_status gemm_tf32x3(cudaStream_t st, const GemmArgs &g, int32_t *info) {
  if (g.M < 0 || g.N < 0 || g.K < 0) return KRONQ_ERR_INVALID_ARG;
  if (g.M == 0 || g.N == 0) return KRONQ_OK;
  if (g.upper_tiles_only && g.M != g.N) return KRONQ_ERR_INVALID_ARG;
  if (wide_ok(g)) return launch<Wide>(st, g, info);
  return launch<Narrow>(st, g, info);
}

size_t gemm_scratch_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return planes_bytes(M, K) + planes_bytes(N, K);
}

kronq_status gemm_f32(cudaStream_t st, const GemmArgs &g, void *scratch,
                      size_t scratch_bytes, int32_t *info) {
  if (g.M < 0 || g.N < 0 || g.K < 0) return KRONQ_ERR_INVALID_ARG;
  if (g.M == 0 || g.N == 0) return KRONQ_OK;
  if (g.upper_tiles_only && g.M != g.N) return KRONQ_ERR_INVALID_ARG;
  if (small_ok(g)) return launch_small(st, g);
  const bool f16 = scratch && g.K > 0 && wide_ok(g) && g.M * g.N * g.K >= kF16MinWork &&
                   scratch_bytes >= gemm_scratch_bytes(g.M, g.N, g.K);
  if (!f16) return gemm_tf32x3(st, g, info);
  uint8_t *w = static_cast<uint8_t *>(scratch);
  Planes pa, pb;
  KQ_TRY(split_operand(st, g.A, g.lda, g.a_mn, g.M, g.K, w, &pa));
  if (same_operand(g)) {
    pb = pa;
  } else {
    KQ_TRY(split_operand(st, g.B, g.ldb, g.b_mn, g.N, g.K, w + planes_bytes(g.M, g.K), &pb));
  }
  return launch<WideH>(st, g, info, &pa, &pb);
}

}  // namespace kronq

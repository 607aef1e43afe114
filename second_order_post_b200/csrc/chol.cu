// Damped inverse Cholesky factor for GPTQ-style OBS [wmrh §四: the per-column
// compensation uses H_X only; the column order needs U with
// Uᵀ U = (H + λI)^-1, U upper].
//
// Route: H + λI = R Rᵀ with R upper (Cholesky taken from the last column
// backwards), then U = R^-1. Both factors come out of one recursion on the
// 2x2 block split H = [[A, B], [Bᵀ, C]]:
//     U22 = inv_chol(C)             (recursive)
//     V   = B U22ᵀ                  (= R12)
//     A  <- A - V Vᵀ                (R11 R11ᵀ)
//     U11 = inv_chol(A)             (recursive)
//     U12 = -U11 (V U22)
// All off-diagonal work runs through gemm_f32, which skips the zero blocks of
// the triangular operands: fp16-split tcgen05 products for the large nodes,
// 3xTF32 for the mid-size ones, plain fp32 FMA on the CUDA cores for the
// smallest. 128x128 diagonal leaves are factored and inverted in registers by
// one CTA. λ = damp_rel * mean(diag H) is added by each leaf to its own
// diagonal (the updates never touch λ, so this equals damping H up front).
#include <mutex>

#include "kernels.cuh"

namespace kronq {
namespace {

constexpr int NB = 128;

__global__ void damping_kernel(const float *H, int64_t d, float damp_rel,
                               float *lambda, int32_t *info) {
  __shared__ double part[32];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < d; i += blockDim.x) s += H[i * d + i];
  s = warp_sum_d(s);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < blockDim.x / 32 ? part[threadIdx.x] : 0.0;
    v = warp_sum_d(v);
    if (threadIdx.x == 0) {
      const double mean = v / double(d);
      if (!isfinite(mean)) report(info, KRONQ_ERR_NONFINITE);
      *lambda = static_cast<float>(double(damp_rel) * mean);
    }
  }
}

// One diagonal leaf at rows/cols [off, off+NB): reads the upper triangle of the
// (already updated) block, adds λ, writes U (upper, zeros below).
//
// Factor and inverse come out of one sweep over the pivots jj = NB-1 .. 0.
// With H = Ŕ D Ŕᵀ (Ŕ unit upper, columns l_j above the diagonal),
// Ŕ = (I + l_{NB-1} e_{NB-1}ᵀ) ... (I + l_0 e_0ᵀ), so X = Ŕ^-1 is the product of
// (I - l_j e_jᵀ) taken from j = 0 on the left to j = NB-1 on the right; pivot jj
// contributes the left factor X <- (I - l_jj e_jjᵀ) X, a rank-1 update of the
// rows above jj, and row jj of X is final when pivot jj is taken. One array M
// holds the Schur complement left of the current column and X from it on, and
// pivot jj applies to every row i < jj and column k >= i
//     M[i][k] -= l[i] * b[k],  l[i] = M[i][jj] / p,
//     b[k] = M[k][jj] (k < jj),  p + 1 (k = jj),  M[jj][k] (k > jj),
// which is the Schur update left of jj, turns column jj into -l, and applies
// the left factor right of it. U = D^-1/2 X.
//
// Each thread keeps one 4x4 tile of the upper triangle in registers. Pivots
// are taken four at a time (the pivot block J = [j0, j0+4) is one tile), in
// two phases separated by barriers:
//   A. The owners of tile column J and tile row J have published them. Every
//      phase-A thread factors the 4x4 pivot block (redundantly, in registers),
//      then thread i < j0 replays the four pivots on row i of the column
//      panel and thread k >= j0+4 on column k of the row panel. Row i gives
//      l_q[i] and the value b_q[i] = M[i][j0+q] that pivot q reads in column
//      i; column k gives b_q[k] = M[j0+q][k], final once pivot q is reached.
//   B. Every other tile above the block row takes the four pivots as one
//      rank-4 update, M[i][k] -= sum_q l_q[i] b_q[k] (q = 3 .. 0, the order of
//      the one-pivot sweep); the panel owners take their final values back.
// Each phase-A chain is one row or column, so a block costs two barriers and
// no thread replays more than its own panel entry.
constexpr int TT = 4;                          // tile edge owned by a thread
constexpr int NT = NB / TT;                    // tile rows and columns
constexpr int NTILES = NT * (NT + 1) / 2;      // upper tiles (I <= K)
constexpr int LTHREADS = (NTILES + 31) / 32 * 32;
static_assert(LTHREADS >= 2 * NB, "phase A needs a thread per panel row and column");

__global__ void __launch_bounds__(LTHREADS)
    chol_leaf_kernel(float *__restrict__ H, int64_t ld, int64_t off,
                     const float *__restrict__ lambda, int32_t *info) {
  __shared__ __align__(16) float colbuf[2][NB][TT];  // M[i][J], rows i < j0+4
  __shared__ __align__(16) float rowbuf[2][TT][NB];  // M[J][k]
  __shared__ __align__(16) float Ls[NB][TT];         // l_q[i], rows i < j0
  __shared__ __align__(16) float Bs[TT][NB];         // b_q[k], k outside J
  __shared__ __align__(16) float blkf[TT][TT];       // the pivot block, factored
  __shared__ float piv[NB];
  const int t = threadIdx.x;
  const bool own = t < NTILES;
  int I = NT, K = NT;  // tile of this thread, row-major over the upper tiles
  if (own) {
    int r = t;
    I = 0;
    while (r >= NT - I) {
      r -= NT - I;
      ++I;
    }
    K = I + r;
  }
  const int r0 = TT * I, c0 = TT * K;
  float m[TT][TT];
  if (own) {
    const float lam = *lambda;
#pragma unroll
    for (int ii = 0; ii < TT; ++ii) {
      const float4 v =
          *reinterpret_cast<const float4 *>(H + (off + r0 + ii) * ld + off + c0);
      m[ii][0] = v.x; m[ii][1] = v.y; m[ii][2] = v.z; m[ii][3] = v.w;
      if (I == K) {
#pragma unroll
        for (int kk = 0; kk < TT; ++kk) {
          if (kk < ii) m[ii][kk] = 0.f;
          if (kk == ii) m[ii][kk] += lam;
        }
      }
    }
  }
  auto publish = [&](int Tj) {
    if (K == Tj) {
#pragma unroll
      for (int ii = 0; ii < TT; ++ii)
        *reinterpret_cast<float4 *>(&colbuf[Tj & 1][r0 + ii][0]) =
            make_float4(m[ii][0], m[ii][1], m[ii][2], m[ii][3]);
    } else if (I == Tj) {
#pragma unroll
      for (int ii = 0; ii < TT; ++ii)
        *reinterpret_cast<float4 *>(&rowbuf[Tj & 1][ii][c0]) =
            make_float4(m[ii][0], m[ii][1], m[ii][2], m[ii][3]);
    }
  };
  if (own) publish(NT - 1);
  __syncthreads();
  bool bad = false;
  for (int Tj = NT - 1; Tj >= 0; --Tj) {
    const int j0 = TT * Tj, par = Tj & 1;
    // ---------------- phase A
    if (t < 2 * NB) {
      float blk[TT][TT];
#pragma unroll
      for (int a = 0; a < TT; ++a) {
        const float4 v = *reinterpret_cast<const float4 *>(&colbuf[par][j0 + a][0]);
        blk[a][0] = v.x; blk[a][1] = v.y; blk[a][2] = v.z; blk[a][3] = v.w;
      }
      float rp[TT], bq[TT][TT], lq[TT][TT];
#pragma unroll
      for (int q = TT - 1; q >= 0; --q) {
        const float p = blk[q][q];
        rp[q] = __frcp_rn(p);
        if (t == 0) {
          piv[j0 + q] = p;
          if (!(p > 0.f) || !isfinite(p)) {
            if (!bad)
              report(info, KRONQ_ERR_NOT_PD | static_cast<int32_t>((off + j0 + q) << 8));
            bad = true;
          }
        }
        float colq[TT], rowq[TT];
#pragma unroll
        for (int a = 0; a < TT; ++a) {
          colq[a] = blk[a][q];
          rowq[a] = blk[q][a];
          bq[q][a] = a < q ? colq[a] : a == q ? p + 1.f : rowq[a];
          lq[q][a] = a < q ? colq[a] * rp[q] : 0.f;
        }
#pragma unroll
        for (int a = 0; a < q; ++a) {
          const float la = lq[q][a];
#pragma unroll
          for (int bb = a; bb < TT; ++bb) blk[a][bb] = fmaf(-la, bq[q][bb], blk[a][bb]);
        }
      }
      if (t < NB) {
        const int i = t;
        if (i < j0) {
          const float4 v = *reinterpret_cast<const float4 *>(&colbuf[par][i][0]);
          float P[TT] = {v.x, v.y, v.z, v.w};
          float Lr[TT];
#pragma unroll
          for (int q = TT - 1; q >= 0; --q) {
            const float l = P[q] * rp[q];
            Lr[q] = l;
            Bs[q][i] = P[q];
#pragma unroll
            for (int a = 0; a < TT; ++a) P[a] = fmaf(-l, bq[q][a], P[a]);
          }
          *reinterpret_cast<float4 *>(&Ls[i][0]) = make_float4(Lr[0], Lr[1], Lr[2], Lr[3]);
          *reinterpret_cast<float4 *>(&colbuf[par][i][0]) = make_float4(P[0], P[1], P[2], P[3]);
        } else if (i == j0) {
          // (not into colbuf: the other phase-A threads may still read it)
#pragma unroll
          for (int a = 0; a < TT; ++a)
            *reinterpret_cast<float4 *>(&blkf[a][0]) =
                make_float4(blk[a][0], blk[a][1], blk[a][2], blk[a][3]);
        }
      } else {
        const int k = t - NB;
        if (k >= j0 + TT) {
          float R[TT];
#pragma unroll
          for (int a = 0; a < TT; ++a) R[a] = rowbuf[par][a][k];
#pragma unroll
          for (int q = TT - 1; q >= 0; --q) {
            Bs[q][k] = R[q];
#pragma unroll
            for (int a = 0; a < q; ++a) R[a] = fmaf(-lq[q][a], R[q], R[a]);
          }
#pragma unroll
          for (int a = 0; a < TT; ++a) rowbuf[par][a][k] = R[a];
        }
      }
    }
    __syncthreads();
    // ---------------- phase B, then the panels of the next block
    if (own) {
      if (I < Tj && K != Tj) {
        float l[TT][TT], b[TT][TT];  // l[ii][q], b[q][kk]
#pragma unroll
        for (int ii = 0; ii < TT; ++ii) {
          const float4 v = *reinterpret_cast<const float4 *>(&Ls[r0 + ii][0]);
          l[ii][0] = v.x; l[ii][1] = v.y; l[ii][2] = v.z; l[ii][3] = v.w;
        }
#pragma unroll
        for (int q = 0; q < TT; ++q) {
          const float4 v = *reinterpret_cast<const float4 *>(&Bs[q][c0]);
          b[q][0] = v.x; b[q][1] = v.y; b[q][2] = v.z; b[q][3] = v.w;
        }
#pragma unroll
        for (int q = TT - 1; q >= 0; --q)
#pragma unroll
          for (int ii = 0; ii < TT; ++ii)
#pragma unroll
            for (int kk = 0; kk < TT; ++kk) m[ii][kk] = fmaf(-l[ii][q], b[q][kk], m[ii][kk]);
      } else if (K == Tj) {
#pragma unroll
        for (int ii = 0; ii < TT; ++ii) {
          const float4 v = I == Tj ? *reinterpret_cast<const float4 *>(&blkf[ii][0])
                                   : *reinterpret_cast<const float4 *>(&colbuf[par][r0 + ii][0]);
          m[ii][0] = v.x; m[ii][1] = v.y; m[ii][2] = v.z; m[ii][3] = v.w;
        }
      } else if (I == Tj) {
#pragma unroll
        for (int ii = 0; ii < TT; ++ii) {
          const float4 v = *reinterpret_cast<const float4 *>(&rowbuf[par][ii][c0]);
          m[ii][0] = v.x; m[ii][1] = v.y; m[ii][2] = v.z; m[ii][3] = v.w;
        }
      }
      if (Tj > 0) publish(Tj - 1);
    }
    __syncthreads();
  }
  if (own) {
#pragma unroll
    for (int ii = 0; ii < TT; ++ii) {
      const int i = r0 + ii;
      const float s = 1.f / sqrtf(piv[i]);
      float o[TT];
#pragma unroll
      for (int kk = 0; kk < TT; ++kk) {
        const int k = c0 + kk;
        o[kk] = k > i ? m[ii][kk] * s : (k == i ? s : 0.f);
      }
      *reinterpret_cast<float4 *>(H + (off + i) * ld + off + c0) =
          make_float4(o[0], o[1], o[2], o[3]);
      if (I != K)  // mirrored tile below the diagonal
        *reinterpret_cast<float4 *>(H + (off + c0 + ii) * ld + off + r0) =
            make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

constexpr int MAXD = 40;  // recursion depth bound (d <= 65536 gives <= 10)

struct Ctx {
  cudaStream_t st;           // critical path (leaves, V, SYRK, U12)
  cudaStream_t side[MAXD];   // T = V U22 of the node at each depth
  cudaEvent_t ev_v[MAXD], ev_t[MAXD];
  float *H;
  int64_t d;
  float *V[MAXD];            // B U22ᵀ of the node at each depth
  float *T[MAXD];            // V U22 of the node at each depth
  void *scr_main;            // GEMM scratch of the critical path
  void *scr_side[MAXD];      // and of each depth's side stream
  size_t scr_main_bytes, scr_side_bytes[MAXD];
  const float *lambda;
  int32_t *info;
  bool root_r;               // keep R12 at the root instead of U12 (no T, no U12)
};

// Streams and events of the recursion, created once per device: the critical
// path runs on a highest-priority stream so that its single-CTA leaves take
// the next free SM ahead of the concurrent T products.
struct CholStreams {
  bool ready = false;
  // held by one call from its fork record to its last join: the fork and
  // join events are shared by every call on the device, so two host threads
  // must not interleave their records and waits
  std::mutex call_mu;
  cudaStream_t main;
  cudaStream_t side[MAXD];
  cudaEvent_t ev_v[MAXD], ev_t[MAXD], fork, join_main, join_side[MAXD];
};

kronq_status chol_streams(CholStreams **out) {
  static CholStreams per_dev[64];
  static std::mutex mu;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return KRONQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  CholStreams &cs = per_dev[dev];
  if (!cs.ready) {
    int lo = 0, hi = 0;
    KQ_CUDA(cudaDeviceGetStreamPriorityRange(&lo, &hi));
    KQ_CUDA(cudaStreamCreateWithPriority(&cs.main, cudaStreamNonBlocking, hi));
    if (cudaEventCreateWithFlags(&cs.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&cs.join_main, cudaEventDisableTiming) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    for (int k = 0; k < MAXD; ++k) {
      if (cudaStreamCreateWithPriority(&cs.side[k], cudaStreamNonBlocking, lo) != cudaSuccess ||
          cudaEventCreateWithFlags(&cs.ev_v[k], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&cs.ev_t[k], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&cs.join_side[k], cudaEventDisableTiming) != cudaSuccess)
        return KRONQ_ERR_CUDA;
    }
    cs.ready = true;
  }
  *out = &cs;
  return KRONQ_OK;
}

inline int64_t first_half(int64_t n) { return (n / NB / 2) * NB; }

kronq_status leaf(const Ctx &c, int64_t off) {
  chol_leaf_kernel<<<1, LTHREADS, 0, c.st>>>(c.H, c.d, off, c.lambda, c.info);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

// Block [off, off+n) of H (n a multiple of NB) -> U of that block, in place.
kronq_status rinv(const Ctx &c, int64_t off, int64_t n, int depth) {
  if (n == NB) return leaf(c, off);
  const int64_t h = first_half(n), m = n - h;
  const int64_t d = c.d;
  float *A11 = c.H + off * d + off;
  float *B12 = c.H + off * d + off + h;
  float *C22 = c.H + (off + h) * d + off + h;
  if (depth >= MAXD - 1) return KRONQ_ERR_UNSUPPORTED;
  float *V = c.V[depth], *T = c.T[depth];
  KQ_TRY(rinv(c, off + h, m, depth + 1));  // C22 -> U22
  {
    GemmArgs g;  // V = B U22ᵀ : V[i][j] = sum_k B[i][k] U22[j][k], k >= j
    g.M = h; g.N = m; g.K = m;
    g.A = B12; g.lda = d;
    g.B = C22; g.ldb = d;
    g.C = V; g.ldc = m;
    g.kflags = KR_B_UPPER;
    KQ_TRY(gemm_f32(c.st, g, c.scr_main, c.scr_main_bytes, c.info));
  }
  const bool keep_r = c.root_r && depth == 0;
  // T = V U22 does not feed the recursion into A11: run it beside it
  if (!keep_r) {
  if (cudaEventRecord(c.ev_v[depth], c.st) != cudaSuccess ||
      cudaStreamWaitEvent(c.side[depth], c.ev_v[depth], 0) != cudaSuccess)
    return KRONQ_ERR_CUDA;
  {
    GemmArgs g;  // T = V U22 : T[i][j] = sum_k V[i][k] U22[k][j], k <= j
    g.M = h; g.N = m; g.K = m;
    g.A = V; g.lda = m;
    g.B = C22; g.ldb = d; g.b_mn = true;
    g.C = T; g.ldc = m;
    g.kflags = KR_B_LOWER;
    KQ_TRY(gemm_f32(c.side[depth], g, c.scr_side[depth], c.scr_side_bytes[depth], c.info));
  }
  KQ_CUDA(cudaEventRecord(c.ev_t[depth], c.side[depth]));
  }
  {
    GemmArgs g;  // A11 -= V Vᵀ (tiles on or above the diagonal)
    g.M = h; g.N = h; g.K = m;
    g.A = V; g.lda = m;
    g.B = V; g.ldb = m;
    g.C = A11; g.ldc = d;
    g.alpha = -1.f; g.beta = 1.f;
    g.upper_tiles_only = true;
    KQ_TRY(gemm_f32(c.st, g, c.scr_main, c.scr_main_bytes, c.info));
  }
  KQ_TRY(rinv(c, off, h, depth + 1));  // A11 -> U11
  if (keep_r) {
    // the caller's OBS crosses the halves with R12 = V itself
    KQ_CUDA(cudaMemcpy2DAsync(B12, static_cast<size_t>(d) * 4, V, static_cast<size_t>(m) * 4,
                          static_cast<size_t>(m) * 4, static_cast<size_t>(h),
                          cudaMemcpyDeviceToDevice, c.st));
  } else {
  KQ_CUDA(cudaStreamWaitEvent(c.st, c.ev_t[depth], 0));
  {
    GemmArgs g;  // U12 = -U11 T : U11[i][k] == 0 for k < i
    g.M = h; g.N = m; g.K = h;
    g.A = A11; g.lda = d;
    g.B = T; g.ldb = m; g.b_mn = true;
    g.C = B12; g.ldc = d;
    g.alpha = -1.f;
    g.kflags = KR_A_UPPER;
    KQ_TRY(gemm_f32(c.st, g, c.scr_main, c.scr_main_bytes, c.info));
  }
  }
  // zeros below the diagonal of this node (the leaves zero their own blocks):
  // triangular operands of the parents' products read U as 128 x 256 tiles
  KQ_CUDA(cudaMemset2DAsync(c.H + (off + h) * d + off, static_cast<size_t>(d) * 4, 0,
                        static_cast<size_t>(h) * 4, static_cast<size_t>(m),
                        c.st));
  return KRONQ_OK;
}

// Workspace layout: [V, T, side-stream GEMM scratch] per recursion depth, the
// critical path's GEMM scratch, then lambda. The largest node at depth i+1 is
// the larger child m_i of the largest node at i, and the node sizes bound the
// products' scratch (V: h x m x m, SYRK: h x h x m, U12: h x m x h, T: h x m x m).
struct CholLayout {
  size_t v[MAXD], t[MAXD], side[MAXD], side_bytes[MAXD];
  size_t main, main_bytes;
  int depths;
  size_t total;
};
CholLayout chol_layout(int64_t d) {
  auto al = [](size_t b) { return (b + 255) / 256 * 256; };
  CholLayout L{};
  size_t off = 0;
  size_t main_bytes = 0;
  int k = 0;
  for (int64_t n = d; n > NB && k < MAXD; ++k) {
    const int64_t h = first_half(n), m = n - h;
    const size_t slot = al(static_cast<size_t>(h) * m * 4);
    L.v[k] = off;
    L.t[k] = off + slot;
    L.side[k] = off + 2 * slot;
    L.side_bytes[k] = al(gemm_scratch_bytes(h, m, m));
    off += 2 * slot + L.side_bytes[k];
    main_bytes = kq_max(main_bytes, kq_max(gemm_scratch_bytes(h, m, m),
                                           kq_max(gemm_scratch_bytes(h, h, m),
                                                  gemm_scratch_bytes(h, m, h))));
    n = m;
  }
  L.depths = k;
  L.main = off;
  L.main_bytes = al(main_bytes);
  L.total = off + L.main_bytes + 256;
  return L;
}

}  // namespace

size_t chol_ws_bytes(int64_t d) { return chol_layout(d).total; }

kronq_status chol_run(cudaStream_t st, float *H, int64_t d, float damp_rel,
                      void *ws, size_t ws_bytes, int32_t *info, bool root_r) {
  const CholLayout lay = chol_layout(d);
  const int depths = lay.depths;
  const size_t need = lay.total;
  if (ws_bytes < need) return KRONQ_ERR_INVALID_ARG;
  CholStreams *cs = nullptr;
  KQ_TRY(chol_streams(&cs));
  std::lock_guard<std::mutex> call_lock(cs->call_mu);
  uint8_t *w = static_cast<uint8_t *>(ws);
  Ctx c;
  c.st = cs->main;
  c.H = H;
  c.d = d;
  auto at = [&](int k, size_t o) {
    return k < depths ? reinterpret_cast<float *>(w + o) : nullptr;
  };
  for (int k = 0; k < MAXD; ++k) {
    c.side[k] = cs->side[k];
    c.ev_v[k] = cs->ev_v[k];
    c.ev_t[k] = cs->ev_t[k];
    c.V[k] = at(k, lay.v[k]);
    c.T[k] = at(k, lay.t[k]);
    c.scr_side[k] = at(k, lay.side[k]);
    c.scr_side_bytes[k] = k < depths ? lay.side_bytes[k] : 0;
  }
  c.scr_main = w + lay.main;
  c.scr_main_bytes = lay.main_bytes;
  float *lambda = reinterpret_cast<float *>(w + need - 256);
  c.lambda = lambda;
  c.info = info;
  c.root_r = root_r && d > NB;
  // fork from the caller's stream
  if (cudaEventRecord(cs->fork, st) != cudaSuccess ||
      cudaStreamWaitEvent(cs->main, cs->fork, 0) != cudaSuccess)
    return KRONQ_ERR_CUDA;
  for (int k = 0; k < depths; ++k)
    KQ_CUDA(cudaStreamWaitEvent(cs->side[k], cs->fork, 0));
  damping_kernel<<<1, 1024, 0, c.st>>>(H, d, damp_rel, lambda, info);
  KQ_CHECK_LAUNCH();
  KQ_TRY(rinv(c, 0, d, 0));
  // join back into the caller's stream (every side stream is idle by now
  // from the main stream's point of view; joining them keeps ws reuse safe)
  if (cudaEventRecord(cs->join_main, cs->main) != cudaSuccess ||
      cudaStreamWaitEvent(st, cs->join_main, 0) != cudaSuccess)
    return KRONQ_ERR_CUDA;
  for (int k = 0; k < depths; ++k)
    if (cudaEventRecord(cs->join_side[k], cs->side[k]) != cudaSuccess ||
        cudaStreamWaitEvent(st, cs->join_side[k], 0) != cudaSuccess)
      return KRONQ_ERR_CUDA;
  return KRONQ_OK;
}

kronq_status chol_inv(cudaStream_t st, float *H, int64_t d, float damp_rel,
                      void *ws, size_t ws_bytes, int32_t *info) {
  return chol_run(st, H, d, damp_rel, ws, ws_bytes, info, false);
}

kronq_status chol_split(cudaStream_t st, float *H, int64_t d, float damp_rel,
                        void *ws, size_t ws_bytes, int32_t *info) {
  return chol_run(st, H, d, damp_rel, ws, ws_bytes, info, true);
}

int64_t chol_split_point(int64_t d) { return first_half(d); }

}  // namespace kronq

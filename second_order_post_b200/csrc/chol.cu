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
// All off-diagonal work runs as fp32-accurate 3xTF32 tcgen05 GEMMs that skip
// the zero blocks of the triangular operands; 128x128 diagonal leaves are
// factored in shared memory by one CTA. λ = damp_rel * mean(diag H) is added
// by each leaf to its own diagonal (the updates never touch λ, so this equals
// damping H up front).
#include "kernels.cuh"

namespace kronq {
namespace {

constexpr int NB = 128;
constexpr int LP = NB + 1;  // padded pitch of the leaf tiles
constexpr int LTHREADS = 512;

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
// Sweep 1, reverse LDLᵀ (H = Ŕ D Ŕᵀ, Ŕ unit upper), blocked by 32 columns from
// the right; for each sub-block [c0, c0+32):
//   (a) warp 0 factors the diagonal sub-block: lane l keeps row c0+l in
//       registers, column entries of other rows arrive by shuffle;
//   (b) one thread per row i < c0 applies the same 32 steps to its panel row;
//   (c) all threads apply the rank-32 update of the leading block.
// Sweep 2, X = Ŕ^-1: four warps invert the diagonal sub-blocks in parallel,
// then the off-diagonal sub-blocks follow block diagonal by block diagonal
// (X_IJ = -X_II Σ_K Ŕ_IK X_KJ) as small shared-memory products.
constexpr int SB = 32;

// C[32x32] = alpha * sum over terms of A_t[32x32] * B_t[32x32] for several
// independent outputs at once (all operands in shared memory, pitch LP).
struct BlkTerm {
  const float *A, *B;
};
__device__ void small_products(int n_out, float **C, const BlkTerm (*terms)[3],
                               const int *n_terms, float alpha) {
  for (int e = threadIdx.x; e < n_out * SB * SB; e += blockDim.x) {
    const int o = e / (SB * SB), r = (e / SB) % SB, c = e % SB;
    float s = 0.f;
    for (int t = 0; t < n_terms[o]; ++t) {
      const float *a = terms[o][t].A + r * LP, *b = terms[o][t].B + c;
#pragma unroll 8
      for (int k = 0; k < SB; ++k) s = fmaf(a[k], b[k * LP], s);
    }
    C[o][r * LP + c] = alpha * s;
  }
}

__global__ void __launch_bounds__(LTHREADS)
    chol_leaf_kernel(float *__restrict__ H, int64_t ld, int64_t off,
                     const float *__restrict__ lambda, int32_t *info) {
  extern __shared__ float sm[];
  float *A = sm;                  // NB x LP: LDLᵀ, then the unit factor
  float *X = A + NB * LP;         // NB x LP: inverse of the unit factor
  float *T = X + NB * LP;         // 3 x SB x LP temporaries
  float *piv = T + 3 * SB * LP;   // NB pivots
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const float lam = *lambda;
  for (int e = t; e < NB * NB; e += LTHREADS) {
    const int r = e / NB, c = e % NB;
    if (c >= r) {
      float v = H[(off + r) * ld + off + c];
      if (c == r) v += lam;
      A[r * LP + c] = v;
    }
  }
  __syncthreads();
  // ================= sweep 1
  for (int J = NB / SB - 1; J >= 0; --J) {
    const int c0 = SB * J;
    if (warp == 0) {  // (a) diagonal sub-block, row c0+lane in registers
      float r[SB];
#pragma unroll
      for (int k = 0; k < SB; ++k) r[k] = (k >= lane) ? A[(c0 + lane) * LP + c0 + k] : 0.f;
      bool bad = false;
#pragma unroll
      for (int jj = SB - 1; jj >= 0; --jj) {
        const float p = __shfl_sync(0xffffffffu, r[jj], jj);
        if (lane == 0) {
          piv[c0 + jj] = p;
          if (!(p > 0.f) || !isfinite(p)) {
            if (!bad) report(info, KRONQ_ERR_NOT_PD | static_cast<int32_t>((off + c0 + jj) << 8));
            bad = true;
          }
        }
        const float f = r[jj] / p;
#pragma unroll
        for (int k = 0; k < jj; ++k) {
          const float ck = __shfl_sync(0xffffffffu, r[jj], k);  // A[c0+k][c0+jj]
          if (lane <= k && lane < jj) r[k] = fmaf(-ck, f, r[k]);
        }
      }
#pragma unroll
      for (int k = 0; k < SB; ++k)
        if (k >= lane) A[(c0 + lane) * LP + c0 + k] = r[k];
    }
    __syncthreads();
    if (c0 == 0) break;
    if (t < c0) {  // (b) panel row t: A[t][c0 .. c0+31]
      float q[SB];
      float *row = A + t * LP + c0;
#pragma unroll
      for (int k = 0; k < SB; ++k) q[k] = row[k];
#pragma unroll
      for (int jj = SB - 1; jj >= 0; --jj) {
        const float f = q[jj] / piv[c0 + jj];
#pragma unroll
        for (int k = 0; k < jj; ++k) q[k] = fmaf(-A[(c0 + k) * LP + c0 + jj], f, q[k]);
      }
#pragma unroll
      for (int k = 0; k < SB; ++k) row[k] = q[k];
    }
    __syncthreads();
    {  // (c) A[i][k] -= sum_jj A[i][c0+jj] A[k][c0+jj] / piv[c0+jj], i <= k < c0
      const int k = t % NB, r0 = t / NB;
      if (k < c0) {
        float g[SB];
#pragma unroll
        for (int jj = 0; jj < SB; ++jj) g[jj] = A[k * LP + c0 + jj] / piv[c0 + jj];
        for (int i = r0; i <= k; i += LTHREADS / NB) {
          const float *ri = A + i * LP + c0;
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int jj = 0; jj < SB; jj += 2) {
            s0 = fmaf(ri[jj], g[jj], s0);
            s1 = fmaf(ri[jj + 1], g[jj + 1], s1);
          }
          A[i * LP + k] -= s0 + s1;
        }
      }
    }
    __syncthreads();
  }
  // unit factor Ŕ[i][k] = A[i][k] / piv[k] (i < k); X = 0
  for (int e = t; e < NB * NB; e += LTHREADS) {
    const int r = e / NB, c = e % NB;
    if (c > r) A[r * LP + c] /= piv[c];
    X[r * LP + c] = 0.f;
  }
  __syncthreads();
  // ================= sweep 2
  if (warp < NB / SB) {  // diagonal inverses, lane = column c0+lane
    const int c0 = SB * warp;
    float x[SB];
#pragma unroll
    for (int i = 0; i < SB; ++i) x[i] = (i == lane) ? 1.f : 0.f;
#pragma unroll
    for (int i = SB - 2; i >= 0; --i) {
      float s = 0.f;
#pragma unroll
      for (int k = i + 1; k < SB; ++k)
        if (k <= lane) s = fmaf(A[(c0 + i) * LP + c0 + k], x[k], s);
      if (i < lane) x[i] = -s;
    }
#pragma unroll
    for (int i = 0; i < SB; ++i)
      if (i <= lane) X[(c0 + i) * LP + c0 + lane] = x[i];
  }
  __syncthreads();
  for (int dist = 1; dist < NB / SB; ++dist) {
    const int n = NB / SB - dist;  // blocks (I, I+dist), I < n
    float *Cs[3];
    BlkTerm terms[3][3];
    int nt[3];
    // T_I = sum_{K=I+1..J} Ŕ_IK X_KJ
    for (int I = 0; I < n; ++I) {
      const int J = I + dist;
      Cs[I] = T + I * SB * LP;
      nt[I] = dist;
      for (int m = 0; m < dist; ++m) {
        const int K = I + 1 + m;
        terms[I][m] = {A + (SB * I) * LP + SB * K, X + (SB * K) * LP + SB * J};
      }
    }
    small_products(n, Cs, terms, nt, 1.f);
    __syncthreads();
    // X_IJ = -X_II T_I
    for (int I = 0; I < n; ++I) {
      const int J = I + dist;
      Cs[I] = X + (SB * I) * LP + SB * J;
      nt[I] = 1;
      terms[I][0] = {X + (SB * I) * LP + SB * I, T + I * SB * LP};
    }
    small_products(n, Cs, terms, nt, -1.f);
    __syncthreads();
  }
  // U(i, c) = X(i, c) / sqrt(piv[i]) for i <= c, zeros below the diagonal
  for (int e = t; e < NB * NB; e += LTHREADS) {
    const int i = e / NB, c = e % NB;
    H[(off + i) * ld + off + c] = (i <= c) ? X[i * LP + c] / sqrtf(piv[i]) : 0.f;
  }
}

__global__ void zero_lower_kernel(float *H, int64_t d) {
  const int64_t r = blockIdx.y;
  for (int64_t c = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; c < r;
       c += int64_t(gridDim.x) * blockDim.x)
    H[r * d + c] = 0.f;
}

struct Ctx {
  cudaStream_t st;
  float *H;
  int64_t d;
  float *V;              // B U22ᵀ of the current node (dead before recursing)
  float *T[40];          // V U22 of the node at each depth (kept across the
                         // recursion into A11)
  const float *lambda;
  int32_t *info;
};

inline int64_t first_half(int64_t n) { return (n / NB / 2) * NB; }

kronq_status leaf(const Ctx &c, int64_t off) {
  const int smem = (2 * NB * LP + 3 * SB * LP + NB) * sizeof(float);
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(chol_leaf_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    attr_done = true;
  }
  chol_leaf_kernel<<<1, LTHREADS, smem, c.st>>>(c.H, c.d, off, c.lambda, c.info);
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
  float *T = c.T[depth];
  KQ_TRY(rinv(c, off + h, m, depth + 1));  // C22 -> U22
  {
    GemmArgs g;  // V = B U22ᵀ : V[i][j] = sum_k B[i][k] U22[j][k], k >= j
    g.M = h; g.N = m; g.K = m;
    g.A = B12; g.lda = d;
    g.B = C22; g.ldb = d;
    g.C = c.V; g.ldc = m;
    g.kflags = KR_B_UPPER;
    KQ_TRY(gemm_tf32x3(c.st, g, c.info));
  }
  {
    GemmArgs g;  // A11 -= V Vᵀ (tiles on or above the diagonal)
    g.M = h; g.N = h; g.K = m;
    g.A = c.V; g.lda = m;
    g.B = c.V; g.ldb = m;
    g.C = A11; g.ldc = d;
    g.alpha = -1.f; g.beta = 1.f;
    g.upper_tiles_only = true;
    KQ_TRY(gemm_tf32x3(c.st, g, c.info));
  }
  {
    GemmArgs g;  // T = V U22 : T[i][j] = sum_k V[i][k] U22[k][j], k <= j
    g.M = h; g.N = m; g.K = m;
    g.A = c.V; g.lda = m;
    g.B = C22; g.ldb = d; g.b_mn = true;
    g.C = T; g.ldc = m;
    g.kflags = KR_B_LOWER;
    KQ_TRY(gemm_tf32x3(c.st, g, c.info));
  }
  KQ_TRY(rinv(c, off, h, depth + 1));  // A11 -> U11
  {
    GemmArgs g;  // U12 = -U11 T : U11[i][k] == 0 for k < i
    g.M = h; g.N = m; g.K = h;
    g.A = A11; g.lda = d;
    g.B = T; g.ldb = m; g.b_mn = true;
    g.C = B12; g.ldc = d;
    g.alpha = -1.f;
    g.kflags = KR_A_UPPER;
    KQ_TRY(gemm_tf32x3(c.st, g, c.info));
  }
  return KRONQ_OK;
}

// Workspace layout: [V: h0*m0][T slot per depth][lambda]. The largest node at
// depth i+1 is the larger child m_i of the largest node at depth i.
size_t chol_layout(int64_t d, size_t *t_off, int *depths) {
  auto al = [](size_t b) { return (b + 255) / 256 * 256; };
  const int64_t h0 = first_half(d);
  size_t off = al(static_cast<size_t>(h0) * (d - h0) * 4);
  int k = 0;
  for (int64_t n = d; n > NB && k < 40; ++k) {
    const int64_t h = first_half(n);
    if (t_off) t_off[k] = off;
    off += al(static_cast<size_t>(h) * (n - h) * 4);
    n = n - h;
  }
  if (depths) *depths = k;
  return off + 256;
}

}  // namespace

size_t chol_ws_bytes(int64_t d) { return chol_layout(d, nullptr, nullptr); }

kronq_status chol_inv(cudaStream_t st, float *H, int64_t d, float damp_rel,
                      void *ws, size_t ws_bytes, int32_t *info) {
  size_t t_off[40];
  int depths = 0;
  const size_t need = chol_layout(d, t_off, &depths);
  if (ws_bytes < need) return KRONQ_ERR_INVALID_ARG;
  uint8_t *w = static_cast<uint8_t *>(ws);
  Ctx c;
  c.st = st;
  c.H = H;
  c.d = d;
  c.V = reinterpret_cast<float *>(w);
  for (int k = 0; k < 40; ++k)
    c.T[k] = k < depths ? reinterpret_cast<float *>(w + t_off[k]) : nullptr;
  float *lambda = reinterpret_cast<float *>(w + need - 256);
  c.lambda = lambda;
  c.info = info;
  damping_kernel<<<1, 1024, 0, st>>>(H, d, damp_rel, lambda, info);
  KQ_CHECK_LAUNCH();
  KQ_TRY(rinv(c, 0, d, 0));
  dim3 grid(static_cast<unsigned>(kq_min<int64_t>(ceil_div(d, 256), 64)),
            static_cast<unsigned>(d));
  zero_lower_kernel<<<grid, 256, 0, st>>>(H, d);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

}  // namespace kronq

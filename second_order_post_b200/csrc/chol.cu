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

// Sweep-1 step for one row: row[k] -= colj[k*LP] * f for k = k0, k0+4, ... < j.
// The row (A[i][k], k < j) and the pivot column (A[k][j]) never share an
// element, so the loads can run ahead of the stores.
__device__ __forceinline__ void ldl_row_step(float *__restrict__ row,
                                             const float *__restrict__ colj,
                                             int k0, int j, float f) {
#pragma unroll 4
  for (int k = k0; k < j; k += 4) row[k] = fmaf(-colj[k * LP], f, row[k]);
}

// One diagonal leaf at rows/cols [off, off+NB): reads the upper triangle of the
// (already updated) block, adds λ, writes U (upper, zeros below).
// Sweep 1, reverse LDLᵀ in shared memory: thread (row i, residue q) updates
// A[i][k] for k ≡ q (mod 4); warps are numbered so that each scheduler holds
// all four row blocks of one residue (balanced). One barrier per column.
// Sweep 2, X = (unit upper)^-1 one column at a time from the bottom row up:
// four lanes of a warp share a column and split the k-sum, no block barrier.
__global__ void __launch_bounds__(LTHREADS)
    chol_leaf_kernel(float *__restrict__ H, int64_t ld, int64_t off,
                     const float *__restrict__ lambda, int32_t *info) {
  extern __shared__ float sm[];
  float *A = sm;                 // NB x LP
  float *X = sm + NB * LP;       // NB x LP
  float *piv = X + NB * LP;      // NB pivots
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
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
  // ---- sweep 1
  {
    const int q = w & 3, i = 32 * (w >> 2) + lane;
    const int k0 = i + ((q - i) & 3);  // first k >= i with k ≡ q (mod 4)
    bool bad = false;
    for (int j = NB - 1; j >= 0; --j) {
      const float p = A[j * LP + j];
      if (t == 0) {
        piv[j] = p;
        if (!(p > 0.f) || !isfinite(p)) {
          if (!bad) report(info, KRONQ_ERR_NOT_PD | static_cast<int32_t>((off + j) << 8));
          bad = true;
        }
      }
      if (i < j) ldl_row_step(A + i * LP, A + j, k0, j, A[i * LP + j] / p);
      __syncthreads();
    }
  }
  // unit upper factor in place: A[i][k] / piv[k], i < k
  for (int e = t; e < NB * NB; e += LTHREADS) {
    const int r = e / NB, c = e % NB;
    if (c > r) A[r * LP + c] /= piv[c];
  }
  __syncthreads();
  // ---- sweep 2: column c of X, lanes 4g..4g+3 of a warp share c
  {
    const int part = lane & 3;
    const int c = 8 * w + (lane >> 2);
    X[c * LP + c] = 1.f;  // X stored transposed: X[c][i] holds X(i, c)
    __syncwarp();
    float *xc = X + c * LP;
    for (int i = NB - 2; i >= 0; --i) {
      float s = 0.f;
      if (i < c) {
        const float *ri = A + i * LP;
        for (int k = i + 1 + part; k <= c; k += 4) s = fmaf(ri[k], xc[k], s);
      }
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (part == 0 && i < c) xc[i] = -s;
      __syncwarp();
    }
  }
  __syncthreads();
  // U(i, c) = X(i, c) / sqrt(piv[i]) for i <= c, zeros below the diagonal
  for (int e = t; e < NB * NB; e += LTHREADS) {
    const int i = e / NB, c = e % NB;
    H[(off + i) * ld + off + c] = (i <= c) ? X[c * LP + i] / sqrtf(piv[i]) : 0.f;
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
  const int smem = (2 * NB * LP + NB) * sizeof(float);
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

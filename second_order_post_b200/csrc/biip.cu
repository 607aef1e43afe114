// Bidirectional incoherence processing (BiIP) [wmrh §三, §八, Q2; aimodeling]:
// a diagonal rescale from diag(H_X), diag(H_G) followed by a seeded orthogonal
// rotation on both sides of W, with H_X and H_G rotated to match:
//   W'   = U_G S_G W S_X U_Xᵀ
//   H_X' = U_X S_X^-1 H_X S_X^-1 U_Xᵀ,   H_G' = U_G S_G^-1 H_G S_G^-1 U_Gᵀ
// with U = (Hhat_had ⊗ Q_m) diag(sign) per side (spec in include/kronq.h).
//
// Every rotation of an R x C row-major matrix M -> P_r diag(cr) M diag(cc) P_cᵀ
// is split into memory passes whose working sets fit in shared memory:
//   row pass      one row chunk of Lc*m_c contiguous columns per CTA (or per
//                 step of a persistent CTA): input factors, Hadamard over the
//                 chunk's a-index, Q_m over each group of m_c contiguous
//                 values (the whole column side when the row fits)
//   column pass   the whole row side in one read and one write: a cluster
//                 of CTAs holds a strip of columns over all rows, Q_m over
//                 each group of rows, the local Hadamard, then the top bits
//                 across the cluster through distributed shared memory
//   row-side Q_m  groups of m_r consecutive rows (m_r > 32, when the column
//   + strided     pass does not apply), then the Hadamard over index bits
//                 whose elements sit at a fixed stride
// The Hadamard factors commute with each other and with Q_m (Kronecker
// structure), and P_r and P_c act on different sides, so the order of the
// passes does not change the result: in place on fp32 with Q_28 on the row
// side (H_X of the pages' 70B shapes) the column pass goes first and takes
// both diagonal factors.
#include <math.h>

#include "kernels.cuh"

namespace kronq {
namespace {


__host__ __device__ inline uint64_t sm64(uint64_t s) {
  uint64_t z = s + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// ------------------------------------------------------------- side preparation
struct SideDev {
  const float *H;  // covariance of this side (diag read)
  int64_t d;
  int rot;         // rotation on
  int scale;       // diagonal scale on
  float expo;
  uint64_t key;    // sm64(sm64(seed) + side)
  float *s;        // out: scale
  float *fw;       // out: sign * s   (factor on W)
  float *fh;       // out: sign / s   (factor on H)
};

__global__ void side_prep_kernel(SideDev a, SideDev b, int32_t *info) {
  const SideDev &p = blockIdx.x == 0 ? a : b;
  __shared__ double part[32];
  __shared__ double mean_sh;
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < p.d; i += blockDim.x) acc += p.H[i * p.d + i];
  acc = warp_sum_d(acc);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < blockDim.x / 32 ? part[threadIdx.x] : 0.0;
    v = warp_sum_d(v);
    if (threadIdx.x == 0) {
      mean_sh = v / double(p.d);
      if (!isfinite(mean_sh)) report(info, KRONQ_ERR_NONFINITE);
    }
  }
  __syncthreads();
  const double floor_v = 1e-8 * mean_sh;
  for (int64_t i = threadIdx.x; i < p.d; i += blockDim.x) {
    double s = 1.0;
    if (p.scale) {
      const double h = p.H[i * p.d + i];
      if (!isfinite(h)) report(info, KRONQ_ERR_NONFINITE);
      s = pow(fmax(h, floor_v), double(p.expo));
    }
    const float sf = static_cast<float>(s);
    float sg = 1.f;
    if (p.rot) sg = (sm64(p.key + static_cast<uint64_t>(i)) >> 63) ? -1.f : 1.f;
    p.s[i] = sf;
    p.fw[i] = sg * sf;
    p.fh[i] = sg / sf;
  }
}

// Q_m = orthogonal factor of the seeded Gaussian m x m matrix (R diag > 0),
// in fp64, one CTA per side, by block classical Gram–Schmidt with
// reorthogonalization: for each block J of QM_NB columns,
//   V <- (I - Q_prev Q_prevᵀ)^2 G_J        (two projection passes)
//   V <- V R^-1, VᵀV = RᵀR (Cholesky)      (twice)
// Every R on the way is upper triangular with a positive diagonal, so the
// columns are those of the unique QR factor.
struct QDev {
  int m;
  uint64_t kq;
  double *G;   // scratch m*m, column-major (column j contiguous)
  float *Q;    // out: Q[b*m + b'] (row-major)
};

constexpr int QM_THREADS = 1024;
constexpr int QM_NB = 16;                 // columns per block
constexpr int QM_LD = QM_NB + 1;          // row stride of the blocks in shared memory
constexpr int QM_MAX = 256;
constexpr size_t QM_SMEM = (2 * QM_MAX * QM_LD + QM_NB * QM_LD) * sizeof(double);

__global__ void __launch_bounds__(QM_THREADS) qm_kernel(QDev a, QDev b) {
  const QDev &p = blockIdx.x == 0 ? a : b;
  const int m = p.m;
  if (m <= 1) {
    if (m == 1 && threadIdx.x == 0) p.Q[0] = 1.f;
    return;
  }
  extern __shared__ double qm_sm[];
  double *V = qm_sm;                       // [r][c], m x QM_NB
  double *Cm = V + QM_MAX * QM_LD;         // [i][c], projection coefficients
  double *S = Cm + QM_MAX * QM_LD;         // [a][c], Gram matrix, then R
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  constexpr int NW = QM_THREADS / 32;
  // Box–Muller normals: G[r][c] with t = r*m + c
  for (int t = threadIdx.x; t < m * m; t += QM_THREADS) {
    const uint64_t x1 = sm64(p.kq + 2ull * t), x2 = sm64(p.kq + 2ull * t + 1ull);
    const double u1 = (double((x1 >> 11)) + 1.0) * 0x1.0p-53;
    const double u2 = double(x2 >> 11) * 0x1.0p-53;
    const int r = t / m, c = t % m;
    p.G[c * m + r] = sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
  }
  __syncthreads();
  for (int j0 = 0; j0 < m; j0 += QM_NB) {
    const int nb = min(QM_NB, m - j0);
    for (int t = threadIdx.x; t < m * QM_NB; t += QM_THREADS) {
      const int c = t / m, r = t % m;
      V[r * QM_LD + c] = c < nb ? p.G[(j0 + c) * m + r] : 0.0;
    }
    __syncthreads();
    for (int pass = 0; pass < 2 && j0 > 0; ++pass) {
      // Cm = Q_prevᵀ V: a warp per earlier column i, lanes over the rows;
      // the 16 sums are then reduced across the warp by halving, after
      // which lane l holds the sum for column (l >> 1) & 15
      for (int i = w; i < j0; i += NW) {
        const double *q = p.G + static_cast<int64_t>(i) * m;
        double acc[QM_NB];
#pragma unroll
        for (int c = 0; c < QM_NB; ++c) acc[c] = 0.0;
        for (int r = lane; r < m; r += 32) {
          const double qr = q[r];
#pragma unroll
          for (int c = 0; c < QM_NB; ++c) acc[c] = fma(qr, V[r * QM_LD + c], acc[c]);
        }
#pragma unroll
        for (int half = QM_NB / 2, bit = 16; half >= 1; half /= 2, bit /= 2) {
          const bool up = lane & bit;
#pragma unroll
          for (int k2 = 0; k2 < half; ++k2) {
            const double send = up ? acc[k2] : acc[k2 + half];
            const double keep = up ? acc[k2 + half] : acc[k2];
            acc[k2] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
          }
        }
        acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 1);
        if ((lane & 1) == 0) Cm[i * QM_LD + ((lane >> 1) & 15)] = acc[0];
      }
      __syncthreads();
      // V -= Q_prev Cm: a thread per (row, quarter of the columns)
      if (threadIdx.x < 4 * m) {
        const int cq = threadIdx.x / m, r = threadIdx.x % m;
        double s4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
        for (int i = 0; i < j0; ++i) {
          const double g = p.G[static_cast<int64_t>(i) * m + r];
          const double *cmi = Cm + i * QM_LD + 4 * cq;
#pragma unroll
          for (int c = 0; c < 4; ++c) s4[c] = fma(g, cmi[c], s4[c]);
        }
        double *vr = V + r * QM_LD + 4 * cq;
#pragma unroll
        for (int c = 0; c < 4; ++c) vr[c] -= s4[c];
      }
      __syncthreads();
    }
    for (int rep = 0; rep < 2; ++rep) {
      // S = VᵀV: four threads per entry, each over every fourth row
      {
        const int e = threadIdx.x >> 2, sl = threadIdx.x & 3;
        const int ra = e / QM_NB, rb = e % QM_NB;
        double s = 0.0;
        for (int r = sl; r < m; r += 4) s = fma(V[r * QM_LD + ra], V[r * QM_LD + rb], s);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        if (sl == 0) S[ra * QM_LD + rb] = s;
      }
      __syncthreads();
      // S = RᵀR in place (R upper, row k of R in row k of S), one warp; the
      // padding columns (nb..) get R = I
      if (w == 0) {
        const int cl = lane & 15;
        for (int k = 0; k < QM_NB; ++k) {
          if (k >= nb) {
            if (lane < QM_NB) S[k * QM_LD + cl] = cl == k ? 1.0 : 0.0;
            __syncwarp();
            continue;
          }
          const double d = sqrt(S[k * QM_LD + k]);
          __syncwarp();
          if (lane < QM_NB && cl > k && cl < nb) S[k * QM_LD + cl] /= d;
          if (lane == 0) S[k * QM_LD + k] = d;
          __syncwarp();
          // trailing update of rows k+1.. (columns > row)
          if (lane < QM_NB && cl > k && cl < nb) {
            const double rkc = S[k * QM_LD + cl];
            for (int a2 = k + 1; a2 <= cl; ++a2) S[a2 * QM_LD + cl] -= S[k * QM_LD + a2] * rkc;
          }
          __syncwarp();
        }
      }
      __syncthreads();
      // V <- V R^-1, a thread per row (forward substitution over columns)
      for (int r = threadIdx.x; r < m; r += QM_THREADS) {
        double *x = V + r * QM_LD;   // this thread's row, solved in place
        for (int c = 0; c < QM_NB; ++c) {
          double v = x[c];
          for (int k = 0; k < c; ++k) v = fma(-x[k], S[k * QM_LD + c], v);
          x[c] = v / S[c * QM_LD + c];
        }
      }
      __syncthreads();
    }
    for (int t = threadIdx.x; t < m * QM_NB; t += QM_THREADS) {
      const int c = t / m, r = t % m;
      if (c < nb) p.G[(j0 + c) * m + r] = V[r * QM_LD + c];
    }
    __syncthreads();
  }
  for (int t = threadIdx.x; t < m * m; t += QM_THREADS) {
    const int bb = t / m, bp = t % m;  // Q[b][b'] = column b', row b
    p.Q[t] = static_cast<float>(p.G[bp * m + bb]);
  }
}

// ------------------------------------------------------------- Hadamard helpers
// In-register Hadamard of R values (unnormalised).
template <int R>
__device__ __forceinline__ void fwht_reg(float (&r)[R]) {
#pragma unroll
  for (int s = 1; s < R; s <<= 1)
#pragma unroll
    for (int i = 0; i < R; ++i)
      if (!(i & s)) {
        const float u = r[i], w = r[i + s];
        r[i] = u + w;
        r[i + s] = u - w;
      }
}

// One radix-R round of a length-L Hadamard over n_vec vectors held in shared
// memory (element j of vector v at X[vbase(v) + j*stride]): combines the R
// elements a + i*h, i < R, for every a whose index bits h .. R*h-1 are clear.
template <int R, class VB>
__device__ void fwht_round(float *X, int n_vec, int L, int h, int stride, VB vbase) {
  const int groups = L / R;
  for (int idx = threadIdx.x; idx < groups * n_vec; idx += blockDim.x) {
    const int v = idx % n_vec, g = idx / n_vec;
    const int a = (g / h) * R * h + (g % h);
    float *x = X + vbase(v) + a * stride;
    float r[R];
#pragma unroll
    for (int i = 0; i < R; ++i) r[i] = x[i * h * stride];
    fwht_reg<R>(r);
#pragma unroll
    for (int i = 0; i < R; ++i) x[i * h * stride] = r[i];
  }
  __syncthreads();
}

// Remaining rounds of a length-L Hadamard whose distances below h are done.
template <class VB>
__device__ void fwht_rest(float *X, int n_vec, int L, int h, int stride, VB vbase) {
  while (h * 16 <= L) {
    fwht_round<16>(X, n_vec, L, h, stride, vbase);
    h *= 16;
  }
  const int rem = L / h;
  if (rem == 2) fwht_round<2>(X, n_vec, L, h, stride, vbase);
  else if (rem == 4) fwht_round<4>(X, n_vec, L, h, stride, vbase);
  else if (rem == 8) fwht_round<8>(X, n_vec, L, h, stride, vbase);
}

// ------------------------------------------------------------- row pass
// One CTA per (row, chunk of L*m contiguous columns) of an R x C matrix:
// out = norm * cr[row] * (Hhat_L ⊗ Q_m)(cc ⊙ x) on the chunk. The chunk lives
// in shared memory (element a*m + b); the first radix-16 Hadamard round runs
// in registers while loading, the Q_m mix runs while storing.
struct RowP {
  const void *in;
  float *out;
  int64_t ld_in, ld_out;
  int in_bf16;
  const float *cr, *cc;
  float norm;
  int L, m;
  const float *Q;  // m x m row-major, null when m == 1
  int64_t chunks;  // chunks per row
};

__device__ __forceinline__ float load_in(const void *p, int bf16, int64_t off) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[off])
              : reinterpret_cast<const float *>(p)[off];
}

template <int R0>
__device__ void row_load_round(const RowP &p, float *X, int64_t row, int64_t c0) {
  const int m = p.m, L = p.L;
  const float rf = p.norm * (p.cr ? p.cr[row] : 1.f);
  const int groups = L / R0;
  for (int idx = threadIdx.x; idx < groups * m; idx += blockDim.x) {
    const int b = idx % m, g = idx / m;
    float r[R0];
#pragma unroll
    for (int i = 0; i < R0; ++i) {
      const int e = (g * R0 + i) * m + b;
      float v = load_in(p.in, p.in_bf16, row * p.ld_in + c0 + e) * rf;
      if (p.cc) v *= p.cc[c0 + e];
      r[i] = v;
    }
    fwht_reg<R0>(r);
#pragma unroll
    for (int i = 0; i < R0; ++i) X[(g * R0 + i) * m + b] = r[i];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(512, 2) row_pass_kernel(RowP p) {
  extern __shared__ float X[];
  const int m = p.m, L = p.L, chunk = L * m;
  const int64_t row = blockIdx.x / p.chunks;
  const int64_t c0 = (blockIdx.x % p.chunks) * int64_t(chunk);
  auto vb = [=](int v) { return v; };
  int h;
  if (L >= 16) {
    row_load_round<16>(p, X, row, c0);
    h = 16;
  } else if (L == 8) {
    row_load_round<8>(p, X, row, c0);
    h = 8;
  } else if (L == 4) {
    row_load_round<4>(p, X, row, c0);
    h = 4;
  } else if (L == 2) {
    row_load_round<2>(p, X, row, c0);
    h = 2;
  } else {
    row_load_round<1>(p, X, row, c0);
    h = 1;
  }
  fwht_rest(X, m, L, h, m, vb);
  float *o = p.out + row * p.ld_out + c0;
  if (p.Q == nullptr) {
    for (int e = threadIdx.x; e < chunk; e += blockDim.x) o[e] = X[e];
    return;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if (m <= 32 && (m % 4) == 0) {
    // lane b owns output b of every group; its row of Q_m stays in registers;
    // two groups per iteration, inputs read as float4 broadcasts
    float q[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) q[k] = (lane < m && k < m) ? p.Q[lane * m + k] : 0.f;
    for (int a = 2 * warp; a < L; a += 2 * nw) {
      const bool two = a + 1 < L;
      const float4 *x0 = reinterpret_cast<const float4 *>(X + a * m);
      const float4 *x1 = reinterpret_cast<const float4 *>(X + (two ? a + 1 : a) * m);
      float y0 = 0.f, y1 = 0.f;
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4) {
        if (4 * k4 < m) {
          const float4 u = x0[k4], v = x1[k4];
          y0 = fmaf(q[4 * k4], u.x, y0);
          y0 = fmaf(q[4 * k4 + 1], u.y, y0);
          y0 = fmaf(q[4 * k4 + 2], u.z, y0);
          y0 = fmaf(q[4 * k4 + 3], u.w, y0);
          y1 = fmaf(q[4 * k4], v.x, y1);
          y1 = fmaf(q[4 * k4 + 1], v.y, y1);
          y1 = fmaf(q[4 * k4 + 2], v.z, y1);
          y1 = fmaf(q[4 * k4 + 3], v.w, y1);
        }
      }
      if (lane < m) {
        o[a * m + lane] = y0;
        if (two) o[(a + 1) * m + lane] = y1;
      }
    }
  } else if (m <= 32) {
    float q[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) q[k] = (lane < m && k < m) ? p.Q[lane * m + k] : 0.f;
    for (int a = warp; a < L; a += nw) {
      const float *x = X + a * m;
      float y = 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k)
        if (k < m) y = fmaf(q[k], x[k], y);
      if (lane < m) o[a * m + lane] = y;
    }
  } else {
    // lanes own outputs b = lane + 32j; Q_m read from global (cached)
    for (int a = warp; a < L; a += nw) {
      const float *x = X + a * m;
      for (int b = lane; b < m; b += 32) {
        const float *qr = p.Q + b * m;
        float y = 0.f;
        for (int k = 0; k < m; ++k) y = fmaf(__ldg(qr + k), x[k], y);
        o[a * m + b] = y;
      }
    }
  }
}

// ------------------------------------------------------------- row-side Q_m
// out[(a*m + b)][c] = sum_k Q[b][k] * in[(a*m + k)][c] for groups of m
// consecutive rows; one thread per column, in place.
__global__ void __launch_bounds__(256)
    rowq_kernel(float *M, int64_t ld, int64_t C, int m, const float *Q) {
  extern __shared__ float sm[];  // Q (m*m), then a [m][64] tile when m > 32
  for (int e = threadIdx.x; e < m * m; e += blockDim.x) {
    sm[e] = Q[e];
    if (m <= 32) sm[m * m + (e % m) * m + e / m] = Q[e];  // Qᵀ
  }
  __syncthreads();
  const int64_t a = blockIdx.y;
  float *base = M + a * m * ld;
  if (m <= 32) {
    const int64_t c = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    if (c >= C) return;
    float x[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) x[k] = k < m ? base[k * ld + c] : 0.f;
    if (m % 4 == 0) {
      // Qᵀ (k-major) in shared memory: 4 outputs per float4 broadcast
      const float4 *qt = reinterpret_cast<const float4 *>(sm + m * m);
      for (int b0 = 0; b0 < m; b0 += 4) {
        float y0 = 0.f, y1 = 0.f, y2 = 0.f, y3 = 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          if (k < m) {
            const float4 qv = qt[(k * m + b0) / 4];
            y0 = fmaf(qv.x, x[k], y0);
            y1 = fmaf(qv.y, x[k], y1);
            y2 = fmaf(qv.z, x[k], y2);
            y3 = fmaf(qv.w, x[k], y3);
          }
        }
        base[b0 * ld + c] = y0;
        base[(b0 + 1) * ld + c] = y1;
        base[(b0 + 2) * ld + c] = y2;
        base[(b0 + 3) * ld + c] = y3;
      }
    } else {
      for (int b = 0; b < m; ++b) {
        const float *qr = sm + b * m;
        float y = 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (k < m) y = fmaf(qr[k], x[k], y);
        base[b * ld + c] = y;
      }
    }
  } else {
    float *T = sm + m * m;  // [m][64]
    const int64_t c0 = blockIdx.x * int64_t(64);
    for (int e = threadIdx.x; e < m * 64; e += blockDim.x) {
      const int k = e / 64, c = e % 64;
      T[e] = (c0 + c < C) ? base[k * ld + c0 + c] : 0.f;
    }
    __syncthreads();
    const int c = threadIdx.x % 64, bq = threadIdx.x / 64;
    if (c0 + c < C) {
      for (int b = bq; b < m; b += blockDim.x / 64) {
        const float *qr = sm + b * m;
        float y = 0.f;
        for (int k = 0; k < m; ++k) y = fmaf(qr[k], T[k * 64 + c], y);
        base[b * ld + c0 + c] = y;
      }
    }
  }
}

// ------------------------------------------------------------- strided pass
// Vector form: cw contiguous columns as float4 lanes; the first Hadamard round
// runs in registers while loading, the last one while storing, and only the
// rounds in between touch shared memory. Needs 16-byte aligned rows.
template <int R>
__device__ __forceinline__ void fwht_reg4(float4 (&r)[R]) {
#pragma unroll
  for (int s = 1; s < R; s <<= 1)
#pragma unroll
    for (int i = 0; i < R; ++i)
      if (!(i & s)) {
        const float4 u = r[i], w = r[i + s];
        r[i] = make_float4(u.x + w.x, u.y + w.y, u.z + w.z, u.w + w.w);
        r[i + s] = make_float4(u.x - w.x, u.y - w.y, u.z - w.z, u.w - w.w);
      }
}

template <int R>
__device__ void round4_load(float4 *X, const float4 *g, int A, int c4n, int64_t smid4,
                            int w4) {
  const int groups = A / R;
  for (int idx = threadIdx.x; idx < groups * c4n; idx += blockDim.x) {
    const int c = idx % c4n, gi = idx / c4n;
    float4 r[R];
#pragma unroll
    for (int i = 0; i < R; ++i)
      r[i] = c < w4 ? g[int64_t(gi * R + i) * smid4 + c] : make_float4(0.f, 0.f, 0.f, 0.f);
    fwht_reg4<R>(r);
#pragma unroll
    for (int i = 0; i < R; ++i) X[(gi * R + i) * c4n + c] = r[i];
  }
  __syncthreads();
}

template <int R>
__device__ void round4_smem(float4 *X, int A, int h, int c4n) {
  const int groups = A / R;
  for (int idx = threadIdx.x; idx < groups * c4n; idx += blockDim.x) {
    const int c = idx % c4n, g = idx / c4n;
    const int a = (g / h) * R * h + (g % h);
    float4 r[R];
#pragma unroll
    for (int i = 0; i < R; ++i) r[i] = X[(a + i * h) * c4n + c];
    fwht_reg4<R>(r);
#pragma unroll
    for (int i = 0; i < R; ++i) X[(a + i * h) * c4n + c] = r[i];
  }
  __syncthreads();
}

template <int R>
__device__ void round4_store(const float4 *X, float4 *g, int A, int h, int c4n,
                             int64_t smid4, int w4) {
  const int groups = A / R;
  for (int idx = threadIdx.x; idx < groups * c4n; idx += blockDim.x) {
    const int c = idx % c4n, gg = idx / c4n;
    const int a = (gg / h) * R * h + (gg % h);
    float4 r[R];
#pragma unroll
    for (int i = 0; i < R; ++i) r[i] = X[(a + i * h) * c4n + c];
    fwht_reg4<R>(r);
    if (c < w4) {
#pragma unroll
      for (int i = 0; i < R; ++i) g[int64_t(a + i * h) * smid4 + c] = r[i];
    }
  }
}

__global__ void __launch_bounds__(512)
    strided_fwht4_kernel(float *base, int64_t so, int64_t n1, int64_t so2, int A,
                         int64_t smid, int64_t inner, int cw, int64_t chunks) {
  extern __shared__ float4 X4[];
  const int64_t o = blockIdx.x / chunks, ch = blockIdx.x % chunks;
  const int64_t c0 = ch * cw;
  const int w4 = static_cast<int>(kq_min<int64_t>(cw, inner - c0)) / 4;
  float4 *g = reinterpret_cast<float4 *>(base + (o % n1) * so + (o / n1) * so2 + c0);
  const int c4n = cw / 4;
  const int64_t smid4 = smid / 4;
  const int R0 = A >= 16 ? 16 : A;
  switch (R0) {
    case 16: round4_load<16>(X4, g, A, c4n, smid4, w4); break;
    case 8: round4_load<8>(X4, g, A, c4n, smid4, w4); break;
    case 4: round4_load<4>(X4, g, A, c4n, smid4, w4); break;
    case 2: round4_load<2>(X4, g, A, c4n, smid4, w4); break;
    default: round4_load<1>(X4, g, A, c4n, smid4, w4); break;
  }
  int h = R0;
  while (A / h > 16) {
    round4_smem<16>(X4, A, h, c4n);
    h *= 16;
  }
  switch (A / h) {
    case 16: round4_store<16>(X4, g, A, h, c4n, smid4, w4); break;
    case 8: round4_store<8>(X4, g, A, h, c4n, smid4, w4); break;
    case 4: round4_store<4>(X4, g, A, h, c4n, smid4, w4); break;
    case 2: round4_store<2>(X4, g, A, h, c4n, smid4, w4); break;
    default: round4_store<1>(X4, g, A, h, c4n, smid4, w4); break;
  }
}

// Scalar form of the strided pass (any alignment).

// View [outer][A][inner] at strides (so, smid, 1); Hadamard (unnormalised) of
// length A along the middle axis; one [A][cw] slab per CTA, first radix-16
// round in registers while loading.
__global__ void __launch_bounds__(512)
    strided_fwht_kernel(float *base, int64_t so, int64_t n1, int64_t so2, int A,
                        int64_t smid, int64_t inner, int cw, int64_t chunks) {
  extern __shared__ float X[];
  const int64_t o = blockIdx.x / chunks, ch = blockIdx.x % chunks;
  const int64_t c0 = ch * cw;
  const int w = static_cast<int>(kq_min<int64_t>(cw, inner - c0));
  float *g = base + (o % n1) * so + (o / n1) * so2 + c0;
  const int R0 = A >= 16 ? 16 : A;
  const int groups = A / R0;
  for (int idx = threadIdx.x; idx < groups * cw; idx += blockDim.x) {
    const int c = idx % cw, gi = idx / cw;
    float r[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i < R0) r[i] = c < w ? g[int64_t(gi * R0 + i) * smid + c] : 0.f;
    if (R0 == 16) fwht_reg<16>(*reinterpret_cast<float(*)[16]>(r));
    else if (R0 == 8) fwht_reg<8>(*reinterpret_cast<float(*)[8]>(r));
    else if (R0 == 4) fwht_reg<4>(*reinterpret_cast<float(*)[4]>(r));
    else if (R0 == 2) fwht_reg<2>(*reinterpret_cast<float(*)[2]>(r));
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (i < R0) X[(gi * R0 + i) * cw + c] = r[i];
  }
  __syncthreads();
  fwht_rest(X, cw, A, R0, cw, [](int v) { return v; });
  for (int e = threadIdx.x; e < A * cw; e += blockDim.x) {
    const int a = e / cw, c = e % cw;
    if (c < w) g[int64_t(a) * smid + c] = X[e];
  }
}

// ------------------------------------------------------------- column pass
// The whole row side of a rotation in one read and one write of the matrix:
// for every column x of an R x C row-major matrix (R = had * m),
//   x <- (Hhat_had ⊗ Q_m) x      (Hadamard unnormalised; the row pass has
//                                 applied the row factors and the norm)
// in place. A strip of 4*W4 contiguous columns is held, over all R rows, in
// the shared memory of a cluster of K CTAs: CTA k holds rows
// [k*RK, (k+1)*RK), RK = (had/K)*m, i.e. Hadamard index a in
// [k*had/K, (k+1)*had/K). Each CTA mixes its groups of m rows with Q_m and
// runs the Hadamard over its local low bits of a; after a cluster barrier the
// high log2(K) bits are one K-point Hadamard across the CTAs, read through
// distributed shared memory, and each CTA writes its share of the positions
// for all K row blocks straight to global memory.
constexpr int CP_THREADS = 256;
constexpr int CP_BUDGET = 112 * 1024;   // dynamic shared memory per CTA (2 per SM)

struct ColP {
  float *M;
  int64_t ld, C;
  int had, m, W4;   // W4: float4 columns per strip
  int box;          // rows per TMA box (divides the rows a CTA holds)
  const float *Q;   // m x m row-major (m > 1, m % 4 == 0), else null
  int32_t *info;
  // diagonal factors applied on the way in (x[r][c] * fr[r] * fc[c]), null
  // for none; only the Q_28 MMA mix applies them
  const float *fr, *fc;
};

// y = Q x for each group of m rows, one thread per (group, column pair); x is
// held in registers, Q rows are read as float4 broadcasts through L1.
__device__ void colpass_qmix(float *X, int AL, int m, int W4, const float *Q) {
  const int W2 = 2 * W4, W = 4 * W4;
  const float4 *Q4 = reinterpret_cast<const float4 *>(Q);
  const int m4 = m / 4;
  for (int t = threadIdx.x; t < AL * W2; t += CP_THREADS) {
    const int al = t / W2, c2 = t % W2;
    float2 *base = reinterpret_cast<float2 *>(X + static_cast<int64_t>(al) * m * W) + c2;
    float2 x[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) x[k] = k < m ? base[k * W2] : make_float2(0.f, 0.f);
    for (int b = 0; b < m; ++b) {
      const float4 *qr = Q4 + b * m4;
      float2 y = make_float2(0.f, 0.f);
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4) {
        if (k4 < m4) {
          const float4 q = __ldg(qr + k4);
          y.x = fmaf(q.x, x[4 * k4].x, y.x);
          y.y = fmaf(q.x, x[4 * k4].y, y.y);
          y.x = fmaf(q.y, x[4 * k4 + 1].x, y.x);
          y.y = fmaf(q.y, x[4 * k4 + 1].y, y.y);
          y.x = fmaf(q.z, x[4 * k4 + 2].x, y.x);
          y.y = fmaf(q.z, x[4 * k4 + 2].y, y.y);
          y.x = fmaf(q.w, x[4 * k4 + 3].x, y.x);
          y.y = fmaf(q.w, x[4 * k4 + 3].y, y.y);
        }
      }
      base[b * W2] = y;
    }
  }
  __syncthreads();
}

// ---- Q_28 mix on the tensor cores (warp MMA m16n8k8, TF32 in three parts)
// fp32 accuracy from TF32 MMAs: x = hi + lo with hi, lo TF32 (rounded to
// nearest), and a*b ~ a_hi*b_hi + a_hi*b_lo + a_lo*b_hi (the dropped a_lo*b_lo
// is below 2^-22 |a b|).
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
  hi = to_tf32(x);
  lo = to_tf32(x - __uint_as_float(hi));
}
// c (16 x 8, fp32) += a (16 x 8, tf32) * b (8 x 8, tf32); per lane (group g =
// lane / 4, t = lane % 4): a = {A[g][t], A[g+8][t], A[g][t+4], A[g+8][t+4]},
// b = {B[t][g], B[t+4][g]}, c = {C[g][2t], C[g][2t+1], C[g+8][2t], C[g+8][2t+1]}.
__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// c (16 x 8) += a (16 x 4) * b (4 x 8), TF32: a = {A[g][t], A[g+8][t]},
// b = {B[t][g]} (the k = 4 shape, for the last 4 of 28)
__device__ __forceinline__ void mma_tf32_k4(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k4.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, "
      "{%4, %5}, {%6}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

// Y = Q X for every group of 28 rows of a strip of W = 8*NTN columns in
// shared memory (X[(g*28 + b)*W + c]), in place: a warp takes whole groups,
// Q (rows padded to 32 with zeros) sits in registers as A fragments, the
// group's 28 x W block supplies the B fragments; k runs as three steps of 8
// and one of 4. With fr / fc (this CTA's rows / the strip's columns) the
// block is scaled on the way in: B = fr[g*28 + k] * X * fc[c].
template <int NT = CP_THREADS, int NTN = 2>
__device__ void colpass_qmix_mma28(float *X, int AL, const float *Q,
                                   const float *fr = nullptr, const float *fc = nullptr) {
  constexpr int W = 8 * NTN;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  constexpr int NWARP = NT / 32;
  float fcol[NTN];
#pragma unroll
  for (int nt = 0; nt < NTN; ++nt) fcol[nt] = fc ? __ldg(fc + nt * 8 + gq) : 1.f;
  uint32_t ah[2][4][4], alo[2][4][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = mt * 16 + gq + ((e & 1) ? 8 : 0);
        const int c = ks * 8 + tq + ((e & 2) ? 4 : 0);
        const float q = (r < 28 && c < 28) ? __ldg(Q + r * 28 + c) : 0.f;
        split_tf32(q, ah[mt][ks][e], alo[mt][ks][e]);
      }
  for (int g = warp; g < AL; g += NWARP) {
    float *xg = X + g * 28 * W;
    float acc[2][NTN][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const int k0 = ks * 8 + tq, k1 = k0 + 4;   // k1 < 28 unless ks == 3
      uint32_t b0h[NTN], b0l[NTN], b1h[NTN], b1l[NTN];
      float r0 = 1.f, r1 = 1.f;
      if (fr) {
        r0 = __ldg(fr + g * 28 + k0);
        if (ks < 3) r1 = __ldg(fr + g * 28 + k1);
      }
#pragma unroll
      for (int nt = 0; nt < NTN; ++nt) {
        const int col = nt * 8 + gq;
        split_tf32(xg[k0 * W + col] * r0 * fcol[nt], b0h[nt], b0l[nt]);
        if (ks < 3) split_tf32(xg[k1 * W + col] * r1 * fcol[nt], b1h[nt], b1l[nt]);
      }
      // the three parts in turn over all accumulators (independent MMAs
      // back to back)
      if (ks < 3) {
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) mma_tf32(acc[mt][nt], alo[mt][ks], b0h[nt], b1h[nt]);
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) mma_tf32(acc[mt][nt], ah[mt][ks], b0l[nt], b1l[nt]);
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) mma_tf32(acc[mt][nt], ah[mt][ks], b0h[nt], b1h[nt]);
      } else {
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
            mma_tf32_k4(acc[mt][nt], alo[mt][3][0], alo[mt][3][1], b0h[nt]);
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
            mma_tf32_k4(acc[mt][nt], ah[mt][3][0], ah[mt][3][1], b0l[nt]);
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt)
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
            mma_tf32_k4(acc[mt][nt], ah[mt][3][0], ah[mt][3][1], b0h[nt]);
      }
    }
    __syncwarp();  // the whole block is read before any lane writes it
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < NTN; ++nt) {
        const int r0 = mt * 16 + gq, n = nt * 8 + 2 * tq;
        if (r0 < 28)
          *reinterpret_cast<float2 *>(xg + r0 * W + n) =
              make_float2(acc[mt][nt][0], acc[mt][nt][1]);
        if (r0 + 8 < 28)
          *reinterpret_cast<float2 *>(xg + (r0 + 8) * W + n) =
              make_float2(acc[mt][nt][2], acc[mt][nt][3]);
      }
    __syncwarp();
  }
  __syncthreads();
}

template <int K>
__global__ void __launch_bounds__(CP_THREADS, 2)
    colpass_kernel(const __grid_constant__ CUtensorMap tm, ColP p) {
  extern __shared__ __align__(128) float4 X4[];
  const int rank = K > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int64_t strip = blockIdx.x / K;
  const int m = p.m, W4 = p.W4;
  const int AL = p.had / K, RK = AL * m;
  const int nvec = RK * W4;
  uint64_t *bar = reinterpret_cast<uint64_t *>(X4 + nvec);
  int *abort_flag = reinterpret_cast<int *>(bar + 1);
  const int64_t row0 = static_cast<int64_t>(rank) * RK;
  const int64_t c0 = strip * 4 * W4;
  // 1. the CTA's row block of the strip, by TMA (columns beyond C read as 0)
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar, 1);
    fence_mbar_init();
    prefetch_tmap(&tm);
    mbar_expect_tx(bar, static_cast<uint32_t>(nvec) * 16u);
    for (int r = 0; r < RK; r += p.box)
      tma_load_2d(X4 + r * W4, &tm, bar, static_cast<int32_t>(c0),
                  static_cast<int32_t>(row0 + r));
  }
  __syncthreads();
  const bool landed = mbar_wait(bar, 0, abort_flag);
  const int good = __syncthreads_and(landed);
  if (!good && threadIdx.x == 0) report(p.info, KRONQ_ERR_TIMEOUT);
  if (good) {
    // 2. Q_m over each group of m consecutive rows
    if (m == 28 && W4 == 4)
      colpass_qmix_mma28<CP_THREADS, 2>(reinterpret_cast<float *>(X4), AL, p.Q,
                                        p.fr ? p.fr + row0 : nullptr,
                                        p.fc ? p.fc + c0 : nullptr);
    else if (m == 28 && W4 == 2)
      colpass_qmix_mma28<CP_THREADS, 1>(reinterpret_cast<float *>(X4), AL, p.Q,
                                        p.fr ? p.fr + row0 : nullptr,
                                        p.fc ? p.fc + c0 : nullptr);
    else if (m > 1)
      colpass_qmix(reinterpret_cast<float *>(X4), AL, m, W4, p.Q);
    // 3. Hadamard over the local bits of a (rows al*m + b, stride m rows)
    if (AL > 1) {
      int h = 1;
      while (AL / h >= 16) {
        round4_smem<16>(X4, AL, h, m * W4);
        h *= 16;
      }
      switch (AL / h) {
        case 8: round4_smem<8>(X4, AL, h, m * W4); break;
        case 4: round4_smem<4>(X4, AL, h, m * W4); break;
        case 2: round4_smem<2>(X4, AL, h, m * W4); break;
        default: break;
      }
    }
  }
  // 4. the high bits of a: a K-point Hadamard across the cluster (every CTA
  // takes the same barriers, also after a timeout)
  if (K > 1) cluster_sync_all();
  if (good) {
    const int per = (nvec + K - 1) / K;
    const int p0 = rank * per, p1 = min(nvec, p0 + per);
    const uint32_t xs = smem_u32(X4);
    for (int q = p0 + threadIdx.x; q < p1; q += CP_THREADS) {
      float4 v[K];
#pragma unroll
      for (int j = 0; j < K; ++j)
        v[j] = (K == 1 || j == rank) ? X4[q]
                                     : ld_dsmem_f4(mapa_shared(xs + 16u * q, j));
      fwht_reg4<K>(v);
      const int r = q / W4, c4 = q % W4;
      const int64_t col = c0 + 4 * c4;
      if (col < p.C) {
#pragma unroll
        for (int j = 0; j < K; ++j)
          __stcs(reinterpret_cast<float4 *>(p.M + (static_cast<int64_t>(j) * RK + r) * p.ld + col),
                 v[j]);
      }
    }
  }
  // no CTA leaves while another may still read its shared memory
  if (K > 1) cluster_sync_all();
  if (!good && threadIdx.x == 0) {
    // let a late copy land before the shared memory is released
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, 0) && globaltimer() - t0 < kWaitLimitNs) {
    }
  }
}

template <int K, int M, int AL, int W4 = 4>
__global__ void __launch_bounds__(CP_THREADS, 2)
    colpass_tpl_kernel(const __grid_constant__ CUtensorMap tm, ColP p);

// Plans and launches the column pass; returns KRONQ_ERR_UNSUPPORTED when the
// shape does not fit it (the caller then takes the two-pass route).
kronq_status launch_colpass(cudaStream_t st, float *M, int64_t ld, int64_t R,
                            int64_t C, int64_t had, int64_t m, const float *Q,
                            int32_t *info, const float *fr = nullptr,
                            const float *fc = nullptr) {
  if (m > 32 || (m > 1 && (m % 4 != 0 || Q == nullptr)) || had < 1 || had * m != R)
    return KRONQ_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(M) % 16 || ld % 4 || C % 4)
    return KRONQ_ERR_UNSUPPORTED;
  int W4 = 0, K = 0;
  for (int w4 : {4, 2, 1}) {
    int k = 1;
    while (static_cast<int64_t>(k) * CP_BUDGET < R * w4 * 16) k *= 2;
    if (k <= 16 && k <= had) {
      W4 = w4;
      K = k;
      break;
    }
  }
  if (K == 0) return KRONQ_ERR_UNSUPPORTED;
  // Q_28 with 16-CTA clusters: 8-CTA clusters of 8-column strips fit more
  // clusters at once (33 against 14 at 28672 rows; 5 % faster there)
  if (m == 28 && K == 16 && W4 == 4 && R * 2 * 16 <= 8 * static_cast<int64_t>(CP_BUDGET) &&
      C % 8 == 0) {
    K = 8;
    W4 = 2;
  }
  // factors ride on the Q_28 MMA mix of whole strips only
  if ((fr || fc) && !(m == 28 && (W4 == 4 || W4 == 2) && C % (4 * W4) == 0))
    return KRONQ_ERR_UNSUPPORTED;
  const int64_t strips = ceil_div(C, 4 * W4);
  if (strips * K > 0x7fffffff) return KRONQ_ERR_UNSUPPORTED;
  const int64_t AL = had / K, RK = AL * m;
  // rows per TMA box: a divisor of RK of at most 256
  int64_t box = 1;
  if (RK <= 256) {
    box = RK;
  } else if (RK % 256 == 0) {
    box = 256;
  } else {
    for (int64_t dv = 1; dv <= m; ++dv)
      if (m % dv == 0 && AL * dv <= 256) box = kq_max(box, AL * dv);
  }
  CUtensorMap tm;
  KQ_TRY(make_tmap_2d(&tm, M, false, static_cast<uint64_t>(C), static_cast<uint64_t>(R),
                      static_cast<uint64_t>(ld), static_cast<uint32_t>(4 * W4),
                      static_cast<uint32_t>(box), TMAP_NONE));
  const int smem = static_cast<int>(RK * W4 * 16 + 64);
  ColP p{M, ld, C, static_cast<int>(had), static_cast<int>(m), W4, static_cast<int>(box), Q,
         info, fr, fc};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(strips * K));
  cfg.blockDim = dim3(CP_THREADS);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(K);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = K > 1 ? 1 : 0;
  auto go = [&](auto kern) -> kronq_status {
    KQ_TRY(smem_attr(kern, CP_BUDGET + 64));
    if (K > 8) KQ_TRY(nonportable_cluster_attr(kern));
    KQ_CUDA(cudaLaunchKernelEx(&cfg, kern, tm, p));
    count_launch();
    return KRONQ_OK;
  };
  if (W4 == 2 && K == 8 && m == 28 && AL == 128) return go(colpass_tpl_kernel<8, 28, 128, 2>);
  if (W4 == 4) {  // the compiled fixed shapes
#define KQ_COL_SHAPE(KK, MM, AA)                                              \
  if (K == KK && m == MM && AL == AA) return go(colpass_tpl_kernel<KK, MM, AA>);
    KQ_COL_SHAPE(16, 28, 64)
    KQ_COL_SHAPE(16, 1, 1024)
    KQ_COL_SHAPE(8, 1, 1024)
    KQ_COL_SHAPE(4, 1, 1024)
    KQ_COL_SHAPE(2, 1, 1024)
    KQ_COL_SHAPE(1, 1, 1024)
    KQ_COL_SHAPE(1, 1, 512)
    KQ_COL_SHAPE(1, 1, 256)
#undef KQ_COL_SHAPE
  }
  switch (K) {
    case 1: return go(colpass_kernel<1>);
    case 2: return go(colpass_kernel<2>);
    case 4: return go(colpass_kernel<4>);
    case 8: return go(colpass_kernel<8>);
    default: return go(colpass_kernel<16>);
  }
}

// ------------------------------------------------------------- fixed shapes
// The shapes of the pages' sublayers (row chunks of L*M floats with M = 1 or
// 28; column strips over R = had*M rows) with every size a compile-time
// constant: the index arithmetic of the inner loops is shifts and multiplies,
// and the Hadamard runs in rounds of radix 32.

// Radix of the next round when n Hadamard points remain (at most rmax):
// everything at once when n <= rmax, else balanced rounds.
__host__ __device__ constexpr int radix_for(int n, int rmax) {
  if (n <= rmax) return n;
  if (n > rmax * rmax) return rmax;
  int r = 1;
  while (r * r < n) r *= 2;
  return r;
}

template <int L, int H>
struct RadixAt {
  static constexpr int R = radix_for(L / H, 32);
};

// distance of the last round of that plan, from distance 1 upward
__host__ __device__ constexpr int last_round_h(int L) {
  int h = 1;
  while (true) {
    const int r = radix_for(L / h, 32);
    if (h * r >= L) return h;
    h *= r;
  }
}

// One round of radix R at distance H over the a-index of an L x M chunk in
// shared memory (element a*M + b), tasks (g, b).
template <int L, int M, int R, int H, int NT>
__device__ __forceinline__ void tround(float *X) {
  constexpr int T = (L / R) * M;
  for (int t = threadIdx.x; t < T; t += NT) {
    const int b = t % M, g = t / M;
    const int a = (g / H) * R * H + (g % H);
    float *x = X + a * M + b;
    float r[R];
#pragma unroll
    for (int i = 0; i < R; ++i) r[i] = x[i * H * M];
    fwht_reg<R>(r);
#pragma unroll
    for (int i = 0; i < R; ++i) x[i * H * M] = r[i];
  }
  __syncthreads();
}

// Rounds from distance H up to (but not including) distance HEND.
template <int L, int M, int H, int HEND, int NT>
__device__ __forceinline__ void trounds(float *X) {
  if constexpr (H < HEND) {
    constexpr int R = RadixAt<L, H>::R;
    tround<L, M, R, H, NT>(X);
    trounds<L, M, H * R, HEND, NT>(X);
  }
}

template <bool BF16>
__device__ __forceinline__ float4 load4(const void *base, int64_t off) {
  if constexpr (BF16) {
    const uint2 u = __ldcs(reinterpret_cast<const uint2 *>(
        reinterpret_cast<const __nv_bfloat16 *>(base) + off));
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
    const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
  } else {
    return __ldcs(reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + off));
  }
}

template <bool BF16>
__device__ __forceinline__ float load1(const void *base, int64_t off) {
  if constexpr (BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base)[off]);
  else return __ldcs(reinterpret_cast<const float *>(base) + off);
}

// Row pass, one CTA per row chunk of L*M contiguous columns:
// out = norm * cr[row] * (Hhat_L ⊗ Q_M)(cc ⊙ x) (unnormalised Hadamard times
// norm). M == 1 (512 threads): vector loads into shared memory, the last
// Hadamard round fused with the store. M == 28 (256 threads): the first round
// (radix 32) fused with the loads; the Q_28 mix on the tensor cores on the way
// out, Y = X Q^T with the chunk as the A operand (L x 28, row-major in shared
// memory) and Q^T in registers as B fragments, each lane storing its pairs of
// outputs.
template <int M>
struct RowThreads {
  static constexpr int N = M == 1 ? 512 : 256;
};

template <int L, int M, bool BF16>
__global__ void __launch_bounds__(RowThreads<M>::N, 2) row_tpl_kernel(RowP p) {
  extern __shared__ float X[];
  constexpr int NT = RowThreads<M>::N;
  constexpr int CH = L * M;
  const int64_t row = blockIdx.x / p.chunks;
  const int64_t c0 = (blockIdx.x % p.chunks) * CH;
  const float rf = p.norm * (p.cr ? p.cr[row] : 1.f);
  const float *cc = p.cc ? p.cc + c0 : nullptr;
  const int64_t in0 = row * p.ld_in + c0;
  float *o = p.out + row * p.ld_out + c0;
  if constexpr (M == 1) {
    float4 *X4 = reinterpret_cast<float4 *>(X);
    for (int e4 = threadIdx.x; e4 < CH / 4; e4 += NT) {
      float4 v = load4<BF16>(p.in, in0 + 4 * e4);
      float4 f = make_float4(rf, rf, rf, rf);
      if (cc) {
        const float4 c = __ldg(reinterpret_cast<const float4 *>(cc) + e4);
        f = make_float4(rf * c.x, rf * c.y, rf * c.z, rf * c.w);
      }
      X4[e4] = make_float4(v.x * f.x, v.y * f.y, v.z * f.z, v.w * f.w);
    }
    __syncthreads();
    constexpr int HL = last_round_h(L);
    constexpr int RL = L / HL;
    trounds<L, 1, 1, HL, NT>(X);
    for (int t = threadIdx.x; t < L / RL; t += NT) {
      const int a = (t / HL) * RL * HL + (t % HL);
      float r[RL];
#pragma unroll
      for (int i = 0; i < RL; ++i) r[i] = X[a + i * HL];
      fwht_reg<RL>(r);
#pragma unroll
      for (int i = 0; i < RL; ++i) o[a + i * HL] = r[i];
    }
  } else {
    static_assert(M == 28 && L % 16 == 0, "the fixed-shape row pass takes M = 28");
    constexpr int R0 = L >= 32 ? 32 : L;
    for (int t = threadIdx.x; t < (L / R0) * M; t += NT) {
      const int b = t % M, g = t / M;
      const int e0 = g * R0 * M + b;
      float r[R0];
#pragma unroll
      for (int i = 0; i < R0; ++i) {
        const int e = e0 + i * M;
        float v = load1<BF16>(p.in, in0 + e) * rf;
        if (cc) v *= __ldg(cc + e);
        r[i] = v;
      }
      fwht_reg<R0>(r);
#pragma unroll
      for (int i = 0; i < R0; ++i) X[e0 + i * M] = r[i];
    }
    __syncthreads();
    trounds<L, M, R0, L, NT>(X);
    // Q_28 mix: B = Q^T (k x n) padded to 32 x 32, hi and lo parts
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    uint32_t bh[4][4][2], bl[4][4][2];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int n = nt * 8 + gq, k = ks * 8 + tq + 4 * e;
          const float q = (n < 28 && k < 28) ? __ldg(p.Q + n * 28 + k) : 0.f;
          split_tf32(q, bh[nt][ks][e], bl[nt][ks][e]);
        }
    constexpr int NW = NT / 32;
    for (int mt = warp; mt < L / 16; mt += NW) {
      float acc[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
      const float *xa = X + (mt * 16 + gq) * 28;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int k0 = ks * 8 + tq, k1 = k0 + 4;
        uint32_t ah[4], al[4];
        split_tf32(xa[k0], ah[0], al[0]);
        split_tf32(xa[8 * 28 + k0], ah[1], al[1]);
        split_tf32(k1 < 28 ? xa[k1] : 0.f, ah[2], al[2]);
        split_tf32(k1 < 28 ? xa[8 * 28 + k1] : 0.f, ah[3], al[3]);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_tf32(acc[nt], al, bh[nt][ks][0], bh[nt][ks][1]);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_tf32(acc[nt], ah, bl[nt][ks][0], bl[nt][ks][1]);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_tf32(acc[nt], ah, bh[nt][ks][0], bh[nt][ks][1]);
      }
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int n = nt * 8 + 2 * tq;
        if (n < 28) {
          const int a0 = mt * 16 + gq;
          *reinterpret_cast<float2 *>(o + a0 * 28 + n) = make_float2(acc[nt][0], acc[nt][1]);
          *reinterpret_cast<float2 *>(o + (a0 + 8) * 28 + n) =
              make_float2(acc[nt][2], acc[nt][3]);
        }
      }
    }
  }
}

// Row pass for fp32 rows of L x 28 with the next rows in flight: one
// persistent CTA per SM holds two row buffers; while one row goes through
// the factors, the Hadamard rounds and the Q_28 mix (warp MMA, stored
// straight to global memory), the bulk copy of a later row lands in the
// other buffer. Qᵀ sits in registers as B fragments for the life of the CTA.
constexpr int RP_THREADS = 512;
int sm_count();

template <int L>
__global__ void __launch_bounds__(RP_THREADS, 1)
    row_pipe28_kernel(RowP p, int64_t items, int32_t *info) {
  extern __shared__ __align__(128) float rp_sm[];
  constexpr int M = 28, CH = L * M, NT = RP_THREADS, NW = NT / 32;
  constexpr uint32_t BYTES = CH * 4;
  uint64_t *full = reinterpret_cast<uint64_t *>(rp_sm + 2 * CH);
  int *abort_flag = reinterpret_cast<int *>(full + 2);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  auto src = [&](int64_t item) {
    return static_cast<const float *>(p.in) + (item / p.chunks) * p.ld_in +
           (item % p.chunks) * CH;
  };
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_mbar_init();
    for (int j = 0; j < 2; ++j) {
      const int64_t it = blockIdx.x + j * static_cast<int64_t>(gridDim.x);
      if (it < items) {
        mbar_expect_tx(&full[j], BYTES);
        bulk_load(rp_sm + j * CH, src(it), BYTES, &full[j]);
      }
    }
  }
  uint32_t bh[4][4][2], bl[4][4][2];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int n = nt * 8 + gq, k = ks * 8 + tq + 4 * e;
        const float q = (n < 28 && k < 28) ? __ldg(p.Q + n * 28 + k) : 0.f;
        split_tf32(q, bh[nt][ks][e], bl[nt][ks][e]);
      }
  __syncthreads();
  int k = 0;
  bool ok = true;
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x, ++k) {
    const int j = k & 1;
    float *X = rp_sm + j * CH;
    const bool landed = mbar_wait(&full[j], (k >> 1) & 1, abort_flag);
    if (!__syncthreads_and(landed)) {
      ok = false;
      break;
    }
    const int64_t row = item / p.chunks, c0 = (item % p.chunks) * CH;
    const float rf = p.norm * (p.cr ? p.cr[row] : 1.f);
    const float *cc = p.cc ? p.cc + c0 : nullptr;
    // factors and the Hadamard bits 0-4 of a
    for (int t = threadIdx.x; t < (L / 32) * M; t += NT) {
      const int b = t % M, g = t / M;
      const int e0 = g * 32 * M + b;
      float r[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int e = e0 + i * M;
        float v = X[e] * rf;
        if (cc) v *= __ldg(cc + e);
        r[i] = v;
      }
      fwht_reg<32>(r);
#pragma unroll
      for (int i = 0; i < 32; ++i) X[e0 + i * M] = r[i];
    }
    __syncthreads();
    trounds<L, M, 32, L, NT>(X);
    // Q_28 mix, Y = X Qᵀ, out by warp MMA
    float *o = p.out + row * p.ld_out + c0;
    for (int mt = warp; mt < L / 16; mt += NW) {
      float acc[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
      const float *xa = X + (mt * 16 + gq) * 28;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int k0 = ks * 8 + tq, k1 = k0 + 4;
        uint32_t ah[4], al[4];
        split_tf32(xa[k0], ah[0], al[0]);
        split_tf32(xa[8 * 28 + k0], ah[1], al[1]);
        split_tf32(k1 < 28 ? xa[k1] : 0.f, ah[2], al[2]);
        split_tf32(k1 < 28 ? xa[8 * 28 + k1] : 0.f, ah[3], al[3]);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_tf32(acc[nt], al, bh[nt][ks][0], bh[nt][ks][1]);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_tf32(acc[nt], ah, bl[nt][ks][0], bl[nt][ks][1]);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma_tf32(acc[nt], ah, bh[nt][ks][0], bh[nt][ks][1]);
      }
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int n = nt * 8 + 2 * tq;
        if (n < 28) {
          const int a0 = mt * 16 + gq;
          __stcs(reinterpret_cast<float2 *>(o + a0 * 28 + n), make_float2(acc[nt][0], acc[nt][1]));
          __stcs(reinterpret_cast<float2 *>(o + (a0 + 8) * 28 + n),
                 make_float2(acc[nt][2], acc[nt][3]));
        }
      }
    }
    __syncthreads();  // every read of this buffer is done
    if (threadIdx.x == 0) {
      const int64_t nx = item + 2 * static_cast<int64_t>(gridDim.x);
      if (nx < items) {
        fence_proxy_async_smem();
        mbar_expect_tx(&full[j], BYTES);
        bulk_load(X, src(nx), BYTES, &full[j]);
      }
    }
  }
  if (!ok && threadIdx.x == 0) {
    report(info, KRONQ_ERR_TIMEOUT);
    // copies still in flight (this iteration's and the next one's) land
    // before the shared memory is released
    for (int d = 0; d < 2; ++d) {
      const int kk = k + d;
      if (blockIdx.x + kk * static_cast<int64_t>(gridDim.x) >= items) continue;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&full[kk & 1], (kk >> 1) & 1) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
  }
}

// Launches the fixed-shape row pass when (L, M, dtype) is one of the
// compiled shapes; KRONQ_ERR_UNSUPPORTED otherwise.
kronq_status launch_row_tpl(cudaStream_t st, const RowP &p, int64_t rows, bool bf16,
                            int32_t *info) {
  const int L = p.L, M = p.m;
  if (reinterpret_cast<uintptr_t>(p.out) % 16 || p.ld_out % 4 || p.ld_in % 4 ||
      reinterpret_cast<uintptr_t>(p.in) % 16 || (p.cc && reinterpret_cast<uintptr_t>(p.cc) % 16) ||
      (M > 1 && p.Q == nullptr))
    return KRONQ_ERR_UNSUPPORTED;
  const int64_t blocks = rows * p.chunks;
  if (blocks > 0x7fffffff) return KRONQ_ERR_UNSUPPORTED;
  if (!bf16 && M == 28 && (L == 1024 || L == 512)) {
    // fp32 rows of the Q_28 shapes: the pipelined persistent form
    const int smem = 2 * L * M * 4 + 64;
    const unsigned grid = static_cast<unsigned>(kq_min<int64_t>(blocks, sm_count()));
    auto pipe = [&](auto kern) -> kronq_status {
      KQ_TRY(smem_attr(kern, smem));
      kern<<<grid, RP_THREADS, smem, st>>>(p, blocks, info);
      KQ_CHECK_LAUNCH();
      return KRONQ_OK;
    };
    return L == 1024 ? pipe(row_pipe28_kernel<1024>) : pipe(row_pipe28_kernel<512>);
  }
  const int smem = L * M * 4;
  auto go = [&](auto kern) -> kronq_status {
    KQ_TRY(smem_attr(kern, smem));
    kern<<<static_cast<unsigned>(blocks), M == 1 ? 512 : 256, smem, st>>>(p);
    KQ_CHECK_LAUNCH();
    return KRONQ_OK;
  };
#define KQ_ROW_SHAPE(LL, MM)                                                  \
  if (L == LL && M == MM)                                                     \
    return bf16 ? go(row_tpl_kernel<LL, MM, true>) : go(row_tpl_kernel<LL, MM, false>);
  KQ_ROW_SHAPE(256, 1)
  KQ_ROW_SHAPE(512, 1)
  KQ_ROW_SHAPE(1024, 1)
  KQ_ROW_SHAPE(2048, 1)
  KQ_ROW_SHAPE(4096, 1)
  KQ_ROW_SHAPE(8192, 1)
  KQ_ROW_SHAPE(16384, 1)
  KQ_ROW_SHAPE(256, 28)
  KQ_ROW_SHAPE(512, 28)
  KQ_ROW_SHAPE(1024, 28)
#undef KQ_ROW_SHAPE
  return KRONQ_ERR_UNSUPPORTED;
}

// rows per TMA box for the column pass: a divisor of RK = AL * M of at most 256
__host__ __device__ constexpr int colpass_box(int AL, int M) {
  const int RK = AL * M;
  if (RK <= 256) return RK;
  if (RK % 256 == 0) return 256;
  int best = 1;
  for (int dv = 1; dv <= M; ++dv)
    if (M % dv == 0 && AL * dv <= 256 && AL * dv > best) best = AL * dv;
  return best;
}

// One Hadamard round over the local a-index of a column strip held as float4
// vectors (V = M * 4 vectors per a).
template <int AL, int V, int R, int H, int NT = CP_THREADS>
__device__ __forceinline__ void tround4(float4 *X4) {
  constexpr int T = (AL / R) * V;
  for (int t = threadIdx.x; t < T; t += NT) {
    const int v = t % V, g = t / V;
    const int a = (g / H) * R * H + (g % H);
    float4 *x = X4 + a * V + v;
    float4 r[R];
#pragma unroll
    for (int i = 0; i < R; ++i) r[i] = x[i * H * V];
    fwht_reg4<R>(r);
#pragma unroll
    for (int i = 0; i < R; ++i) x[i * H * V] = r[i];
  }
  __syncthreads();
}

template <int AL, int V, int H, int NT = CP_THREADS>
__device__ __forceinline__ void trounds4(float4 *X4) {
  if constexpr (H < AL) {
    constexpr int R = radix_for(AL / H, 16);
    tround4<AL, V, R, H, NT>(X4);
    trounds4<AL, V, H * R, NT>(X4);
  }
}

// Column pass (see colpass_kernel) with K, M, the local Hadamard length AL
// and the strip width (4*W4 columns) fixed at compile time.
template <int K, int M, int AL, int W4>
__global__ void __launch_bounds__(CP_THREADS, 2)
    colpass_tpl_kernel(const __grid_constant__ CUtensorMap tm, ColP p) {
  extern __shared__ __align__(128) float4 X4[];
  constexpr int RK = AL * M, NV = RK * W4, BOX = colpass_box(AL, M);
  const int rank = K > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int64_t strip = blockIdx.x / K;
  uint64_t *bar = reinterpret_cast<uint64_t *>(X4 + NV);
  int *abort_flag = reinterpret_cast<int *>(bar + 1);
  const int64_t row0 = static_cast<int64_t>(rank) * RK;
  const int64_t c0 = strip * 4 * W4;
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar, 1);
    fence_mbar_init();
    prefetch_tmap(&tm);
    mbar_expect_tx(bar, static_cast<uint32_t>(NV) * 16u);
#pragma unroll 1
    for (int r = 0; r < RK; r += BOX)
      tma_load_2d(X4 + r * W4, &tm, bar, static_cast<int32_t>(c0),
                  static_cast<int32_t>(row0 + r));
  }
  __syncthreads();
  const bool landed = mbar_wait(bar, 0, abort_flag);
  const int good = __syncthreads_and(landed);
  if (!good && threadIdx.x == 0) report(p.info, KRONQ_ERR_TIMEOUT);
  if (good) {
    if constexpr (M == 28) {
      static_assert(W4 == 2 || W4 == 4, "the Q_28 mix takes strips of 8 or 16 columns");
      colpass_qmix_mma28<CP_THREADS, W4 / 2>(reinterpret_cast<float *>(X4), AL, p.Q,
                                             p.fr ? p.fr + row0 : nullptr,
                                             p.fc ? p.fc + c0 : nullptr);
    } else if constexpr (M > 1) {
      colpass_qmix(reinterpret_cast<float *>(X4), AL, M, W4, p.Q);
    }
    trounds4<AL, M * W4, 1>(X4);
  }
  if (K > 1) cluster_sync_all();
  if (good) {
    constexpr int PER = (NV + K - 1) / K;
    const int p0 = rank * PER, p1 = min(NV, p0 + PER);
    const uint32_t xs = smem_u32(X4);
    for (int q = p0 + threadIdx.x; q < p1; q += CP_THREADS) {
      float4 v[K];
#pragma unroll
      for (int j = 0; j < K; ++j)
        v[j] = (K == 1 || j == rank) ? X4[q]
                                     : ld_dsmem_f4(mapa_shared(xs + 16u * q, j));
      fwht_reg4<K>(v);
      const int r = q / W4, c4 = q % W4;
      const int64_t col = c0 + 4 * c4;
      if (col < p.C) {
#pragma unroll
        for (int j = 0; j < K; ++j)
          __stcs(reinterpret_cast<float4 *>(p.M + (static_cast<int64_t>(j) * RK + r) * p.ld + col),
                 v[j]);
      }
    }
  }
  if (K > 1) cluster_sync_all();
  if (!good && threadIdx.x == 0) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, 0) && globaltimer() - t0 < kWaitLimitNs) {
    }
  }
}

// ------------------------------------------------------------- large Q_m
// For 32 < m (the 172 of 11008 = 64 * 172) the Q_m mix is a small GEMM per
// group, Y = Q X, and runs as one: Qᵀ stays in shared memory for the life of
// a persistent CTA (one per SM) and each thread accumulates a 4 x 4 tile of
// outputs, two 16-byte shared loads per 16 FMA.
constexpr int QB_THREADS = 256;
constexpr int QB_CW = 64;                 // columns per work item (column side)
constexpr int QB_SMEM_FLOATS = 227 * 1024 / 4;

__device__ void load_qt(float *Qt, const float *Q, int m, int mp) {
  for (int e = threadIdx.x; e < mp * mp; e += QB_THREADS) {
    const int k = e / mp, b = e % mp;
    Qt[e] = (k < m && b < m) ? Q[b * m + k] : 0.f;
  }
}

// Column side: each group of m consecutive rows of M (R x C, in place) is
// replaced by Q_m times it; work items are (group, 64-column tile).
__global__ void __launch_bounds__(QB_THREADS, 1)
    qmix_rows_kernel(float *M, int64_t ld, int64_t C, int m, int64_t groups,
                     const float *Q) {
  extern __shared__ float4 qb_sm4[];
  const int mp = (m + 3) & ~3, nb4 = mp / 4;
  float *Qt = reinterpret_cast<float *>(qb_sm4);
  float4 *Qt4 = qb_sm4;
  float4 *X4 = qb_sm4 + mp * nb4;           // [mp][QB_CW / 4]
  constexpr int NC4 = QB_CW / 4;
  load_qt(Qt, Q, m, mp);
  const int64_t ctiles = (C + QB_CW - 1) / QB_CW;
  const int64_t items = groups * ctiles;
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
    const int64_t a = item / ctiles, c0 = (item % ctiles) * QB_CW;
    float *base = M + a * m * ld;
    __syncthreads();
    for (int e4 = threadIdx.x; e4 < mp * NC4; e4 += QB_THREADS) {
      const int k = e4 / NC4, c4 = e4 % NC4;
      const int64_t col = c0 + 4 * c4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k < m && col < C) v = *reinterpret_cast<const float4 *>(base + k * ld + col);
      X4[e4] = v;
    }
    __syncthreads();
    for (int t = threadIdx.x; t < nb4 * NC4; t += QB_THREADS) {
      const int b4 = t / NC4, c4 = t % NC4;
      float4 acc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k = 0; k < m; ++k) {
        const float4 q = Qt4[k * nb4 + b4], x = X4[k * NC4 + c4];
        const float qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i].x = fmaf(qq[i], x.x, acc[i].x);
          acc[i].y = fmaf(qq[i], x.y, acc[i].y);
          acc[i].z = fmaf(qq[i], x.z, acc[i].z);
          acc[i].w = fmaf(qq[i], x.w, acc[i].w);
        }
      }
      const int64_t col = c0 + 4 * c4;
      if (col < C) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int b = 4 * b4 + i;
          if (b < m) *reinterpret_cast<float4 *>(base + b * ld + col) = acc[i];
        }
      }
    }
  }
}

// Row pass for 32 < m: work items are row chunks of L*m contiguous columns:
// load with the factors, Hadamard over a in shared memory, then
// Y[a][b] = sum_k X[a][k] Q[b][k] written straight to global memory.
__global__ void __launch_bounds__(QB_THREADS, 1) row_big_kernel(RowP p, int64_t items) {
  extern __shared__ float4 qb_sm4[];
  const int m = p.m, L = p.L, mp = (m + 3) & ~3, nb4 = mp / 4;
  const int CH = L * m;
  float *Qt = reinterpret_cast<float *>(qb_sm4);
  const float4 *Qt4 = qb_sm4;
  float *X = Qt + mp * mp;
  load_qt(Qt, p.Q, m, mp);
  auto vb = [](int v) { return v; };
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
    const int64_t row = item / p.chunks, c0 = (item % p.chunks) * CH;
    const float rf = p.norm * (p.cr ? p.cr[row] : 1.f);
    __syncthreads();
    for (int e = threadIdx.x; e < CH; e += QB_THREADS) {
      float v = load_in(p.in, p.in_bf16, row * p.ld_in + c0 + e) * rf;
      if (p.cc) v *= p.cc[c0 + e];
      X[e] = v;
    }
    __syncthreads();
    fwht_rest(X, m, L, 1, m, vb);
    float *o = p.out + row * p.ld_out + c0;
    const int na4 = (L + 3) / 4;
    for (int t = threadIdx.x; t < na4 * nb4; t += QB_THREADS) {
      const int a4 = t / nb4, b4 = t % nb4;
      float4 acc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      const int a0 = 4 * a4;
      const float *x0 = X + a0 * m;
      for (int k = 0; k < m; ++k) {
        const float4 q = Qt4[k * nb4 + b4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float xv = a0 + i < L ? x0[i * m + k] : 0.f;
          acc[i].x = fmaf(xv, q.x, acc[i].x);
          acc[i].y = fmaf(xv, q.y, acc[i].y);
          acc[i].z = fmaf(xv, q.z, acc[i].z);
          acc[i].w = fmaf(xv, q.w, acc[i].w);
        }
      }
      const int b0 = 4 * b4;
      if (b0 < m) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (a0 + i < L) *reinterpret_cast<float4 *>(o + (a0 + i) * m + b0) = acc[i];
      }
    }
  }
}

// ---- the same two mixes on the tensor cores (warp MMA m16n8k8, TF32 in
// three parts, as for Q_28). The unit of work is a 32 x 16 block of the
// product (two m tiles by two n tiles); Q_m sits in shared memory in the
// order the fragments are read, so that a lane's values are contiguous.
constexpr int QT_THREADS = 512;
constexpr int QT_MAX_L = 64;              // Hadamard positions per row chunk

__host__ __device__ constexpr int qt_xs_row(int m) { return (m + 7) / 8 * 8 + 4; }
__host__ __device__ constexpr int qt_xs_col(int cw) { return cw + 8; }

// C (MT*16 x NT*8) = A (MT*16 x KS*8) * B (KS*8 x NT*8) over 2 x 2 tile
// units; loadA(mt, ks, a[4]) and loadB(nt, ks, b[2]) return fragments as
// floats (zero outside the operands), store(mt, nt, c[4]) takes the result.
template <class LA, class LB, class ST>
__device__ __forceinline__ void mma3_units(int MT, int NT, int KS, LA loadA, LB loadB,
                                           ST store) {
  const int warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const int MP = (MT + 1) / 2, NP = (NT + 1) / 2;
  for (int u = warp; u < MP * NP; u += nwarp) {
    const int mt0 = 2 * (u % MP), nt0 = 2 * (u / MP);
    const bool m1 = mt0 + 1 < MT, n1 = nt0 + 1 < NT;
    float acc[2][2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
#pragma unroll 2
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t ah[2][4], alo[2][4], bh[2][2], bl[2][2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        if (i == 0 || m1) loadA(mt0 + i, ks, a);
#pragma unroll
        for (int e = 0; e < 4; ++e) split_tf32(a[e], ah[i][e], alo[i][e]);
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float b[2] = {0.f, 0.f};
        if (j == 0 || n1) loadB(nt0 + j, ks, b);
#pragma unroll
        for (int e = 0; e < 2; ++e) split_tf32(b[e], bh[j][e], bl[j][e]);
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) mma_tf32(acc[i][j], alo[i], bh[j][0], bh[j][1]);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) mma_tf32(acc[i][j], ah[i], bl[j][0], bl[j][1]);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) mma_tf32(acc[i][j], ah[i], bh[j][0], bh[j][1]);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        if ((i == 0 || m1) && (j == 0 || n1)) store(mt0 + i, nt0 + j, acc[i][j]);
  }
}

// Row pass for 32 < m on the tensor cores: as row_big_kernel, with the chunk
// held as X[a][k] (row stride qt_xs_row(m), columns m.. zero) and
// Y = X Qᵀ: B[k][n] = Q[n][k], stored per (n tile, k step, lane) as 2 floats.
__global__ void __launch_bounds__(QT_THREADS, 1) row_big_mma_kernel(RowP p, int64_t items) {
  extern __shared__ float4 qb_sm4[];
  const int m = p.m, L = p.L;
  const int KS = (m + 7) / 8, NT = KS, MT = L / 16, XS = qt_xs_row(m);
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  float *Qb = reinterpret_cast<float *>(qb_sm4);
  float *X = Qb + NT * KS * 64;
  for (int e = threadIdx.x; e < NT * KS * 64; e += QT_THREADS) {
    const int f = e & 1, ln = (e >> 1) & 31, blk = e >> 6;
    const int nt = blk / KS, ks = blk % KS;
    const int n = nt * 8 + (ln >> 2), k = ks * 8 + (ln & 3) + 4 * f;
    Qb[e] = (n < m && k < m) ? p.Q[n * m + k] : 0.f;
  }
  for (int e = threadIdx.x; e < L * (XS - m); e += QT_THREADS) {
    const int a = e / (XS - m), k = m + e % (XS - m);
    X[a * XS + k] = 0.f;
  }
  const int CH = L * m;
  auto vb = [](int v) { return v; };
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
    const int64_t row = item / p.chunks, c0 = (item % p.chunks) * CH;
    const float rf = p.norm * (p.cr ? p.cr[row] : 1.f);
    __syncthreads();
    {
      // four float4 loads per thread in flight (m % 4 == 0: a float4 never
      // straddles two groups)
      const int n4 = CH / 4;
      const int64_t in0 = row * p.ld_in + c0;
      const float4 *cc4 = p.cc ? reinterpret_cast<const float4 *>(p.cc + c0) : nullptr;
      for (int e4 = threadIdx.x; e4 < n4; e4 += 4 * QT_THREADS) {
        float4 v[4], f[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int idx = e4 + u * QT_THREADS;
          v[u] = f[u] = make_float4(1.f, 1.f, 1.f, 1.f);
          if (idx < n4) {
            v[u] = p.in_bf16 ? load4<true>(p.in, in0 + 4 * idx) : load4<false>(p.in, in0 + 4 * idx);
            if (cc4) f[u] = __ldg(cc4 + idx);
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int idx = e4 + u * QT_THREADS;
          if (idx < n4) {
            const int e = 4 * idx, a = e / m, b = e - a * m;
            *reinterpret_cast<float4 *>(X + a * XS + b) =
                make_float4(v[u].x * rf * f[u].x, v[u].y * rf * f[u].y, v[u].z * rf * f[u].z,
                            v[u].w * rf * f[u].w);
          }
        }
      }
    }
    __syncthreads();
    fwht_rest(X, m, L, 1, XS, vb);
    float *o = p.out + row * p.ld_out + c0;
    mma3_units(
        MT, NT, KS,
        [&](int mt, int ks, float (&a)[4]) {
          const float *x = X + (mt * 16 + gq) * XS + ks * 8 + tq;
          a[0] = x[0];
          a[1] = x[8 * XS];
          a[2] = x[4];
          a[3] = x[8 * XS + 4];
        },
        [&](int nt, int ks, float (&b)[2]) {
          const float2 v = reinterpret_cast<const float2 *>(Qb)[(nt * KS + ks) * 32 + lane];
          b[0] = v.x;
          b[1] = v.y;
        },
        [&](int mt, int nt, const float (&c)[4]) {
          const int a = mt * 16 + gq, b = nt * 8 + 2 * tq;
          if (b < m) {
            *reinterpret_cast<float2 *>(o + a * m + b) = make_float2(c[0], c[1]);
            *reinterpret_cast<float2 *>(o + (a + 8) * m + b) = make_float2(c[2], c[3]);
          }
        });
  }
}

// Column side for 32 < m on the tensor cores: each group of m rows of a
// strip of CW columns, Y = Q X, with X[k][c] in shared memory (row stride
// qt_xs_col(CW), rows m.. zero) and A[b][k] = Q[b][k] stored per (m tile,
// k step, lane) as 4 floats.
__global__ void __launch_bounds__(QT_THREADS, 1)
    qmix_rows_mma_kernel(float *M, int64_t ld, int64_t C, int m, int64_t groups, int CW,
                         const float *Q) {
  extern __shared__ float4 qb_sm4[];
  const int KS = (m + 7) / 8, MT = (m + 15) / 16, NT = CW / 8, XS = qt_xs_col(CW);
  const int lane = threadIdx.x & 31, gq = lane >> 2, tq = lane & 3;
  float *Qa = reinterpret_cast<float *>(qb_sm4);
  float *X = Qa + MT * KS * 128;
  for (int e = threadIdx.x; e < MT * KS * 128; e += QT_THREADS) {
    const int f = e & 3, ln = (e >> 2) & 31, blk = e >> 7;
    const int mt = blk / KS, ks = blk % KS;
    const int b = mt * 16 + (ln >> 2) + 8 * (f & 1), k = ks * 8 + (ln & 3) + 4 * (f >> 1);
    Qa[e] = (b < m && k < m) ? Q[b * m + k] : 0.f;
  }
  for (int e = threadIdx.x; e < (KS * 8 - m) * XS; e += QT_THREADS) X[m * XS + e] = 0.f;
  const int64_t ctiles = (C + CW - 1) / CW;
  const int64_t items = groups * ctiles;
  const int cw4 = CW / 4;
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
    const int64_t a = item / ctiles, c0 = (item % ctiles) * CW;
    float *base = M + a * m * ld + c0;
    __syncthreads();
    for (int e4 = threadIdx.x; e4 < m * cw4; e4 += 4 * QT_THREADS) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = e4 + u * QT_THREADS;
        const int k = idx / cw4, c = 4 * (idx % cw4);
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (idx < m * cw4 && c0 + c < C) v[u] = *reinterpret_cast<const float4 *>(base + k * ld + c);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = e4 + u * QT_THREADS;
        const int k = idx / cw4, c = 4 * (idx % cw4);
        if (idx < m * cw4) *reinterpret_cast<float4 *>(X + k * XS + c) = v[u];
      }
    }
    __syncthreads();
    mma3_units(
        MT, NT, KS,
        [&](int mt, int ks, float (&av)[4]) {
          const float4 v = reinterpret_cast<const float4 *>(Qa)[(mt * KS + ks) * 32 + lane];
          av[0] = v.x;
          av[1] = v.y;
          av[2] = v.z;
          av[3] = v.w;
        },
        [&](int nt, int ks, float (&b)[2]) {
          const float *x = X + (ks * 8 + tq) * XS + nt * 8 + gq;
          b[0] = x[0];
          b[1] = x[4 * XS];
        },
        [&](int mt, int nt, const float (&c)[4]) {
          const int b = mt * 16 + gq, c2 = nt * 8 + 2 * tq;
          if (c0 + c2 < C) {
            if (b < m) *reinterpret_cast<float2 *>(base + b * ld + c2) = make_float2(c[0], c[1]);
            if (b + 8 < m)
              *reinterpret_cast<float2 *>(base + (b + 8) * ld + c2) = make_float2(c[2], c[3]);
          }
        });
  }
}

// shared memory of the two kernels above
size_t row_big_mma_smem(int m, int L) {
  const size_t ks = (m + 7) / 8;
  return (ks * ks * 64 + static_cast<size_t>(L) * qt_xs_row(m)) * 4;
}
size_t qmix_mma_smem(int m, int cw) {
  const size_t ks = (m + 7) / 8, mt = (m + 15) / 16;
  return (mt * ks * 128 + ks * 8 * qt_xs_col(cw)) * 4;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// ------------------------------------------------------------- planning
struct SideRot {
  int64_t d, had, m;
  bool rot;
  const float *Q;  // device Q_m (m > 1 and rot) or null
};

constexpr int64_t ROW_CHUNK_MAX = 28672;  // floats of one row chunk (112 KB)
constexpr int SLAB_FLOATS = 32768;        // floats of one strided slab
constexpr int64_t MAX_A = 1024;           // Hadamard length of one strided pass

// Hadamard of length A (power of two) along the middle axis of the view
// [outer][A][inner] (strides so, smid, 1). Lengths above MAX_A are split into
// two balanced factors Hhat_A = Hhat_hi ⊗ Hhat_lo, one pass each; each pass
// sees its independent vectors on a two-level outer index.
kronq_status launch_strided(cudaStream_t st, float *base, int64_t outer,
                            int64_t so, int64_t A, int64_t smid, int64_t inner) {
  KQ_TRY(smem_attr(strided_fwht_kernel, SLAB_FLOATS * 4));
  KQ_TRY(smem_attr(strided_fwht4_kernel, SLAB_FLOATS * 4));
  if (A <= 1) return KRONQ_OK;
  const bool vec = reinterpret_cast<uintptr_t>(base) % 16 == 0 && so % 4 == 0 &&
                   smid % 4 == 0 && inner % 4 == 0;
  auto pass = [&](int64_t a, int64_t stride, int64_t n2, int64_t so2) -> kronq_status {
    int64_t cw = kq_min<int64_t>(inner, kq_min<int64_t>(256, SLAB_FLOATS / a));
    cw = kq_max<int64_t>(1, cw);
    const int64_t chunks = ceil_div(inner, cw);
    const int64_t blocks = outer * n2 * chunks;
    if (blocks > 0x7fffffff) return KRONQ_ERR_UNSUPPORTED;
    if (vec && cw % 4 == 0)
      strided_fwht4_kernel<<<static_cast<unsigned>(blocks), 512,
                             static_cast<size_t>(a * cw * 4), st>>>(
          base, so, outer, so2, static_cast<int>(a), stride, inner,
          static_cast<int>(cw), chunks);
    else
      strided_fwht_kernel<<<static_cast<unsigned>(blocks), 512,
                            static_cast<size_t>(a * cw * 4), st>>>(
          base, so, outer, so2, static_cast<int>(a), stride, inner,
          static_cast<int>(cw), chunks);
    KQ_CHECK_LAUNCH();
    return KRONQ_OK;
  };
  if (A <= MAX_A) return pass(A, smid, 1, 0);
  int64_t lo = 1;
  while (lo * lo < A) lo *= 2;  // lo >= sqrt(A), both factors <= MAX_A
  const int64_t hi = A / lo;
  if (lo > MAX_A || hi > MAX_A) return KRONQ_ERR_UNSUPPORTED;
  // low factor: elements smid apart; vectors (outer, high position)
  KQ_TRY(pass(lo, smid, hi, lo * smid));
  // high factor: elements lo*smid apart; vectors (outer, low position)
  return pass(hi, lo * smid, lo, smid);
}

// out = P_r diag(cr) in diag(cc) P_cᵀ for an R x C row-major matrix.
kronq_status rotate(cudaStream_t st, const void *in, bool in_bf16, int64_t ld_in,
                    float *out, int64_t ld_out, int64_t R, int64_t C,
                    const SideRot &sr, const SideRot &sc, const float *cr,
                    const float *cc, int32_t *info) {
  const int64_t had_r = sr.rot ? sr.had : 1, m_r = sr.rot ? sr.m : 1;
  const int64_t had_c = sc.rot ? sc.had : 1, m_c = sc.rot ? sc.m : 1;
  // In place on fp32 with Q_28 on the row side, the row side goes first and
  // takes both diagonal factors (a load per row and per column of its strip);
  // the row pass then runs without factors (the per-element column factor
  // would otherwise be an L2 read per element of every row).
  bool row_side_done = false;
  if (in == out && !in_bf16 && ld_in == ld_out && sr.rot && m_r == 28 && (cr || cc)) {
    const kronq_status s0 =
        launch_colpass(st, out, ld_out, R, C, had_r, m_r, sr.Q, info, cr, cc);
    if (s0 == KRONQ_OK) {
      row_side_done = true;
      cr = nullptr;
      cc = nullptr;
    } else if (s0 != KRONQ_ERR_UNSUPPORTED) {
      return s0;
    }
  }
  // ---- row pass over chunks of Lc * m_c contiguous columns
  int64_t Lc = 1;
  const int64_t mpc = (m_c + 3) / 4 * 4;
  // large Q_m on the column side: the persistent GEMM-style row pass, whose
  // shared memory holds Q_mᵀ next to the chunk
  const bool big = sc.rot && m_c > 32 && m_c % 4 == 0 && ld_out % 4 == 0 &&
                   reinterpret_cast<uintptr_t>(out) % 16 == 0 &&
                   mpc * mpc + m_c <= QB_SMEM_FLOATS;
  bool big_mma = false;
  if (big) {
    while (Lc * 2 <= had_c && mpc * mpc + Lc * 2 * m_c <= QB_SMEM_FLOATS) Lc *= 2;
    // the tensor-core form: chunks of up to QT_MAX_L Hadamard positions,
    // whole 16-row tiles
    const int64_t Lm = kq_min<int64_t>(had_c, QT_MAX_L);
    const bool in_vec = reinterpret_cast<uintptr_t>(in) % 16 == 0 && ld_in % 4 == 0 &&
                        (!cc || reinterpret_cast<uintptr_t>(cc) % 16 == 0);
    if (in_vec && Lm % 16 == 0 &&
        row_big_mma_smem(static_cast<int>(m_c), static_cast<int>(Lm)) <=
            static_cast<size_t>(227 * 1024)) {
      big_mma = true;
      Lc = Lm;
    }
  } else if (sc.rot) {
    while (Lc * 2 <= had_c && Lc * 2 * m_c <= ROW_CHUNK_MAX) Lc *= 2;
  } else {
    // no column rotation: chunks are only a unit of work
    while (Lc * 2 <= 8192 && C % (Lc * 2) == 0) Lc *= 2;
  }
  const int64_t chunk = Lc * m_c;
  {
    RowP p{};
    p.in = in; p.out = out; p.ld_in = ld_in; p.ld_out = ld_out;
    p.in_bf16 = in_bf16; p.cr = cr; p.cc = cc;
    p.norm = static_cast<float>(1.0 / sqrt(double(had_r) * double(had_c)));
    p.L = static_cast<int>(sc.rot ? Lc : chunk);
    p.m = static_cast<int>(sc.rot ? m_c : 1);
    if (!sc.rot) p.L = static_cast<int>(chunk), p.m = 1;
    p.Q = (sc.rot && m_c > 1) ? sc.Q : nullptr;
    p.chunks = C / chunk;
    size_t smem = static_cast<size_t>(chunk) * 4;
    KQ_TRY(smem_attr(row_pass_kernel, static_cast<int>(ROW_CHUNK_MAX * 4)));
    if (C % chunk) return KRONQ_ERR_UNSUPPORTED;
    const int64_t blocks = R * p.chunks;
    if (blocks > 0x7fffffff) return KRONQ_ERR_UNSUPPORTED;
    // without a column rotation the chunk is a plain scaled copy: L = chunk
    // with no Hadamard would be wrong, so run it as m = chunk, L = 1
    if (!sc.rot) {
      p.L = 1;
      p.m = static_cast<int>(chunk);
      p.Q = nullptr;
    }
    if (big_mma) {
      const int smem = static_cast<int>(row_big_mma_smem(p.m, p.L));
      KQ_TRY(smem_attr(row_big_mma_kernel, smem));
      const int64_t items = R * p.chunks;
      const unsigned grid = static_cast<unsigned>(kq_min<int64_t>(items, sm_count()));
      row_big_mma_kernel<<<grid, QT_THREADS, smem, st>>>(p, items);
      KQ_CHECK_LAUNCH();
    } else if (big) {
      const int smem = static_cast<int>((mpc * mpc + chunk) * 4);
      KQ_TRY(smem_attr(row_big_kernel, smem));
      const int64_t items = R * p.chunks;
      const unsigned grid = static_cast<unsigned>(kq_min<int64_t>(items, sm_count()));
      row_big_kernel<<<grid, QB_THREADS, smem, st>>>(p, items);
      KQ_CHECK_LAUNCH();
    }
    const kronq_status fast = big ? KRONQ_OK : launch_row_tpl(st, p, R, in_bf16, info);
    if (big) {
    } else if (fast != KRONQ_ERR_UNSUPPORTED) {
      KQ_TRY(fast);
    } else {
      row_pass_kernel<<<static_cast<unsigned>(blocks), 512, smem, st>>>(p);
      KQ_CHECK_LAUNCH();
    }
  }
  // ---- column-side Hadamard bits beyond the chunk
  if (sc.rot && had_c / Lc > 1)
    KQ_TRY(launch_strided(st, out, R, ld_out, had_c / Lc, chunk, chunk));
  if (row_side_done) return KRONQ_OK;
  // ---- row side in one pass (cluster column pass) where the shape allows
  if (sr.rot && (had_r > 1 || m_r > 1)) {
    const kronq_status s = launch_colpass(st, out, ld_out, R, C, had_r, m_r,
                                          m_r > 1 ? sr.Q : nullptr, info);
    if (s != KRONQ_ERR_UNSUPPORTED) return s;
  }
  // ---- otherwise two passes: Q_m over groups of m_r consecutive rows, then
  // the Hadamard
  const bool rows_aligned = ld_out % 4 == 0 && C % 4 == 0 &&
                            reinterpret_cast<uintptr_t>(out) % 16 == 0;
  if (sr.rot && m_r > 32 && m_r % 4 == 0 && rows_aligned &&
      qmix_mma_smem(static_cast<int>(m_r), QB_CW) <= static_cast<size_t>(227 * 1024)) {
    const int smem = static_cast<int>(qmix_mma_smem(static_cast<int>(m_r), QB_CW));
    KQ_TRY(smem_attr(qmix_rows_mma_kernel, smem));
    const int64_t items = had_r * ceil_div(C, QB_CW);
    const unsigned grid = static_cast<unsigned>(kq_min<int64_t>(items, sm_count()));
    qmix_rows_mma_kernel<<<grid, QT_THREADS, smem, st>>>(out, ld_out, C, static_cast<int>(m_r),
                                                         had_r, QB_CW, sr.Q);
    KQ_CHECK_LAUNCH();
  } else if (sr.rot && m_r > 32 && m_r % 4 == 0 && rows_aligned &&
             (m_r + 3) / 4 * 4 * ((m_r + 3) / 4 * 4 + QB_CW) <= QB_SMEM_FLOATS) {
    const int mp = static_cast<int>((m_r + 3) / 4 * 4);
    const int smem = (mp * mp + mp * QB_CW) * 4;
    KQ_TRY(smem_attr(qmix_rows_kernel, smem));
    const int64_t items = had_r * ceil_div(C, QB_CW);
    const unsigned grid = static_cast<unsigned>(kq_min<int64_t>(items, sm_count()));
    qmix_rows_kernel<<<grid, QB_THREADS, smem, st>>>(out, ld_out, C, static_cast<int>(m_r),
                                                     had_r, sr.Q);
    KQ_CHECK_LAUNCH();
  } else if (sr.rot && m_r > 1) {
    // Q_m, then Qᵀ (m <= 32) or a [m][64] input tile (m > 32)
    const size_t smem =
        (static_cast<size_t>(m_r) * m_r + (m_r > 32 ? m_r * 64 : m_r * m_r)) * 4;
    if (smem > 227 * 1024) return KRONQ_ERR_UNSUPPORTED;
    KQ_TRY(smem_attr(rowq_kernel, 227 * 1024));
    const int64_t cols = m_r > 32 ? 64 : 256;
    dim3 grid(static_cast<unsigned>(ceil_div(C, cols)), static_cast<unsigned>(had_r));
    rowq_kernel<<<grid, 256, smem, st>>>(out, ld_out, C, static_cast<int>(m_r), sr.Q);
    KQ_CHECK_LAUNCH();
  }
  if (sr.rot && had_r > 1)
    KQ_TRY(launch_strided(st, out, m_r, ld_out, had_r, m_r * ld_out, C));
  return KRONQ_OK;
}

}  // namespace

size_t biip_ws_bytes(int64_t d_out, int64_t d_in, const kronq_opts &o) {
  auto al = [](size_t b) { return (b + 255) / 256 * 256; };
  size_t b = 0;
  b += 2 * al(static_cast<size_t>(d_in) * 4);
  b += 2 * al(static_cast<size_t>(d_out) * 4);
  b += al(static_cast<size_t>(o.rot_in.m) * o.rot_in.m * 4);
  b += al(static_cast<size_t>(o.rot_out.m) * o.rot_out.m * 4);
  b += al(static_cast<size_t>(o.rot_in.m) * o.rot_in.m * 8);
  b += al(static_cast<size_t>(o.rot_out.m) * o.rot_out.m * 8);
  return b + 256;
}

kronq_status biip(cudaStream_t st, const kronq_opts &o, const void *W,
                  bool w_bf16, int64_t d_out, int64_t d_in, float *W_rot,
                  float *H_X, float *H_G, float *s_x, float *s_g, void *ws,
                  size_t ws_bytes, int32_t *info) {
  if (ws_bytes < biip_ws_bytes(d_out, d_in, o)) return KRONQ_ERR_INVALID_ARG;
  auto al = [](size_t b) { return (b + 255) / 256 * 256; };
  uint8_t *w = static_cast<uint8_t *>(ws);
  float *fxw = reinterpret_cast<float *>(w); w += al(d_in * 4);
  float *fxh = reinterpret_cast<float *>(w); w += al(d_in * 4);
  float *fgw = reinterpret_cast<float *>(w); w += al(d_out * 4);
  float *fgh = reinterpret_cast<float *>(w); w += al(d_out * 4);
  const int mx = static_cast<int>(o.rot_in.m), mg = static_cast<int>(o.rot_out.m);
  float *Qx = reinterpret_cast<float *>(w); w += al(size_t(mx) * mx * 4);
  float *Qg = reinterpret_cast<float *>(w); w += al(size_t(mg) * mg * 4);
  double *Gx = reinterpret_cast<double *>(w); w += al(size_t(mx) * mx * 8);
  double *Gg = reinterpret_cast<double *>(w);

  const bool rot_x = !(o.flags & KRONQ_FLAG_NO_ROT_IN);
  const bool rot_g = !(o.flags & KRONQ_FLAG_NO_ROT_OUT);
  const bool scale = !(o.flags & KRONQ_FLAG_NO_SCALE);
  const uint64_t k0 = sm64(o.seed);
  SideDev sx{H_X, d_in, rot_x, scale, o.scale_exp, sm64(k0 + 0), s_x, fxw, fxh};
  SideDev sg{H_G, d_out, rot_g, scale, o.scale_exp, sm64(k0 + 1), s_g, fgw, fgh};
  side_prep_kernel<<<2, 1024, 0, st>>>(sx, sg, info);
  KQ_CHECK_LAUNCH();
  const uint64_t qkey = 0xA5A5A5A5A5A5A5A5ull;
  QDev qx{rot_x ? mx : 1, sx.key ^ qkey, Gx, Qx};
  QDev qg{rot_g ? mg : 1, sg.key ^ qkey, Gg, Qg};
  KQ_TRY(smem_attr(qm_kernel, static_cast<int>(QM_SMEM)));
  qm_kernel<<<2, QM_THREADS, QM_SMEM, st>>>(qx, qg);
  KQ_CHECK_LAUNCH();

  SideRot rx{d_in, o.rot_in.had, o.rot_in.m, rot_x, Qx};
  SideRot rg{d_out, o.rot_out.had, o.rot_out.m, rot_g, Qg};
  // W' = U_G (S_G W S_X) U_Xᵀ: rows use the output side, columns the input side
  KQ_TRY(rotate(st, W, w_bf16, d_in, W_rot, d_in, d_out, d_in, rg, rx, fgw, fxw, info));
  // H_X' = U_X S_X^-1 H_X S_X^-1 U_Xᵀ, H_G' likewise (in place)
  KQ_TRY(rotate(st, H_X, false, d_in, H_X, d_in, d_in, d_in, rx, rx, fxh, fxh, info));
  KQ_TRY(rotate(st, H_G, false, d_out, H_G, d_out, d_out, d_out, rg, rg, fgh, fgh, info));
  return KRONQ_OK;
}


// ------------------------------------------------------------- reuse by the
// quantized-layer matvec: one side's rotation applied along rows, and the
// factors of both sides
namespace {
__global__ void side_factor_kernel(const float *s, int64_t d, int rot, uint64_t key,
                                   float *f) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < d;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float sg = (rot && (sm64(key + static_cast<uint64_t>(i)) >> 63)) ? -1.f : 1.f;
    f[i] = sg / s[i];
  }
}
__global__ void transpose_small_kernel(const float *a, float *at, int m) {
  for (int e = threadIdx.x; e < m * m; e += blockDim.x) at[(e % m) * m + e / m] = a[e];
}
}  // namespace

// ---- a few whole rows (the tokens of a matvec): out = norm (Hhat ⊗ Q_m)
// (cc ⊙ x) per row, each row spread over a cluster of K CTAs. CTA k holds
// the Hadamard positions a in [k*AL, (k+1)*AL) (elements a*m + b), mixes each
// group with Q_m, runs the Hadamard over its local a, and the top log2(K)
// bits are one K-point Hadamard across the cluster (distributed shared
// memory), written straight out.
constexpr int VR_THREADS = 256;

__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

template <int K>
__global__ void __launch_bounds__(VR_THREADS)
    vec_rot_kernel(const float *in, float *out, int64_t C, int had, int m, const float *Q,
                   const float *cc, float norm) {
  extern __shared__ __align__(16) float vr_sm[];
  const int rank = K > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int64_t row = blockIdx.x / K;
  const int AL = had / K, n = AL * m;
  float *X = vr_sm, *Y = vr_sm + n;
  const int64_t e0 = static_cast<int64_t>(rank) * n;
  const float *x = in + row * C + e0;
  for (int e = threadIdx.x; e < n; e += VR_THREADS)
    X[e] = x[e] * norm * (cc ? __ldg(cc + e0 + e) : 1.f);
  __syncthreads();
  float *Z = X;
  if (m > 1) {   // Y[a][b] = sum_k Q[b][k] X[a][k]
    for (int t = threadIdx.x; t < n; t += VR_THREADS) {
      const int a = t / m, b = t - a * m;
      const float *xa = X + a * m, *qb = Q + b * m;
      float acc = 0.f;
      for (int k = 0; k < m; ++k) acc = fmaf(__ldg(qb + k), xa[k], acc);
      Y[t] = acc;
    }
    __syncthreads();
    Z = Y;
  }
  if (AL > 1) fwht_rest(Z, m, AL, 1, m, [](int v) { return v; });
  if (K > 1) cluster_sync_all();
  const int per = (n + K - 1) / K;
  const uint32_t zs = smem_u32(Z);
  for (int q = rank * per + threadIdx.x; q < min(n, (rank + 1) * per); q += VR_THREADS) {
    float v[K];
#pragma unroll
    for (int j = 0; j < K; ++j)
      v[j] = (K == 1 || j == rank) ? Z[q] : ld_dsmem_f32(mapa_shared(zs + 4u * q, j));
    fwht_reg<K>(v);
#pragma unroll
    for (int j = 0; j < K; ++j) out[row * C + static_cast<int64_t>(j) * n + q] = v[j];
  }
  // no CTA leaves while another may still read its shared memory
  if (K > 1) cluster_sync_all();
}

// Launches vec_rot_kernel when it applies (a rotation of whole rows, out not
// aliasing in, m <= 32); KRONQ_ERR_UNSUPPORTED otherwise.
kronq_status launch_vec_rot(cudaStream_t st, const float *in, float *out, int64_t R, int64_t C,
                            int64_t had, int64_t m, const float *Q, const float *cc) {
  if (R < 1 || R > 64 || in == out || m > 32 || had < 2 || had * m != C || (m > 1 && !Q))
    return KRONQ_ERR_UNSUPPORTED;
  const int K = static_cast<int>(kq_min<int64_t>(16, had));
  const int64_t n = had / K * m;
  const int smem = static_cast<int>(2 * n * 4);
  if (smem > 48 * 1024) return KRONQ_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(R * K));
  cfg.blockDim = dim3(VR_THREADS);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(K);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float norm = static_cast<float>(1.0 / sqrt(double(had)));
  auto go = [&](auto kern) -> kronq_status {
    if (K > 8) KQ_TRY(nonportable_cluster_attr(kern));
    KQ_CUDA(cudaLaunchKernelEx(&cfg, kern, in, out, C, static_cast<int>(had), static_cast<int>(m),
                               Q, cc, norm));
    count_launch();
    return KRONQ_OK;
  };
  switch (K) {
    case 2: return go(vec_rot_kernel<2>);
    case 4: return go(vec_rot_kernel<4>);
    case 8: return go(vec_rot_kernel<8>);
    default: return go(vec_rot_kernel<16>);
  }
}

kronq_status rotate_rows(cudaStream_t st, const float *in, float *out, int64_t R,
                         int64_t C, bool rot, int64_t had, int64_t m, const float *Q,
                         const float *cc, int32_t *info) {
  if (rot) {
    const kronq_status s = launch_vec_rot(st, in, out, R, C, had, m, Q, cc);
    if (s != KRONQ_ERR_UNSUPPORTED) return s;
  }
  const SideRot none{R, 1, 1, false, nullptr};
  const SideRot sc{C, rot ? had : C, rot ? m : 1, rot, Q};
  return rotate(st, in, false, C, out, C, R, C, none, sc, nullptr, cc, info);
}

kronq_status rotation_factors(cudaStream_t st, const kronq_opts &o, const float *s_x,
                              const float *s_g, int64_t d_out, int64_t d_in, float *fx,
                              float *fg, float *Qx, float *QgT, float *Qg, double *G) {
  const bool rot_x = !(o.flags & KRONQ_FLAG_NO_ROT_IN);
  const bool rot_g = !(o.flags & KRONQ_FLAG_NO_ROT_OUT);
  const uint64_t k0 = sm64(o.seed);
  const uint64_t kx = sm64(k0 + 0), kg = sm64(k0 + 1);
  side_factor_kernel<<<static_cast<unsigned>(kq_min<int64_t>(ceil_div(d_in, 256), 1024)), 256,
                       0, st>>>(s_x, d_in, rot_x, kx, fx);
  KQ_CHECK_LAUNCH();
  side_factor_kernel<<<static_cast<unsigned>(kq_min<int64_t>(ceil_div(d_out, 256), 1024)), 256,
                       0, st>>>(s_g, d_out, rot_g, kg, fg);
  KQ_CHECK_LAUNCH();
  const uint64_t qkey = 0xA5A5A5A5A5A5A5A5ull;
  const int mx = rot_x ? static_cast<int>(o.rot_in.m) : 1;
  const int mg = rot_g ? static_cast<int>(o.rot_out.m) : 1;
  QDev qx{mx, kx ^ qkey, G, Qx};
  QDev qg{mg, kg ^ qkey, G + 256 * 256, Qg};
  KQ_TRY(smem_attr(qm_kernel, static_cast<int>(QM_SMEM)));
  qm_kernel<<<2, QM_THREADS, QM_SMEM, st>>>(qx, qg);
  KQ_CHECK_LAUNCH();
  transpose_small_kernel<<<1, 256, 0, st>>>(Qg, QgT, mg);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

}  // namespace kronq

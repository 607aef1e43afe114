// Bidirectional incoherence processing (BiIP) [wmrh §三, §八, Q2; aimodeling]:
// a diagonal rescale from diag(H_X), diag(H_G) followed by a seeded orthogonal
// rotation on both sides of W, with H_X and H_G rotated to match:
//   W'   = U_G S_G W S_X U_Xᵀ
//   H_X' = U_X S_X^-1 H_X S_X^-1 U_Xᵀ,   H_G' = U_G S_G^-1 H_G S_G^-1 U_Gᵀ
// with U = (Hhat_had ⊗ Q_m) diag(sign) per side (spec in include/kronq.h).
//
// Every rotation of an R x C row-major matrix M -> P_r diag(cr) M diag(cc) P_cᵀ
// is split into memory passes whose working sets fit in shared memory:
//   row pass      one row chunk of Lc*m_c contiguous columns per CTA: input
//                 factors, Hadamard over the chunk's a-index, Q_m over each
//                 group of m_c contiguous values (the whole column side when
//                 the row fits in 112 KB)
//   row-side Q_m  groups of m_r consecutive rows, one thread per column
//   strided pass  Hadamard over index bits whose elements sit at a fixed
//                 stride (within a row, or across rows); one [A][cw] slab per
//                 CTA with cw contiguous columns
// The Hadamard factors commute with each other and with Q_m (Kronecker
// structure), so the order of the passes does not change the result.
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
// by classical Gram–Schmidt applied twice per column, in fp64. One CTA per side.
struct QDev {
  int m;
  uint64_t kq;
  double *G;   // scratch m*m, column-major (column j contiguous)
  float *Q;    // out: Q[b*m + b'] (row-major)
};

__global__ void qm_kernel(QDev a, QDev b) {
  const QDev &p = blockIdx.x == 0 ? a : b;
  const int m = p.m;
  if (m <= 1) {
    if (m == 1 && threadIdx.x == 0) p.Q[0] = 1.f;
    return;
  }
  __shared__ double v[256];
  __shared__ double coef[256];
  __shared__ double part[32];
  const int nw = blockDim.x / 32, w = threadIdx.x / 32, lane = threadIdx.x & 31;
  // Box–Muller normals: G[r][c] with t = r*m + c
  for (int t = threadIdx.x; t < m * m; t += blockDim.x) {
    const uint64_t x1 = sm64(p.kq + 2ull * t), x2 = sm64(p.kq + 2ull * t + 1ull);
    const double u1 = (double((x1 >> 11)) + 1.0) * 0x1.0p-53;
    const double u2 = double(x2 >> 11) * 0x1.0p-53;
    const int r = t / m, c = t % m;
    p.G[c * m + r] = sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
  }
  __syncthreads();
  for (int j = 0; j < m; ++j) {
    for (int r = threadIdx.x; r < m; r += blockDim.x) v[r] = p.G[j * m + r];
    __syncthreads();
    for (int pass = 0; pass < 2; ++pass) {
      for (int i = w; i < j; i += nw) {
        double s = 0.0;
        for (int r = lane; r < m; r += 32) s += p.G[i * m + r] * v[r];
        s = warp_sum_d(s);
        if (lane == 0) coef[i] = s;
      }
      __syncthreads();
      for (int r = threadIdx.x; r < m; r += blockDim.x) {
        double s = v[r];
        for (int i = 0; i < j; ++i) s -= coef[i] * p.G[i * m + r];
        v[r] = s;
      }
      __syncthreads();
    }
    double s = 0.0;
    for (int r = threadIdx.x; r < m; r += blockDim.x) s += v[r] * v[r];
    s = warp_sum_d(s);
    if (lane == 0) part[w] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
      double t = 0.0;
      for (int k = 0; k < nw; ++k) t += part[k];
      part[0] = 1.0 / sqrt(t);
    }
    __syncthreads();
    const double inv = part[0];
    for (int r = threadIdx.x; r < m; r += blockDim.x) p.G[j * m + r] = v[r] * inv;
    __syncthreads();
  }
  for (int t = threadIdx.x; t < m * m; t += blockDim.x) {
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
                    const float *cc) {
  const int64_t had_r = sr.rot ? sr.had : 1, m_r = sr.rot ? sr.m : 1;
  const int64_t had_c = sc.rot ? sc.had : 1, m_c = sc.rot ? sc.m : 1;
  // ---- row pass over chunks of Lc * m_c contiguous columns
  int64_t Lc = 1;
  if (sc.rot) {
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
    row_pass_kernel<<<static_cast<unsigned>(blocks), 512, smem, st>>>(p);
    KQ_CHECK_LAUNCH();
  }
  // ---- column-side Hadamard bits beyond the chunk
  if (sc.rot && had_c / Lc > 1)
    KQ_TRY(launch_strided(st, out, R, ld_out, had_c / Lc, chunk, chunk));
  // ---- row side: Q_m over groups of m_r consecutive rows, then the Hadamard
  if (sr.rot && m_r > 1) {
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
  qm_kernel<<<2, 256, 0, st>>>(qx, qg);
  KQ_CHECK_LAUNCH();

  SideRot rx{d_in, o.rot_in.had, o.rot_in.m, rot_x, Qx};
  SideRot rg{d_out, o.rot_out.had, o.rot_out.m, rot_g, Qg};
  // W' = U_G (S_G W S_X) U_Xᵀ: rows use the output side, columns the input side
  KQ_TRY(rotate(st, W, w_bf16, d_in, W_rot, d_in, d_out, d_in, rg, rx, fgw, fxw));
  // H_X' = U_X S_X^-1 H_X S_X^-1 U_Xᵀ, H_G' likewise (in place)
  KQ_TRY(rotate(st, H_X, false, d_in, H_X, d_in, d_in, d_in, rx, rx, fxh, fxh));
  KQ_TRY(rotate(st, H_G, false, d_out, H_G, d_out, d_out, d_out, rg, rg, fgh, fgh));
  return KRONQ_OK;
}

}  // namespace kronq

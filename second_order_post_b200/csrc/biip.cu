// Bidirectional incoherence processing (BiIP) [wmrh §三, §八, Q2; aimodeling]:
// a diagonal rescale from diag(H_X), diag(H_G) followed by a seeded orthogonal
// rotation on both sides of W, with H_X and H_G rotated to match:
//   W'   = U_G S_G W S_X U_Xᵀ
//   H_X' = U_X S_X^-1 H_X S_X^-1 U_Xᵀ,   H_G' = U_G S_G^-1 H_G S_G^-1 U_Gᵀ
// with U = (Hhat_had ⊗ Q_m) diag(sign) per side (spec in include/kronq.h).
//
// Every rotation of an R x C row-major matrix M -> P_r diag(cr) M diag(cc) P_cᵀ
// is split into memory passes whose working sets fit in shared memory:
//   tile pass     one (kr*Lr*mr) x (kc*Lc*mc) tile per CTA: input factors,
//                 Hadamard over the low Lc (Lr) index bits and Q_m on the
//                 contiguous (consecutive-row) factor of each side
//   strided pass  Hadamard over the remaining high index bits, whose elements
//                 sit at a fixed stride (within a row, or across rows); one
//                 [A][cw] slab per CTA with cw contiguous columns
// The Hadamard factors commute with each other and with Q_m (Kronecker
// structure), so the order of the passes does not change the result.
#include <math.h>

#include "kernels.cuh"

namespace kronq {
namespace {

constexpr int TILE_BUDGET = 12288;   // floats per tile buffer
constexpr int SLAB_BUDGET = 32768;   // floats per strided slab
constexpr int MAX_A = 1024;          // Hadamard length of one strided pass

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

// ------------------------------------------------------------- tile pass
struct TileP {
  const void *in;
  float *out;
  int64_t ld_in, ld_out;
  int in_bf16;
  const float *cr, *cc;  // row / column factors (null = 1)
  float norm;
  int kr, Lr, mr;        // tile rows = kr * Lr * mr
  int kc, Lc, mc;        // tile cols = kc * Lc * mc
  const float *Qr, *Qc;  // Q_m of the row side / column side (null = skip)
  int64_t tiles_c;
};

__device__ __forceinline__ float ld_in(const TileP &p, int64_t off) {
  return p.in_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p.in)[off])
                   : reinterpret_cast<const float *>(p.in)[off];
}

// Radix-2 Hadamard butterflies over n_vec vectors of length L; element j of
// vector v lives at base(v) + j*stride.
template <class Base>
__device__ void fwht_smem(float *X, int n_vec, int L, int stride, Base base) {
  for (int h = 1; h < L; h <<= 1) {
    const int half = L >> 1;
    const int total = n_vec * half;
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
      const int v = idx % n_vec, pidx = idx / n_vec;
      const int a = (pidx / h) * 2 * h + (pidx % h);
      float *x = X + base(v) + a * stride;
      const float u = x[0], w = x[h * stride];
      x[0] = u + w;
      x[h * stride] = u - w;
    }
    __syncthreads();
  }
}

// y = Q x for n_vec vectors of length m (element b at base(v) + b*stride);
// output written to Y at the same positions. Four outputs per thread.
template <class Base>
__device__ void qmix_smem(const float *X, float *Y, const float *Q, int n_vec,
                          int m, int stride, Base base) {
  const int nb4 = (m + 3) / 4;
  const int total = n_vec * nb4;
  for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
    const int v = idx % n_vec, b0 = (idx / n_vec) * 4;
    const int bo = base(v);
    float y0 = 0.f, y1 = 0.f, y2 = 0.f, y3 = 0.f;
    const float *q0 = Q + b0 * m;
    for (int k = 0; k < m; ++k) {
      const float x = X[bo + k * stride];
      y0 = fmaf(q0[k], x, y0);
      if (b0 + 1 < m) y1 = fmaf(q0[m + k], x, y1);
      if (b0 + 2 < m) y2 = fmaf(q0[2 * m + k], x, y2);
      if (b0 + 3 < m) y3 = fmaf(q0[3 * m + k], x, y3);
    }
    Y[bo + b0 * stride] = y0;
    if (b0 + 1 < m) Y[bo + (b0 + 1) * stride] = y1;
    if (b0 + 2 < m) Y[bo + (b0 + 2) * stride] = y2;
    if (b0 + 3 < m) Y[bo + (b0 + 3) * stride] = y3;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(512) tile_pass_kernel(TileP p) {
  extern __shared__ float sm[];
  const int TR = p.kr * p.Lr * p.mr, TC = p.kc * p.Lc * p.mc;
  const int TCP = TC + ((TC & 1) ? 0 : 1);
  const bool stage = (p.Qr != nullptr) || (p.Qc != nullptr);
  float *T = sm;
  float *S = sm + TR * TCP;
  float *qsm = stage ? S + TR * TCP : sm + TR * TCP;
  const float *Qr = p.Qr, *Qc = p.Qc;
  // small Q_m into shared memory
  {
    float *q = qsm;
    if (p.Qc && p.mc * p.mc <= 4096) {
      for (int e = threadIdx.x; e < p.mc * p.mc; e += blockDim.x) q[e] = p.Qc[e];
      Qc = q;
      q += p.mc * p.mc;
    }
    if (p.Qr && p.mr * p.mr <= 4096) {
      for (int e = threadIdx.x; e < p.mr * p.mr; e += blockDim.x) q[e] = p.Qr[e];
      Qr = q;
    }
  }
  const int64_t tr = blockIdx.x / p.tiles_c, tc = blockIdx.x % p.tiles_c;
  const int64_t r0 = tr * TR, c0 = tc * TC;
  for (int e = threadIdx.x; e < TR * TC; e += blockDim.x) {
    const int r = e / TC, c = e % TC;
    float v = ld_in(p, (r0 + r) * p.ld_in + c0 + c) * p.norm;
    if (p.cr) v *= p.cr[r0 + r];
    if (p.cc) v *= p.cc[c0 + c];
    T[r * TCP + c] = v;
  }
  __syncthreads();
  // ---- column side (within each row): Hadamard over a'_lo, then Q_c over b'
  const int Lc = p.Lc, mc = p.mc, Lr = p.Lr, mr = p.mr;
  if (Lc > 1) {
    const int nv = TR * p.kc * mc;
    fwht_smem(T, nv, Lc, mc, [=](int v) {
      const int b = v % mc, t2 = v / mc, kb = t2 % p.kc, r = t2 / p.kc;
      return r * TCP + kb * Lc * mc + b;
    });
  }
  if (Qc) {
    const int nv = TR * p.kc * Lc;
    qmix_smem(T, S, Qc, nv, mc, 1, [=](int v) {
      const int r = v % TR, g = v / TR;  // g = kb*Lc + a
      return r * TCP + g * mc;
    });
    float *t = T; T = S; S = t;
  }
  // ---- row side (across rows): Hadamard over a_lo, then Q_r over b
  if (Lr > 1) {
    const int nv = TC * p.kr * mr;
    fwht_smem(T, nv, Lr, mr * TCP, [=](int v) {
      const int c = v % TC, t2 = v / TC, b = t2 % mr, kb = t2 / mr;
      return (kb * Lr * mr + b) * TCP + c;
    });
  }
  if (Qr) {
    const int nv = TC * p.kr * Lr;
    qmix_smem(T, S, Qr, nv, mr, TCP, [=](int v) {
      const int c = v % TC, g = v / TC;  // g = kb*Lr + a
      return g * mr * TCP + c;
    });
    float *t = T; T = S; S = t;
  }
  for (int e = threadIdx.x; e < TR * TC; e += blockDim.x) {
    const int r = e / TC, c = e % TC;
    p.out[(r0 + r) * p.ld_out + c0 + c] = T[r * TCP + c];
  }
}

// ------------------------------------------------------------- strided pass
// View [outer][A][inner] at strides (so, sm, 1); Hadamard (unnormalised) of
// length A along the middle axis; one [A][cw] slab per CTA.
__global__ void __launch_bounds__(512)
    strided_fwht_kernel(float *base, int64_t so, int A, int64_t smid,
                        int64_t inner, int cw, int64_t chunks) {
  extern __shared__ float X[];
  const int64_t o = blockIdx.x / chunks, ch = blockIdx.x % chunks;
  const int64_t c0 = ch * cw;
  const int w = static_cast<int>(kq_min<int64_t>(cw, inner - c0));
  float *g = base + o * so + c0;
  for (int e = threadIdx.x; e < A * cw; e += blockDim.x) {
    const int a = e / cw, c = e % cw;
    X[e] = c < w ? g[a * smid + c] : 0.f;
  }
  __syncthreads();
  // radix-4 stages, then one radix-2 stage if log2(A) is odd
  int h = 1;
  for (; 4 * h <= A; h *= 4) {
    const int quads = A / 4;
    for (int idx = threadIdx.x; idx < quads * cw; idx += blockDim.x) {
      const int c = idx % cw, q = idx / cw;
      const int a = (q / h) * 4 * h + (q % h);
      float *x = X + a * cw + c;
      const float x0 = x[0], x1 = x[h * cw], x2 = x[2 * h * cw], x3 = x[3 * h * cw];
      const float s0 = x0 + x1, d0 = x0 - x1, s1 = x2 + x3, d1 = x2 - x3;
      x[0] = s0 + s1;
      x[h * cw] = d0 + d1;
      x[2 * h * cw] = s0 - s1;
      x[3 * h * cw] = d0 - d1;
    }
    __syncthreads();
  }
  if (h < A) {
    for (int idx = threadIdx.x; idx < (A / 2) * cw; idx += blockDim.x) {
      const int c = idx % cw, q = idx / cw;
      const int a = (q / h) * 2 * h + (q % h);
      float *x = X + a * cw + c;
      const float u = x[0], v = x[h * cw];
      x[0] = u + v;
      x[h * cw] = u - v;
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < A * cw; e += blockDim.x) {
    const int a = e / cw, c = e % cw;
    if (c < w) g[a * smid + c] = X[e];
  }
}

// ------------------------------------------------------------- planning
struct SideRot {
  int64_t d, had, m;
  bool rot;
  const float *Q;  // device Q_m (m > 1 and rot) or null
};

int64_t pow2_floor(int64_t x) {
  int64_t p = 1;
  while (p * 2 <= x) p *= 2;
  return p;
}

kronq_status launch_tile(cudaStream_t st, const TileP &p, int64_t R, int64_t C) {
  const int TR = p.kr * p.Lr * p.mr, TC = p.kc * p.Lc * p.mc;
  const int TCP = TC + ((TC & 1) ? 0 : 1);
  const bool stage = p.Qr || p.Qc;
  size_t smem = static_cast<size_t>(TR) * TCP * 4 * (stage ? 2 : 1);
  if (p.Qc && p.mc * p.mc <= 4096) smem += p.mc * p.mc * 4;
  if (p.Qr && p.mr * p.mr <= 4096) smem += p.mr * p.mr * 4;
  if (smem > 227 * 1024) return KRONQ_ERR_UNSUPPORTED;
  if (R % TR || C % TC) return KRONQ_ERR_UNSUPPORTED;
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(tile_pass_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    attr_done = true;
  }
  TileP q = p;
  q.tiles_c = C / TC;
  const int64_t tiles = (R / TR) * (C / TC);
  tile_pass_kernel<<<static_cast<unsigned>(tiles), 512, smem, st>>>(q);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

// Hadamard of length A (power of two) along a strided axis, split into
// passes of at most MAX_A each (Hhat_A = Hhat_A1 ⊗ Hhat_A2).
kronq_status launch_strided(cudaStream_t st, float *base, int64_t outer,
                            int64_t so, int64_t A, int64_t smid, int64_t inner) {
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(strided_fwht_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SLAB_BUDGET * 4) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    attr_done = true;
  }
  int64_t stride = smid;
  while (A > 1) {
    const int64_t a = kq_min<int64_t>(A, MAX_A);
    // this pass covers the lowest log2(a) bits of the remaining index
    const int64_t cw = kq_max<int64_t>(1, kq_min<int64_t>(inner, kq_min<int64_t>(256, SLAB_BUDGET / a)));
    const int64_t chunks = ceil_div(inner, cw);
    // outer index enumerates (outer, high index bits beyond this pass)
    const int64_t hi = A / a;
    // treat (outer, hi) as one outer axis when they are regularly strided:
    // element (o, j, t, c) at o*so + (j*a + t)*stride + c for j < hi, t < a
    for (int64_t j = 0; j < hi; ++j) {
      const int64_t blocks = outer * chunks;
      if (blocks > 0x7fffffff) return KRONQ_ERR_UNSUPPORTED;
      strided_fwht_kernel<<<static_cast<unsigned>(blocks), 512,
                            static_cast<size_t>(a * cw * 4), st>>>(
          base + j * a * stride, so, static_cast<int>(a), stride, inner,
          static_cast<int>(cw), chunks);
      KQ_CHECK_LAUNCH();
    }
    stride *= a;
    A /= a;
  }
  return KRONQ_OK;
}

// out = P_r diag(cr) in diag(cc) P_cᵀ for an R x C matrix (row-major).
kronq_status rotate(cudaStream_t st, const void *in, bool in_bf16, int64_t ld_in,
                    float *out, int64_t ld_out, int64_t R, int64_t C,
                    const SideRot &sr, const SideRot &sc, const float *cr,
                    const float *cc) {
  const int64_t had_r = sr.rot ? sr.had : 1, m_r = sr.rot ? sr.m : 1;
  const int64_t had_c = sc.rot ? sc.had : 1, m_c = sc.rot ? sc.m : 1;
  const bool qr = sr.rot && sr.m > 1, qc = sc.rot && sc.m > 1;
  const int64_t budget = TILE_BUDGET;
  // column side block: Lc * m_c, capped at 1024 floats and at the budget / m_r
  int64_t Lc = 1, Lr = 1, kc = 1, kr = 1;
  bool split = false;  // Q on both sides does not fit one tile
  if (qr && qc && m_r * m_c > budget) split = true;
  if (sc.rot) {
    const int64_t cap = split ? budget / 32 : kq_min<int64_t>(1024, budget / m_r);
    Lc = pow2_floor(kq_max<int64_t>(1, cap / m_c));
    while (had_c % Lc) Lc /= 2;
  }
  const int64_t tcb = Lc * m_c;
  if (!sc.rot || tcb < 32) {
    kc = 1;
    while (kc * tcb < 32 && C % (2 * kc * tcb) == 0) kc *= 2;
  }
  const int64_t TC = kc * tcb;
  if (!split) {
    if (sr.rot) {
      Lr = pow2_floor(kq_max<int64_t>(1, budget / (TC * m_r)));
      while (had_r % Lr) Lr /= 2;
      Lr = kq_min<int64_t>(Lr, had_r);
    }
    const int64_t trb = Lr * m_r;
    kr = 1;
    while (2 * kr * trb * TC <= budget && R % (2 * kr * trb) == 0 && kr * trb < 256)
      kr *= 2;
    TileP p{};
    p.in = in; p.out = out; p.ld_in = ld_in; p.ld_out = ld_out;
    p.in_bf16 = in_bf16; p.cr = cr; p.cc = cc;
    p.norm = static_cast<float>(1.0 / sqrt(double(had_r) * double(had_c)));
    p.kr = kr; p.Lr = Lr; p.mr = m_r; p.kc = kc; p.Lc = Lc; p.mc = m_c;
    p.Qr = qr ? sr.Q : nullptr;
    p.Qc = qc ? sc.Q : nullptr;
    KQ_TRY(launch_tile(st, p, R, C));
  } else {
    // pass 1: column side only (rows independent)
    TileP p{};
    p.in = in; p.out = out; p.ld_in = ld_in; p.ld_out = ld_out;
    p.in_bf16 = in_bf16; p.cr = cr; p.cc = cc;
    p.norm = static_cast<float>(1.0 / sqrt(double(had_r) * double(had_c)));
    kr = 1;
    while (2 * kr * TC <= budget && R % (2 * kr) == 0 && kr < 64) kr *= 2;
    p.kr = kr; p.Lr = 1; p.mr = 1; p.kc = kc; p.Lc = Lc; p.mc = m_c;
    p.Qc = sc.Q;
    KQ_TRY(launch_tile(st, p, R, C));
    // pass 2: row side only (columns independent), in place on out
    TileP q{};
    q.in = out; q.out = out; q.ld_in = ld_out; q.ld_out = ld_out;
    q.in_bf16 = 0; q.norm = 1.f;
    Lr = pow2_floor(kq_max<int64_t>(1, budget / (32 * m_r)));
    while (had_r % Lr) Lr /= 2;
    int64_t kc2 = 1;
    while (Lr * m_r * 2 * kc2 <= budget && C % (2 * kc2) == 0 && kc2 < 32) kc2 *= 2;
    q.kr = 1; q.Lr = Lr; q.mr = m_r; q.kc = kc2; q.Lc = 1; q.mc = 1;
    q.Qr = sr.Q;
    KQ_TRY(launch_tile(st, q, R, C));
  }
  // remaining Hadamard bits
  const int64_t Ac = had_c / Lc, Ar = had_r / Lr;
  if (Ac > 1) KQ_TRY(launch_strided(st, out, R, ld_out, Ac, tcb, tcb));
  if (Ar > 1) {
    const int64_t blk = Lr * m_r;  // rows per block
    KQ_TRY(launch_strided(st, out, blk, ld_out, Ar, blk * ld_out, C));
  }
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

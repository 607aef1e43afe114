// The quantized sublayer applied to activations [aimodeling: packed low-bit
// weights used through a fused dequant + BiIP matvec; wmrh Q2: the two
// Hadamard transforms per layer at inference]:
//   y = S_G^-1 U_G^T W_hat' U_X S_X^-1 x
// for a few tokens x (rows of X, B x d_in), with W_hat' never expanded in
// memory: the codes are unpacked in registers inside the product.
//
//   1. x2 = U_X S_X^-1 x      the BiIP row pass (Hadamard ⊗ Q_m of the input
//                             side, with the factors sign/s applied first)
//   2. y1 = W_hat' x2         dequant GEMV: per row and group,
//                             scale * (sum_c q_c x2_c - zero * sum_c x2_c)
//   3. y  = S_G^-1 U_G^T y1   the BiIP row pass with Q_m^T of the output
//                             side, then the factors sign/s
//
// The GEMV streams the packed codes (bits/8 bytes per weight) once per
// token: a CTA owns 16 rows, its warps split the columns in chunks, and each
// lane takes 16 (or, at 3 bits, 32) consecutive columns, i.e. whole code
// words. A lane keeps its slice of x2 in registers and first loads the code
// words of all 16 rows, so that 16 independent loads per lane are in flight;
// codes become floats by the exact bit-pattern trick (2^23 + q) - 2^23.
#include "kernels.cuh"

namespace kronq {
namespace {

constexpr int MV_THREADS = 512;
constexpr int MV_WARPS = MV_THREADS / 32;
constexpr int MV_ROWS = 16;                      // rows per CTA

// Columns a lane takes per chunk: 16 for 2 and 4 bits (one or two whole code
// words), 32 for 3 bits (three words).
template <int BITS>
struct MvShape {
  static constexpr int COLS = BITS == 3 ? 32 : 16;
  static constexpr int WORDS = COLS * BITS / 32;
  static constexpr int CHUNK = 32 * COLS;
};

// float of a small unsigned integer q < 2^23: the bit pattern 2^23 + q as a
// float, minus 2^23 (exact)
__device__ __forceinline__ float small_uint_to_float(uint32_t q) {
  return __uint_as_float(q | 0x4B000000u) - 8388608.0f;
}

// One token: y1[row] = sum_g scale * (sum_c q_c x_c - zero * sum_c x_c) for
// the CTA's MV_ROWS rows; the warps of a CTA split the columns in chunks and
// meet in shared memory at the end.
template <int BITS>
__global__ void __launch_bounds__(MV_THREADS, BITS == 3 ? 1 : 2)
    dequant_gemv_kernel(const uint32_t *__restrict__ codes, const float *__restrict__ scales,
                        const uint8_t *__restrict__ zeros, int d_out, int d_in, int group,
                        const float *__restrict__ x2, float *__restrict__ y1) {
  using S = MvShape<BITS>;
  __shared__ float part[MV_WARPS][MV_ROWS];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r0 = blockIdx.x * MV_ROWS;
  const int nr = min(MV_ROWS, d_out - r0);
  const int64_t words_row = static_cast<int64_t>(BITS) * d_in / 32;
  const int ng = d_in / group;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  float acc[MV_ROWS];
#pragma unroll
  for (int k = 0; k < MV_ROWS; ++k) acc[k] = 0.f;
  const int nchunks = (d_in + S::CHUNK - 1) / S::CHUNK;
  for (int ch = warp; ch < nchunks; ch += MV_WARPS) {
    const int col = ch * S::CHUNK + S::COLS * lane;
    if (col >= d_in) continue;
    float xv[S::COLS];
    float xsum = 0.f;
    const float4 *x4 = reinterpret_cast<const float4 *>(x2 + col);
#pragma unroll
    for (int q = 0; q < S::COLS / 4; ++q) {
      const float4 v = __ldg(x4 + q);
      xv[4 * q] = v.x;
      xv[4 * q + 1] = v.y;
      xv[4 * q + 2] = v.z;
      xv[4 * q + 3] = v.w;
      xsum += (v.x + v.y) + (v.z + v.w);
    }
    const int g = col / group;
    const int64_t w0 = static_cast<int64_t>(col) * BITS / 32;
    // all rows' code words first: MV_ROWS independent loads in flight
    uint32_t w[MV_ROWS][S::WORDS];
#pragma unroll
    for (int k = 0; k < MV_ROWS; ++k) {
      const int64_t row = r0 + kq_min(k, nr - 1);
      const uint32_t *p = codes + row * words_row + w0;
#pragma unroll
      for (int t = 0; t < S::WORDS; ++t) w[k][t] = __ldg(p + t);
    }
#pragma unroll
    for (int k = 0; k < MV_ROWS; ++k) {
      const int64_t row = r0 + kq_min(k, nr - 1);
      const float sc = __ldg(scales + row * ng + g);
      const float z = static_cast<float>(__ldg(zeros + row * ng + g));
      float dot = 0.f;
#pragma unroll
      for (int j = 0; j < S::COLS; ++j) {
        const int bit = j * BITS, wi = bit >> 5, sh = bit & 31;
        uint32_t q;
        if (sh + BITS <= 32) {
          q = (w[k][wi] >> sh) & MASK;
        } else {   // a 3-bit code across two words
          q = ((w[k][wi] >> sh) | (w[k][wi + 1] << (32 - sh))) & MASK;
        }
        dot = fmaf(small_uint_to_float(q), xv[j], dot);
      }
      acc[k] = fmaf(sc, dot - z * xsum, acc[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < MV_ROWS; ++k) {
    const float v = warp_sum(acc[k]);
    if (lane == 0) part[warp][k] = v;
  }
  __syncthreads();
  if (threadIdx.x < nr) {
    float v = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < MV_WARPS; ++w2) v += part[w2][threadIdx.x];
    y1[r0 + threadIdx.x] = v;
  }
}

// ---- 2- and 4-bit codes: two codes per packed fp32 pair instruction
// A code q_j at bits [b*j, b*j + b) of a 16-bit half word w16 becomes a float
// exactly as ((w16 & mask_j) | bits(2^23)) - 2^23 = q_j * 2^(b*j): no shift
// per code. The matching x value is stored pre-scaled by 2^(-b*j) (exact), so
// the product is q_j * x_j. Pairs of codes go through one packed subtract and
// one packed FMA (fp32x2) into a two-lane accumulator.
__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  return (static_cast<unsigned long long>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

template <int BITS>
struct MvShapeX2 {
  static constexpr int COLS = 32 / BITS, WORDS = 1, CHUNK = 32 * COLS;
};

template <int BITS>
__global__ void __launch_bounds__(MV_THREADS, 2)
    dequant_gemv_x2_kernel(const uint32_t *__restrict__ codes, const float *__restrict__ scales,
                           const uint8_t *__restrict__ zeros, int d_out, int d_in, int group,
                           const float *__restrict__ x2, float *__restrict__ y1) {
  static_assert(BITS == 2 || BITS == 4, "codes must not straddle 16-bit halves");
  using S = MvShapeX2<BITS>;                  // one code word a lane per row
  constexpr int PER16 = 16 / BITS;            // codes per 16-bit half word
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  constexpr uint32_t MAGIC = 0x4B000000u;     // bits of 2^23
  __shared__ float part[MV_WARPS][MV_ROWS];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r0 = blockIdx.x * MV_ROWS;
  const int nr = min(MV_ROWS, d_out - r0);
  const int64_t words_row = static_cast<int64_t>(BITS) * d_in / 32;
  const int ng = d_in / group;
  const unsigned long long neg2 = pack2(-8388608.0f, -8388608.0f);
  float acc[MV_ROWS];
#pragma unroll
  for (int k = 0; k < MV_ROWS; ++k) acc[k] = 0.f;
  const int nchunks = (d_in + S::CHUNK - 1) / S::CHUNK;
  for (int ch = warp; ch < nchunks; ch += MV_WARPS) {
    const int col = ch * S::CHUNK + S::COLS * lane;
    if (col >= d_in) continue;
    // x pre-scaled by 2^(-BITS * position in its half word), as pairs
    unsigned long long xp[S::COLS / 2];
    float xsum = 0.f;
    const float4 *x4 = reinterpret_cast<const float4 *>(x2 + col);
#pragma unroll
#pragma unroll
    for (int q = 0; q < S::COLS / 4; ++q) {
      const float4 v = __ldg(x4 + q);
      xsum += (v.x + v.y) + (v.z + v.w);
      const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j0 = 4 * q + 2 * h, j1 = j0 + 1;
        // times 2^(-BITS * position): exact (a power of two)
        xp[j0 / 2] = pack2(e[2 * h] * __int_as_float((127 - BITS * (j0 % PER16)) << 23),
                           e[2 * h + 1] * __int_as_float((127 - BITS * (j1 % PER16)) << 23));
      }
    }
    const int g = col / group;
    const int64_t w0 = static_cast<int64_t>(col) * BITS / 32;
    uint32_t w[MV_ROWS][S::WORDS];
#pragma unroll
    for (int k = 0; k < MV_ROWS; ++k) {
      const int64_t row = r0 + kq_min(k, nr - 1);
      const uint32_t *p = codes + row * words_row + w0;
#pragma unroll
      for (int t = 0; t < S::WORDS; ++t) w[k][t] = __ldg(p + t);
    }
#pragma unroll
    for (int k = 0; k < MV_ROWS; ++k) {
      const int64_t row = r0 + kq_min(k, nr - 1);
      const float sc = __ldg(scales + row * ng + g);
      const float z = static_cast<float>(__ldg(zeros + row * ng + g));
      unsigned long long a2 = 0ull;
#pragma unroll
      for (int t = 0; t < S::WORDS; ++t) {
#pragma unroll
        for (int hw = 0; hw < 2; ++hw) {
          const uint32_t h16 = hw ? (w[k][t] >> 16) : w[k][t];
#pragma unroll
          for (int i = 0; i < PER16; i += 2) {
            const uint32_t lo = (h16 & (MASK << (BITS * i))) | MAGIC;
            const uint32_t hi = (h16 & (MASK << (BITS * (i + 1)))) | MAGIC;
            const int j = (t * 2 + hw) * PER16 + i;   // column within the lane's 16
            a2 = fma2(add2(pack2(__uint_as_float(lo), __uint_as_float(hi)), neg2), xp[j / 2], a2);
          }
        }
      }
      const float dot = __uint_as_float(static_cast<uint32_t>(a2)) +
                        __uint_as_float(static_cast<uint32_t>(a2 >> 32));
      acc[k] = fmaf(sc, dot - z * xsum, acc[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < MV_ROWS; ++k) {
    const float v = warp_sum(acc[k]);
    if (lane == 0) part[warp][k] = v;
  }
  __syncthreads();
  if (threadIdx.x < nr) {
    float v = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < MV_WARPS; ++w2) v += part[w2][threadIdx.x];
    y1[r0 + threadIdx.x] = v;
  }
}

__global__ void scale_cols_kernel(const float *in, const float *f, float *out, int64_t B,
                                  int64_t d) {
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < B * d;
       e += int64_t(gridDim.x) * blockDim.x)
    out[e] = in[e] * f[e % d];
}

size_t al256(size_t b) { return (b + 255) / 256 * 256; }

struct Desc {
  float *fx, *fg, *Qx, *QgT, *Qg;
  double *G;
};

Desc desc_layout(void *p, int64_t d_out, int64_t d_in) {
  uint8_t *w = static_cast<uint8_t *>(p);
  Desc d;
  d.fx = reinterpret_cast<float *>(w); w += al256(d_in * 4);
  d.fg = reinterpret_cast<float *>(w); w += al256(d_out * 4);
  d.Qx = reinterpret_cast<float *>(w); w += al256(256 * 256 * 4);
  d.QgT = reinterpret_cast<float *>(w); w += al256(256 * 256 * 4);
  d.Qg = reinterpret_cast<float *>(w); w += al256(256 * 256 * 4);
  d.G = reinterpret_cast<double *>(w);
  return d;
}

template <int BITS>
kronq_status launch_gemv(cudaStream_t st, const uint32_t *codes, const float *scales,
                         const uint8_t *zeros, int64_t d_out, int64_t d_in, int group,
                         const float *x2, float *y1) {
  const int64_t grid = ceil_div(d_out, MV_ROWS);
  if constexpr (BITS == 3) {
    dequant_gemv_kernel<BITS><<<static_cast<unsigned>(grid), MV_THREADS, 0, st>>>(
        codes, scales, zeros, static_cast<int>(d_out), static_cast<int>(d_in), group, x2, y1);
  } else {
    dequant_gemv_x2_kernel<BITS><<<static_cast<unsigned>(grid), MV_THREADS, 0, st>>>(
        codes, scales, zeros, static_cast<int>(d_out), static_cast<int>(d_in), group, x2, y1);
  }
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

}  // namespace

size_t matvec_desc_bytes(int64_t d_out, int64_t d_in) {
  return al256(d_in * 4) + al256(d_out * 4) + 3 * al256(256 * 256 * 4) +
         al256(2 * 256 * 256 * 8) + 256;
}

size_t matvec_ws_bytes(int64_t d_out, int64_t d_in, int64_t B) {
  return al256(static_cast<size_t>(B) * d_in * 4) + 2 * al256(static_cast<size_t>(B) * d_out * 4) +
         256;
}

kronq_status matvec_prepare(cudaStream_t st, const kronq_opts &o, const float *s_x,
                            const float *s_g, int64_t d_out, int64_t d_in, void *desc) {
  const Desc d = desc_layout(desc, d_out, d_in);
  return rotation_factors(st, o, s_x, s_g, d_out, d_in, d.fx, d.fg, d.Qx, d.QgT, d.Qg, d.G);
}

kronq_status dequant_matvec(cudaStream_t st, const kronq_opts &o, const void *desc,
                            const uint32_t *codes, const float *scales, const uint8_t *zeros,
                            int64_t d_out, int64_t d_in, const float *x, int64_t B, float *y,
                            void *ws, int32_t *info) {
  const Desc d = desc_layout(const_cast<void *>(desc), d_out, d_in);
  const bool rot_x = !(o.flags & KRONQ_FLAG_NO_ROT_IN);
  const bool rot_g = !(o.flags & KRONQ_FLAG_NO_ROT_OUT);
  uint8_t *w = static_cast<uint8_t *>(ws);
  float *x2 = reinterpret_cast<float *>(w); w += al256(static_cast<size_t>(B) * d_in * 4);
  float *y1 = reinterpret_cast<float *>(w); w += al256(static_cast<size_t>(B) * d_out * 4);
  float *y2 = reinterpret_cast<float *>(w);
  // 1. x2 = U_X S_X^-1 x
  KQ_TRY(rotate_rows(st, x, x2, B, d_in, rot_x, o.rot_in.had, o.rot_in.m, d.Qx, d.fx, info));
  // 2. y1 = W_hat' x2, one pass over the codes per token
  for (int64_t b = 0; b < B; ++b) {
    const float *xb = x2 + b * d_in;
    float *yb = y1 + b * d_out;
    if (o.bits == 2)
      KQ_TRY(launch_gemv<2>(st, codes, scales, zeros, d_out, d_in, o.group, xb, yb));
    else if (o.bits == 3)
      KQ_TRY(launch_gemv<3>(st, codes, scales, zeros, d_out, d_in, o.group, xb, yb));
    else
      KQ_TRY(launch_gemv<4>(st, codes, scales, zeros, d_out, d_in, o.group, xb, yb));
  }
  // 3. y = S_G^-1 U_G^T y1: Hadamard ⊗ Q_m^T, then sign / s
  KQ_TRY(rotate_rows(st, y1, y2, B, d_out, rot_g, o.rot_out.had, o.rot_out.m, d.QgT, nullptr,
                     info));
  const int64_t n = B * d_out;
  scale_cols_kernel<<<static_cast<unsigned>(kq_min<int64_t>(ceil_div(n, 256), 1024)), 256, 0,
                      st>>>(y2, d.fg, y, B, d_out);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

}  // namespace kronq

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

// packed fp32 pairs (two lanes in one 64-bit register)
__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  unsigned long long d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ float2 unpack2(unsigned long long v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
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

// The streaming GEMV for 2- and 4-bit codes: every warp streams whole rows, a
// row block of MV3_RB rows at a time, 16 bytes of code words per lane and row
// per step (all rows' loads in flight at once); the lane's x values are read
// once per step (L1-resident: x is the same for every row) for all the
// block's rows.
//   A code q at bits [b*i, b*i + b) of a 16-bit half word h becomes a float
// exactly as ((h & mask_i) | bits(2^23)) - 2^23 = q * 2^(b*i): no shift per
// code. x is scaled by 2^(-b*i) on the way in (exact), so the product is
// q * x. Pairs of codes take one packed subtract and one packed FMA (fp32x2)
// into a two-lane accumulator.
constexpr int MV3_THREADS = 256;
constexpr int MV3_RB = 8;                        // rows per row block of a warp

template <int BITS>
struct Mv3 {
  static constexpr int WORDS = 4;                      // code words per lane and step
  static constexpr int LCOLS = WORDS * 32 / BITS;      // columns per lane and step
  static constexpr int TILE = 32 * LCOLS;              // columns per warp step
};

// 2^(-k) for 0 <= k <= 126, exact
__device__ __forceinline__ float pow2_neg(int k) { return __int_as_float((127 - k) << 23); }

template <int BITS>
__global__ void __launch_bounds__(MV3_THREADS, 2)
    dequant_gemv3_kernel(const uint32_t *__restrict__ codes, const float *__restrict__ scales,
                         const uint8_t *__restrict__ zeros, int d_out, int d_in, int group,
                         int rblk, const float *__restrict__ x2, float *__restrict__ y1) {
  using S = Mv3<BITS>;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  constexpr uint32_t MAGIC = 0x4B000000u;        // bits of 2^23
  __shared__ float part[MV3_THREADS / 32][MV3_RB];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarp = MV3_THREADS / 32, cs_n = nwarp / rblk;
  const int rb = warp % rblk, cs = warp / rblk;
  const int row0 = (blockIdx.x * rblk + rb) * MV3_RB;
  const int64_t words_row = static_cast<int64_t>(BITS) * d_in / 32;
  const int ng = d_in / group;
  const unsigned long long neg2 = pack2(-8388608.0f, -8388608.0f);
  // one packed step: codes at bits sh0 of h0 and sh1 of h1 against the x pair
  auto step = [&](unsigned long long &acc2, uint32_t h0, int sh0, uint32_t h1, int sh1,
                  unsigned long long xp) {
    const uint32_t lo = (h0 & (MASK << sh0)) | MAGIC;
    const uint32_t hi = (h1 & (MASK << sh1)) | MAGIC;
    acc2 = fma2(add2(pack2(__uint_as_float(lo), __uint_as_float(hi)), neg2), xp, acc2);
  };
  float acc[MV3_RB];
#pragma unroll
  for (int k = 0; k < MV3_RB; ++k) acc[k] = 0.f;
  const int ntiles = (d_in + S::TILE - 1) / S::TILE;
  for (int t = cs; t < ntiles; t += cs_n) {
    const int c = t * S::TILE + lane * S::LCOLS;
    if (c >= d_in) continue;
    uint32_t w[MV3_RB][S::WORDS];
#pragma unroll
    for (int k = 0; k < MV3_RB; ++k) {
      const int row = min(row0 + k, d_out - 1);
      const uint32_t *p = codes + row * words_row + static_cast<int64_t>(c) * BITS / 32;
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
      w[k][0] = v.x;
      w[k][1] = v.y;
      w[k][2] = v.z;
      w[k][3] = v.w;
    }
    unsigned long long a2[MV3_RB];
#pragma unroll
    for (int k = 0; k < MV3_RB; ++k) a2[k] = 0ull;
    float xsum = 0.f;
    {
      constexpr int PER16 = 16 / BITS;           // codes per 16-bit half word
#pragma unroll
      for (int hwi = 0; hwi < 8; ++hwi) {        // half words of the 4 code words
        const int j0 = hwi * PER16;
        float xv[PER16];
#pragma unroll
        for (int q = 0; q < PER16 / 4; ++q) {
          const float4 v = __ldg(reinterpret_cast<const float4 *>(x2 + c + j0) + q);
          xv[4 * q] = v.x;
          xv[4 * q + 1] = v.y;
          xv[4 * q + 2] = v.z;
          xv[4 * q + 3] = v.w;
        }
#pragma unroll
        for (int i = 0; i < PER16; i += 2) {
          xsum += xv[i] + xv[i + 1];
          const unsigned long long xp =
              pack2(xv[i] * pow2_neg(BITS * i), xv[i + 1] * pow2_neg(BITS * (i + 1)));
#pragma unroll
          for (int k = 0; k < MV3_RB; ++k) {
            const uint32_t h = (hwi & 1) ? (w[k][hwi >> 1] >> 16) : w[k][hwi >> 1];
            step(a2[k], h, BITS * i, h, BITS * (i + 1), xp);
          }
        }
      }
    }
    const int g = c / group;
#pragma unroll
    for (int k = 0; k < MV3_RB; ++k) {
      const int row = min(row0 + k, d_out - 1);
      const float sc = __ldg(scales + static_cast<int64_t>(row) * ng + g);
      const float z = static_cast<float>(__ldg(zeros + static_cast<int64_t>(row) * ng + g));
      const float2 d2 = unpack2(a2[k]);
      const float dot = d2.x + d2.y;
      acc[k] = fmaf(sc, dot - z * xsum, acc[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < MV3_RB; ++k) {
    const float v = warp_sum(acc[k]);
    if (lane == 0) part[warp][k] = v;
  }
  __syncthreads();
  if (threadIdx.x < rblk * MV3_RB) {
    const int rbi = threadIdx.x / MV3_RB, k = threadIdx.x % MV3_RB;
    const int row = (blockIdx.x * rblk + rbi) * MV3_RB + k;
    if (row < d_out) {
      float v = 0.f;
      for (int c2 = 0; c2 < cs_n; ++c2) v += part[c2 * rblk + rbi][k];
      y1[row] = v;
    }
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
  if constexpr (BITS != 3) {
    constexpr int64_t LCOLS = Mv3<BITS>::LCOLS;
    if (d_in % LCOLS == 0 && group % LCOLS == 0) {
      // row blocks per CTA (the other warps split the columns): the largest
      // that still gives every SM two CTAs
      int rblk = 4;
      while (rblk > 1 && ceil_div(d_out, int64_t(rblk) * MV3_RB) < 2 * 148) rblk /= 2;
      const int64_t grid3 = ceil_div(d_out, int64_t(rblk) * MV3_RB);
      dequant_gemv3_kernel<BITS><<<static_cast<unsigned>(grid3), MV3_THREADS, 0, st>>>(
          codes, scales, zeros, static_cast<int>(d_out), static_cast<int>(d_in), group, rblk,
          x2, y1);
      KQ_CHECK_LAUNCH();
      return KRONQ_OK;
    }
  }
  const int64_t grid = ceil_div(d_out, MV_ROWS);
  dequant_gemv_kernel<BITS><<<static_cast<unsigned>(grid), MV_THREADS, 0, st>>>(
      codes, scales, zeros, static_cast<int>(d_out), static_cast<int>(d_in), group, x2, y1);
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

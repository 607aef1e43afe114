// Blocked column-wise OBS quantize-and-compensate [gptget-en Methodology:
// extends GPTQ's column-wise OBS; wmrh §四: the per-column update is GPTAQ's
// and H_G does not enter it, so rows are independent given U; wmrh §五:
// W2/W3/W4 with 128-column groups].
//
// Per 128-column block j0 (one launch of obs_block_kernel): eight lanes share
// one row, lane p of the eight holding the columns 8i + p (i < 16) in
// registers, so that every lane has about the same number of updates left at
// any column. U[j0:j0+128, j0:j0+128] sits in shared memory, permuted so that
// each lane's columns of a U row are contiguous. The sweep over the block's
// 128 columns is unrolled, so every register index is a compile-time
// constant. For each column j: group (scale, zero) at a group start,
// q = clamp(rint(w/scale)+zero), err = (w - w_hat)/U[j][j] (the row's eight
// lanes all compute them from the owner's weight), w_k -= err * U[j][k] for
// the block's k > j. The errors go to E; the columns right of the block are
// updated lazily by 3xTF32 GEMMs: within a super-block of S columns after
// every block (W[:, blk_end:sb_end] -= E_blk U[blk, blk_end:sb_end]), and
// once per super-block for everything right of it
// (W[:, sb_end:] -= E_sb U[sb, sb_end:]). Codes are packed in registers
// during the sweep (little-endian bitstream per row).
#include <utility>

#include "kernels.cuh"

namespace kronq {
namespace {

constexpr int OB = 128;                    // block width
constexpr int QLPR = 8;                    // lanes per row
constexpr int QNI = OB / QLPR;             // columns (registers) per lane
constexpr int QWARPS = 8;
constexpr int OTHREADS = 32 * QWARPS;
constexpr int OROWS = QWARPS * (32 / QLPR);  // rows per CTA
constexpr int QUP = QNI + 4;               // one lane's run of a U row (padded)
constexpr int QUROW = QLPR * QUP;          // floats per permuted U row
constexpr int OSMEM = (OB * QUROW + OB) * 4;
constexpr int SUPER = 1024;                // super-block width

// State of one lane during the sweep of a block.
template <int BITS>
struct SweepState {
  static constexpr int NW = OB * BITS / 32;  // code words of the block per row
  float w[QNI], err[QNI];
  uint32_t cw[NW];
  float scale, rscale, zero;
};

// Where a row's group parameters go: scales[gi], zeros[gi] for the group gi
// that starts at block column J is gi = g0 + J / group.
struct GroupOut {
  float *scales;
  uint8_t *zeros;
  int64_t g0;
  bool store;
};

// Column J of the block (every register index is a compile-time constant).
template <int BITS, int J>
__device__ __forceinline__ void obs_column(SweepState<BITS> &S, const float *Up,
                                           const float *inv, int p, int lane0,
                                           int group, const GroupOut &go) {
  constexpr int io = J / QLPR, po = J % QLPR;
  constexpr float maxq = static_cast<float>((1 << BITS) - 1);
  if constexpr (J % 32 == 0) {
    if (J % group == 0) {
      // group start: (scale, zero) from the row's current weights of the group
      float mn = INFINITY, mx = -INFINITY;
#pragma unroll
      for (int i = io; i < QNI; ++i) {
        if (QLPR * i < J + group) {
          mn = fminf(mn, S.w[i]);
          mx = fmaxf(mx, S.w[i]);
        }
      }
#pragma unroll
      for (int o = 1; o < QLPR; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      const float xmin = fminf(mn, 0.f), xmax = fmaxf(mx, 0.f);
      if (xmax == xmin) {
        S.scale = 1.f;
        S.zero = 0.f;
      } else {
        S.scale = (xmax - xmin) / maxq;
        S.zero = rintf(-xmin / S.scale);
      }
      S.rscale = 1.f / S.scale;
      if (go.store) {
        const int64_t gi = go.g0 + J / group;
        go.scales[gi] = S.scale;
        go.zeros[gi] = static_cast<uint8_t>(S.zero);
      }
    }
  }
  const float4 *u4 = reinterpret_cast<const float4 *>(Up + J * QUROW + p * QUP);
  const float iu = inv[J];
  const float wj = __shfl_sync(0xffffffffu, S.w[io], lane0 | po);
  // w/scale as a product with the group's reciprocal: it can differ from
  // the quotient only within an ulp of a rounding tie
  const float q = fminf(fmaxf(rintf(wj * S.rscale) + S.zero, 0.f), maxq);
  const float wh = S.scale * (q - S.zero);
  const float e = (wj - wh) * iu;
  {
    const uint32_t qi = static_cast<uint32_t>(q);
    constexpr int bit = J * BITS, k = bit / 32, s = bit % 32;
    S.cw[k] |= qi << s;
    if constexpr (s + BITS > 32) S.cw[k + 1] |= qi >> (32 - s);
  }
#pragma unroll
  for (int a = io / 4; a < QNI / 4; ++a) {
    const float4 u = u4[a];
    const float uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = 4 * a + c;
      if (i == io) {
        // the column itself: the owner keeps w_hat and the error, the row's
        // lanes right of it update their column of the same i
        if (p > po) S.w[i] = fmaf(-e, uu[c], S.w[i]);
        else if (p == po) {
          S.w[i] = wh;
          S.err[i] = e;
        }
      } else if (i > io) {
        S.w[i] = fmaf(-e, uu[c], S.w[i]);
      }
    }
  }
}

template <int BITS, int... J>
__device__ __forceinline__ void obs_sweep(std::integer_sequence<int, J...>,
                                          SweepState<BITS> &S, const float *Up,
                                          const float *inv, int p, int lane0, int group,
                                          const GroupOut &go) {
  (obs_column<BITS, J>(S, Up, inv, p, lane0, group, go), ...);
}

// One 128-column block for OROWS rows per CTA (32 / QLPR rows per warp).
template <int BITS>
__global__ void __launch_bounds__(OTHREADS)
    obs_block_kernel(float *__restrict__ W, int64_t ldw,
                     const float *__restrict__ U, int64_t ldu, int64_t j0,
                     int64_t d_out, int group,
                     float *__restrict__ E, int64_t lde, int64_t e_col,
                     uint32_t *__restrict__ codes, int64_t ldq,
                     float *__restrict__ scales, uint8_t *__restrict__ zeros,
                     int64_t ngroups) {
  extern __shared__ __align__(16) float Up[];  // Up[j][p][i] = U[j][QLPR*i + p]
  float *inv = Up + OB * QUROW;                // 1/U[j][j]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = lane & (QLPR - 1), lane0 = lane & ~(QLPR - 1);
  const int64_t row = int64_t(blockIdx.x) * OROWS + warp * (32 / QLPR) + lane / QLPR;
  const bool ok = row < d_out;
  SweepState<BITS> S;
#pragma unroll
  for (int i = 0; i < QNI; ++i) {
    S.w[i] = ok ? W[row * ldw + j0 + QLPR * i + p] : 0.f;
    S.err[i] = 0.f;
  }
  // U block: float4 loads of a row's 4 consecutive columns (one per lane
  // phase), eight in flight per thread, scattered into the permuted layout
  constexpr int C4 = OB / 4;                        // float4s per U row
  constexpr int BATCH = 8;
  static_assert((OB * C4) % (OTHREADS * BATCH) == 0, "U block batches");
  for (int e0 = threadIdx.x; e0 < OB * C4; e0 += OTHREADS * BATCH) {
    float4 v[BATCH];
#pragma unroll
    for (int b = 0; b < BATCH; ++b) {
      const int e = e0 + b * OTHREADS, r = e / C4, c4 = e % C4;
      v[b] = __ldg(reinterpret_cast<const float4 *>(U + (j0 + r) * ldu + j0) + c4);
    }
#pragma unroll
    for (int b = 0; b < BATCH; ++b) {
      const int e = e0 + b * OTHREADS, r = e / C4, c4 = e % C4;
      const float vv[4] = {v[b].x, v[b].y, v[b].z, v[b].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int c = 4 * c4 + q;
        Up[r * QUROW + (c % QLPR) * QUP + c / QLPR] = vv[q];
      }
    }
  }
#pragma unroll
  for (int k = 0; k < SweepState<BITS>::NW; ++k) S.cw[k] = 0u;
  S.scale = 1.f;
  S.rscale = 1.f;
  S.zero = 0.f;
  __syncthreads();
  if (threadIdx.x < OB) {
    const int j = threadIdx.x;
    inv[j] = 1.f / Up[j * QUROW + (j % QLPR) * QUP + j / QLPR];
  }
  __syncthreads();
  const GroupOut go{scales + row * ngroups, zeros + row * ngroups, j0 / group,
                    p == 0 && ok};
  obs_sweep<BITS>(std::make_integer_sequence<int, OB>{}, S, Up, inv, p, lane0, group, go);
  if (!ok) return;
#pragma unroll
  for (int i = 0; i < QNI; ++i) {
    W[row * ldw + j0 + QLPR * i + p] = S.w[i];
    E[row * lde + e_col + QLPR * i + p] = S.err[i];
  }
  uint32_t *cr = codes + row * ldq + (j0 * BITS) / 32;
#pragma unroll
  for (int k = 0; k < SweepState<BITS>::NW; ++k)
    if (k / BITS == p) cr[k] = S.cw[k];
}

__global__ void diff_inplace_kernel(float *__restrict__ A, int64_t lda,
                                    const float *__restrict__ B, int64_t ldb,
                                    int64_t rows, int64_t cols) {
  for (int64_t r = blockIdx.y; r < rows; r += gridDim.y)
    for (int64_t c = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; c < cols;
         c += int64_t(gridDim.x) * blockDim.x)
      A[r * lda + c] -= B[r * ldb + c];
}

}  // namespace

// Workspace: the errors E (d_out x S), then scratch for the super-block
// products (d_out x (d_in - S) x S at most).
size_t quant_ws_bytes(int64_t d_out, int64_t d_in, const kronq_opts &) {
  const int64_t S = kq_min<int64_t>(d_in, SUPER);
  const size_t e = (static_cast<size_t>(d_out) * S * 4 + 255) / 256 * 256;
  return e + gemm_scratch_bytes(d_out, d_in - S, S) + 256;
}

// OBS over the n columns of a strided view: W (pitch ldw), its U block
// (pitch ldu), and the codes / scales / zeros of those columns (row pitches
// ldq words and lds groups of the full arrays).
kronq_status quantize_view(cudaStream_t st, const kronq_opts &o, const QuantView &v,
                           void *ws, size_t ws_bytes, int32_t *info) {
  const int64_t d_out = v.d_out, n = v.n;
  if (ws_bytes < quant_ws_bytes(d_out, n, o)) return KRONQ_ERR_INVALID_ARG;
  const int64_t S = kq_min<int64_t>(n, SUPER);
  float *E = static_cast<float *>(ws);
  const size_t e_bytes = (static_cast<size_t>(d_out) * S * 4 + 255) / 256 * 256;
  void *scr = static_cast<uint8_t *>(ws) + e_bytes;
  const size_t scr_bytes = ws_bytes - e_bytes;
  KQ_TRY(smem_attr(obs_block_kernel<2>, OSMEM));
  KQ_TRY(smem_attr(obs_block_kernel<3>, OSMEM));
  KQ_TRY(smem_attr(obs_block_kernel<4>, OSMEM));
  auto block_kernel = o.bits == 2 ? obs_block_kernel<2>
                      : o.bits == 3 ? obs_block_kernel<3>
                                    : obs_block_kernel<4>;
  if (o.bits < 2 || o.bits > 4) return KRONQ_ERR_INVALID_ARG;
  float *W = v.W;
  const float *U = v.U;
  const unsigned grid = static_cast<unsigned>(ceil_div(d_out, OROWS));
  for (int64_t sb0 = 0; sb0 < n; sb0 += S) {
    const int64_t sb1 = kq_min<int64_t>(n, sb0 + S);
    for (int64_t j0 = sb0; j0 < sb1; j0 += OB) {
      block_kernel<<<grid, OTHREADS, OSMEM, st>>>(
          W, v.ldw, U, v.ldu, j0, d_out, o.group, E, S, j0 - sb0, v.codes,
          v.ldq, v.scales, v.zeros, v.lds);
      KQ_CHECK_LAUNCH();
      if (j0 + OB < sb1) {
        GemmArgs g;
        g.M = d_out; g.N = sb1 - j0 - OB; g.K = OB;
        g.A = E + (j0 - sb0); g.lda = S;
        g.B = U + j0 * v.ldu + j0 + OB; g.ldb = v.ldu; g.b_mn = true;
        g.C = W + j0 + OB; g.ldc = v.ldw;
        g.alpha = -1.f; g.beta = 1.f;
        KQ_TRY(gemm_tf32x3(st, g, info));
      }
    }
    if (sb1 < n) {
      GemmArgs g;
      g.M = d_out; g.N = n - sb1; g.K = sb1 - sb0;
      g.A = E; g.lda = S;
      g.B = U + sb0 * v.ldu + sb1; g.ldb = v.ldu; g.b_mn = true;
      g.C = W + sb1; g.ldc = v.ldw;
      g.alpha = -1.f; g.beta = 1.f;
      KQ_TRY(gemm_f32(st, g, scr, scr_bytes, info));
    }
  }
  return KRONQ_OK;
}

kronq_status quantize(cudaStream_t st, const kronq_opts &o, float *W,
                      const float *U, int64_t d_out, int64_t d_in,
                      uint32_t *codes, float *scales, uint8_t *zeros,
                      void *ws, size_t ws_bytes, int32_t *info) {
  QuantView v{W, d_in, U, d_in, codes, o.bits * d_in / 32, scales, zeros,
              d_in / o.group, d_out, d_in};
  return quantize_view(st, o, v, ws, ws_bytes, info);
}

// ---------------------------------------------------------------- split form
// OBS on the output of chol_split, F = [U11, R12; 0, U22] (H + λI = R Rᵀ with
// R upper, U = R^-1, split at h). The sweep over the first h columns uses
// U11. Its results enter the second half through R12 alone: the GPTQ
// recursion gives E·U = W − Ŵ for the scaled errors E, so E = (W − Ŵ)·R,
// and the second half starts from
//     W2 + ((W1 − Ŵ1) R12) U22,
// after which the sweep over the second half uses U22. The result equals the
// one-pass sweep with the full U (same decisions; the products differ by
// rounding).
size_t quant_split_ws_bytes(int64_t d_out, int64_t d_in, int64_t h, const kronq_opts &o) {
  auto al = [](size_t b) { return (b + 255) / 256 * 256; };
  const int64_t m = d_in - h;
  const size_t save = al(static_cast<size_t>(d_out) * h * 4);
  const size_t p = al(static_cast<size_t>(d_out) * m * 4);
  const size_t sweep = kq_max(quant_ws_bytes(d_out, h, o), quant_ws_bytes(d_out, m, o));
  const size_t cross = kq_max(gemm_scratch_bytes(d_out, m, h), gemm_scratch_bytes(d_out, m, m));
  return save + p + kq_max(sweep, cross) + 256;
}

kronq_status quantize_split(cudaStream_t st, const kronq_opts &o, float *W,
                            const float *F, int64_t d_out, int64_t d_in, int64_t h,
                            uint32_t *codes, float *scales, uint8_t *zeros,
                            void *ws, size_t ws_bytes, int32_t *info) {
  if (ws_bytes < quant_split_ws_bytes(d_out, d_in, h, o)) return KRONQ_ERR_INVALID_ARG;
  auto al = [](size_t b) { return (b + 255) / 256 * 256; };
  const int64_t m = d_in - h;
  uint8_t *w = static_cast<uint8_t *>(ws);
  float *W1 = reinterpret_cast<float *>(w);               // W1, then W1 − Ŵ1
  w += al(static_cast<size_t>(d_out) * h * 4);
  float *P = reinterpret_cast<float *>(w);                // (W1 − Ŵ1) R12
  w += al(static_cast<size_t>(d_out) * m * 4);
  const size_t rest = ws_bytes - (static_cast<size_t>(w - static_cast<uint8_t *>(ws)));
  const int64_t ldq = o.bits * d_in / 32, lds = d_in / o.group;
  KQ_CUDA(cudaMemcpy2DAsync(W1, static_cast<size_t>(h) * 4, W, static_cast<size_t>(d_in) * 4,
                        static_cast<size_t>(h) * 4, static_cast<size_t>(d_out),
                        cudaMemcpyDeviceToDevice, st));
  QuantView v1{W, d_in, F, d_in, codes, ldq, scales, zeros, lds, d_out, h};
  KQ_TRY(quantize_view(st, o, v1, w, rest, info));
  {  // W1 − Ŵ1
    dim3 grid(static_cast<unsigned>(kq_min<int64_t>(ceil_div(h, 256), 16)),
              static_cast<unsigned>(kq_min<int64_t>(d_out, 65535)));
    diff_inplace_kernel<<<grid, 256, 0, st>>>(W1, h, W, d_in, d_out, h);
    KQ_CHECK_LAUNCH();
  }
  {
    GemmArgs g;  // P = (W1 − Ŵ1) R12
    g.M = d_out; g.N = m; g.K = h;
    g.A = W1; g.lda = h;
    g.B = F + h; g.ldb = d_in; g.b_mn = true;
    g.C = P; g.ldc = m;
    KQ_TRY(gemm_f32(st, g, w, rest, info));
  }
  {
    GemmArgs g;  // W2 += P U22 : U22[k][j] == 0 for k > j
    g.M = d_out; g.N = m; g.K = m;
    g.A = P; g.lda = m;
    g.B = F + h * d_in + h; g.ldb = d_in; g.b_mn = true;
    g.C = W + h; g.ldc = d_in;
    g.beta = 1.f;
    g.kflags = KR_B_LOWER;
    KQ_TRY(gemm_f32(st, g, w, rest, info));
  }
  QuantView v2{W + h, d_in, F + h * d_in + h, d_in, codes + o.bits * h / 32, ldq,
               scales + h / o.group, zeros + h / o.group, lds, d_out, m};
  return quantize_view(st, o, v2, w, rest, info);
}

}  // namespace kronq

// Blocked column-wise OBS quantize-and-compensate [gptget-en Methodology:
// extends GPTQ's column-wise OBS; wmrh §四: the per-column update is GPTAQ's
// and H_G does not enter it, so rows are independent given U; wmrh §五:
// W2/W3/W4 with 128-column groups].
//
// Per 128-column block j0 (one launch of obs_block_kernel): each warp owns one
// row at a time, the block's 128 weights of the row live in 4 registers per
// lane, U[j0:j0+128, j0:j0+128] sits in shared memory. For each column j:
// group (scale, zero) at a group start, q = clamp(rint(w/scale)+zero),
// err = (w - w_hat)/U[j][j], w_k -= err * U[j][k] for the block's k > j.
// The errors go to E; the columns right of the block are updated lazily by
// 3xTF32 GEMMs: within a super-block of S columns after every block
// (W[:, blk_end:sb_end] -= E_blk U[blk, blk_end:sb_end]), and once per
// super-block for everything right of it (W[:, sb_end:] -= E_sb U[sb, sb_end:]).
// Codes are packed in the same pass (little-endian bitstream per row).
#include "kernels.cuh"

namespace kronq {
namespace {

constexpr int OB = 128;        // block width
constexpr int OTHREADS = 256;  // 8 warps
constexpr int RPW = 4;         // rows per warp, swept together
constexpr int OROWS = (OTHREADS / 32) * RPW;
constexpr int SUPER = 1024;    // super-block width
constexpr int OSMEM = (OB * OB + OB) * 4;

// Columns [32*SLOT, 32*SLOT + 32) of the block for the warp's RPW rows. With
// the register slot fixed at compile time, columns left of the chunk need no
// update and columns right of it are updated without predicates.
template <int SLOT>
__device__ __forceinline__ void obs_chunk(float (&w)[RPW][4], float (&err)[RPW][4],
                                          float (&scale)[RPW], float (&rscale)[RPW],
                                          float (&zero)[RPW], const float *Us,
                                          const float *inv, uint8_t (*qs)[OB],
                                          int lane, int group, float maxq,
                                          int64_t row0, int64_t d_out, int64_t j0,
                                          float *scales, uint8_t *zeros,
                                          int64_t ngroups) {
  constexpr int jb = 32 * SLOT;
  if (jb % group == 0) {
    // group start: (scale, zero) from the rows' current weights of the group
    float mn[RPW], mx[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      mn[r] = INFINITY;
      mx[r] = -INFINITY;
#pragma unroll
      for (int s = SLOT; s < 4; ++s) {
        if (32 * s < jb + group) {
          mn[r] = fminf(mn[r], w[r][s]);
          mx[r] = fmaxf(mx[r], w[r][s]);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        mn[r] = fminf(mn[r], __shfl_xor_sync(0xffffffffu, mn[r], o));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], o));
      }
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const float xmin = fminf(mn[r], 0.f), xmax = fmaxf(mx[r], 0.f);
      if (xmax == xmin) {
        scale[r] = 1.f;
        zero[r] = 0.f;
      } else {
        scale[r] = (xmax - xmin) / maxq;
        zero[r] = rintf(-xmin / scale[r]);
      }
      rscale[r] = 1.f / scale[r];
      if (lane == 0 && row0 + r < d_out) {
        const int64_t gi = (j0 + jb) / group;
        scales[(row0 + r) * ngroups + gi] = scale[r];
        zeros[(row0 + r) * ngroups + gi] = static_cast<uint8_t>(zero[r]);
      }
    }
  }
  for (int jj = 0; jj < 32; ++jj) {
    const int j = jb + jj;
    const float *urow = Us + j * OB + lane;
    float u[4];
#pragma unroll
    for (int s = SLOT; s < 4; ++s) u[s] = urow[32 * s];
    const float iu = inv[j];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const float wj = __shfl_sync(0xffffffffu, w[r][SLOT], jj);
      // w/scale as a product with the group's reciprocal: it can differ from
      // the quotient only within an ulp of a rounding tie
      const float q = fminf(fmaxf(rintf(wj * rscale[r]) + zero[r], 0.f), maxq);
      const float wh = scale[r] * (q - zero[r]);
      const float e = (wj - wh) * iu;
      if (lane > jj) w[r][SLOT] = fmaf(-e, u[SLOT], w[r][SLOT]);
#pragma unroll
      for (int s = SLOT + 1; s < 4; ++s) w[r][s] = fmaf(-e, u[s], w[r][s]);
      if (lane == jj) {
        w[r][SLOT] = wh;
        err[r][SLOT] = e;
        qs[r][j] = static_cast<uint8_t>(q);
      }
    }
  }
}

// One 128-column block for OROWS rows per CTA. Each warp sweeps its 4 rows
// together (independent dependency chains), lane l holding columns
// l, l+32, l+64, l+96 of each row.
__global__ void __launch_bounds__(OTHREADS)
    obs_block_kernel(float *__restrict__ W, int64_t ldw,
                     const float *__restrict__ U, int64_t ldu, int64_t j0,
                     int64_t d_out, int bits, int group,
                     float *__restrict__ E, int64_t lde, int64_t e_col,
                     uint32_t *__restrict__ codes, int64_t ldq,
                     float *__restrict__ scales, uint8_t *__restrict__ zeros,
                     int64_t ngroups) {
  extern __shared__ float Us[];                 // OB x OB, then 1/U[j][j]
  float *inv = Us + OB * OB;
  __shared__ uint8_t qsm[OTHREADS / 32][RPW][OB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < OB * OB; e += OTHREADS) {
    const int r = e / OB, c = e % OB;
    Us[e] = U[(j0 + r) * ldu + j0 + c];
  }
  __syncthreads();
  if (threadIdx.x < OB) inv[threadIdx.x] = 1.f / Us[threadIdx.x * OB + threadIdx.x];
  __syncthreads();
  const float maxq = static_cast<float>((1 << bits) - 1);
  const int64_t row0 = int64_t(blockIdx.x) * OROWS + warp * RPW;
  float w[RPW][4], err[RPW][4];
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const bool ok = row0 + r < d_out;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      w[r][s] = ok ? W[(row0 + r) * ldw + j0 + lane + 32 * s] : 0.f;
      err[r][s] = 0.f;
    }
  }
  float scale[RPW], rscale[RPW], zero[RPW];
  uint8_t (*qs)[OB] = qsm[warp];
  obs_chunk<0>(w, err, scale, rscale, zero, Us, inv, qs, lane, group, maxq, row0,
               d_out, j0, scales, zeros, ngroups);
  obs_chunk<1>(w, err, scale, rscale, zero, Us, inv, qs, lane, group, maxq, row0,
               d_out, j0, scales, zeros, ngroups);
  obs_chunk<2>(w, err, scale, rscale, zero, Us, inv, qs, lane, group, maxq, row0,
               d_out, j0, scales, zeros, ngroups);
  obs_chunk<3>(w, err, scale, rscale, zero, Us, inv, qs, lane, group, maxq, row0,
               d_out, j0, scales, zeros, ngroups);
  __syncwarp();
  const int nwords = OB * bits / 32;
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const int64_t row = row0 + r;
    if (row >= d_out) break;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      W[row * ldw + j0 + lane + 32 * s] = w[r][s];
      E[row * lde + e_col + lane + 32 * s] = err[r][s];
    }
    if (lane < nwords) {
      uint32_t word = 0;
      const int bit0 = 32 * lane;
      const int c_lo = bit0 / bits, c_hi = min(OB - 1, (bit0 + 31) / bits);
      for (int c = c_lo; c <= c_hi; ++c) {
        const int sh = c * bits - bit0;
        const uint32_t code = qsm[warp][r][c];
        word |= sh >= 0 ? (code << sh) : (code >> (-sh));
      }
      codes[row * ldq + (j0 * bits) / 32 + lane] = word;
    }
  }
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
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(obs_block_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             OSMEM) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    attr_done = true;
  }
  float *W = v.W;
  const float *U = v.U;
  const unsigned grid = static_cast<unsigned>(ceil_div(d_out, OROWS));
  for (int64_t sb0 = 0; sb0 < n; sb0 += S) {
    const int64_t sb1 = kq_min<int64_t>(n, sb0 + S);
    for (int64_t j0 = sb0; j0 < sb1; j0 += OB) {
      obs_block_kernel<<<grid, OTHREADS, OSMEM, st>>>(
          W, v.ldw, U, v.ldu, j0, d_out, o.bits, o.group, E, S, j0 - sb0, v.codes,
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
  if (cudaMemcpy2DAsync(W1, static_cast<size_t>(h) * 4, W, static_cast<size_t>(d_in) * 4,
                        static_cast<size_t>(h) * 4, static_cast<size_t>(d_out),
                        cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return KRONQ_ERR_CUDA;
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

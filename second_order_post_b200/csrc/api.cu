// The C ABI of libkronq.so (declared in include/kronq.h): argument validation
// and dispatch to the kernels. No call allocates device memory.
#include <math.h>

#include <algorithm>
#include <numeric>
#include <vector>

#include "kernels.cuh"

using namespace kronq;

namespace {

bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

bool rot_ok(const kronq_rot &r, int64_t d) {
  return is_pow2(r.had) && r.m >= 1 && r.m <= 256 && r.had * r.m == d;
}

bool aligned(const void *p, size_t a) {
  return reinterpret_cast<uintptr_t>(p) % a == 0;
}

}  // namespace

extern "C" {

const char *kronq_status_string(kronq_status s) {
  switch (s) {
    case KRONQ_OK: return "ok";
    case KRONQ_ERR_INVALID_ARG: return "invalid argument";
    case KRONQ_ERR_UNSUPPORTED: return "unsupported shape or layout";
    case KRONQ_ERR_NOT_PD: return "matrix not positive definite";
    case KRONQ_ERR_NONFINITE: return "non-finite value";
    case KRONQ_ERR_TIMEOUT: return "device wait timed out";
    case KRONQ_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

kronq_status kronq_accum_cov(kronq_stream_t stream, const void *A,
                             kronq_dtype dtype, int64_t n, int64_t d,
                             int64_t lda, float alpha, float beta, float *H,
                             int32_t *info_dev) {
  if (!H || !info_dev || d <= 0 || n < 0 || lda < d || (n > 0 && !A))
    return KRONQ_ERR_INVALID_ARG;
  if (dtype != KRONQ_F32 && dtype != KRONQ_BF16) return KRONQ_ERR_INVALID_ARG;
  if (d > (int64_t(1) << 20) || n > (int64_t(1) << 31)) return KRONQ_ERR_UNSUPPORTED;
  if (dtype == KRONQ_BF16 && (d % 128 || lda % 8 || !aligned(A, 16)))
    return KRONQ_ERR_UNSUPPORTED;
  KQ_TRY(require_sm100());
  cudaStream_t st = as_stream(stream);
  KQ_TRY(launch_set_int(st, info_dev, 0));
  if (dtype == KRONQ_BF16)
    return cov_bf16(st, static_cast<const __nv_bfloat16 *>(A), n, d, lda, alpha,
                    beta, H, info_dev);
  return cov_f32(st, static_cast<const float *>(A), n, d, lda, alpha, beta, H);
}

kronq_status kronq_sensitivity(kronq_stream_t stream, const float *H_X,
                               int64_t d_in, const float *H_G, int64_t d_out,
                               double *out_dev) {
  if (!H_X || !H_G || !out_dev || d_in <= 0 || d_out <= 0)
    return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(require_sm100());
  return launch_sensitivity(as_stream(stream), H_X, d_in, H_G, d_out, out_dev);
}

size_t kronq_workspace_bytes(kronq_ws_kind which, int64_t d_out, int64_t d_in,
                             const kronq_opts *opts) {
  if (d_out <= 0 || d_in <= 0) return 0;
  switch (which) {
    case KRONQ_WS_BIIP:
      if (!opts || opts->rot_in.m < 1 || opts->rot_in.m > 256 ||
          opts->rot_out.m < 1 || opts->rot_out.m > 256)
        return 0;
      return biip_ws_bytes(d_out, d_in, *opts);
    case KRONQ_WS_CHOL:
      if (d_in % 128) return 0;
      return chol_ws_bytes(d_in);
    case KRONQ_WS_QUANT:
      if (!opts) return 0;
      return quant_ws_bytes(d_out, d_in, *opts);
    case KRONQ_WS_LOSS:
      return loss_ws_bytes(d_out, d_in);
    case KRONQ_WS_QUANT_SPLIT:
      if (!opts || d_in % 128 || d_in < 256) return 0;
      return quant_split_ws_bytes(d_out, d_in, chol_split_point(d_in), *opts);
  }
  return 0;
}

kronq_status kronq_biip(kronq_stream_t stream, const kronq_opts *opts,
                        const void *W, kronq_dtype wdtype, int64_t d_out,
                        int64_t d_in, float *W_rot, float *H_X, float *H_G,
                        float *s_x, float *s_g, void *ws, size_t ws_bytes,
                        int32_t *info_dev) {
  if (!opts || !W || !W_rot || !H_X || !H_G || !s_x || !s_g || !ws ||
      !info_dev || d_out <= 0 || d_in <= 0)
    return KRONQ_ERR_INVALID_ARG;
  if (wdtype != KRONQ_F32 && wdtype != KRONQ_BF16) return KRONQ_ERR_INVALID_ARG;
  if (!(opts->scale_exp >= 0.f && opts->scale_exp <= 4.f)) return KRONQ_ERR_INVALID_ARG;
  const bool rot_x = !(opts->flags & KRONQ_FLAG_NO_ROT_IN);
  const bool rot_g = !(opts->flags & KRONQ_FLAG_NO_ROT_OUT);
  if (rot_x && !rot_ok(opts->rot_in, d_in)) return KRONQ_ERR_UNSUPPORTED;
  if (rot_g && !rot_ok(opts->rot_out, d_out)) return KRONQ_ERR_UNSUPPORTED;
  if (d_in % 32 || d_in > 65536 || d_out > 65536)
    return KRONQ_ERR_UNSUPPORTED;
  if (!aligned(ws, 256)) return KRONQ_ERR_INVALID_ARG;
  kronq_opts o = *opts;
  if (!rot_x) o.rot_in = {d_in, 1};
  if (!rot_g) o.rot_out = {d_out, 1};
  if (ws_bytes < biip_ws_bytes(d_out, d_in, o)) return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(require_sm100());
  cudaStream_t st = as_stream(stream);
  KQ_TRY(launch_set_int(st, info_dev, 0));
  return biip(st, o, W, wdtype == KRONQ_BF16, d_out, d_in, W_rot, H_X, H_G, s_x,
              s_g, ws, ws_bytes, info_dev);
}

kronq_status kronq_chol_inv(kronq_stream_t stream, float *H, int64_t d,
                            float damp_rel, void *ws, size_t ws_bytes,
                            int32_t *info_dev) {
  if (!H || !ws || !info_dev || d <= 0 || !(damp_rel >= 0.f) || !isfinite(damp_rel))
    return KRONQ_ERR_INVALID_ARG;
  if (d % 128 || d > 65536) return KRONQ_ERR_UNSUPPORTED;
  if (!aligned(ws, 256) || !aligned(H, 16)) return KRONQ_ERR_INVALID_ARG;
  if (ws_bytes < chol_ws_bytes(d)) return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(require_sm100());
  cudaStream_t st = as_stream(stream);
  KQ_TRY(launch_set_int(st, info_dev, 0));
  return chol_inv(st, H, d, damp_rel, ws, ws_bytes, info_dev);
}

kronq_status kronq_quantize_sublayer(kronq_stream_t stream,
                                     const kronq_opts *opts, float *W_rot,
                                     const float *U, int64_t d_out,
                                     int64_t d_in, uint32_t *codes,
                                     float *scales, uint8_t *zeros, void *ws,
                                     size_t ws_bytes, int32_t *info_dev) {
  if (!opts || !W_rot || !U || !codes || !scales || !zeros || !ws ||
      !info_dev || d_out <= 0 || d_in <= 0)
    return KRONQ_ERR_INVALID_ARG;
  if (opts->bits < 2 || opts->bits > 4) return KRONQ_ERR_INVALID_ARG;
  if (opts->group != 32 && opts->group != 64 && opts->group != 128)
    return KRONQ_ERR_UNSUPPORTED;
  if (opts->block != 128 || d_in % 128) return KRONQ_ERR_UNSUPPORTED;
  if (!aligned(ws, 256) || !aligned(W_rot, 16) || !aligned(U, 16))
    return KRONQ_ERR_INVALID_ARG;
  if (ws_bytes < quant_ws_bytes(d_out, d_in, *opts)) return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(require_sm100());
  cudaStream_t st = as_stream(stream);
  KQ_TRY(launch_set_int(st, info_dev, 0));
  return quantize(st, *opts, W_rot, U, d_out, d_in, codes, scales, zeros, ws,
                  ws_bytes, info_dev);
}

kronq_status kronq_chol_split(kronq_stream_t stream, float *H, int64_t d,
                              float damp_rel, void *ws, size_t ws_bytes,
                              int32_t *info_dev) {
  if (!H || !ws || !info_dev || d <= 0 || !(damp_rel >= 0.f) || !isfinite(damp_rel))
    return KRONQ_ERR_INVALID_ARG;
  if (d % 128 || d < 256 || d > 65536) return KRONQ_ERR_UNSUPPORTED;
  if (!aligned(ws, 256) || !aligned(H, 16)) return KRONQ_ERR_INVALID_ARG;
  if (ws_bytes < chol_ws_bytes(d)) return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(require_sm100());
  cudaStream_t st = as_stream(stream);
  KQ_TRY(launch_set_int(st, info_dev, 0));
  return chol_split(st, H, d, damp_rel, ws, ws_bytes, info_dev);
}

int64_t kronq_chol_split_point(int64_t d) { return d >= 256 ? chol_split_point(d) : 0; }

kronq_status kronq_quantize_split(kronq_stream_t stream, const kronq_opts *opts,
                                  float *W_rot, const float *F, int64_t d_out,
                                  int64_t d_in, uint32_t *codes, float *scales,
                                  uint8_t *zeros, void *ws, size_t ws_bytes,
                                  int32_t *info_dev) {
  if (!opts || !W_rot || !F || !codes || !scales || !zeros || !ws || !info_dev ||
      d_out <= 0 || d_in <= 0)
    return KRONQ_ERR_INVALID_ARG;
  if (opts->bits < 2 || opts->bits > 4) return KRONQ_ERR_INVALID_ARG;
  if (opts->group != 32 && opts->group != 64 && opts->group != 128)
    return KRONQ_ERR_UNSUPPORTED;
  if (opts->block != 128 || d_in % 128 || d_in < 256) return KRONQ_ERR_UNSUPPORTED;
  if (!aligned(ws, 256) || !aligned(W_rot, 16) || !aligned(F, 16))
    return KRONQ_ERR_INVALID_ARG;
  const int64_t h = chol_split_point(d_in);
  if (ws_bytes < quant_split_ws_bytes(d_out, d_in, h, *opts)) return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(require_sm100());
  cudaStream_t st = as_stream(stream);
  KQ_TRY(launch_set_int(st, info_dev, 0));
  return quantize_split(st, *opts, W_rot, F, d_out, d_in, h, codes, scales, zeros, ws,
                        ws_bytes, info_dev);
}

kronq_status kronq_layer_loss(kronq_stream_t stream, const float *W_ref,
                              const float *W_hat, const float *H_X,
                              const float *H_G, int64_t d_out, int64_t d_in,
                              double *loss_dev, void *ws, size_t ws_bytes,
                              int32_t *info_dev) {
  if (!W_ref || !W_hat || !H_X || !H_G || !loss_dev || !ws || !info_dev ||
      d_out <= 0 || d_in <= 0)
    return KRONQ_ERR_INVALID_ARG;
  if (d_in % 128 || d_out % 128) return KRONQ_ERR_UNSUPPORTED;
  if (!aligned(ws, 256) || !aligned(W_ref, 16) || !aligned(W_hat, 16) ||
      !aligned(H_X, 16) || !aligned(H_G, 16))
    return KRONQ_ERR_INVALID_ARG;
  if (ws_bytes < loss_ws_bytes(d_out, d_in)) return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(require_sm100());
  cudaStream_t st = as_stream(stream);
  KQ_TRY(launch_set_int(st, info_dev, 0));
  return layer_loss(st, W_ref, W_hat, H_X, H_G, d_out, d_in, loss_dev, ws,
                    ws_bytes, info_dev);
}

size_t kronq_matvec_desc_bytes(const kronq_opts *opts, int64_t d_out, int64_t d_in) {
  if (!opts || d_out <= 0 || d_in <= 0) return 0;
  return matvec_desc_bytes(d_out, d_in);
}

size_t kronq_matvec_workspace_bytes(int64_t d_out, int64_t d_in, int64_t n_tokens) {
  if (d_out <= 0 || d_in <= 0 || n_tokens <= 0) return 0;
  return matvec_ws_bytes(d_out, d_in, n_tokens);
}

namespace {
kronq_status check_matvec_opts(const kronq_opts *opts, int64_t d_out, int64_t d_in) {
  if (opts->bits < 2 || opts->bits > 4) return KRONQ_ERR_INVALID_ARG;
  if (opts->group != 32 && opts->group != 64 && opts->group != 128)
    return KRONQ_ERR_UNSUPPORTED;
  const bool rot_x = !(opts->flags & KRONQ_FLAG_NO_ROT_IN);
  const bool rot_g = !(opts->flags & KRONQ_FLAG_NO_ROT_OUT);
  if (rot_x && !rot_ok(opts->rot_in, d_in)) return KRONQ_ERR_UNSUPPORTED;
  if (rot_g && !rot_ok(opts->rot_out, d_out)) return KRONQ_ERR_UNSUPPORTED;
  if (d_in % opts->group || d_in % 32 || d_in > 65536 || d_out > 65536)
    return KRONQ_ERR_UNSUPPORTED;
  return KRONQ_OK;
}
}  // namespace

kronq_status kronq_matvec_prepare(kronq_stream_t stream, const kronq_opts *opts,
                                  const float *s_x, const float *s_g, int64_t d_out,
                                  int64_t d_in, void *desc, size_t desc_bytes) {
  if (!opts || !s_x || !s_g || !desc || d_out <= 0 || d_in <= 0) return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(check_matvec_opts(opts, d_out, d_in));
  if (!aligned(desc, 256) || desc_bytes < matvec_desc_bytes(d_out, d_in))
    return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(require_sm100());
  return matvec_prepare(as_stream(stream), *opts, s_x, s_g, d_out, d_in, desc);
}

kronq_status kronq_dequant_matvec(kronq_stream_t stream, const kronq_opts *opts,
                                  const void *desc, const uint32_t *codes,
                                  const float *scales, const uint8_t *zeros, int64_t d_out,
                                  int64_t d_in, const float *x, int64_t n_tokens, float *y,
                                  void *ws, size_t ws_bytes, int32_t *info_dev) {
  if (!opts || !desc || !codes || !scales || !zeros || !x || !y || !ws || !info_dev ||
      d_out <= 0 || d_in <= 0 || n_tokens <= 0)
    return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(check_matvec_opts(opts, d_out, d_in));
  if (n_tokens > 4096) return KRONQ_ERR_UNSUPPORTED;
  if (!aligned(desc, 256) || !aligned(ws, 256) || !aligned(codes, 16) || !aligned(x, 16) ||
      !aligned(y, 16) || ws_bytes < matvec_ws_bytes(d_out, d_in, n_tokens))
    return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(require_sm100());
  cudaStream_t st = as_stream(stream);
  KQ_TRY(launch_set_int(st, info_dev, 0));
  return dequant_matvec(st, *opts, desc, codes, scales, zeros, d_out, d_in, x, n_tokens, y, ws,
                        info_dev);
}

kronq_status kronq_selftest_timeout(kronq_stream_t stream, uint64_t limit_ns,
                                    int32_t *info_dev) {
  if (!info_dev || limit_ns == 0 || limit_ns > kSelftestMaxNs)
    return KRONQ_ERR_INVALID_ARG;
  KQ_TRY(require_sm100());
  cudaStream_t st = as_stream(stream);
  KQ_TRY(launch_set_int(st, info_dev, 0));
  return launch_selftest_timeout(st, limit_ns, info_dev);
}

kronq_status kronq_gemm_f32(kronq_stream_t stream, int64_t M, int64_t N,
                            int64_t K, float alpha, const float *A, int64_t lda,
                            int a_mn, const float *B, int64_t ldb, int b_mn,
                            float beta, float *C, int64_t ldc, void *ws,
                            size_t ws_bytes, int32_t *info_dev) {
  if (M < 0 || N < 0 || K < 0 || !info_dev) return KRONQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return KRONQ_OK;
  if (!C || (K > 0 && (!A || !B))) return KRONQ_ERR_INVALID_ARG;
  const int64_t a_rows = a_mn ? K : M, a_cols = a_mn ? M : K;
  const int64_t b_rows = b_mn ? K : N, b_cols = b_mn ? N : K;
  if (ldc < N || (K > 0 && (lda < a_cols || ldb < b_cols))) return KRONQ_ERR_INVALID_ARG;
  if (!aligned(C, 16) || ldc % 4 || (K > 0 && (!aligned(A, 16) || !aligned(B, 16) ||
                                                lda % 4 || ldb % 4)))
    return KRONQ_ERR_UNSUPPORTED;
  if (K > 0) {
    auto overlap = [](const float *p, int64_t rows, int64_t ld, int64_t cols,
                      const float *q, int64_t qrows, int64_t qld, int64_t qcols) {
      const float *pe = p + (rows - 1) * ld + cols, *qe = q + (qrows - 1) * qld + qcols;
      return p < qe && q < pe;
    };
    if (overlap(C, M, ldc, N, A, a_rows, lda, a_cols) ||
        overlap(C, M, ldc, N, B, b_rows, ldb, b_cols))
      return KRONQ_ERR_INVALID_ARG;
  }
  KQ_TRY(require_sm100());
  cudaStream_t st = as_stream(stream);
  KQ_TRY(launch_set_int(st, info_dev, 0));
  GemmArgs g;
  g.M = M; g.N = N; g.K = K;
  g.A = A; g.lda = lda; g.a_mn = a_mn != 0;
  g.B = B; g.ldb = ldb; g.b_mn = b_mn != 0;
  g.C = C; g.ldc = ldc;
  g.alpha = alpha; g.beta = beta;
  if (ws && !aligned(ws, 256)) return KRONQ_ERR_INVALID_ARG;
  return gemm_f32(st, g, ws, ws ? ws_bytes : 0, info_dev);
}

size_t kronq_gemm_f32_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return gemm_scratch_bytes(M, N, K);
}

kronq_status kronq_allocate_bits(const double *score, const int64_t *numel,
                                 int n, double avg_budget, int *bits_out) {
  if (!score || !numel || !bits_out || n <= 0 || !(avg_budget >= 2.0))
    return KRONQ_ERR_INVALID_ARG;
  double total = 0.0;
  for (int i = 0; i < n; ++i) {
    if (numel[i] <= 0 || !isfinite(score[i])) return KRONQ_ERR_INVALID_ARG;
    total += static_cast<double>(numel[i]);
  }
  std::vector<int> order(n);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return score[a] > score[b]; });
  for (int i = 0; i < n; ++i) bits_out[i] = 2;
  double used = 2.0 * total;
  const double cap = avg_budget * total;
  for (int from = 2; from <= 3; ++from) {
    for (int k = 0; k < n; ++k) {
      const int i = order[k];
      if (bits_out[i] == from && used + static_cast<double>(numel[i]) <= cap) {
        bits_out[i] = from + 1;
        used += static_cast<double>(numel[i]);
      }
    }
  }
  return KRONQ_OK;
}

uint64_t kronq_kernel_launches(void) { return launches(); }

const char *kronq_last_cuda_error(void) {
  return cudaGetErrorString(static_cast<cudaError_t>(last_cuda_error()));
}

}  // extern "C"

// Internal launcher interfaces between the C-ABI layer (api.cu) and the
// kernels. Nothing here is exported.
#pragma once

#include "common.cuh"

namespace kronq {

// ---------------------------------------------------------------- GEMM
// C = beta*C + alpha * A * B^T in fp32 with 3xTF32 tcgen05 MMAs.
//   A is M x K: stored row-major (A[i*lda+k], K-major) or, with a_mn, as
//   K x M (A[k*lda+i]). B is N x K: B[j*ldb+k], or with b_mn B[k*ldb+j].
// Per-tile K ranges skip blocks that a triangular operand keeps at zero.
enum : uint32_t {
  KR_A_UPPER = 1u,  // A[i][k] == 0 for k < i  -> k starts at the tile's m0
  KR_B_UPPER = 2u,  // B[j][k] == 0 for k < j  -> k starts at the tile's n0
  KR_B_LOWER = 4u,  // B[j][k] == 0 for k > j  -> k ends at n0 + 128
  KR_A_LOWER = 8u   // A[i][k] == 0 for k > i  -> k ends at m0 + 128
};

struct GemmArgs {
  int64_t M = 0, N = 0, K = 0;
  const float *A = nullptr;
  int64_t lda = 0;
  bool a_mn = false;
  const float *B = nullptr;
  int64_t ldb = 0;
  bool b_mn = false;
  float *C = nullptr;
  int64_t ldc = 0;
  float alpha = 1.f, beta = 0.f;
  uint32_t kflags = 0;
  bool upper_tiles_only = false;  // square C: only tiles with m0 <= n0
};

kronq_status gemm_tf32x3(cudaStream_t st, const GemmArgs &g, int32_t *info);
// Same product; large ones run on the fp16-split path when `scratch` holds at
// least gemm_scratch_bytes(M, N, K) bytes (256-byte aligned), the rest on
// gemm_tf32x3. The scratch is in use until the product completes on `st`.
kronq_status gemm_f32(cudaStream_t st, const GemmArgs &g, void *scratch,
                      size_t scratch_bytes, int32_t *info);
size_t gemm_scratch_bytes(int64_t M, int64_t N, int64_t K);

// ---------------------------------------------------------------- covariance
kronq_status cov_bf16(cudaStream_t st, const __nv_bfloat16 *A, int64_t n,
                      int64_t d, int64_t lda, float alpha, float beta,
                      float *H, int32_t *info);
kronq_status cov_f32(cudaStream_t st, const float *A, int64_t n, int64_t d,
                     int64_t lda, float alpha, float beta, float *H);
kronq_status scale_matrix(cudaStream_t st, float *H, int64_t n_elems,
                          float beta);

// ---------------------------------------------------------------- misc
kronq_status launch_sensitivity(cudaStream_t st, const float *hx, int64_t dx,
                                const float *hg, int64_t dg, double *out);
kronq_status launch_set_int(cudaStream_t st, int32_t *p, int32_t v);
kronq_status launch_selftest_timeout(cudaStream_t st, uint64_t limit_ns,
                                     int32_t *info);
uint64_t launches();
int last_cuda_error();

// ---------------------------------------------------------------- Cholesky
size_t chol_ws_bytes(int64_t d);
kronq_status chol_inv(cudaStream_t st, float *H, int64_t d, float damp_rel,
                      void *ws, size_t ws_bytes, int32_t *info);
// Same recursion, but the root keeps R12 (= V) in place of U12:
// H <- [U11, R12; 0, U22] split at chol_split_point(d).
kronq_status chol_split(cudaStream_t st, float *H, int64_t d, float damp_rel,
                        void *ws, size_t ws_bytes, int32_t *info);
int64_t chol_split_point(int64_t d);

// ---------------------------------------------------------------- BiIP
size_t biip_ws_bytes(int64_t d_out, int64_t d_in, const kronq_opts &o);
kronq_status biip(cudaStream_t st, const kronq_opts &o, const void *W,
                  bool w_bf16, int64_t d_out, int64_t d_in, float *W_rot,
                  float *H_X, float *H_G, float *s_x, float *s_g, void *ws,
                  size_t ws_bytes, int32_t *info);

// Rows of an R x C matrix through one side's rotation:
// out[r] = (Hhat_had ⊗ Q_m)(cc ⊙ in[r]) / sqrt(had) (a plain cc-scaled copy
// when rot is false; cc may be null).
kronq_status rotate_rows(cudaStream_t st, const float *in, float *out, int64_t R,
                         int64_t C, bool rot, int64_t had, int64_t m, const float *Q,
                         const float *cc, int32_t *info);
// fx = sign_x / s_x, fg = sign_g / s_g, Q_m of both sides (Qg and its
// transpose QgT); G: 2 * 256 * 256 doubles of scratch.
kronq_status rotation_factors(cudaStream_t st, const kronq_opts &o, const float *s_x,
                              const float *s_g, int64_t d_out, int64_t d_in, float *fx,
                              float *fg, float *Qx, float *QgT, float *Qg, double *G);

// ---------------------------------------------------------------- OBS
size_t quant_ws_bytes(int64_t d_out, int64_t d_in, const kronq_opts &o);
kronq_status quantize(cudaStream_t st, const kronq_opts &o, float *W,
                      const float *U, int64_t d_out, int64_t d_in,
                      uint32_t *codes, float *scales, uint8_t *zeros,
                      void *ws, size_t ws_bytes, int32_t *info);
struct QuantView {
  float *W;
  int64_t ldw;
  const float *U;
  int64_t ldu;
  uint32_t *codes;
  int64_t ldq;       // words per row of the full code array
  float *scales;
  uint8_t *zeros;
  int64_t lds;       // groups per row of the full scale / zero arrays
  int64_t d_out, n;  // rows, columns of the view
};
kronq_status quantize_view(cudaStream_t st, const kronq_opts &o, const QuantView &v,
                           void *ws, size_t ws_bytes, int32_t *info);
size_t quant_split_ws_bytes(int64_t d_out, int64_t d_in, int64_t h, const kronq_opts &o);
kronq_status quantize_split(cudaStream_t st, const kronq_opts &o, float *W,
                            const float *F, int64_t d_out, int64_t d_in, int64_t h,
                            uint32_t *codes, float *scales, uint8_t *zeros,
                            void *ws, size_t ws_bytes, int32_t *info);

// ---------------------------------------------------------------- matvec
size_t matvec_desc_bytes(int64_t d_out, int64_t d_in);
size_t matvec_ws_bytes(int64_t d_out, int64_t d_in, int64_t B);
kronq_status matvec_prepare(cudaStream_t st, const kronq_opts &o, const float *s_x,
                            const float *s_g, int64_t d_out, int64_t d_in, void *desc);
kronq_status dequant_matvec(cudaStream_t st, const kronq_opts &o, const void *desc,
                            const uint32_t *codes, const float *scales, const uint8_t *zeros,
                            int64_t d_out, int64_t d_in, const float *x, int64_t B, float *y,
                            void *ws, int32_t *info);

// ---------------------------------------------------------------- loss
size_t loss_ws_bytes(int64_t d_out, int64_t d_in);
kronq_status layer_loss(cudaStream_t st, const float *W_ref,
                        const float *W_hat, const float *H_X, const float *H_G,
                        int64_t d_out, int64_t d_in, double *loss, void *ws,
                        size_t ws_bytes, int32_t *info);

}  // namespace kronq

// Kronecker-factored layer loss tr(H_G dW H_X dWᵀ) = vec(dW)ᵀ (H_X ⊗ H_G) vec(dW)
// [aimodeling: H ≈ H_X ⊗ H_G; wmrh §二], used to measure a quantized layer:
// P = dW H_X and Q = H_G dW on the 3xTF32 GEMM, then sum(P ⊙ Q) in fp64.
#include "kernels.cuh"

namespace kronq {
namespace {

__global__ void diff_kernel(const float *a, const float *b, float *out, int64_t n) {
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n;
       e += int64_t(gridDim.x) * blockDim.x)
    out[e] = a[e] - b[e];
}

__global__ void dot_kernel(const float *p, const float *q, int64_t n, double *out) {
  __shared__ double part[32];
  double s = 0.0;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < n;
       e += int64_t(gridDim.x) * blockDim.x)
    s += double(p[e]) * double(q[e]);
  s = warp_sum_d(s);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < blockDim.x / 32 ? part[threadIdx.x] : 0.0;
    v = warp_sum_d(v);
    if (threadIdx.x == 0) atomicAdd(out, v);
  }
}

}  // namespace

// Workspace: D, P, Q (d_out x d_in each), then scratch for the two products.
size_t loss_ws_bytes(int64_t d_out, int64_t d_in) {
  const size_t one = (static_cast<size_t>(d_out) * d_in * 4 + 255) / 256 * 256;
  return 3 * one + kq_max(gemm_scratch_bytes(d_out, d_in, d_in),
                          gemm_scratch_bytes(d_out, d_in, d_out)) + 256;
}

kronq_status layer_loss(cudaStream_t st, const float *W_ref, const float *W_hat,
                        const float *H_X, const float *H_G, int64_t d_out,
                        int64_t d_in, double *loss, void *ws, size_t ws_bytes,
                        int32_t *info) {
  if (ws_bytes < loss_ws_bytes(d_out, d_in)) return KRONQ_ERR_INVALID_ARG;
  const size_t one = (static_cast<size_t>(d_out) * d_in * 4 + 255) / 256 * 256;
  uint8_t *w = static_cast<uint8_t *>(ws);
  float *D = reinterpret_cast<float *>(w);
  float *P = reinterpret_cast<float *>(w + one);
  float *Q = reinterpret_cast<float *>(w + 2 * one);
  void *scr = w + 3 * one;
  const size_t scr_bytes = ws_bytes - 3 * one;
  const int64_t n = d_out * d_in;
  const unsigned blocks = static_cast<unsigned>(kq_min<int64_t>(ceil_div(n, 256), 148 * 8));
  diff_kernel<<<blocks, 256, 0, st>>>(W_ref, W_hat, D, n);
  KQ_CHECK_LAUNCH();
  GemmArgs g;  // P = D H_X
  g.M = d_out; g.N = d_in; g.K = d_in;
  g.A = D; g.lda = d_in;
  g.B = H_X; g.ldb = d_in;
  g.C = P; g.ldc = d_in;
  KQ_TRY(gemm_f32(st, g, scr, scr_bytes, info));
  GemmArgs h;  // Q = H_G D
  h.M = d_out; h.N = d_in; h.K = d_out;
  h.A = H_G; h.lda = d_out;
  h.B = D; h.ldb = d_in; h.b_mn = true;
  h.C = Q; h.ldc = d_in;
  KQ_TRY(gemm_f32(st, h, scr, scr_bytes, info));
  KQ_CUDA(cudaMemsetAsync(loss, 0, sizeof(double), st));
  dot_kernel<<<blocks, 256, 0, st>>>(P, Q, n, loss);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

}  // namespace kronq

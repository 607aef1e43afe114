// kronq_biip_noalloc: the BiIP step for callers that cannot hand the library
// a device workspace.
//
// Some callers cannot allocate device memory at the point where they rotate a
// layer:
//   - serving and training frameworks that reserve all of HBM up front for
//     their own pool allocator, where an extra cudaMalloc fails or fragments
//     the pool;
//   - plugin hosts that only pass a plugin its input and output buffers;
//   - latency-sensitive loops where cudaMalloc/cudaFree would synchronise the
//     device.
// For them this entry point keeps its scratch (the per-side diagonal factors
// and the seeded Q_m factors) in a file-scope device array instead of a
// caller workspace. The array is part of the module image: every GPU that
// loads libkronq.so holds it, 4 MiB, until the process exits.
//
// The array's name is only a host-side stand-in in host code. Its device
// address is looked up once per device with cudaGetSymbolAddress, with that
// device current, on the first call made on that device, and cached.
#include <mutex>

#include "kernels.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_biip_scratch[kScratchBytes];

void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_biip_scratch on the current device (set up once).
kronq_status scratch_on_current_device(void **out) {
  int dev = -1;
  KQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return KRONQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_biip_scratch) != cudaSuccess || p == nullptr)
      return KRONQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return KRONQ_OK;
}

bool pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }

bool factor_ok(const kronq_rot &r, int64_t d) {
  return pow2(r.had) && r.m >= 1 && r.m <= 256 && r.had * r.m == d;
}

}  // namespace

extern "C" kronq_status kronq_biip_noalloc(
    kronq_stream_t stream, const kronq_opts *opts, const void *W,
    kronq_dtype wdtype, int64_t d_out, int64_t d_in, float *W_rot, float *H_X,
    float *H_G, float *s_x, float *s_g, int32_t *info_dev) {
  using namespace kronq;
  if (!opts || !W || !W_rot || !H_X || !H_G || !s_x || !s_g || !info_dev ||
      d_out <= 0 || d_in <= 0)
    return KRONQ_ERR_INVALID_ARG;
  if (wdtype != KRONQ_F32 && wdtype != KRONQ_BF16) return KRONQ_ERR_INVALID_ARG;
  if (!(opts->scale_exp >= 0.f && opts->scale_exp <= 4.f)) return KRONQ_ERR_INVALID_ARG;
  const bool rot_x = !(opts->flags & KRONQ_FLAG_NO_ROT_IN);
  const bool rot_g = !(opts->flags & KRONQ_FLAG_NO_ROT_OUT);
  if (rot_x && !factor_ok(opts->rot_in, d_in)) return KRONQ_ERR_UNSUPPORTED;
  if (rot_g && !factor_ok(opts->rot_out, d_out)) return KRONQ_ERR_UNSUPPORTED;
  if (d_in % 32 || d_in > 65536 || d_out > 65536) return KRONQ_ERR_UNSUPPORTED;
  kronq_opts o = *opts;
  if (!rot_x) o.rot_in = {d_in, 1};
  if (!rot_g) o.rot_out = {d_out, 1};
  // The fixed array bounds what this entry point accepts.
  if (biip_ws_bytes(d_out, d_in, o) > kScratchBytes) return KRONQ_ERR_UNSUPPORTED;
  KQ_TRY(require_sm100());
  void *scratch = nullptr;
  KQ_TRY(scratch_on_current_device(&scratch));
  cudaStream_t st = as_stream(stream);
  KQ_TRY(launch_set_int(st, info_dev, 0));
  // Every scratch byte the kernels read is written earlier in the same call,
  // so nothing has to be cleared between calls.
  return biip(st, o, W, wdtype == KRONQ_BF16, d_out, d_in, W_rot, H_X, H_G, s_x,
              s_g, scratch, kScratchBytes, info_dev);
}

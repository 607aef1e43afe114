// Small helpers: device check, TMA tensor maps, sensitivity traces.
#include <cudaTypedefs.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <set>
#include <map>
#include <tuple>
#include <utility>

#include "kernels.cuh"

namespace kronq {
namespace {

__global__ void sensitivity_kernel(const float *hx, int64_t dx, const float *hg,
                                   int64_t dg, double *out) {
  __shared__ double part[2][32];
  double sx = 0.0, sg = 0.0;
  for (int64_t i = threadIdx.x; i < dx; i += blockDim.x) sx += hx[i * dx + i];
  for (int64_t i = threadIdx.x; i < dg; i += blockDim.x) sg += hg[i * dg + i];
  sx = warp_sum_d(sx);
  sg = warp_sum_d(sg);
  if ((threadIdx.x & 31) == 0) {
    part[0][threadIdx.x >> 5] = sx;
    part[1][threadIdx.x >> 5] = sg;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, b = 0.0;
    for (int k = 0; k < int(blockDim.x / 32); ++k) {
      a += part[0][k];
      b += part[1][k];
    }
    out[0] = a;
    out[1] = b;
    out[2] = a * b;
  }
}

__global__ void set_int_kernel(int32_t *p, int32_t v) { *p = v; }

// One thread waits, through the library's bounded mbarrier wait, on a barrier
// that nothing ever completes: the wait must give up after limit_ns and the
// kernel must report KRONQ_ERR_TIMEOUT and return.
__global__ void selftest_timeout_kernel(uint64_t limit_ns, int32_t *info) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait(&bar, 0, &abort_flag, limit_ns)) report(info, KRONQ_ERR_TIMEOUT);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault,
                                &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

namespace {
std::atomic<uint64_t> g_launches{0};
}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {
std::atomic<int> g_last_cuda{0};
}
kronq_status cuda_fail(cudaError_t e) {
  g_last_cuda.store(static_cast<int>(e), std::memory_order_relaxed);
  return KRONQ_ERR_CUDA;
}
int last_cuda_error() { return g_last_cuda.load(std::memory_order_relaxed); }

uint64_t launches() { return g_launches.load(std::memory_order_relaxed); }

namespace {
constexpr int kMaxDev = 64;
// per device: 0 = not checked yet, 1 = sm_100, 2 = another architecture
std::atomic<int> g_arch_ok[kMaxDev];
}  // namespace

kronq_status require_sm100() {
  int dev = -1;
  KQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDev) return KRONQ_ERR_UNSUPPORTED;
  int state = g_arch_ok[dev].load(std::memory_order_acquire);
  if (state == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return KRONQ_ERR_CUDA;
    state = (major == 10 && minor == 0) ? 1 : 2;
    g_arch_ok[dev].store(state, std::memory_order_release);
  }
  return state == 1 ? KRONQ_OK : KRONQ_ERR_CUDA;
}

namespace {
std::mutex g_attr_mu;
}  // namespace

// The dynamic shared-memory limit of a kernel only ever rises: a launch with
// fewer bytes than the current limit needs no change, and lowering it would
// break a later launch of the same kernel with more.
kronq_status set_max_dyn_smem(const void *func, int bytes) {
  int dev = -1;
  KQ_CUDA(cudaGetDevice(&dev));
  static std::map<std::pair<int, const void *>, int> limit;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  int &cur = limit[std::make_pair(dev, func)];
  if (bytes <= cur) return KRONQ_OK;
  KQ_CUDA(cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  cur = bytes;
  return KRONQ_OK;
}

kronq_status set_nonportable_cluster(const void *func) {
  int dev = -1;
  KQ_CUDA(cudaGetDevice(&dev));
  static std::set<std::pair<int, const void *>> done;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  const auto key = std::make_pair(dev, func);
  if (done.count(key)) return KRONQ_OK;
  KQ_CUDA(cudaFuncSetAttribute(func, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
  done.insert(key);
  return KRONQ_OK;
}

kronq_status make_tmap_2d(CUtensorMap *map, const void *base, bool bf16,
                          uint64_t inner, uint64_t outer, uint64_t pitch_elems,
                          uint32_t box_inner, uint32_t box_outer,
                          int swz) {
  const uint64_t es = bf16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0) return KRONQ_ERR_UNSUPPORTED;
  if ((pitch_elems * es) % 16 != 0) return KRONQ_ERR_UNSUPPORTED;
  auto fn = encode_fn();
  if (!fn) return KRONQ_ERR_CUDA;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_elems * es};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map,
                  bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz == TMAP_SW128_32B ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                  : swz == TMAP_SW64    ? CU_TENSOR_MAP_SWIZZLE_64B
                  : swz == TMAP_NONE    ? CU_TENSOR_MAP_SWIZZLE_NONE
                                        : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? KRONQ_OK : KRONQ_ERR_CUDA;
}

kronq_status launch_sensitivity(cudaStream_t st, const float *hx, int64_t dx,
                                const float *hg, int64_t dg, double *out) {
  sensitivity_kernel<<<1, 1024, 0, st>>>(hx, dx, hg, dg, out);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

kronq_status launch_selftest_timeout(cudaStream_t st, uint64_t limit_ns,
                                     int32_t *info) {
  selftest_timeout_kernel<<<1, 32, 0, st>>>(limit_ns, info);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

kronq_status launch_set_int(cudaStream_t st, int32_t *p, int32_t v) {
  set_int_kernel<<<1, 1, 0, st>>>(p, v);
  KQ_CHECK_LAUNCH();
  return KRONQ_OK;
}

}  // namespace kronq

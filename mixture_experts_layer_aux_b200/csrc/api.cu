// api.cu -- status strings, the device status word, and host helpers shared by
// the entry points (SM count, TMA tensor-map encoding via the driver entry point,
// so the library itself does not link libcuda).
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

// One status word per device (each GPU that loads the library holds its own copy).
__device__ int g_moe_status = 0;

namespace moe_host {

static constexpr int kMaxDev = 64;

int* device_status_ptr() {
  static int* ptrs[kMaxDev] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    (void)cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_moe_status) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

int num_sms() {
  static int sms[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    (void)cudaGetLastError();
    return 148;
  }
  if (!sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = 148;
    }
    sms[dev] = n;
  }
  return sms[dev];
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      (void)cudaGetLastError();
  });
  return fn;
}

// 2-D tiled map over a row-major [outer, inner] tensor with a row stride in
// bytes; box = box_inner x box_outer elements, 128-byte swizzle, zero fill
// out of bounds.
bool encode_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_2d_plain(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                          uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace moe_host

extern "C" const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null pointer or inconsistent size";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape or dtype not handled by the kernels";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT: pointer not 16-byte aligned";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA call or kernel launch failed";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE: a kernel recorded a device-side failure";
    default: return "unknown moe status";
  }
}

extern "C" int moe_get_device_status(int32_t* word_out, int clear) {
  if (!word_out) return MOE_ERR_INVALID_ARG;
  int* p = moe_host::device_status_ptr();
  if (!p) return MOE_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  *word_out = v;
  if (clear && v != 0) {
    int z = 0;
    if (cudaMemcpy(p, &z, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return v == 0 ? MOE_OK : MOE_ERR_DEVICE;
}

namespace {
constexpr int DEV_WAIT_TIMEOUT_SELFTEST = 0x1F0;  // device status code of moe_selftest_wait_timeout

// One thread waits, through the bounded wait every GEMM role uses, on an mbarrier that nothing completes
// (the phase of parity 0 of a fresh barrier); the wait gives up after MOE_WAIT_NS and records its code.
__global__ void wait_selftest_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
    (void)mbar_wait(&bar, 0, &abort_flag, status, DEV_WAIT_TIMEOUT_SELFTEST);
  }
}
}  // namespace

extern "C" int moe_selftest_wait_timeout(void* stream) {
  int* p = moe_host::device_status_ptr();
  if (!p) return MOE_ERR_CUDA;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(p);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

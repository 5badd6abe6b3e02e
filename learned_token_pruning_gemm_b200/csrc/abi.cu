// Library-wide pieces of the C ABI: status strings, the per-device status word
// that kernels write when a device-side check fails, tensor-map encoding and the
// bounded-wait self test.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace {

// One word per device (a __device__ variable exists once per device context).
__device__ int g_status_word;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices];
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

}  // namespace

namespace tg {

int* status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dt, uint32_t rank, const void* base,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swz) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return false;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t bdim[5], estr[5];
  for (uint32_t i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estr[i] = 1;
    if (i + 1 < rank) gstr[i] = strides_bytes[i];
  }
  CUresult r = g_encode(map, dt, rank, const_cast<void*>(base), gdim, gstr, bdim, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool ensure_smem(const void* fn, int bytes) {
  struct Entry {
    int dev;
    const void* fn;
    int bytes;
  };
  static Entry cache[256];
  static int n = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  for (int i = 0; i < n; ++i)
    if (cache[i].dev == dev && cache[i].fn == fn && cache[i].bytes >= bytes) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  if (n < 256) cache[n++] = Entry{dev, fn, bytes};
  return true;
}

tg_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TG_OK : TG_ERR_CUDA;
}

}  // namespace tg

namespace {

// Waits on a flag that nothing sets, with the library's bounded wait on an
// mbarrier whose phase never completes. Records TG_ERR_TIMEOUT and returns.
__global__ void selftest_wait_kernel(int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tg::mbar_init(&bar, 1);
    abort_flag = 0;
    tg::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) tg::mbar_wait(&bar, 0, status, &abort_flag, limit_ns);
  __syncthreads();
}

}  // namespace

extern "C" {

int tg_abi_version(void) { return 5; }

int tg_debug_build(void) { return tg::kDebug ? 1 : 0; }

const char* tg_status_string(tg_status s) {
  switch (s) {
    case TG_OK: return "TG_OK";
    case TG_ERR_INVALID_ARG: return "TG_ERR_INVALID_ARG";
    case TG_ERR_UNSUPPORTED: return "TG_ERR_UNSUPPORTED";
    case TG_ERR_MISALIGNED: return "TG_ERR_MISALIGNED";
    case TG_ERR_WORKSPACE: return "TG_ERR_WORKSPACE";
    case TG_ERR_CUDA: return "TG_ERR_CUDA";
    case TG_ERR_TIMEOUT: return "TG_ERR_TIMEOUT";
    case TG_ERR_DEVICE_CHECK: return "TG_ERR_DEVICE_CHECK";
    case TG_ERR_DEBUG_BOUNDS: return "TG_ERR_DEBUG_BOUNDS";
  }
  return "TG_ERR_UNKNOWN";
}

tg_status tg_device_status(tg_stream_t stream, int reset) {
  int* p = tg::status_word();
  if (!p) return TG_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return TG_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return TG_ERR_CUDA;
  if (reset) {
    int z = 0;
    if (cudaMemcpy(p, &z, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return TG_ERR_CUDA;
  }
  return static_cast<tg_status>(v);
}

tg_status tg_selftest_bounded_wait(int64_t timeout_ns, tg_stream_t stream) {
  if (timeout_ns < 1000 || timeout_ns > 10000000000ll) return TG_ERR_INVALID_ARG;
  int* st = tg::status_word();
  if (!st) return TG_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, stream>>>(st, static_cast<uint64_t>(timeout_ns));
  return tg::launch_status();
}

}  // extern "C"

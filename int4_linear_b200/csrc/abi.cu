// Status strings, per-thread error messages, the device timeout word,
// tensor-map encoding and the timeout test hook.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "fq_device.cuh"
#include "fq_host.h"

namespace fq {

namespace {
thread_local char g_msg[512];

// One word per device, read and cleared by fq_check_device_error.
__device__ unsigned g_timeout_word;

constexpr int kMaxDevices = 64;
unsigned* g_word_ptr[kMaxDevices];
int g_sm_count[kMaxDevices];
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
}  // namespace

fq_status fail(fq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

void clear_error() { g_msg[0] = 0; }

static int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
  return d;
}

unsigned* device_error_word() {
  const int d = current_device();
  if (d < 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_word_ptr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_timeout_word) != cudaSuccess) return nullptr;
    g_word_ptr[d] = static_cast<unsigned*>(p);
  }
  return g_word_ptr[d];
}

int sm_count() {
  const int d = current_device();
  if (d < 0) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sm_count[d]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    g_sm_count[d] = n;
  }
  return g_sm_count[d];
}

fq_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return FQ_OK;
}

fq_status make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint64_t inner, uint64_t rows,
                       uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return fail(FQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
  }
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(FQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for %llu x %llu, box %u x %u", int(r),
                (unsigned long long)inner, (unsigned long long)rows, box_inner, box_rows);
  return FQ_OK;
}

// One CTA waits on a barrier nothing arrives at and gives up after limit_ns.
__global__ void debug_wait_kernel(uint64_t limit_ns, unsigned* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait(&bar, 0, limit_ns)) record_error(err, kErrTimeoutDebug);
  }
  __syncthreads();
}

}  // namespace fq

extern "C" {

const char* fq_status_string(fq_status s) {
  switch (s) {
    case FQ_OK: return "ok";
    case FQ_ERR_INVALID: return "invalid argument";
    case FQ_ERR_UNSUPPORTED: return "unsupported parameters";
    case FQ_ERR_CUDA: return "CUDA error";
    case FQ_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* fq_last_error(void) { return fq::g_msg; }

fq_status fq_check_device_error(void* stream) {
  const cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fq::fail(FQ_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  unsigned* w = fq::device_error_word();
  if (!w) return fq::fail(FQ_ERR_CUDA, "device error word unavailable");
  unsigned v = 0;
  if (cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return fq::fail(FQ_ERR_CUDA, "reading the device error word failed");
  if (v != 0) {
    const unsigned zero = 0;
    cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    return fq::fail(FQ_ERR_TIMEOUT, "a device wait gave up (code 0x%x)", v);
  }
  fq::clear_error();
  return FQ_OK;
}

fq_status fq_debug_wait_timeout(unsigned limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 100000) return fq::fail(FQ_ERR_INVALID, "limit_us must be in [1, 100000]");
  unsigned* w = fq::device_error_word();
  if (!w) return fq::fail(FQ_ERR_CUDA, "device error word unavailable");
  fq::debug_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(uint64_t(limit_us) * 1000ull, w);
  return fq::check_launch("debug_wait_kernel");
}

}  // extern "C"

// vca_status.cu -- status word, error strings, wait limit, tensor-map encoding
// and the bounded-wait self-test.
#include <stdarg.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "vca_device.cuh"
#include "vca_host.h"

namespace vca {

static thread_local char g_msg[512] = "";
static std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
}

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(); }

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(VCA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return VCA_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return fail(VCA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t gd[5], gs[5];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) gs[i] = strides_bytes[i];
  }
  CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(VCA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return VCA_OK;
}

// One block, one thread: waits on an mbarrier nobody arrives on.
__global__ void wait_timeout_kernel(DevStatus* st, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, &abort_flag, st, limit_ns, 9001);
  __syncthreads();
}

}  // namespace vca

using namespace vca;

extern "C" {

size_t vca_status_bytes(void) { return sizeof(DevStatus); }

int vca_reset_status(void* ws, vca_stream_t stream) {
  if (!ws) return fail(VCA_ERR_WORKSPACE, "vca_reset_status: null workspace");
  if (cudaMemsetAsync(ws, 0, sizeof(DevStatus), (cudaStream_t)stream) != cudaSuccess)
    return fail(VCA_ERR_CUDA, "vca_reset_status: cudaMemsetAsync failed");
  return VCA_OK;
}

int vca_check_status(void* ws, vca_stream_t stream, int* where, int* info) {
  if (!ws) return fail(VCA_ERR_WORKSPACE, "vca_check_status: null workspace");
  DevStatus h;
  cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return fail(VCA_ERR_CUDA, "vca_check_status: %s", cudaGetErrorString(e));
  if (where) *where = h.where;
  if (info) *info = h.info;
  if (h.code != 0) {
    cudaMemsetAsync(ws, 0, sizeof(DevStatus), (cudaStream_t)stream);
    cudaStreamSynchronize((cudaStream_t)stream);
    return fail(h.code, "device status %d at tag %d (info %d)", h.code, h.where, h.info);
  }
  return VCA_OK;
}

const char* vca_last_error(void) { return g_msg; }

void vca_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns ? ns : 1); }

int vca_debug_wait_timeout(void* ws, uint64_t limit_ns, vca_stream_t stream) {
  if (!ws) return fail(VCA_ERR_WORKSPACE, "vca_debug_wait_timeout: null workspace");
  wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((DevStatus*)ws, limit_ns);
  return check_launch("wait_timeout_kernel");
}

}  // extern "C"

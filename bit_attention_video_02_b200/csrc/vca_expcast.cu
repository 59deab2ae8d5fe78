// vca_expcast.cu -- ExpCast-FP8 reference map and the E4M3 encoder.
//
// ExpCast-FP8 ("VC-Attention: Training-Free Low-Bit Attention Speeds Video
// Diffusion Up to 3.6x", ExpCast-FP8 bullet; "Nunchux AI Introduces
// VC-Attention..." abstract): an E4M3 byte read as an integer is about
// 8*log2(v) + 56, so the byte of p = 2^z is written with one fp32 FMA,
// 8*z + 56 + beta (beta = -0.35), rounded to nearest even and clamped to the
// finite non-negative codes [0, 126].
#include "vca_device.cuh"
#include "vca_host.h"

namespace vca {

__device__ __forceinline__ uint32_t expcast_code(float z) {
  if (isnan(z)) return 0x7Fu;
  float a = __fmaf_rn(8.0f, z, 55.65f);
  float r = rintf(a);
  r = fminf(fmaxf(r, 0.0f), 126.0f);
  return (uint32_t)r;
}

__global__ void expcast_kernel(const float* __restrict__ z, uint8_t* __restrict__ codes, int64_t n) {
  int64_t n4 = n / 4;
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const float4* z4 = reinterpret_cast<const float4*>(z);
  uint32_t* c4 = reinterpret_cast<uint32_t*>(codes);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 v = z4[i];
    c4[i] = expcast_code(v.x) | (expcast_code(v.y) << 8) | (expcast_code(v.z) << 16) |
            (expcast_code(v.w) << 24);
  }
  for (int64_t i = n4 * 4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    codes[i] = (uint8_t)expcast_code(z[i]);
}

__global__ void e4m3_encode_kernel(const float* __restrict__ x, uint8_t* __restrict__ out,
                                   int64_t n) {
  int64_t n4 = n / 4;
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const float4* x4 = reinterpret_cast<const float4*>(x);
  uint32_t* o4 = reinterpret_cast<uint32_t*>(out);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 v = x4[i];
    o4[i] = (uint32_t)cvt_e4m3x2(v.x, v.y) | ((uint32_t)cvt_e4m3x2(v.z, v.w) << 16);
  }
  for (int64_t i = n4 * 4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = (uint8_t)(cvt_e4m3x2(x[i], 0.0f) & 0xFF);
}

static int grid_for(int64_t n) {
  int64_t g = (n / 4 + 255) / 256;
  if (g < 1) g = 1;
  if (g > 148 * 16) g = 148 * 16;
  return (int)g;
}

}  // namespace vca

using namespace vca;

extern "C" int vca_expcast_ref(const float* z, uint8_t* codes, int64_t n, vca_stream_t stream) {
  if (n < 0) return fail(VCA_ERR_INVALID, "vca_expcast_ref: n < 0");
  if (n == 0) return VCA_OK;
  if (!z || !codes) return fail(VCA_ERR_INVALID, "vca_expcast_ref: null pointer");
  if (!aligned16(z) || !aligned16(codes))
    return fail(VCA_ERR_INVALID, "vca_expcast_ref: pointers must be 16-byte aligned");
  expcast_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(z, codes, n);
  return check_launch("expcast_kernel");
}

extern "C" int vca_e4m3_encode(const float* x, uint8_t* out, int64_t n, vca_stream_t stream) {
  if (n < 0) return fail(VCA_ERR_INVALID, "vca_e4m3_encode: n < 0");
  if (n == 0) return VCA_OK;
  if (!x || !out) return fail(VCA_ERR_INVALID, "vca_e4m3_encode: null pointer");
  if (!aligned16(x) || !aligned16(out))
    return fail(VCA_ERR_INVALID, "vca_e4m3_encode: pointers must be 16-byte aligned");
  e4m3_encode_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(x, out, n);
  return check_launch("e4m3_encode_kernel");
}

// Conversion between bf16 latent-cache rows and the MXFP8 rows of gdla_fp8.cuh (one warp per
// row; lane b < 18 owns block b): for a bf16 cache written by the prefill, for the exchange of
// context parallelism at half the bytes, and for tests.
#include "gdla_fp8.cuh"
#include "gdla_internal.h"

namespace gdla {

__global__ void __launch_bounds__(256) mxfp8_quantize_kernel(const __nv_bfloat16* __restrict__ in,
                                                             long long rows, uint8_t* __restrict__ out) {
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  uint8_t* dst = out + row * FP8_ROW_BYTES;
  if (lane >= 18) {
    dst[FP8_SCALE_OFF + lane] = 0;              // bytes 594 .. 607
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(in + row * FP8_ROW_VALUES + 32 * lane);
  float v[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 w = src[i];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * i + 2 * e] = __uint_as_float(u[e] << 16);
      v[8 * i + 2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int k = mx_block_exp(amax);
  const float inv = exp2i(-k);
  uint32_t q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    q[i] = uint32_t(e4m3x2_from(v[4 * i] * inv, v[4 * i + 1] * inv)) |
           (uint32_t(e4m3x2_from(v[4 * i + 2] * inv, v[4 * i + 3] * inv)) << 16);
  uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * lane);
  d4[0] = make_uint4(q[0], q[1], q[2], q[3]);
  d4[1] = make_uint4(q[4], q[5], q[6], q[7]);
  dst[FP8_SCALE_OFF + lane] = uint8_t(k + 127);
}

__global__ void __launch_bounds__(256) mxfp8_dequantize_kernel(const uint8_t* __restrict__ in, long long rows,
                                                               __nv_bfloat16* __restrict__ out) {
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows || lane >= 18) return;
  const uint8_t* src = in + row * FP8_ROW_BYTES;
  const float s = exp2i(int(src[FP8_SCALE_OFF + lane]) - 127);
  const uint4* c4 = reinterpret_cast<const uint4*>(src + 32 * lane);
  const uint4 a = c4[0], b = c4[1];
  const uint32_t c[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t o[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t x = f16x2_from_e4m3x2(uint16_t(c[i] >> (16 * h)));
      const float lo = __half2float(__ushort_as_half(uint16_t(x & 0xFFFFu))) * s;
      const float hi = __half2float(__ushort_as_half(uint16_t(x >> 16))) * s;
      o[2 * i + h] = pack_bf162(lo, hi);
    }
  }
  uint4* d4 = reinterpret_cast<uint4*>(out + row * FP8_ROW_VALUES + 32 * lane);
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
}

int launch_mxfp8_quantize(const void* in, long long rows, void* out, cudaStream_t st) {
  if (rows <= 0) return 0;
  mxfp8_quantize_kernel<<<unsigned((rows + 7) / 8), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(in), rows,
                                                                    static_cast<uint8_t*>(out));
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

int launch_mxfp8_dequantize(const void* in, long long rows, void* out, cudaStream_t st) {
  if (rows <= 0) return 0;
  mxfp8_dequantize_kernel<<<unsigned((rows + 7) / 8), 256, 0, st>>>(static_cast<const uint8_t*>(in), rows,
                                                                      static_cast<__nv_bfloat16*>(out));
  return cudaPeekAtLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace gdla

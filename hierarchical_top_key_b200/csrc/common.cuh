// common.cuh - types, element access and number-format helpers shared by the
// libhisa kernels (one translation unit: libhisa.cu includes every .cuh).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/hisa.h"

namespace hisa {

enum : int { DT_F32 = HISA_F32, DT_BF16 = HISA_BF16, DT_E4M3 = HISA_E4M3 };

template <int DT> struct Elem;
template <> struct Elem<DT_F32>  { static constexpr int bytes = 4; };
template <> struct Elem<DT_BF16> { static constexpr int bytes = 2; };
template <> struct Elem<DT_E4M3> { static constexpr int bytes = 1; };

// Device status word: kernels that give up a bounded wait record a code here.
__device__ int g_status;

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_status, 0, code); }

// ---------------------------------------------------------------- decode

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

__device__ __forceinline__ float e4m3_to_float(uint32_t code) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
  return __half2float(__half(h));
}

// Unpack one 16-byte vector of elements to floats (code values for E4M3).
template <int DT> struct Vec16 {
  static constexpr int n = 16 / Elem<DT>::bytes;
  __device__ __forceinline__ static void unpack(const uint4& v, float* out);
};
template <> __device__ __forceinline__ void Vec16<DT_F32>::unpack(const uint4& v, float* o) {
  o[0] = __uint_as_float(v.x); o[1] = __uint_as_float(v.y);
  o[2] = __uint_as_float(v.z); o[3] = __uint_as_float(v.w);
}
template <> __device__ __forceinline__ void Vec16<DT_BF16>::unpack(const uint4& v, float* o) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = __uint_as_float(w[i] << 16);
    o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
template <> __device__ __forceinline__ void Vec16<DT_E4M3>::unpack(const uint4& v, float* o) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) o[4 * i + j] = e4m3_to_float((w[i] >> (8 * j)) & 0xFF);
  }
}

// ---------------------------------------------------------------- encode

// float64 -> bfloat16 bits, round to nearest even in one step (finite input).
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x));
  const uint32_t sign = static_cast<uint32_t>(b >> 63) << 15;
  const double a = fabs(x);
  if (a < ldexp(1.0, -126)) {                     // below 2^-126: multiples of 2^-133
    const double n = rint(ldexp(a, 133));           // exact scaling, then ties-to-even
    return static_cast<uint16_t>(sign | static_cast<uint32_t>(n));
  }
  // keep 7 of the 52 stored mantissa bits; round on the 45 dropped ones
  const uint64_t mag = b & 0x7FFFFFFFFFFFFFFFull;
  const uint64_t lsb = (mag >> 45) & 1ull;
  const uint64_t rounded = mag + 0x0FFFFFFFFFFFull + lsb;   // 2^44 - 1 + lsb
  const uint64_t top = rounded >> 45;                         // exp11 | mant7
  const int64_t exp11 = static_cast<int64_t>(top >> 7);
  const uint32_t mant7 = static_cast<uint32_t>(top & 0x7F);
  const int64_t exp8 = exp11 - 1023 + 127;
  if (exp8 >= 255) return static_cast<uint16_t>(sign | 0x7F80u);
  return static_cast<uint16_t>(sign | (static_cast<uint32_t>(exp8) << 7) | mant7);
}

// fp32 -> E4M3 code, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint8_t float_to_e4m3(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

// ---------------------------------------------------------------- ordering keys

// Order-preserving map fp32 -> uint32 (larger float -> larger key); -0 maps
// like +0.  Finite scores map to keys >= 0x00800000, so key 0 can mark an
// absent candidate.
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace hisa

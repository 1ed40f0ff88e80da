// pool.cuh - segment means of consecutive key rows: HISA block pooling and
// StreamIndex-style key compression (same arithmetic, different group rule).
//
// HBM-bound streaming kernel.  Each thread owns one 16-byte column vector of
// one output row and walks the rows of its group; the threads of a warp cover
// whole key rows, so every load instruction reads contiguous rows.  Sums are
// fp64 (exact for bf16/E4M3 inputs and for fp32 inputs within 2^29 of each
// other), and the mean is rounded once to the output format.
#pragma once
#include "common.cuh"

namespace hisa {

// out row o of sequence b averages in rows [o*G, min(o*G+G, n_in)).
// DT_E4M3: inputs are codes with one scale per row; the fp64 mean of the
// dequantised rows is rounded to fp32 and re-quantised with one scale per
// output row (absmax/448, 1 when zero).
template <int DT>
__global__ void __launch_bounds__(256) segment_mean_kernel(
    const uint8_t* __restrict__ in, const float* __restrict__ in_scale,
    uint8_t* __restrict__ out, float* __restrict__ out_scale,
    int batch, int n_in, int n_out, int d, int G, int o_first, int o_count) {
  constexpr int VE = Vec16<DT>::n;             // elements per 16-byte vector
  const int vecs = d / VE;                     // threads per output row (power of 2, <= 32)
  const int64_t row_bytes = static_cast<int64_t>(d) * Elem<DT>::bytes;
  const int64_t total = static_cast<int64_t>(batch) * o_count * vecs;
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < ceil_div(total, 32) * 32;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const bool live = g < total;
    const int64_t lrow = live ? g / vecs : 0;            // flattened (b, o - o_first)
    const int v = static_cast<int>(g % vecs);
    const int b = static_cast<int>(lrow / o_count);
    const int o = o_first + static_cast<int>(lrow % o_count);
    const int64_t orow = static_cast<int64_t>(b) * n_out + o;   // output row in [batch, n_out]
    const int r0 = o * G;
    const int r1 = min(r0 + G, n_in);
    double acc[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] = 0.0;
    if (live) {
      const uint8_t* base = in + (static_cast<int64_t>(b) * n_in) * row_bytes + v * 16;
#pragma unroll 4
      for (int r = r0; r < r1; ++r) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(base + r * row_bytes));
        float f[VE];
        Vec16<DT>::unpack(raw, f);
        if (DT == DT_E4M3) {
          const double sc = static_cast<double>(__ldg(in_scale + static_cast<int64_t>(b) * n_in + r));
#pragma unroll
          for (int e = 0; e < VE; ++e) acc[e] += static_cast<double>(f[e]) * sc;
        } else {
#pragma unroll
          for (int e = 0; e < VE; ++e) acc[e] += static_cast<double>(f[e]);
        }
      }
    }
    const double cnt = static_cast<double>(max(r1 - r0, 1));
    uint8_t* dst = out + orow * row_bytes + v * 16;
    if (DT == DT_F32) {
      if (live) {
        float4 r;
        r.x = static_cast<float>(acc[0] / cnt); r.y = static_cast<float>(acc[1] / cnt);
        r.z = static_cast<float>(acc[2] / cnt); r.w = static_cast<float>(acc[3] / cnt);
        *reinterpret_cast<float4*>(dst) = r;
      }
    } else if (DT == DT_BF16) {
      if (live) {
        uint32_t p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          p[i] = static_cast<uint32_t>(f64_to_bf16_rne(acc[2 * i] / cnt)) |
                 (static_cast<uint32_t>(f64_to_bf16_rne(acc[2 * i + 1] / cnt)) << 16);
        *reinterpret_cast<uint4*>(dst) = make_uint4(p[0], p[1], p[2], p[3]);
      }
    } else {
      // E4M3: the `vecs` threads of a row are consecutive lanes of one warp
      float m[VE];
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < VE; ++e) {
        m[e] = static_cast<float>(acc[e] / cnt);
        amax = fmaxf(amax, fabsf(m[e]));
      }
      for (int off = 1; off < vecs; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
      if (live) {
        uint32_t p[4] = {0, 0, 0, 0};
#pragma unroll
        for (int e = 0; e < VE; ++e)
          p[e / 4] |= static_cast<uint32_t>(float_to_e4m3(__fdiv_rn(m[e], scale))) << (8 * (e % 4));
        *reinterpret_cast<uint4*>(dst) = make_uint4(p[0], p[1], p[2], p[3]);
        if (v == 0) out_scale[orow] = scale;
      }
    }
  }
}

// Per-row E4M3 quantisation of bf16 / fp32 rows: one warp per row.
template <int DT>
__global__ void __launch_bounds__(256) quantize_rows_kernel(
    const uint8_t* __restrict__ x, int64_t rows, int cols, uint8_t* __restrict__ codes,
    float* __restrict__ scale) {
  constexpr int VE = Vec16<DT>::n;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int vecs = cols / VE;
  const int64_t row_bytes = static_cast<int64_t>(cols) * Elem<DT>::bytes;
  for (int64_t r = warp; r < rows; r += nwarps) {
    const uint8_t* src = x + r * row_bytes;
    float amax = 0.f;
    for (int v = lane; v < vecs; v += 32) {
      float f[VE];
      Vec16<DT>::unpack(__ldg(reinterpret_cast<const uint4*>(src + v * 16)), f);
#pragma unroll
      for (int e = 0; e < VE; ++e) amax = fmaxf(amax, fabsf(f[e]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    uint8_t* dst = codes + r * cols;
    for (int v = lane; v < vecs; v += 32) {
      float f[VE];
      Vec16<DT>::unpack(__ldg(reinterpret_cast<const uint4*>(src + v * 16)), f);
      uint32_t p[VE / 4 > 0 ? VE / 4 : 1] = {};
#pragma unroll
      for (int e = 0; e < VE; ++e)
        p[e / 4] |= static_cast<uint32_t>(float_to_e4m3(__fdiv_rn(f[e], sc))) << (8 * (e % 4));
      if (VE == 8) {
        *reinterpret_cast<uint2*>(dst + v * 8) = make_uint2(p[0], p[1]);
      } else {
        *reinterpret_cast<uint32_t*>(dst + v * 4) = p[0];
      }
    }
    if (lane == 0) scale[r] = sc;
  }
}

}  // namespace hisa

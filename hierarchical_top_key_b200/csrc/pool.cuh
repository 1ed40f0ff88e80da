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

// Write one 16-byte vector of a mean row: acc holds the float64 sums of its
// elements over cnt rows; the row is rounded to the storage type (E4M3: the
// row's absmax/448 scale, reduced over the `vecs` consecutive lanes holding
// the row, which all call this together; only `live` lanes store).
template <int DT>
__device__ __forceinline__ void write_mean(const double (&acc)[Vec16<DT>::n], double cnt, uint8_t* dst,
                                           float* scale_out, int v, int vecs, bool live) {
  constexpr int VE = Vec16<DT>::n;
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
      if (v == 0) *scale_out = scale;
    }
  }
}

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
    write_mean<DT>(acc, cnt, out + orow * row_bytes + v * 16, out_scale ? out_scale + orow : nullptr, v, vecs, live);
  }
}

// Block means over paged keys: block o of sequence b is page pages[b * n_out + o]
// of `in` ([num_pages, G, d], scales [num_pages, G]); its first
// min(G, n_in - o * G) rows are keys.  Same arithmetic and rounding as
// segment_mean_kernel.  A page entry outside [0, num_pages) leaves the output
// row untouched and records HISA_ERR_INVALID_ARG in the status word.
template <int DT>
__global__ void __launch_bounds__(256) paged_block_mean_kernel(
    const uint8_t* __restrict__ in, const float* __restrict__ in_scale, const int32_t* __restrict__ pages,
    int num_pages, uint8_t* __restrict__ out, float* __restrict__ out_scale,
    int batch, int n_in, int n_out, int d, int G, int o_first, int o_count) {
  constexpr int VE = Vec16<DT>::n;
  const int vecs = d / VE;
  const int64_t row_bytes = static_cast<int64_t>(d) * Elem<DT>::bytes;
  const int64_t total = static_cast<int64_t>(batch) * o_count * vecs;
  for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < ceil_div(total, 32) * 32;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const bool live = g < total;
    const int64_t lrow = live ? g / vecs : 0;
    const int v = static_cast<int>(g % vecs);
    const int b = static_cast<int>(lrow / o_count);
    const int o = o_first + static_cast<int>(lrow % o_count);
    const int64_t orow = static_cast<int64_t>(b) * n_out + o;
    const int nrows = max(0, min(G, n_in - o * G));
    bool ok = live;
    int pg = 0;
    if (live) {
      pg = __ldg(pages + orow);
      if (pg < 0 || pg >= num_pages) {
        ok = false;
        if (v == 0) record_status(HISA_ERR_INVALID_ARG);
      }
    }
    double acc[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] = 0.0;
    if (ok) {
      const uint8_t* base = in + static_cast<int64_t>(pg) * G * row_bytes + v * 16;
#pragma unroll 4
      for (int r = 0; r < nrows; ++r) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(base + r * row_bytes));
        float f[VE];
        Vec16<DT>::unpack(raw, f);
        if (DT == DT_E4M3) {
          const double sc = static_cast<double>(__ldg(in_scale + static_cast<int64_t>(pg) * G + r));
#pragma unroll
          for (int e = 0; e < VE; ++e) acc[e] += static_cast<double>(f[e]) * sc;
        } else {
#pragma unroll
          for (int e = 0; e < VE; ++e) acc[e] += static_cast<double>(f[e]);
        }
      }
    }
    write_mean<DT>(acc, static_cast<double>(max(nrows, 1)), out + orow * row_bytes + v * 16,
                   out_scale ? out_scale + orow : nullptr, v, vecs, ok);
  }
}

// The same means with one CTA per output row, for long groups (few output
// rows of many keys): the group's rows are split over `parts` threads per
// column vector, and the fp64 partial sums are added in a fixed order (the
// sums are exact, so the result equals the one-thread walk's).
template <int DT>
__global__ void __launch_bounds__(256) segment_mean_wide_kernel(
    const uint8_t* __restrict__ in, const float* __restrict__ in_scale,
    uint8_t* __restrict__ out, float* __restrict__ out_scale,
    int batch, int n_in, int n_out, int d, int G, int o_first, int o_count) {
  constexpr int VE = Vec16<DT>::n;
  __shared__ double part_sum[256 * VE];
  const int vecs = d / VE;
  const int parts = 256 / vecs;
  const int v = threadIdx.x % vecs, part = threadIdx.x / vecs;
  const int64_t row_bytes = static_cast<int64_t>(d) * Elem<DT>::bytes;
  for (int64_t lrow = blockIdx.x; lrow < static_cast<int64_t>(batch) * o_count; lrow += gridDim.x) {
    const int b = static_cast<int>(lrow / o_count);
    const int o = o_first + static_cast<int>(lrow % o_count);
    const int64_t orow = static_cast<int64_t>(b) * n_out + o;
    const int r0 = o * G, r1 = min(r0 + G, n_in);
    double acc[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] = 0.0;
    const uint8_t* base = in + (static_cast<int64_t>(b) * n_in) * row_bytes + v * 16;
#pragma unroll 4
    for (int r = r0 + part; r < r1; r += parts) {
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
    __syncthreads();
#pragma unroll
    for (int e = 0; e < VE; ++e) part_sum[threadIdx.x * VE + e] = acc[e];
    __syncthreads();
    if (threadIdx.x < 32) {                       // lanes 0..vecs-1 hold the row
      double tot[VE];
#pragma unroll
      for (int e = 0; e < VE; ++e) tot[e] = 0.0;
      if (threadIdx.x < vecs)
        for (int pt = 0; pt < parts; ++pt)
#pragma unroll
          for (int e = 0; e < VE; ++e) tot[e] += part_sum[(pt * vecs + threadIdx.x) * VE + e];
      write_mean<DT>(tot, static_cast<double>(max(r1 - r0, 1)), out + orow * row_bytes + threadIdx.x * 16,
                     out_scale ? out_scale + orow : nullptr, threadIdx.x, vecs, threadIdx.x < vecs);
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

// Fully visible blocks per query: blocks 0..c_t-1, c_t = (n_t - 1) / B.
__global__ void visible_blocks_kernel(const int32_t* __restrict__ n_visible, int64_t rows, int L, int B,
                                      int32_t* __restrict__ out) {
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < rows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int n = max(0, min(n_visible[r], L));
    out[r] = n > 0 ? (n - 1) / B : 0;
  }
}

// Block list of the three-level indexer: the current block c_t first, then
// the selected blocks (sel rows of width m-1, -1 padded), then -1 padding.
__global__ void assemble_blocks_kernel(const int32_t* __restrict__ n_visible, const int32_t* __restrict__ sel,
                                       int64_t rows, int L, int B, int top_m, int32_t* __restrict__ out) {
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < rows;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int n = max(0, min(n_visible[r], L));
    int32_t* o = out + r * top_m;
    if (n == 0) {
      for (int i = 0; i < top_m; ++i) o[i] = -1;
      continue;
    }
    o[0] = (n - 1) / B;
    int j = 1;
    for (int i = 0; i < top_m - 1; ++i) {
      const int32_t b = sel ? sel[r * (top_m - 1) + i] : -1;
      if (b >= 0) o[j++] = b;
    }
    for (; j < top_m; ++j) o[j] = -1;
  }
}

}  // namespace hisa

// sort.cuh - order of the scored top-k output.
//
// The selection kernels emit each query's k indices as a set, in whatever
// order their passes produce them.  When the caller asks for scores, the row
// is returned sorted by (score desc, index asc), the order that defines the
// top-k itself, with the -1 / -inf padding last.  One CTA sorts one row at a
// time in shared memory: each (score, index) pair becomes one 64-bit key,
// the order-preserving image of the score in the high word and the
// complement of the index in the low word, so that a plain descending sort of
// the keys is the required order; padding (-inf, -1) maps below every real
// entry.  Bitonic network over the row padded to a power of two.
#pragma once
#include "common.cuh"

namespace hisa {

constexpr int kSortThreads = 1024;
constexpr int kSortMaxK = 16384;     // longest row sorted on chip (128 KB of keys)

__device__ __forceinline__ uint64_t scored_key(float score, int32_t idx) {
  return (static_cast<uint64_t>(float_key(score)) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(idx));
}

__global__ void __launch_bounds__(kSortThreads) sort_scored_rows_kernel(int32_t* __restrict__ idx,
                                                                        float* __restrict__ score, int64_t rows,
                                                                        int k, int n_pow2) {
  extern __shared__ __align__(16) uint64_t sk[];
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    int32_t* ri = idx + row * k;
    float* rs = score + row * k;
    for (int i = threadIdx.x; i < n_pow2; i += blockDim.x) sk[i] = i < k ? scored_key(rs[i], ri[i]) : 0ull;
    __syncthreads();
    // descending bitonic sort: stage (size, stride); each thread handles
    // pairs (i, i ^ stride) with i < partner
    for (int size = 2; size <= n_pow2; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int p = threadIdx.x; p < (n_pow2 >> 1); p += blockDim.x) {
          const int i = 2 * p - (p & (stride - 1));      // lower element of the pair
          const int j = i + stride;
          const bool desc = (i & size) == 0;               // direction of this bitonic run
          const uint64_t a = sk[i], b = sk[j];
          if ((a < b) == desc) { sk[i] = b; sk[j] = a; }
        }
        __syncthreads();
      }
    }
    for (int i = threadIdx.x; i < k; i += blockDim.x) {
      const uint64_t key = sk[i];
      const int32_t id = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(key & 0xFFFFFFFFull));
      ri[i] = id;
      rs[i] = id < 0 ? -__int_as_float(0x7f800000) : key_float(static_cast<uint32_t>(key >> 32));
    }
    __syncthreads();
  }
}

inline int sort_pow2(int k) {
  int n = 1;
  while (n < k) n <<= 1;
  return n < 2 ? 2 : n;
}

}  // namespace hisa

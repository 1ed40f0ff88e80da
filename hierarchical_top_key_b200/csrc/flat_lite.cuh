// flat_lite.cuh - flat DSA indexer top-k without materialising score rows
// (the sampled-threshold, write-back-only-promising-candidates scheme of
// "LITETOPK" in the Indexer-TopK abstract).
//
// 1. Every stride-th key is scored (the dense kernel over a strided view of the
//    keys); per query the r-th largest of those sample scores becomes its
//    threshold, r chosen so that the keys at or above it outnumber k with
//    overwhelming probability under uniform sampling.
// 2. The dense kernel scores every visible key again and appends only the
//    (position, ordering key) pairs at or above the query's threshold.
// 3. flat_pairs_select_kernel takes the exact top-k of the pairs.  When fewer
//    than k pairs passed, or more than the buffer holds, the estimate failed:
//    the query goes on a list, and flat_fallback_kernel rescores its whole
//    visible prefix on CUDA cores and selects from that.  Either way the result
//    is the exact top-k by (score desc, position asc).
#pragma once
#include "common.cuh"
#include "select.cuh"
#include "score_simt.cuh"

namespace hisa {

// Per query: the compaction threshold from its sample scores (row lr of
// `sample`, sample j = key j*stride).  Queries whose whole visible prefix fits
// the pair buffer take every key (threshold 1).
template <int KPT>
__global__ void __launch_bounds__(128) flat_thresh_kernel(
    const float* __restrict__ sample, int64_t sld, const int32_t* __restrict__ n_visible, int64_t row0,
    int64_t nrows, int L, int stride, int cap, int r_target, uint32_t* __restrict__ thresh) {
  __shared__ uint32_t red[4];
  for (int64_t lr = blockIdx.x; lr < nrows; lr += gridDim.x) {
    const int n = max(0, min(__ldg(n_visible + row0 + lr), L));
    if (n <= cap) {
      if (threadIdx.x == 0) thresh[lr] = 1u;
      continue;
    }
    const int ns = (n + stride - 1) / stride;
    const float* row = sample + lr * sld;
    uint32_t key[KPT];
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      const int i = threadIdx.x + u * 128;
      key[u] = i < ns ? float_key(__ldg(row + i)) : 0u;
    }
    const uint32_t T = cta_rth_largest<128, KPT>(key, static_cast<uint32_t>(min(r_target, ns)), red);
    if (threadIdx.x == 0) thresh[lr] = max(T, 1u);
  }
}

// Exact top-k of each query's pairs; failed estimates go on the fallback list.
template <int KPT>
__global__ void __launch_bounds__(256) flat_pairs_select_kernel(
    const uint2* __restrict__ pairs, const uint32_t* __restrict__ counts, int cap,
    const int32_t* __restrict__ n_visible, int64_t row0, int64_t nrows, int L, int k,
    int32_t* __restrict__ out_idx, float* __restrict__ out_score, uint32_t* __restrict__ fail_count,
    int32_t* __restrict__ fail_rows) {
  __shared__ uint32_t red[8];
  __shared__ uint32_t slot_ctr;
  const int tid = threadIdx.x, lane = tid & 31;
  for (int64_t lr = blockIdx.x; lr < nrows; lr += gridDim.x) {
    const int64_t r = row0 + lr;
    const int n = max(0, min(__ldg(n_visible + r), L));
    const uint32_t c = counts[lr];
    int32_t* oi = out_idx + r * k;
    float* os = out_score ? out_score + r * k : nullptr;
    const bool every_key = n <= cap;                    // threshold 1: every visible key is a pair
    if (!every_key && (c < static_cast<uint32_t>(k) || c > static_cast<uint32_t>(cap))) {
      if (tid == 0) fail_rows[atomicAdd(fail_count, 1u)] = static_cast<int32_t>(lr);
      continue;
    }
    const uint32_t m = min(c, static_cast<uint32_t>(cap));
    const uint2* pr = pairs + lr * cap;
    if (m <= static_cast<uint32_t>(k)) {                // every pair, then padding
      for (int i = tid; i < k; i += 256) {
        if (static_cast<uint32_t>(i) < m) {
          const uint2 e = pr[i];
          oi[i] = static_cast<int32_t>(e.x);
          if (os) os[i] = key_float(e.y);
        } else {
          oi[i] = -1;
          if (os) os[i] = -__int_as_float(0x7f800000);
        }
      }
      continue;
    }
    uint32_t key[KPT], pos[KPT];
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      const uint32_t i = tid + u * 256;
      if (i < m) {
        const uint2 e = pr[i];
        pos[u] = e.x;
        key[u] = e.y;
      } else {
        pos[u] = 0xFFFFFFFFu;
        key[u] = 0u;
      }
    }
    const uint32_t T = cta_rth_largest<256, KPT>(key, static_cast<uint32_t>(k), red);
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      gt += key[u] > T ? 1u : 0u;
      eq += key[u] == T ? 1u : 0u;
    }
    gt = cta_sum<256>(gt, red);
    eq = cta_sum<256>(eq, red);
    const uint32_t need = static_cast<uint32_t>(k) - gt;   // places for keys equal to T, lowest positions first
    uint32_t P = 0xFFFFFFFFu;
    if (eq > need) {
      // the smallest position P with `need` equal keys at or below it
      P = 0u;
      for (int bit = 30; bit >= 0; --bit) {
        const uint32_t test = P | ((1u << bit) - 1u);
        uint32_t cnt = 0;
#pragma unroll
        for (int u = 0; u < KPT; ++u) cnt += (key[u] == T && pos[u] <= test) ? 1u : 0u;
        if (cta_sum<256>(cnt, red) < need) P |= 1u << bit;
      }
    }
    if (tid == 0) slot_ctr = 0;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      const bool take = key[u] > T || (key[u] == T && key[u] != 0u && pos[u] <= P);
      const uint32_t ball = __ballot_sync(0xffffffffu, take);
      uint32_t base = 0;
      if (lane == 0 && ball) base = atomicAdd(&slot_ctr, static_cast<uint32_t>(__popc(ball)));
      base = __shfl_sync(0xffffffffu, base, 0) + __popc(ball & ((1u << lane) - 1u));
      if (take) {
        oi[base] = static_cast<int32_t>(pos[u]);
        if (os) os[base] = key_float(key[u]);
      }
    }
    __syncthreads();
  }
}

// The queries whose estimate failed: score the whole visible prefix on CUDA
// cores into this CTA's scratch row, then select from it.
template <int DT, int HT>
__global__ void __launch_bounds__(kSimtThreads) flat_fallback_kernel(
    const uint8_t* __restrict__ q, const float* __restrict__ q_scale, const float* __restrict__ w,
    const uint8_t* __restrict__ keys, const float* __restrict__ k_scale, const int32_t* __restrict__ n_visible,
    int64_t row0, int Q, int H, int d, int L, int k, const uint32_t* __restrict__ fail_count,
    const int32_t* __restrict__ fail_rows, float* __restrict__ scratch, int32_t* __restrict__ out_idx,
    float* __restrict__ out_score) {
  using T = SimtTile<DT, HT>;
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ SelectSmem sel;
  float* qs = reinterpret_cast<float*>(smem);
  float* ws = qs + HT * d;
  uint8_t* tile = reinterpret_cast<uint8_t*>(ws + HT);
  float* srow = scratch + static_cast<int64_t>(blockIdx.x) * L;
  const uint32_t nf = *fail_count;
  for (uint32_t f = blockIdx.x; f < nf; f += gridDim.x) {
    const int64_t r = row0 + fail_rows[f];
    const int b = static_cast<int>(r / Q);
    const int n = max(0, min(n_visible[r], L));
    __syncthreads();
    T::load_query(q + r * static_cast<int64_t>(H) * d * Elem<DT>::bytes, w + r * H, H, d, qs, ws);
    const uint8_t* kseq = keys + static_cast<int64_t>(b) * L * d * Elem<DT>::bytes;
    const float qsc = DT == DT_E4M3 ? q_scale[r] : 1.f;
    for (int s0 = 0; s0 < n; s0 += kSimtThreads) {
      const int cnt = min(kSimtThreads, n - s0);
      __syncthreads();
      T::stage_keys(kseq, d, cnt, [&](int j) { return static_cast<int64_t>(s0 + j); }, tile);
      __syncthreads();
      if (static_cast<int>(threadIdx.x) < cnt) {
        float v = T::score_row(qs, ws, tile, d, threadIdx.x);
        if (DT == DT_E4M3) v *= qsc * k_scale[static_cast<int64_t>(b) * L + s0 + threadIdx.x];
        srow[s0 + threadIdx.x] = v;
      }
    }
    __syncthreads();
    int32_t* oi = out_idx + r * k;
    float* os = out_score ? out_score + r * k : nullptr;
    auto key_at = [&](int i) { return float_key(srow[i]); };
    auto emit = [&](uint32_t slot, int i, uint32_t key) {
      oi[slot] = i;
      if (os) os[slot] = key_float(key);
    };
    const uint32_t nv = block_topk(key_at, n, static_cast<uint32_t>(k), emit, sel);
    for (int i = static_cast<int>(nv) + threadIdx.x; i < k; i += blockDim.x) {
      oi[i] = -1;
      if (os) os[i] = -__int_as_float(0x7f800000);
    }
  }
}

}  // namespace hisa

// score_simt.cuh - CUDA-core (fp32 FMA) indexer scoring.
//
// I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:]), with E4M3 scales folded in
// at the end (q_scale[t] * k_scale[s] * sum_h ...; positive scales commute
// with ReLU).  This path computes every dot product in fp32 on the CUDA cores
// and is the path for fp32 inputs, where a tensor-core format (tf32) would
// round the inputs.
//
// A CTA holds one query's q (fp32, [HT][d]) and w in shared memory and scores
// a tile of up to 256 keys per step, one key per thread; the key rows are
// staged in their storage format with a 16-byte row pad so that each thread's
// 16-byte reads of its own row are bank-conflict free, and q is read as
// broadcast float4s.
#pragma once
#include "common.cuh"
#include "select.cuh"

namespace hisa {

constexpr int kSimtThreads = 256;

template <int DT, int HT>
struct SimtTile {
  static constexpr int VE = Vec16<DT>::n;
  // smem layout (bytes): q [HT][d] f32 | w [HT] f32 | key tile [256][row_bytes+16]
  __host__ __device__ static int row_stride(int d) { return d * Elem<DT>::bytes + 16; }
  __host__ __device__ static size_t smem_bytes(int d) {
    return static_cast<size_t>(HT) * d * 4 + HT * 4 + static_cast<size_t>(kSimtThreads) * row_stride(d);
  }

  // Stage q[t] and w[t] (heads >= H are zero) into shared memory.
  __device__ static void load_query(const uint8_t* q_row, const float* w_row, int H, int d,
                                    float* qs, float* ws) {
    const int nv = d / VE;
    for (int i = threadIdx.x; i < HT * nv; i += blockDim.x) {
      const int h = i / nv, v = i % nv;
      float f[VE];
      if (h < H) {
        Vec16<DT>::unpack(__ldg(reinterpret_cast<const uint4*>(q_row + (static_cast<int64_t>(h) * d + v * VE) *
                                                                            Elem<DT>::bytes)), f);
      } else {
#pragma unroll
        for (int e = 0; e < VE; ++e) f[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < VE; ++e) qs[h * d + v * VE + e] = f[e];
    }
    for (int h = threadIdx.x; h < HT; h += blockDim.x) ws[h] = h < H ? w_row[h] : 0.f;
  }

  // Copy key rows into the tile: row j of the tile <- key row src_row(j), for
  // j < count (src_row(j) < 0 leaves the row unset).
  template <class SrcRow>
  __device__ static void stage_keys(const uint8_t* keys, int d, int count, SrcRow src_row, uint8_t* tile) {
    const int row_bytes = d * Elem<DT>::bytes;
    const int nv = row_bytes / 16;
    const int stride = row_stride(d);
    for (int i = threadIdx.x; i < count * nv; i += blockDim.x) {
      const int j = i / nv, v = i % nv;
      const int64_t s = src_row(j);
      if (s >= 0)
        *reinterpret_cast<uint4*>(tile + j * stride + v * 16) =
            __ldg(reinterpret_cast<const uint4*>(keys + s * row_bytes + v * 16));
    }
  }

  // Score of the key in tile row j (this thread's row) against the staged query.
  __device__ static float score_row(const float* qs, const float* ws, const uint8_t* tile, int d, int j) {
    const uint8_t* kr = tile + j * row_stride(d);
    float acc[HT];
#pragma unroll
    for (int h = 0; h < HT; ++h) acc[h] = 0.f;
    for (int c = 0; c < d; c += VE) {
      float kv[VE];
      Vec16<DT>::unpack(*reinterpret_cast<const uint4*>(kr + c * Elem<DT>::bytes), kv);
#pragma unroll
      for (int h = 0; h < HT; ++h) {
        const float4* qp = reinterpret_cast<const float4*>(qs + h * d + c);
#pragma unroll
        for (int e4 = 0; e4 < VE / 4; ++e4) {
          const float4 qv = qp[e4];
          acc[h] = fmaf(qv.x, kv[4 * e4 + 0], acc[h]);
          acc[h] = fmaf(qv.y, kv[4 * e4 + 1], acc[h]);
          acc[h] = fmaf(qv.z, kv[4 * e4 + 2], acc[h]);
          acc[h] = fmaf(qv.w, kv[4 * e4 + 3], acc[h]);
        }
      }
    }
    float s = 0.f;
#pragma unroll
    for (int h = 0; h < HT; ++h) s = fmaf(ws[h], fmaxf(acc[h], 0.f), s);
    return s;
  }
};

// Dense causal scoring into fp32 rows: CTA (x = row in chunk, y = key chunk)
// writes out[row][s] for s in its chunk with s < vis(row), where vis is
// n_visible (flat indexer over keys) or (n_visible-1)/B (coarse stage over
// pooled blocks, only fully visible blocks).
template <int DT, int HT>
__global__ void __launch_bounds__(kSimtThreads) score_rows_simt_kernel(
    const uint8_t* __restrict__ q, const float* __restrict__ q_scale, const float* __restrict__ w,
    const uint8_t* __restrict__ keys, const float* __restrict__ k_scale,
    const int32_t* __restrict__ n_visible, int block_div, int Q, int H, int d, int L,
    int64_t row0, float* __restrict__ out, int64_t ld_out, int keys_per_cta) {
  using T = SimtTile<DT, HT>;
  extern __shared__ __align__(16) uint8_t smem[];
  float* qs = reinterpret_cast<float*>(smem);
  float* ws = qs + HT * d;
  uint8_t* tile = reinterpret_cast<uint8_t*>(ws + HT);
  const int64_t r = row0 + blockIdx.x;
  const int b = static_cast<int>(r / Q);
  const int nv = n_visible[r];
  const int vis = block_div > 0 ? (nv > 0 ? (nv - 1) / block_div : 0) : nv;
  const int s_begin = blockIdx.y * keys_per_cta;
  const int s_end = min(min(s_begin + keys_per_cta, vis), L);
  if (s_begin >= s_end) return;
  T::load_query(q + r * static_cast<int64_t>(H) * d * Elem<DT>::bytes, w + r * H, H, d, qs, ws);
  const uint8_t* kseq = keys + static_cast<int64_t>(b) * L * d * Elem<DT>::bytes;
  const float qsc = DT == DT_E4M3 ? q_scale[r] : 1.f;
  float* orow = out + static_cast<int64_t>(blockIdx.x) * ld_out;
  for (int s0 = s_begin; s0 < s_end; s0 += kSimtThreads) {
    const int cnt = min(kSimtThreads, s_end - s0);
    __syncthreads();
    T::stage_keys(kseq, d, cnt, [&](int j) { return static_cast<int64_t>(s0 + j); }, tile);
    __syncthreads();
    if (static_cast<int>(threadIdx.x) < cnt) {
      float v = T::score_row(qs, ws, tile, d, threadIdx.x);
      if (DT == DT_E4M3) v *= qsc * k_scale[static_cast<int64_t>(b) * L + s0 + threadIdx.x];
      orow[s0 + threadIdx.x] = v;
    }
  }
}

// Fused HISA refinement stage on CUDA cores: one CTA per query.  Scores the
// visible keys of the retained blocks into a shared-memory candidate buffer
// (as ordering keys; 0 = absent), then selects the top-k in shared memory.
template <int DT, int HT>
__global__ void __launch_bounds__(kSimtThreads) token_stage_simt_kernel(
    const uint8_t* __restrict__ q, const float* __restrict__ q_scale, const float* __restrict__ w,
    const uint8_t* __restrict__ keys, const float* __restrict__ k_scale,
    const int32_t* __restrict__ n_visible, const int32_t* __restrict__ block_idx, int Q, int H,
    int d, int L, int B, int top_m, int top_k, int32_t* __restrict__ out_idx,
    float* __restrict__ out_score) {
  using T = SimtTile<DT, HT>;
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ SelectSmem sel;
  __shared__ int32_t blk[256];
  __shared__ int nblk_s;
  float* qs = reinterpret_cast<float*>(smem);
  float* ws = qs + HT * d;
  uint8_t* tile = reinterpret_cast<uint8_t*>(ws + HT);
  uint32_t* cand = reinterpret_cast<uint32_t*>(tile + kSimtThreads * T::row_stride(d));
  const int64_t r = blockIdx.x;
  const int b = static_cast<int>(r / Q);
  const int n = max(0, min(n_visible[r], L));
  const int nb = static_cast<int>(ceil_div(L, B));
  // retained blocks: valid, visible, deduplicated, ascending (so candidate
  // position order is key order and ties resolve to the lower key)
  if (threadIdx.x == 0) {
    int cnt = 0;
    for (int i = 0; i < top_m; ++i) {
      const int bi = block_idx[r * top_m + i];
      if (bi < 0 || bi >= nb || bi * B >= n) continue;
      int pos = cnt;
      bool dup = false;
      for (int j = 0; j < cnt; ++j) dup |= blk[j] == bi;
      if (dup) continue;
      while (pos > 0 && blk[pos - 1] > bi) { blk[pos] = blk[pos - 1]; --pos; }
      blk[pos] = bi;
      ++cnt;
    }
    nblk_s = cnt;
  }
  T::load_query(q + r * static_cast<int64_t>(H) * d * Elem<DT>::bytes, w + r * H, H, d, qs, ws);
  __syncthreads();
  const int nblk = nblk_s;
  const int ncand = nblk * B;
  const uint8_t* kseq = keys + static_cast<int64_t>(b) * L * d * Elem<DT>::bytes;
  const float qsc = DT == DT_E4M3 ? q_scale[r] : 1.f;
  auto key_of = [&](int c) -> int64_t {        // candidate position -> key index, -1 if not visible
    const int64_t s = static_cast<int64_t>(blk[c / B]) * B + c % B;
    return s < n ? s : -1;
  };
  for (int c0 = 0; c0 < ncand; c0 += kSimtThreads) {
    const int cnt = min(kSimtThreads, ncand - c0);
    __syncthreads();
    T::stage_keys(kseq, d, cnt, [&](int j) { return key_of(c0 + j); }, tile);
    __syncthreads();
    if (static_cast<int>(threadIdx.x) < cnt) {
      const int64_t s = key_of(c0 + threadIdx.x);
      uint32_t key = 0u;
      if (s >= 0) {
        float v = T::score_row(qs, ws, tile, d, threadIdx.x);
        if (DT == DT_E4M3) v *= qsc * k_scale[static_cast<int64_t>(b) * L + s];
        key = float_key(v);
      }
      cand[c0 + threadIdx.x] = key;
    }
  }
  __syncthreads();
  int32_t* oi = out_idx + r * top_k;
  float* os = out_score ? out_score + r * top_k : nullptr;
  auto key_at = [&](int i) { return cand[i]; };
  auto emit = [&](uint32_t slot, int i, uint32_t key) {
    oi[slot] = static_cast<int32_t>(key_of(i));
    if (os) os[slot] = key_float(key);
  };
  const uint32_t nv = block_topk(key_at, ncand, static_cast<uint32_t>(top_k), emit, sel);
  for (int i = static_cast<int>(nv) + threadIdx.x; i < top_k; i += blockDim.x) {
    oi[i] = -1;
    if (os) os[i] = -__int_as_float(0x7f800000);
  }
}

}  // namespace hisa

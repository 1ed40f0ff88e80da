// select.cuh - block-wide exact top-k selection on order-preserving uint32
// keys (radix select, 8 bits per pass), ties resolved to the lower position.
//
// The selection finds the key T of the k-th largest element by four
// histogram passes (one digit each, most significant first), then emits every
// element with key > T (in any order) and the lowest-positioned elements with
// key == T, which fill the remaining slots.  Key 0 marks an absent element and
// is never emitted.  Keys are read through a functor, so the same code serves
// rows in global memory (flat scores, block scores) and candidate buffers in
// shared memory (the fused refinement stage).
#pragma once
#include "common.cuh"

namespace hisa {

// A set of threads that selects together: the whole CTA, or a run of whole
// warps synchronised by a named barrier.
struct CtaGroup {
  __device__ __forceinline__ static int tid() { return threadIdx.x; }
  __device__ __forceinline__ static int size() { return blockDim.x; }
  __device__ __forceinline__ static void sync() { __syncthreads(); }
};
template <int BASE, int N, int ID>
struct WarpRange {
  static_assert(BASE % 32 == 0 && N % 32 == 0, "whole warps");
  __device__ __forceinline__ static int tid() { return static_cast<int>(threadIdx.x) - BASE; }
  __device__ __forceinline__ static int size() { return N; }
  __device__ __forceinline__ static void sync() { asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(N) : "memory"); }
};

struct SelectSmem {
  uint32_t hist[256];
  uint32_t warp_cnt[32];
  uint32_t digit;
  uint32_t above;
  uint32_t at_digit;       // histogram count of the chosen digit (last pass: elements equal to T)
  uint32_t n_gt_slots;     // running slot counter for key > T
  uint32_t eq_base;        // equal-to-T elements seen in earlier chunks
  uint32_t n_valid;
};

// Block-wide exclusive prefix of a 0/1 flag over the threads (in thread
// order); returns the prefix and writes the block total to *total.
template <class Grp = CtaGroup>
__device__ __forceinline__ uint32_t block_flag_prefix(bool flag, SelectSmem& sm, uint32_t* total) {
  const int lane = Grp::tid() & 31, wid = Grp::tid() >> 5, nw = Grp::size() >> 5;
  const uint32_t ball = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) sm.warp_cnt[wid] = __popc(ball);
  Grp::sync();
  uint32_t off = 0, tot = 0;
  for (int i = 0; i < nw; ++i) {
    const uint32_t c = sm.warp_cnt[i];
    off += (i < wid) ? c : 0;
    tot += c;
  }
  Grp::sync();
  *total = tot;
  return off + __popc(ball & ((1u << lane) - 1u));
}

// Count of keys != 0 among positions [0, n).
template <class KeyAt, class Grp = CtaGroup>
__device__ uint32_t block_count_valid(KeyAt key_at, int n, SelectSmem& sm) {
  uint32_t c = 0;
  for (int i = Grp::tid(); i < n; i += Grp::size()) c += key_at(i) != 0u;
  c = __reduce_add_sync(0xffffffffu, c);
  if (Grp::tid() == 0) sm.n_valid = 0;
  Grp::sync();
  if ((Grp::tid() & 31) == 0) atomicAdd(&sm.n_valid, c);
  Grp::sync();
  const uint32_t v = sm.n_valid;
  Grp::sync();
  return v;
}

// Emit(slot, position, key) for the k largest keys among [0, n).  Requires
// blockDim.x to be a multiple of 32 (<= 1024) and more than k valid keys.
// Returns nothing; every slot 0..k-1 is emitted exactly once.
template <class KeyAt, class Emit, class Grp = CtaGroup>
__device__ void block_radix_topk(KeyAt key_at, int n, uint32_t k, Emit emit, SelectSmem& sm) {
  uint32_t prefix = 0, remaining = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int i = Grp::tid(); i < 256; i += Grp::size()) sm.hist[i] = 0;
    Grp::sync();
    for (int i = Grp::tid(); i < n; i += Grp::size()) {
      const uint32_t key = key_at(i);
      if (key != 0u && ((key ^ prefix) & hi_mask) == 0u) atomicAdd(&sm.hist[(key >> shift) & 255u], 1u);
    }
    Grp::sync();
    if (Grp::tid() < 32) {
      // lane l holds bins 255-8l .. 248-8l (descending), suffix sums across lanes
      const int lane = Grp::tid();
      uint32_t h[8], t = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { h[j] = sm.hist[255 - 8 * lane - j]; t += h[j]; }
      uint32_t incl = t;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const uint32_t excl = incl - t;
      const uint32_t ball = __ballot_sync(0xffffffffu, incl >= remaining);
      const int src = __ffs(ball) - 1;
      if (lane == src) {
        uint32_t c = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (c + h[j] >= remaining) { sm.digit = 255 - 8 * lane - j; sm.above = c; sm.at_digit = h[j]; break; }
          c += h[j];
        }
      }
    }
    Grp::sync();
    prefix |= sm.digit << shift;
    remaining -= sm.above;
    Grp::sync();
  }
  // prefix is the k-th largest key; `remaining` elements equal to it are taken
  const uint32_t T = prefix, need_eq = remaining, n_gt = k - remaining;
  const uint32_t n_eq = sm.at_digit;
  if (Grp::tid() == 0) { sm.n_gt_slots = 0; sm.eq_base = 0; }
  Grp::sync();
  if (need_eq == n_eq) {
    // no tie is cut at the boundary: every key >= T is taken, in any order
    for (int base = 0; base < n; base += Grp::size()) {
      const int i = base + Grp::tid();
      const uint32_t key = i < n ? key_at(i) : 0u;
      const bool take = key >= T && key != 0u;
      const uint32_t ball = __ballot_sync(0xffffffffu, take);
      uint32_t base_slot = 0;
      if ((Grp::tid() & 31) == 0 && ball) base_slot = atomicAdd(&sm.n_gt_slots, __popc(ball));
      base_slot = __shfl_sync(0xffffffffu, base_slot, 0);
      if (take) emit(base_slot + __popc(ball & ((1u << (Grp::tid() & 31)) - 1u)), i, key);
    }
    Grp::sync();
    return;
  }
  for (int base = 0; base < n; base += Grp::size()) {
    const int i = base + Grp::tid();
    const uint32_t key = i < n ? key_at(i) : 0u;
    if (key > T) {
      const uint32_t slot = atomicAdd(&sm.n_gt_slots, 1u);
      emit(slot, i, key);
    }
    uint32_t tot;
    const uint32_t rank = block_flag_prefix<Grp>(key == T && key != 0u, sm, &tot);
    const uint32_t r = sm.eq_base + rank;
    if (key == T && key != 0u && r < need_eq) emit(n_gt + r, i, key);
    Grp::sync();
    if (Grp::tid() == 0) sm.eq_base += tot;
    Grp::sync();
  }
}

// Emit every valid key (key != 0) among [0, n) in position order into slots
// 0..n_valid-1 (used when there are no more than k of them).
template <class KeyAt, class Emit, class Grp = CtaGroup>
__device__ void block_emit_all(KeyAt key_at, int n, Emit emit, SelectSmem& sm) {
  if (Grp::tid() == 0) sm.eq_base = 0;
  Grp::sync();
  for (int base = 0; base < n; base += Grp::size()) {
    const int i = base + Grp::tid();
    const uint32_t key = i < n ? key_at(i) : 0u;
    uint32_t tot;
    const uint32_t rank = block_flag_prefix<Grp>(key != 0u, sm, &tot);
    if (key != 0u) emit(sm.eq_base + rank, i, key);
    Grp::sync();
    if (Grp::tid() == 0) sm.eq_base += tot;
    Grp::sync();
  }
}

// ---------------------------------------------------------------- row kernels

// Flat DSA top-k over fp32 score rows: row r holds scores of keys 0..n_r-1.
__global__ void __launch_bounds__(512) flat_select_kernel(
    const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_visible,
    int64_t row0, int L, int top_k, int32_t* __restrict__ out_idx, float* __restrict__ out_score) {
  __shared__ SelectSmem sm;
  const int64_t r = row0 + blockIdx.x;
  const float* row = scores + static_cast<int64_t>(blockIdx.x) * ld;
  const int n = max(0, min(n_visible[r], L));
  int32_t* oi = out_idx + r * top_k;
  float* os = out_score ? out_score + r * top_k : nullptr;
  auto key_at = [&](int i) { return float_key(row[i]); };
  auto emit = [&](uint32_t slot, int i, uint32_t key) {
    oi[slot] = i;
    if (os) os[slot] = key_float(key);
  };
  if (n <= top_k) {
    for (int i = threadIdx.x; i < top_k; i += blockDim.x) {
      oi[i] = i < n ? i : -1;
      if (os) os[i] = i < n ? row[i] : -__int_as_float(0x7f800000);
    }
    return;
  }
  block_radix_topk(key_at, n, static_cast<uint32_t>(top_k), emit, sm);
}

// HISA block selection over fp32 block-score rows: row r holds scores of the
// fully visible blocks 0..c_r-1; the current block c_r is always kept.
__global__ void __launch_bounds__(512) block_select_kernel(
    const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_visible,
    int64_t row0, int L, int block_size, int top_m, int32_t* __restrict__ out_idx) {
  __shared__ SelectSmem sm;
  const int64_t r = row0 + blockIdx.x;
  const float* row = scores + static_cast<int64_t>(blockIdx.x) * ld;
  const int n = max(0, min(n_visible[r], L));
  const int c = n > 0 ? (n - 1) / block_size : -1;
  int32_t* oi = out_idx + r * top_m;
  if (c + 1 <= top_m) {                    // every visible block (or none)
    for (int i = threadIdx.x; i < top_m; i += blockDim.x) oi[i] = i <= c ? i : -1;
    return;
  }
  if (threadIdx.x == 0) oi[0] = c;
  if (top_m == 1) return;
  auto key_at = [&](int i) { return float_key(row[i]); };
  auto emit = [&](uint32_t slot, int i, uint32_t) { oi[1 + slot] = i; };
  block_radix_topk(key_at, c, static_cast<uint32_t>(top_m - 1), emit, sm);
}

}  // namespace hisa

// select.cuh - block-wide exact top-k selection on order-preserving uint32
// keys, ties resolved to the lower position.  Key 0 marks an absent element
// and is never emitted.  Keys are read through a functor, so the same code
// serves rows in global memory (flat scores, block scores) and candidate
// buffers in shared memory (the fused refinement stage).
//
// Two selectors, tried in this order where the caller has the row's key range:
//  - linear bins (scan_topk, two_pass_topk, two_pass_topk_rows): a histogram
//    of up to 2048 equal-width bins over [kmin, kmax], a block-parallel search
//    for the bin holding the k-th place, one counting pass and a block scan,
//    then one write pass; the members of the boundary bin are gathered into a
//    small buffer and ranked exactly.  Returns false when that bin overflows
//    its buffer, and the caller falls back to
//  - radix select (block_topk_range, block_topk): digits of 11 bits, most
//    significant first, over only the bits in which kmin and kmax differ, so
//    the number of histogram passes varies with the row (at most three for 32
//    bits); it finds the key T of the k-th largest element, then emits every
//    element with key > T in any order and the lowest-positioned elements with
//    key == T into the remaining slots.
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

constexpr int kDigitBits = 11;
constexpr int kDigitBins = 1 << kDigitBits;

struct SelectSmem {
  uint32_t hist[kDigitBins];
  uint32_t warp_cnt[32];
  uint32_t kmin, kmax, n_valid;
  uint32_t digit;
  uint32_t above;
  uint32_t at_digit;       // histogram count of the chosen digit
  uint32_t n_slots;        // running slot counter for unordered emission
  uint32_t eq_base;        // equal-to-T elements seen in earlier chunks
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

// Emit every key >= T (and != 0) into slots taken from a shared counter, in
// no particular order.  One warp-aggregated atomic per warp and chunk.
template <class KeyAt, class Emit, class Grp>
__device__ void emit_at_least(KeyAt key_at, int n, uint32_t T, Emit emit, SelectSmem& sm) {
  if (Grp::tid() == 0) sm.n_slots = 0;
  Grp::sync();
  const int lane = Grp::tid() & 31;
  for (int base = 0; base < n; base += Grp::size()) {
    const int i = base + Grp::tid();
    const uint32_t key = i < n ? key_at(i) : 0u;
    const bool take = key >= T && key != 0u;
    const uint32_t ball = __ballot_sync(0xffffffffu, take);
    uint32_t slot0 = 0;
    if (lane == 0 && ball) slot0 = atomicAdd(&sm.n_slots, __popc(ball));
    slot0 = __shfl_sync(0xffffffffu, slot0, 0);
    if (take) emit(slot0 + __popc(ball & ((1u << lane) - 1u)), i, key);
  }
  Grp::sync();
}

// Sum of one value per thread over a CTA of NT threads; every thread gets it.
template <int NT>
__device__ __forceinline__ uint32_t cta_sum(uint32_t v, uint32_t* red) {
  v = __reduce_add_sync(0xffffffffu, v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  uint32_t t = 0;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) t += red[i];
  __syncthreads();
  return t;
}

template <int NT>
__device__ __forceinline__ uint32_t cta_max(uint32_t v, uint32_t* red) {
  v = __reduce_max_sync(0xffffffffu, v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  uint32_t t = 0;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) t = max(t, red[i]);
  __syncthreads();
  return t;
}

template <int NT>
__device__ __forceinline__ uint32_t cta_min(uint32_t v, uint32_t* red) {
  v = __reduce_min_sync(0xffffffffu, v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  uint32_t t = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) t = min(t, red[i]);
  __syncthreads();
  return t;
}

// The r-th largest of the CTA's keys (KPT per thread, 0 = absent; r >= 1 and
// at most the number of present keys): bit by bit from the highest bit where
// the smallest and largest keys differ, keeping a bit when at least r keys
// are >= the value with it set.
template <int NT, int KPT>
__device__ uint32_t cta_rth_largest(const uint32_t (&key)[KPT], uint32_t r, uint32_t* red) {
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
  for (int u = 0; u < KPT; ++u)
    if (key[u] != 0u) { lo = min(lo, key[u]); hi = max(hi, key[u]); }
  lo = cta_min<NT>(lo, red);
  hi = cta_max<NT>(hi, red);
  if (lo >= hi) return hi;
  const int top = 31 - __clz(lo ^ hi);
  uint32_t T = hi & ~((2u << top) - 1u);
  for (int bit = top; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    uint32_t c = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) c += key[u] >= cand ? 1u : 0u;
    if (cta_sum<NT>(c, red) >= r) T = cand;
  }
  return T;
}

// The bin holding the k-th place of sm.hist[0, nbins) counted from the top:
// sets sm.digit, sm.above (elements in higher bins) and sm.at_digit (the
// bin's count).  Each thread sums a run of bins, one block scan orders the
// runs, and the thread whose run crosses k walks it.  Ends with a sync.
template <class Grp>
__device__ __forceinline__ void bin_search(SelectSmem& sm, int nbins, uint32_t k) {
  const int tid = Grp::tid(), nt = Grp::size(), lane = tid & 31;
  const int per = (nbins + nt - 1) / nt;             // every bin belongs to one thread's run
  const int top = nbins - 1 - tid * per;
  uint32_t t = 0;
#pragma unroll 8
  for (int j = 0; j < per; ++j)
    if (top - j >= 0) t += sm.hist[top - j];
  uint32_t incl = t;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) sm.warp_cnt[tid >> 5] = incl;
  Grp::sync();
  uint32_t woff = 0;
  for (int wi = 0; wi < (tid >> 5); ++wi) woff += sm.warp_cnt[wi];
  incl += woff;
  const uint32_t excl = incl - t;
  if (t > 0 && excl < k && incl >= k) {
    uint32_t c = excl;
    for (int j = 0; j < per && top - j >= 0; ++j) {
      const uint32_t h = sm.hist[top - j];
      if (c + h >= k) { sm.digit = top - j; sm.above = c; sm.at_digit = h; break; }
      c += h;
    }
  }
  Grp::sync();
}

// Top-k of the keys at positions [0, n) (key 0 = absent): calls
// Emit(slot, position, key) exactly once for each slot 0..min(k, valid)-1 and
// returns the number of valid keys.  Ties at the k-th place go to the lower
// position.  Radix select on the bits that vary between the smallest and the
// largest key, 11 bits per pass; spreading the digits over that range keeps
// histogram atomics on distinct bins.
// As block_topk below, with the range and count of the valid keys given.
template <class KeyAt, class Emit, class Grp = CtaGroup>
__device__ uint32_t block_topk_range(KeyAt key_at, int n, uint32_t k, Emit emit, SelectSmem& sm, uint32_t kmin,
                                     uint32_t kmax, uint32_t n_valid);

template <class KeyAt, class Emit, class Grp = CtaGroup>
__device__ uint32_t block_topk(KeyAt key_at, int n, uint32_t k, Emit emit, SelectSmem& sm) {
  const int lane = Grp::tid() & 31;
  // ---- range and count of the valid keys
  uint32_t lo = 0xFFFFFFFFu, hi = 0u, cnt = 0;
  for (int i = Grp::tid(); i < n; i += Grp::size()) {
    const uint32_t key = key_at(i);
    if (key != 0u) { lo = min(lo, key); hi = max(hi, key); ++cnt; }
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if (Grp::tid() == 0) { sm.kmin = 0xFFFFFFFFu; sm.kmax = 0u; sm.n_valid = 0u; }
  Grp::sync();
  if (lane == 0) { atomicMin(&sm.kmin, lo); atomicMax(&sm.kmax, hi); atomicAdd(&sm.n_valid, cnt); }
  Grp::sync();
  const uint32_t kmin = sm.kmin, kmax = sm.kmax, n_valid = sm.n_valid;
  Grp::sync();
  return block_topk_range<KeyAt, Emit, Grp>(key_at, n, k, emit, sm, kmin, kmax, n_valid);
}

template <class KeyAt, class Emit, class Grp>
__device__ uint32_t block_topk_range(KeyAt key_at, int n, uint32_t k, Emit emit, SelectSmem& sm, uint32_t kmin,
                                     uint32_t kmax, uint32_t n_valid) {
  const int lane = Grp::tid() & 31;
  if (n_valid <= k) {
    emit_at_least<KeyAt, Emit, Grp>(key_at, n, 1u, emit, sm);
    return n_valid;
  }
  // ---- digits below the common prefix of kmin and kmax
  int shift = kmin == kmax ? 0 : 32 - __clz(kmin ^ kmax);
  uint32_t prefix = kmax & (shift == 32 ? 0u : ~((1u << shift) - 1u));
  uint32_t remaining = k, n_eq = n_valid;
  while (shift > 0) {
    const int dig = min(kDigitBits, shift);
    shift -= dig;
    const int nbins = 1 << dig;
    const uint32_t dmask = static_cast<uint32_t>(nbins - 1);
    for (int i = Grp::tid(); i < nbins; i += Grp::size()) sm.hist[i] = 0;
    Grp::sync();
    for (int base = 0; base < n; base += Grp::size()) {
      const int i = base + Grp::tid();
      const uint32_t key = i < n ? key_at(i) : 0u;
      const bool act = key != 0u && (static_cast<uint64_t>(key ^ prefix) >> (shift + dig)) == 0;
      if (act) atomicAdd(&sm.hist[(key >> shift) & dmask], 1u);
    }
    Grp::sync();
    bin_search<Grp>(sm, nbins, remaining);
    prefix |= sm.digit << shift;
    remaining -= sm.above;
    n_eq = sm.at_digit;
    Grp::sync();
    if (n_eq == remaining) {
      // the whole boundary bin is taken: every key >= prefix (lower bits 0) is in
      emit_at_least<KeyAt, Emit, Grp>(key_at, n, prefix, emit, sm);
      return n_valid;
    }
  }
  // prefix == T, the k-th largest key; `remaining` of the n_eq keys equal to T
  // are taken, the lowest positions first
  const uint32_t T = prefix, need_eq = remaining, n_gt = k - remaining;
  if (Grp::tid() == 0) { sm.n_slots = 0; sm.eq_base = 0; }
  Grp::sync();
  for (int base = 0; base < n; base += Grp::size()) {
    const int i = base + Grp::tid();
    const uint32_t key = i < n ? key_at(i) : 0u;
    const bool gt = key > T;
    const uint32_t ball = __ballot_sync(0xffffffffu, gt);
    uint32_t slot0 = 0;
    if (lane == 0 && ball) slot0 = atomicAdd(&sm.n_slots, __popc(ball));
    slot0 = __shfl_sync(0xffffffffu, slot0, 0);
    if (gt) emit(slot0 + __popc(ball & ((1u << lane) - 1u)), i, key);
    uint32_t tot;
    const uint32_t rank = block_flag_prefix<Grp>(key == T, sm, &tot);
    const uint32_t r = sm.eq_base + rank;
    if (key == T && r < need_eq) emit(n_gt + r, i, key);
    Grp::sync();
    if (Grp::tid() == 0) sm.eq_base += tot;
    Grp::sync();
    if (sm.eq_base >= need_eq && base + Grp::size() < n) {
      // every tied key needed is placed; the rest only contributes keys > T
      for (int b2 = base + Grp::size(); b2 < n; b2 += Grp::size()) {
        const int i2 = b2 + Grp::tid();
        const uint32_t key2 = i2 < n ? key_at(i2) : 0u;
        const bool gt2 = key2 > T;
        const uint32_t ball2 = __ballot_sync(0xffffffffu, gt2);
        uint32_t s2 = 0;
        if (lane == 0 && ball2) s2 = atomicAdd(&sm.n_slots, __popc(ball2));
        s2 = __shfl_sync(0xffffffffu, s2, 0);
        if (gt2) emit(s2 + __popc(ball2 & ((1u << lane) - 1u)), i2, key2);
      }
      break;
    }
  }
  Grp::sync();
  (void)n_eq;
  return n_valid;
}

// ---------------------------------------------------------------- row kernels

// Two-pass top-k over positions [0, n) whose valid keys lie in [kmin, kmax]
// (key 0 marks an absent position and is skipped).  Pass 1: histogram over
// 2048 bins spaced linearly in score value between the smallest and largest
// score (a monotone map, so whole bins are ordered; linear spacing spreads
// the bulk of the scores, where ordering-key bits would pile it into the few
// bins of a handful of exponents).  Pass 2: every key above the boundary bin is emitted;
// the boundary bin's (key, position) pairs go to an on-chip buffer of `cap`
// entries (a power of two), where the remaining places are chosen exactly
// (larger key first, then lower position).  Returns false, having emitted
// nothing, when the boundary bin would overflow the buffer; the caller then
// falls back to block_topk_range.
template <class KeyAt, class Emit, class Grp>
__device__ bool two_pass_topk(KeyAt key_at, int n, uint32_t k, Emit emit, SelectSmem& sm, uint32_t* buf_key,
                              int32_t* buf_pos, uint32_t* buf_count, int cap, uint32_t kmin, uint32_t kmax) {
  const int lane = Grp::tid() & 31;
  const int nbins = kDigitBins;
  const float smin = key_float(kmin), smax = key_float(kmax);
  float scale = smax > smin ? static_cast<float>(nbins) / (smax - smin) : 0.f;
  if (!(scale < 1e30f)) scale = 0.f;                 // overflowing or degenerate range: one bin
  auto bin_of = [&](uint32_t key) -> uint32_t {
    const int b = static_cast<int>((key_float(key) - smin) * scale);
    return static_cast<uint32_t>(min(max(b, 0), nbins - 1));
  };
  for (int i = Grp::tid(); i < nbins; i += Grp::size()) sm.hist[i] = 0;
  if (Grp::tid() == 0) { *buf_count = 0; sm.n_slots = 0; }
  Grp::sync();
  for (int i = Grp::tid(); i < n; i += Grp::size()) {
    const uint32_t key = key_at(i);
    if (key != 0u) atomicAdd(&sm.hist[bin_of(key)], 1u);
  }
  Grp::sync();
  uint32_t remaining = k;
  bin_search<Grp>(sm, nbins, remaining);
  const uint32_t D = sm.digit, above = sm.above, n_eq = sm.at_digit;
  remaining -= above;
  Grp::sync();
  const bool take_bin = n_eq == remaining;
  if (!take_bin && n_eq > static_cast<uint32_t>(cap)) return false;
  // pass 2: emit keys above the boundary bin; buffer the bin (or take all of it)
  for (int base = 0; base < n; base += Grp::size()) {
    const int i = base + Grp::tid();
    const uint32_t key = i < n ? key_at(i) : 0u;
    const bool valid = key != 0u;
    const uint32_t dg = valid ? bin_of(key) : 0u;
    const bool gt = valid && (dg > D || (take_bin && dg == D));
    const uint32_t ball = __ballot_sync(0xffffffffu, gt);
    uint32_t slot0 = 0;
    if (lane == 0 && ball) slot0 = atomicAdd(&sm.n_slots, __popc(ball));
    slot0 = __shfl_sync(0xffffffffu, slot0, 0);
    if (gt) emit(slot0 + __popc(ball & ((1u << lane) - 1u)), i, key);
    if (!take_bin) {
      const bool eq = valid && dg == D;
      const uint32_t be = __ballot_sync(0xffffffffu, eq);
      uint32_t b0 = 0;
      if (lane == 0 && be) b0 = atomicAdd(buf_count, __popc(be));
      b0 = __shfl_sync(0xffffffffu, b0, 0);
      if (eq) {
        const uint32_t at = b0 + __popc(be & ((1u << lane) - 1u));
        buf_key[at] = key;
        buf_pos[at] = i;
      }
    }
  }
  Grp::sync();
  if (take_bin) return true;
  // choose `remaining` of the n_eq buffered keys: larger key first, then lower position
  const int nb = static_cast<int>(n_eq);
  if (nb <= 256) {
    for (int e = Grp::tid(); e < nb; e += Grp::size()) {
      const uint32_t ke = buf_key[e];
      const int pe = buf_pos[e];
      uint32_t rank = 0;
      for (int f = 0; f < nb; ++f) {
        const uint32_t kf = buf_key[f];
        rank += (kf > ke || (kf == ke && buf_pos[f] < pe)) ? 1u : 0u;
      }
      if (rank < remaining) emit(above + rank, pe, ke);
    }
  } else {
    // bitonic sort of the buffer (padded to a power of two) by (key desc, position asc)
    int np2 = 1;
    while (np2 < nb) np2 <<= 1;
    for (int i = nb + Grp::tid(); i < np2; i += Grp::size()) { buf_key[i] = 0u; buf_pos[i] = 0x7FFFFFFF; }
    Grp::sync();
    for (int size = 2; size <= np2; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = Grp::tid(); i < np2 / 2; i += Grp::size()) {
          const int lo = 2 * i - (i & (stride - 1));
          const int hi = lo + stride;
          const bool desc = (lo & size) == 0;          // this run sorts "best first"
          const uint32_t ka = buf_key[lo], kb = buf_key[hi];
          const int pa = buf_pos[lo], pb = buf_pos[hi];
          const bool b_better = kb > ka || (kb == ka && pb < pa);
          if (b_better == desc) {
            buf_key[lo] = kb; buf_key[hi] = ka;
            buf_pos[lo] = pb; buf_pos[hi] = pa;
          }
        }
        Grp::sync();
      }
    }
    for (int e = Grp::tid(); e < static_cast<int>(remaining); e += Grp::size()) emit(above + e, buf_pos[e], buf_key[e]);
  }
  Grp::sync();
  return true;
}

// Block-wide exclusive prefix sums of two per-thread counts (thread order);
// totals go to *ta and *tb.
template <class Grp>
__device__ __forceinline__ void block_scan2(uint32_t a, uint32_t b, uint32_t* pa, uint32_t* pb, uint32_t* ta,
                                            uint32_t* tb, SelectSmem& sm) {
  const int lane = Grp::tid() & 31, wid = Grp::tid() >> 5, nw = Grp::size() >> 5;
  uint32_t ia = a, ib = b;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t oa = __shfl_up_sync(0xffffffffu, ia, off);
    const uint32_t ob = __shfl_up_sync(0xffffffffu, ib, off);
    if (lane >= off) { ia += oa; ib += ob; }
  }
  if (lane == 31) { sm.warp_cnt[wid] = ia; sm.hist[wid] = ib; }   // hist is free here: the bins are consumed
  Grp::sync();
  uint32_t wa = 0, wb = 0, sa = 0, sb = 0;
  for (int i = 0; i < nw; ++i) {
    const uint32_t ca = sm.warp_cnt[i], cb = sm.hist[i];
    if (i < wid) { wa += ca; wb += cb; }
    sa += ca;
    sb += cb;
  }
  Grp::sync();
  *pa = wa + ia - a;
  *pb = wb + ib - b;
  *ta = sa;
  *tb = sb;
}

// Like two_pass_topk, for keys cheap to read three times (shared memory):
// thread i owns positions i, i+size, ...; pass 2 only counts, one block scan
// gives every thread its output offsets, pass 3 writes.  No returning atomics
// or per-element shuffles; loops are unrolled four-wide so the loads of four
// positions are in flight together.  `nbins` (<= kDigitBins) linear bins.
template <class KeyAt, class Emit, class Grp>
__device__ bool scan_topk(KeyAt key_at, int n, uint32_t k, Emit emit, SelectSmem& sm, uint32_t* buf_key,
                          int32_t* buf_pos, int cap, uint32_t kmin, uint32_t kmax, int nbins = kDigitBins) {
  const int lane = Grp::tid() & 31;
  const int tid = Grp::tid(), nt = Grp::size();
  const float smin = key_float(kmin), smax = key_float(kmax);
  float scale = smax > smin ? static_cast<float>(nbins) / (smax - smin) : 0.f;
  if (!(scale < 1e30f)) scale = 0.f;
  const uint32_t top_bin = static_cast<uint32_t>(nbins - 1);
  // bin = nearest integer to (score - smin) * scale, by adding 2^23 and reading
  // the low mantissa bits (exact for values below 2^22, monotone in the score);
  // this keeps the float-to-int conversion pipe free
  const float bias = 8388608.0f - smin * scale;
  auto bin_of = [&](uint32_t key) -> uint32_t {
    // signed difference: a value rounded just below 2^23 gives -1 -> bin 0
    const int b = static_cast<int>(__float_as_uint(fmaf(key_float(key), scale, bias)) - 0x4B000000u);
    return min(static_cast<uint32_t>(max(b, 0)), top_bin);
  };
  for (int i = tid; i < nbins; i += nt) sm.hist[i] = 0;
  Grp::sync();
  // pass 1: histogram
  for (int base = tid; base < n; base += 4 * nt) {
    uint32_t kv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) kv[u] = base + u * nt < n ? key_at(base + u * nt) : 0u;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (kv[u] != 0u) atomicAdd(&sm.hist[bin_of(kv[u])], 1u);
  }
  Grp::sync();
  uint32_t remaining = k;
  bin_search<Grp>(sm, nbins, remaining);
  const uint32_t D = sm.digit, above = sm.above, n_eq = sm.at_digit;
  remaining -= above;
  const bool take_bin = n_eq == remaining;
  if (!take_bin && n_eq > static_cast<uint32_t>(cap)) return false;
  const uint32_t gt_floor = take_bin ? D : D + 1;        // bins >= gt_floor are emitted outright
  // pass 2: count what this thread emits and buffers
  uint32_t cg = 0, ce = 0;
  for (int base = tid; base < n; base += 4 * nt) {
    uint32_t kv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) kv[u] = base + u * nt < n ? key_at(base + u * nt) : 0u;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (kv[u] == 0u) continue;
      const uint32_t b = bin_of(kv[u]);
      cg += b >= gt_floor ? 1u : 0u;
      ce += b == D && !take_bin ? 1u : 0u;
    }
  }
  uint32_t og, oe, tg, te;
  block_scan2<Grp>(cg, ce, &og, &oe, &tg, &te, sm);
  // pass 3: write
  for (int base = tid; base < n; base += 4 * nt) {
    uint32_t kv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) kv[u] = base + u * nt < n ? key_at(base + u * nt) : 0u;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (kv[u] == 0u) continue;
      const uint32_t b = bin_of(kv[u]);
      if (b >= gt_floor) {
        emit(og++, base + u * nt, kv[u]);
      } else if (b == D) {
        buf_key[oe] = kv[u];
        buf_pos[oe] = base + u * nt;
        ++oe;
      }
    }
  }
  Grp::sync();
  if (take_bin) return true;
  // the remaining places among the buffered keys: larger key first, then lower position
  const int nb = static_cast<int>(n_eq);
  for (int e = tid; e < nb; e += nt) {
    const uint32_t ke = buf_key[e];
    const int pe = buf_pos[e];
    uint32_t rank = 0;
    for (int f = 0; f < nb; ++f) {
      const uint32_t kf = buf_key[f];
      rank += (kf > ke || (kf == ke && buf_pos[f] < pe)) ? 1u : 0u;
    }
    if (rank < remaining) emit(above + rank, pe, ke);
  }
  Grp::sync();
  return true;
}

constexpr int kTwoPassCap = 4096;

struct TwoPassSmem {
  uint32_t key[kTwoPassCap];
  int32_t pos[kTwoPassCap];
  uint32_t count;
};

// two_pass_topk over a 16-byte aligned fp32 row, reading it as float4 and two
// of them per thread per step: a row of scores is streamed from DRAM, and one
// 4-byte load in flight per thread leaves the selection latency-bound at a
// fraction of the bandwidth.  Same contract as two_pass_topk.
template <class Emit, class Grp>
__device__ bool two_pass_topk_rows(const float* __restrict__ row, int n, uint32_t k, Emit emit, SelectSmem& sm,
                                   uint32_t* buf_key, int32_t* buf_pos, uint32_t* buf_count, int cap,
                                   uint32_t kmin, uint32_t kmax) {
  const int lane = Grp::tid() & 31, tid = Grp::tid(), nt = Grp::size();
  const int nbins = kDigitBins;
  const float smin = key_float(kmin), smax = key_float(kmax);
  float scale = smax > smin ? static_cast<float>(nbins) / (smax - smin) : 0.f;
  if (!(scale < 1e30f)) scale = 0.f;
  // bin = nearest integer to (score - smin) * scale, by adding 2^23 and reading
  // the low mantissa bits: monotone in the score (so in the ordering key) and
  // free of the float-to-int conversion; computed from the score itself
  const float bias = 8388608.0f - smin * scale;
  const uint32_t top_bin = static_cast<uint32_t>(nbins - 1);
  auto bin_of = [&](float v) -> uint32_t {
    const int b = static_cast<int>(__float_as_uint(fmaf(v, scale, bias)) - 0x4B000000u);
    return min(static_cast<uint32_t>(max(b, 0)), top_bin);
  };
  // -0 scores bin like +0 (their ordering keys are equal); scores past n are skipped
  auto load8 = [&](int p0, float (&v)[8], uint32_t& valid) {
    valid = 0u;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int p = p0 + 4 * h;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (p + 3 < n) {
        x = __ldcg(reinterpret_cast<const float4*>(row + p));
        valid |= 0xFu << (4 * h);
      } else {
        if (p < n) { x.x = __ldcg(row + p); valid |= 1u << (4 * h); }
        if (p + 1 < n) { x.y = __ldcg(row + p + 1); valid |= 2u << (4 * h); }
        if (p + 2 < n) { x.z = __ldcg(row + p + 2); valid |= 4u << (4 * h); }
      }
      v[4 * h + 0] = x.x; v[4 * h + 1] = x.y; v[4 * h + 2] = x.z; v[4 * h + 3] = x.w;
    }
  };
  for (int i = tid; i < nbins; i += nt) sm.hist[i] = 0;
  if (tid == 0) { *buf_count = 0; sm.n_slots = 0; }
  Grp::sync();
  for (int p0 = 8 * tid; p0 < n; p0 += 8 * nt) {
    float v[8];
    uint32_t valid;
    load8(p0, v, valid);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if ((valid >> u) & 1u) atomicAdd(&sm.hist[bin_of(v[u])], 1u);
  }
  Grp::sync();
  uint32_t remaining = k;
  bin_search<Grp>(sm, nbins, remaining);
  const uint32_t D = sm.digit, above = sm.above, n_eq = sm.at_digit;
  remaining -= above;
  Grp::sync();
  const bool take_bin = n_eq == remaining;
  if (!take_bin && n_eq > static_cast<uint32_t>(cap)) return false;
  const uint32_t gt_floor = take_bin ? D : D + 1;
  // pass 2: emit keys from the bins above the boundary (or from it too when
  // all of it is taken) and buffer the boundary bin; most warp-steps find
  // nothing to do and skip the slot bookkeeping
  for (int b0 = 0; b0 < n; b0 += 8 * nt) {
    const int p0 = b0 + 8 * tid;
    float v[8];
    uint32_t valid;
    load8(p0, v, valid);
    uint32_t gt_mask = 0u, eq_mask = 0u;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t b = bin_of(v[u]);
      const bool ok = (valid >> u) & 1u;
      gt_mask |= (ok && b >= gt_floor) ? 1u << u : 0u;
      eq_mask |= (ok && !take_bin && b == D) ? 1u << u : 0u;
    }
    if (__any_sync(0xffffffffu, gt_mask != 0u)) {
      // this warp's emissions for the step: count, one reservation, prefix
      const uint32_t cnt = __popc(gt_mask);
      uint32_t incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      uint32_t base = 0;
      if (lane == 31) base = atomicAdd(&sm.n_slots, incl);
      base = __shfl_sync(0xffffffffu, base, 31) + incl - cnt;
      for (uint32_t m = gt_mask; m; m &= m - 1) {
        const int u = __ffs(m) - 1;
        emit(base++, p0 + u, float_key(v[u]));
      }
    }
    if (__any_sync(0xffffffffu, eq_mask != 0u)) {
      const uint32_t cnt = __popc(eq_mask);
      uint32_t incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      uint32_t base = 0;
      if (lane == 31) base = atomicAdd(buf_count, incl);
      base = __shfl_sync(0xffffffffu, base, 31) + incl - cnt;
      for (uint32_t m = eq_mask; m; m &= m - 1) {
        const int u = __ffs(m) - 1;
        buf_key[base] = float_key(v[u]);
        buf_pos[base] = p0 + u;
        ++base;
      }
    }
  }
  Grp::sync();
  if (take_bin) return true;
  const int nb = static_cast<int>(n_eq);
  for (int e = tid; e < nb; e += nt) {
    const uint32_t ke = buf_key[e];
    const int pe = buf_pos[e];
    uint32_t rank = 0;
    for (int f = 0; f < nb; ++f) {
      const uint32_t kf = buf_key[f];
      rank += (kf > ke || (kf == ke && buf_pos[f] < pe)) ? 1u : 0u;
    }
    if (rank < remaining) emit(above + rank, pe, ke);
  }
  Grp::sync();
  return true;
}

// Top-k of the union of `parts` top-k lists per row (idx -1 = empty slot),
// by (score desc, index asc): the refinement stage split over several CTAs
// per query writes each part's own top-k, and since every element of the
// query's top-k is in its part's top-k, the top-k of the union is exact.
template <int KPT>
__global__ void __launch_bounds__(256) merge_parts_kernel(const int32_t* __restrict__ part_idx,
                                                          const float* __restrict__ part_score, int parts,
                                                          int64_t rows, int k, int32_t* __restrict__ out_idx,
                                                          float* __restrict__ out_score) {
  __shared__ uint32_t red[8];
  __shared__ uint32_t slot_ctr;
  const int tid = threadIdx.x, lane = tid & 31;
  const int m_all = parts * k;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int32_t* pi = part_idx + r * m_all;
    const float* ps = part_score + r * m_all;
    uint32_t key[KPT], pos[KPT];
    uint32_t valid = 0;
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      const int i = tid + u * 256;
      const int32_t x = i < m_all ? pi[i] : -1;
      pos[u] = x >= 0 ? static_cast<uint32_t>(x) : 0xFFFFFFFFu;
      key[u] = x >= 0 ? max(float_key(ps[i]), 1u) : 0u;
      valid += x >= 0 ? 1u : 0u;
    }
    valid = cta_sum<256>(valid, red);
    int32_t* oi = out_idx + r * k;
    float* os = out_score ? out_score + r * k : nullptr;
    uint32_t T = 0u, P = 0xFFFFFFFFu;
    if (valid > static_cast<uint32_t>(k)) {
      T = cta_rth_largest<256, KPT>(key, static_cast<uint32_t>(k), red);
      uint32_t gt = 0, eq = 0;
#pragma unroll
      for (int u = 0; u < KPT; ++u) {
        gt += key[u] > T ? 1u : 0u;
        eq += key[u] == T ? 1u : 0u;
      }
      gt = cta_sum<256>(gt, red);
      eq = cta_sum<256>(eq, red);
      const uint32_t need = static_cast<uint32_t>(k) - gt;
      if (eq > need) {
        P = 0u;
        for (int bit = 30; bit >= 0; --bit) {
          const uint32_t test = P | ((1u << bit) - 1u);
          uint32_t cnt = 0;
#pragma unroll
          for (int u = 0; u < KPT; ++u) cnt += (key[u] == T && pos[u] <= test) ? 1u : 0u;
          if (cta_sum<256>(cnt, red) < need) P |= 1u << bit;
        }
      }
    }
    if (tid == 0) slot_ctr = 0;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      const bool take = key[u] != 0u && (key[u] > T || (key[u] == T && pos[u] <= P));
      const uint32_t ball = __ballot_sync(0xffffffffu, take);
      uint32_t base = 0;
      if (lane == 0 && ball) base = atomicAdd(&slot_ctr, static_cast<uint32_t>(__popc(ball)));
      base = __shfl_sync(0xffffffffu, base, 0) + __popc(ball & ((1u << lane) - 1u));
      if (take) {
        oi[base] = static_cast<int32_t>(pos[u]);
        if (os) os[base] = ps[tid + u * 256];
      }
    }
    __syncthreads();
    const uint32_t filled = min(valid, static_cast<uint32_t>(k));
    for (int i = static_cast<int>(filled) + tid; i < k; i += 256) {
      oi[i] = -1;
      if (os) os[i] = -__int_as_float(0x7f800000);
    }
    __syncthreads();
  }
}

// Flat DSA top-k over fp32 score rows: row r holds scores of keys 0..n_r-1.
// `minmax` (nullable) holds, per row, the smallest and largest ordering key
// the scoring kernel wrote; with it the row is read twice (histogram, then
// emission), without it the generic multi-pass selection runs.
__global__ void __launch_bounds__(512) flat_select_kernel(
    const float* __restrict__ scores, int64_t ld, const uint32_t* __restrict__ minmax,
    const int32_t* __restrict__ n_visible, int64_t row0, int L, int top_k, int32_t* __restrict__ out_idx,
    float* __restrict__ out_score) {
  __shared__ SelectSmem sm;
  extern __shared__ __align__(16) uint8_t flat_dyn[];
  TwoPassSmem& tp = *reinterpret_cast<TwoPassSmem*>(flat_dyn);
  const int64_t r = row0 + blockIdx.x;
  const float* row = scores + static_cast<int64_t>(blockIdx.x) * ld;
  const int n = max(0, min(n_visible[r], L));
  int32_t* oi = out_idx + r * top_k;
  float* os = out_score ? out_score + r * top_k : nullptr;
  auto emit = [&](uint32_t slot, int i, uint32_t key) {
    oi[slot] = i;
    if (os) os[slot] = key_float(key);
  };
  auto key_at = [&](int i) { return float_key(__ldcg(row + i)); };
  uint32_t nv = static_cast<uint32_t>(n);
  bool done = false;
  if (minmax != nullptr && n > top_k) {
    // vectorised two passes (boundary bins up to 256 keys), then the general
    // two passes (up to kTwoPassCap), then the radix select
    done = two_pass_topk_rows<decltype(emit), CtaGroup>(row, n, static_cast<uint32_t>(top_k), emit, sm, tp.key,
                                                         tp.pos, &tp.count, 256, minmax[2 * blockIdx.x],
                                                         minmax[2 * blockIdx.x + 1]);
    if (!done)
      done = two_pass_topk<decltype(key_at), decltype(emit), CtaGroup>(
          key_at, n, static_cast<uint32_t>(top_k), emit, sm, tp.key, tp.pos, &tp.count, kTwoPassCap,
          minmax[2 * blockIdx.x], minmax[2 * blockIdx.x + 1]);
  }
  if (!done) nv = block_topk(key_at, n, static_cast<uint32_t>(top_k), emit, sm);
  for (int i = static_cast<int>(nv) + threadIdx.x; i < top_k; i += blockDim.x) {
    oi[i] = -1;
    if (os) os[i] = -__int_as_float(0x7f800000);
  }
}

// (smallest, largest) ordering-key pairs start empty.
__global__ void init_minmax_kernel(uint32_t* minmax, int64_t rows) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < rows;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    minmax[2 * i] = 0xFFFFFFFFu;
    minmax[2 * i + 1] = 0u;
  }
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
  block_topk(key_at, c, static_cast<uint32_t>(top_m - 1), emit, sm);
}

// The same selection with one warp per row, for rows of at most 32 * KPL
// block scores: each lane keeps its KPL keys (positions lane, lane + 32, ...)
// in registers; the (m-1)-th largest key T is found bit by bit from the top,
// each step counting the keys >= the candidate value across the warp; keys
// above T are emitted by ballot, then the lowest positions among the keys
// equal to T fill the remaining places.
template <int KPL>
__global__ void __launch_bounds__(256) block_select_warp_kernel(
    const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_visible, int64_t row0,
    int64_t nrows, int L, int block_size, int top_m, int32_t* __restrict__ out_idx) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t lr = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5; lr < nrows; lr += warps) {
    const int64_t r = row0 + lr;
    const float* row = scores + lr * ld;
    const int n = max(0, min(__ldg(n_visible + r), L));
    const int c = n > 0 ? (n - 1) / block_size : -1;
    int32_t* oi = out_idx + r * top_m;
    if (c + 1 <= top_m) {                    // every visible block (or none)
      for (int i = lane; i < top_m; i += 32) oi[i] = i <= c ? i : -1;
      continue;
    }
    if (lane == 0) oi[0] = c;
    const uint32_t k = static_cast<uint32_t>(top_m - 1);
    if (k == 0) continue;
    uint32_t key[KPL];
    uint32_t kmax = 0u, kmin = 0xFFFFFFFFu;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const int i = lane + 32 * j;
      key[j] = i < c ? float_key(__ldg(row + i)) : 0u;
      if (i < c) { kmax = max(kmax, key[j]); kmin = min(kmin, key[j]); }
    }
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    // bits above the highest one where kmin and kmax differ are common to all keys
    const int top_bit = kmin == kmax ? -1 : 31 - __clz(kmin ^ kmax);
    uint32_t T = top_bit < 0 ? kmax : (kmax & ~((2u << top_bit) - 1u));
    for (int bit = top_bit; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      uint32_t cnt = 0;
#pragma unroll
      for (int j = 0; j < KPL; ++j) cnt += key[j] >= cand ? 1u : 0u;
      if (__reduce_add_sync(0xffffffffu, cnt) >= k) T = cand;
    }
    // T is the k-th largest key: emit the keys above it, then the lowest
    // positions among those equal to it
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t base = 1;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const uint32_t ball = __ballot_sync(0xffffffffu, key[j] > T);
      if (key[j] > T) oi[base + __popc(ball & lt)] = lane + 32 * j;
      base += __popc(ball);
    }
    const uint32_t need = k + 1 - base;      // places left for keys equal to T
    uint32_t seen = 0;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
      const uint32_t ball = __ballot_sync(0xffffffffu, key[j] == T && key[j] != 0u);
      const uint32_t rank = seen + __popc(ball & lt);
      if (key[j] == T && key[j] != 0u && rank < need) oi[base + rank] = lane + 32 * j;
      seen += __popc(ball);
    }
  }
}

}  // namespace hisa

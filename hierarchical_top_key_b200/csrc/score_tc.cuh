// score_tc.cuh - tensor-core (tcgen05) dense causal indexer scoring for the
// flat DSA indexer and the HISA coarse stage.
//
// One MMA tile computes D[s, (t,h)] = k[s,:] . q[t,h,:] for 128 keys s (the
// A operand, M = 128) against a group of G queries x H heads (the B operand,
// N = G*H = 256), K = head_dim, accumulating in fp32 in TMEM.  The epilogue
// reduces over heads inside each thread (TMEM lane = key), so the indexer
// score I[t,s] = sum_h w[t,h] * max(D[s,(t,h)], 0) costs one max and one FMA
// per accumulator element and no cross-thread traffic; E4M3 scales are applied
// to the reduced score.  Scores are written as fp32 rows (one per query) for
// the row-wise top-k that follows; the [queries, heads, keys] tensor never
// exists outside TMEM.
//
// Persistent, warp-specialised CTA (one per SM):
//   warp 10     unit set-up: visibility, weights and scales of each work unit
//               into a ring of four shared-memory slots, ahead of the others
//   warp 0      TMA producer: q group (one or two buffers) and key tiles (ring)
//   warp 1      TMEM owner and MMA issuer (one thread)
//   warps 2..9  epilogue: TMEM -> registers -> weighted ReLU sum -> global
// Two TMEM accumulators (2 x 256 columns) let the MMA of tile i+1 overlap the
// epilogue of tile i.  Work units are (query group, chunk of key tiles) in a
// static schedule; the set-up warp publishes the non-empty ones in order and
// ends the ring with an empty unit.  Units with few key tiles (the coarse
// stage has one or two per query group) are then no longer paced by global
// loads in the producer, the issuer and the epilogue.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace hisa {

constexpr int kDenseTileM = 128;
constexpr int kDenseN = 256;
constexpr int kDenseEpiWarps = 8;
constexpr int kDenseSetupWarp = 2 + kDenseEpiWarps;
constexpr int kDenseThreads = 32 * (kDenseSetupWarp + 1);
constexpr int kDenseSlots = 4;
constexpr int kDenseMaxG = 16;            // queries per group (H >= 16)

// One published work unit.  ntiles == 0 ends the ring.
struct alignas(16) DenseSlot {
  int b, t0, nq, tile0, ntiles, pad0, pad1, pad2;
  int vis[kDenseMaxG];                    // visible key rows of each query of the group
  float qsc[kDenseMaxG];                  // E4M3 q scales (1 otherwise)
  uint32_t thr[kDenseMaxG];               // compaction thresholds (ordering keys)
  float w[kDenseN];                       // [G][H] head weights (0 past the last query)
};

struct DenseParams {
  int Q, H, d, L;           // L: key rows per sequence (keys, or pooled blocks)
  int G;                    // queries per group (kDenseN / H)
  int groups_per_seq;
  int block_div;            // 0: flat (vis = n); > 0: coarse (vis = (n-1)/block_div)
  int vis_stride;           // > 1: the key rows are every vis_stride-th key (vis = ceil(n / vis_stride))
  int kc_tiles;             // key tiles per work unit
  int max_chunks;           // units per group
  int stages;               // key-tile ring depth (<= 8)
  int q_bufs;               // q group buffers (1 or 2)
  int64_t gg0;              // first (sequence, group) handled by this launch
  int ngroups;
  int64_t row0;             // output row of query (b, t) is b*Q + t - row0
  const float* w;
  const int32_t* n_visible;
  const float* q_scale;
  const float* k_scale;
  float* out;
  int64_t ld;
  uint32_t* minmax;         // nullable: per output row, (min, max) ordering key written
  int64_t ksc_ld;           // E4M3 key scales: key row s of sequence b has scale k_scale[b*ksc_ld + s*ksc_step]
  int ksc_step;
  // Compaction (thresh != nullptr): instead of score rows, each output row r
  // receives the (key row, ordering key) pairs whose key is >= thresh[r],
  // appended at pairs[r*cap ...] in any order; counts[r] counts them all
  // (beyond cap the pairs are dropped but still counted).
  const uint32_t* thresh;
  uint2* pairs;
  uint32_t* counts;
  int cap;
};

struct DenseUnit {
  int b, t0, nq, tile0, ntiles;
};

__device__ __forceinline__ int dense_vis(const DenseParams& p, int n) {
  int v = p.block_div > 0 ? (n > 0 ? (n - 1) / p.block_div : 0) : n;
  if (p.vis_stride > 1) v = n > 0 ? (n + p.vis_stride - 1) / p.vis_stride : 0;
  return max(0, min(v, p.L));
}

// Unit u of the schedule: groups in descending order (longest causal
// prefixes first), then chunks of kc_tiles key tiles.

// Snake order over rounds of gridDim.x units balances the causal triangle.
__device__ __forceinline__ int64_t dense_unit_index(int64_t round) {
  const int64_t base = round * gridDim.x;
  return base + ((round & 1) ? (gridDim.x - 1 - blockIdx.x) : blockIdx.x);
}

template <int DT, int H>
__global__ void __launch_bounds__(kDenseThreads, 1) dense_score_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap, const DenseParams p) {
  using namespace sm100;
  constexpr int G = kDenseN / H;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int row_bytes = p.d * Elem<DT>::bytes;           // 128 or 256
  const int panels = row_bytes / 128;
  const int panel_elems = 128 / Elem<DT>::bytes;
  const uint32_t q_bytes = kDenseN * row_bytes;          // per q buffer
  const uint32_t k_bytes = kDenseTileM * row_bytes;      // per key stage
  uint8_t* q_buf = smem;                                 // [q_bufs][panels][256][128B]
  uint8_t* k_buf = smem + p.q_bufs * q_bytes;            // [stages][panels][128][128B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(k_buf + p.stages * k_bytes);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + p.stages;
  uint64_t* q_full = bars + 2 * p.stages;                // [2]
  uint64_t* q_empty = q_full + 2;                        // [2]
  uint64_t* acc_full = q_empty + 2;                      // [2]
  uint64_t* acc_empty = acc_full + 2;                    // [2]
  uint64_t* unit_full = acc_empty + 2;                   // [kDenseSlots]
  uint64_t* unit_empty = unit_full + kDenseSlots;        // [kDenseSlots]
  uint64_t* drain = unit_empty + kDenseSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  DenseSlot* slots = reinterpret_cast<DenseSlot*>((reinterpret_cast<uintptr_t>(tmem_slot + 2) + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) { mbar_init(k_full + s, 1); mbar_init(k_empty + s, 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1); mbar_init(q_empty + i, 1);
      mbar_init(acc_full + i, 1); mbar_init(acc_empty + i, kDenseEpiWarps);
    }
    for (int i = 0; i < kDenseSlots; ++i) { mbar_init(unit_full + i, 1); mbar_init(unit_empty + i, kDenseEpiWarps); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  if (warp == 0 && lane == 0) { tma_prefetch_desc(&qmap); tma_prefetch_desc(&kmap); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int64_t total_units = static_cast<int64_t>(p.ngroups) * p.max_chunks;

  if (warp == kDenseSetupWarp) {
    // ------------------------------------------------------------ unit set-up
    int un = 0;
    bool ok = true;
    for (int64_t r = 0; ok && r * gridDim.x < total_units; ++r) {
      const int64_t u = dense_unit_index(r);
      if (u >= total_units) continue;
      const int64_t gg = p.gg0 + (p.ngroups - 1 - u / p.max_chunks);
      const int chunk = static_cast<int>(u % p.max_chunks);
      const int b = static_cast<int>(gg / p.groups_per_seq);
      const int t0 = static_cast<int>(gg % p.groups_per_seq) * p.G;
      const int nq = min(p.G, p.Q - t0);
      const int64_t qrow0 = static_cast<int64_t>(b) * p.Q + t0;
      const int vis = lane < nq ? dense_vis(p, __ldg(p.n_visible + qrow0 + lane)) : 0;
      const int vmax = __reduce_max_sync(0xffffffffu, vis);
      const int tile0 = chunk * p.kc_tiles;
      const int ntiles = min(p.kc_tiles, (vmax + kDenseTileM - 1) / kDenseTileM - tile0);
      if (ntiles <= 0) continue;
      const int sl = un % kDenseSlots;
      int okl = 1;
      if (lane == 0) okl = mbar_wait(unit_empty + sl, ((un / kDenseSlots) & 1) ^ 1, abort_flag) ? 1 : 0;
      if (!(ok = __shfl_sync(0xffffffffu, okl, 0) != 0)) break;
      DenseSlot& S = slots[sl];
      if (lane == 0) { S.b = b; S.t0 = t0; S.nq = nq; S.tile0 = tile0; S.ntiles = ntiles; }
      if (lane < kDenseMaxG) {
        S.vis[lane] = vis;
        S.qsc[lane] = (DT == DT_E4M3 && lane < nq) ? __ldg(p.q_scale + qrow0 + lane) : 1.f;
        S.thr[lane] = (p.thresh != nullptr && lane < nq) ? __ldg(p.thresh + qrow0 + lane - p.row0) : 0u;
      }
      for (int i = lane; i < G * H; i += 32) {
        const int j = i / H;
        S.w[i] = j < nq ? __ldg(p.w + (qrow0 + j) * p.H + (i % H)) : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(unit_full + sl);
      ++un;
    }
    if (ok) {   // the empty unit that ends the ring
      const int sl = un % kDenseSlots;
      int okl = 1;
      if (lane == 0) okl = mbar_wait(unit_empty + sl, ((un / kDenseSlots) & 1) ^ 1, abort_flag) ? 1 : 0;
      if (__shfl_sync(0xffffffffu, okl, 0) != 0 && lane == 0) {
        slots[sl].ntiles = 0;
        mbar_arrive(unit_full + sl);
      }
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int st = 0;
      uint32_t kph = 0;
      int un = 0;
      int8_t last_ph[8];
      for (int s = 0; s < 8; ++s) last_ph[s] = -1;
      int8_t last_qph[2] = {-1, -1};
      bool ok = true;
      while (ok) {
        const int sl = un % kDenseSlots;
        if (!(ok = mbar_wait(unit_full + sl, (un / kDenseSlots) & 1, abort_flag))) break;
        DenseUnit U;
        U.b = slots[sl].b; U.t0 = slots[sl].t0; U.tile0 = slots[sl].tile0; U.ntiles = slots[sl].ntiles;
        if (U.ntiles == 0) break;
        const int qb = un % p.q_bufs;
        if (!(ok = mbar_wait(q_empty + qb, ((un / p.q_bufs) & 1) ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(q_full + qb, q_bytes);
        const int qrow = (U.b * p.Q + U.t0) * p.H;
        for (int pn = 0; pn < panels; ++pn)
          tma_load_2d(q_buf + qb * q_bytes + pn * (kDenseN * 128), &qmap, q_full + qb, pn * panel_elems, qrow);
        last_qph[qb] = static_cast<int8_t>((un / p.q_bufs) & 1);
        for (int i = 0; i < U.ntiles; ++i) {
          if (!(ok = mbar_wait(k_empty + st, kph ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(k_full + st, k_bytes);
          const int krow = U.b * p.L + (U.tile0 + i) * kDenseTileM;
          for (int pn = 0; pn < panels; ++pn)
            tma_load_2d(k_buf + st * k_bytes + pn * (kDenseTileM * 128), &kmap, k_full + st, pn * panel_elems, krow);
          last_ph[st] = static_cast<int8_t>(kph);
          if (++st == p.stages) { st = 0; kph ^= 1; }
        }
        ++un;
      }
      if (!ok) {   // drain the copies this thread issued before leaving
        for (int s = 0; s < p.stages; ++s)
          if (last_ph[s] >= 0) mbar_drain(k_full + s, static_cast<uint32_t>(last_ph[s]));
        for (int i = 0; i < 2; ++i)
          if (last_qph[i] >= 0) mbar_drain(q_full + i, static_cast<uint32_t>(last_qph[i]));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc(kDenseTileM, kDenseN, DT == DT_BF16 ? 1u : 0u);
      const int ksteps = row_bytes / 32;       // 32 bytes of K per MMA (16 bf16 / 32 e4m3)
      int st = 0, ab = 0;
      uint32_t kph = 0, aph = 0;
      int un = 0;
      bool ok = true;
      while (ok) {
        const int sl = un % kDenseSlots;
        if (!(ok = mbar_wait(unit_full + sl, (un / kDenseSlots) & 1, abort_flag))) break;
        DenseUnit U;
        U.ntiles = slots[sl].ntiles;
        if (U.ntiles == 0) break;
        const int qb = un % p.q_bufs;
        if (!(ok = mbar_wait(q_full + qb, (un / p.q_bufs) & 1, abort_flag))) break;
        tc_fence_after();
        const uint64_t q_desc = desc_k_sw128(smem_u32(q_buf + qb * q_bytes));
        for (int i = 0; i < U.ntiles; ++i) {
          if (!(ok = mbar_wait(acc_empty + ab, aph ^ 1, abort_flag))) break;
          if (!(ok = mbar_wait(k_full + st, kph, abort_flag))) break;
          tc_fence_after();
          const uint64_t k_desc = desc_k_sw128(smem_u32(k_buf + st * k_bytes));
          const uint32_t d_tmem = tmem_base + ab * kDenseN;
          if (ksteps == 8) mma_tile_sw128<DT, 8, kDenseTileM, kDenseN>(d_tmem, k_desc, q_desc, idesc);
          else mma_tile_sw128<DT, 4, kDenseTileM, kDenseN>(d_tmem, k_desc, q_desc, idesc);
          mma_commit(k_empty + st);
          mma_commit(acc_full + ab);
          if (++st == p.stages) { st = 0; kph ^= 1; }
          ab ^= 1;
          aph ^= ab == 0 ? 1u : 0u;
        }
        if (ok) mma_commit(q_empty + qb);
        ++un;
      }
      mma_commit(drain);
      mbar_drain(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // The unit's weights, visibility and scales come from its slot; lane 0
    // alone waits on the barriers, and each warp releases the slot when it
    // is done with the unit.
    const int e = warp - 2;
    const int quarter = warp & 3;                 // TMEM lanes this warp may access
    const int half = e >> 2;                      // which half of the group's queries
    constexpr int QPT = G / 2;                    // queries per thread
    int64_t tc = 0;
    int un = 0;
    bool ok = true;
    while (ok) {
      const int sl = un % kDenseSlots;
      int okl = 1;
      if (lane == 0) okl = mbar_wait(unit_full + sl, (un / kDenseSlots) & 1, abort_flag) ? 1 : 0;
      if (!(ok = __shfl_sync(0xffffffffu, okl, 0) != 0)) break;
      const DenseSlot& S = slots[sl];
      DenseUnit U;
      U.b = S.b; U.t0 = S.t0; U.nq = S.nq; U.tile0 = S.tile0; U.ntiles = S.ntiles;
      if (U.ntiles == 0) break;
      const int64_t qrow0 = static_cast<int64_t>(U.b) * p.Q + U.t0;
      const float* w_w = S.w + half * QPT * H;
      const float* qsc_w = S.qsc + half * QPT;
      const int* vis_w = S.vis + half * QPT;
      const uint32_t* thr_w = S.thr + half * QPT;
      uint32_t kmin[QPT], kmax[QPT];
#pragma unroll
      for (int jq = 0; jq < QPT; ++jq) { kmin[jq] = 0xFFFFFFFFu; kmax[jq] = 0u; }
      // compaction: a tile's appends are reserved (lane 0's atomic) while the
      // tile is scored and written out one tile later, so the atomic's latency
      // hides behind the next tile's work
      uint32_t pball[QPT], pkey[QPT], pbase[QPT];
      int ps = 0;
#pragma unroll
      for (int jq = 0; jq < QPT; ++jq) pball[jq] = 0u;
      auto flush = [&]() {
#pragma unroll
        for (int jq = 0; jq < QPT; ++jq) {
          if (pball[jq] == 0u) continue;
          const uint32_t slot = __shfl_sync(0xffffffffu, pbase[jq], 0) + __popc(pball[jq] & ((1u << lane) - 1u));
          if (((pball[jq] >> lane) & 1u) && slot < static_cast<uint32_t>(p.cap))
            p.pairs[(qrow0 + half * QPT + jq - p.row0) * p.cap + slot] = make_uint2(ps, pkey[jq]);
          pball[jq] = 0u;
        }
      };
      for (int i = 0; i < U.ntiles; ++i, ++tc) {
        const int ab = static_cast<int>(tc & 1);
        int okl = 1;
        if (lane == 0) okl = mbar_wait(acc_full + ab, static_cast<uint32_t>((tc >> 1) & 1), abort_flag) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
        if (!ok) break;
        tc_fence_after();
        const int s = (U.tile0 + i) * kDenseTileM + quarter * 32 + lane;
        float ksc = 1.f;
        if (DT == DT_E4M3 && s < p.L)
          ksc = __ldg(p.k_scale + static_cast<int64_t>(U.b) * p.ksc_ld + static_cast<int64_t>(s) * p.ksc_step);
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + ab * kDenseN;
        uint32_t nball[QPT], nkey[QPT], nbase[QPT];
#pragma unroll
        for (int jq = 0; jq < QPT; ++jq) {
          const int j = half * QPT + jq;
          const float* wq = w_w + jq * H;
          float acc = 0.f;
          if (H >= 32) {
            // the query's H columns in one batch of TMEM loads, one wait, then
            // four independent accumulation chains over float4 weights
            uint32_t v[H];
#pragma unroll
            for (int c0 = 0; c0 < H; c0 += 32)
              tmem_ld32(t_row + j * H + c0, *reinterpret_cast<uint32_t(*)[32]>(v + c0));
            tmem_wait_ld();
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
            const float4* w4 = reinterpret_cast<const float4*>(wq);
#pragma unroll
            for (int e = 0; e < H / 4; ++e) {
              const float4 wv = w4[e];
              a4[0] = fmaf(wv.x, fmaxf(__uint_as_float(v[4 * e + 0]), 0.f), a4[0]);
              a4[1] = fmaf(wv.y, fmaxf(__uint_as_float(v[4 * e + 1]), 0.f), a4[1]);
              a4[2] = fmaf(wv.z, fmaxf(__uint_as_float(v[4 * e + 2]), 0.f), a4[2]);
              a4[3] = fmaf(wv.w, fmaxf(__uint_as_float(v[4 * e + 3]), 0.f), a4[3]);
            }
            acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
          } else {
            uint32_t v[16];
            tmem_ld16(t_row + j * H, v);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) acc = fmaf(wq[c], fmaxf(__uint_as_float(v[c]), 0.f), acc);
          }
          if (DT == DT_E4M3) acc *= qsc_w[jq] * ksc;
          const uint32_t key = float_key(acc);
          if (p.thresh != nullptr) {
            // warp-aggregated append of this tile's keys that pass the row's threshold
            const bool take = s < vis_w[jq] && key >= thr_w[jq] && key != 0u;
            nball[jq] = __ballot_sync(0xffffffffu, take);
            nkey[jq] = key;
            nbase[jq] = (lane == 0 && nball[jq] != 0u)
                            ? atomicAdd(p.counts + (qrow0 + j - p.row0), static_cast<uint32_t>(__popc(nball[jq])))
                            : 0u;
          } else if (s < vis_w[jq]) {
            p.out[(qrow0 + j - p.row0) * p.ld + s] = acc;
            kmin[jq] = min(kmin[jq], key);
            kmax[jq] = max(kmax[jq], key);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + ab);
        if (p.thresh != nullptr) {
          flush();          // the previous tile's appends, reserved one tile ago
#pragma unroll
          for (int jq = 0; jq < QPT; ++jq) { pball[jq] = nball[jq]; pkey[jq] = nkey[jq]; pbase[jq] = nbase[jq]; }
          ps = s;
        }
      }
      if (p.thresh != nullptr) flush();
      if (ok && p.minmax != nullptr) {
#pragma unroll
        for (int jq = 0; jq < QPT; ++jq) {
          const uint32_t lo = __reduce_min_sync(0xffffffffu, kmin[jq]);
          const uint32_t hi = __reduce_max_sync(0xffffffffu, kmax[jq]);
          const int j = half * QPT + jq;
          if (lane == 0 && j < U.nq && hi != 0u) {
            atomicMin(p.minmax + 2 * (qrow0 + j - p.row0), lo);
            atomicMax(p.minmax + 2 * (qrow0 + j - p.row0) + 1, hi);
          }
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(unit_empty + sl);
      ++un;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// Bytes of dynamic shared memory the dense kernel needs.
inline size_t dense_smem_bytes(int row_bytes, int stages, int q_bufs) {
  return 1024 /*alignment slack*/ + q_bufs * static_cast<size_t>(kDenseN) * row_bytes +
         static_cast<size_t>(stages) * kDenseTileM * row_bytes + 8 * (2 * stages + 9 + 2 * kDenseSlots) + 8 + 16 +
         kDenseSlots * sizeof(DenseSlot);
}

}  // namespace hisa

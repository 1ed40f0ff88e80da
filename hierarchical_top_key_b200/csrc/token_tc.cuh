// token_tc.cuh - fused HISA refinement stage on tensor cores.
//
// For each query t: the keys of its retained blocks are gathered by TMA
// (each block is a contiguous run of B key rows, so one tile load per block),
// scored against q[t] with tcgen05 (M = 128 candidate keys, N = H heads,
// K = head_dim, fp32 accumulators in TMEM), reduced over heads with the
// weighted ReLU in-thread, kept in shared memory as ordering keys, and the
// top-k is selected on chip.  Candidate scores never reach global memory.
//
// Persistent, warp-specialised CTA (one per SM), queries processed as a
// pipeline of jobs:
//   warp 0       job set-up (whole warp: read, filter, dedupe and sort the
//                block list; stage w[t]), running up to four jobs ahead
//   warps 1, 2   MMA issuers, alternate tiles (warp 1 owns TMEM).  An M=128,
//                N=64 MMA is bound by per-thread issue, not by the tensor
//                core, so two issuers nearly double the rate.
//   warp 3       TMA issuer: q[t] and one tile load per retained block
//   warps 4..11  scorers, two groups of four on alternate tiles: TMEM ->
//                weighted ReLU sum -> candidate keys in smem, plus each
//                job's key range and valid count
//   warps 12..15 selector: histogram + counting-scan top-k over the candidate keys
// Rings: job slots (4), q buffers (2), key stages, TMEM accumulators (8 x H
// columns), candidate buffers (2).  Blocks are sorted ascending so candidate
// position order is key order, which makes ties resolve to the lower key.
#pragma once
#include "common.cuh"
#include "select.cuh"
#include "sm100.cuh"

namespace hisa {

constexpr int kTokTileM = 128;
constexpr int kTokJobs = 4;
constexpr int kTokAcc = 8;                        // TMEM accumulators (multiple of the issuer count)
constexpr int kTokIssuers = 2;                    // MMA issuer warps 1..kTokIssuers
constexpr int kTokTmaWarp = 1 + kTokIssuers;
constexpr int kTokScorerBase = kTokTmaWarp + 1;   // first scorer warp
constexpr int kTokScorerWarps = 4;                // per group; one warp per TMEM lane quarter
constexpr int kTokScoreGroups = 2;
constexpr int kTokSelectWarps = 4;
constexpr int kTokSelectBase = 32 * (kTokScorerBase + kTokScorerWarps * kTokScoreGroups);
constexpr int kTokThreads = kTokSelectBase + 32 * kTokSelectWarps;
constexpr int kTokBinCap = 256;                   // boundary-bin buffer of the selector
constexpr int kTokMaxBlocks = 256;                // top_m limit
constexpr int kTokMaxBitmapWords = 256;           // blocks per sequence limit / 32

struct TokenParams {
  int64_t rows;            // batch * Q
  int Q, H, d, L, B, top_m, top_k;
  int nb;                  // ceil(L / B)
  int max_cand;            // top_m * B rounded up to whole tiles
  int stages;
  const float* w;
  const int32_t* n_visible;
  const int32_t* block_idx;
  const float* q_scale;
  const float* k_scale;
  int32_t* out_idx;        // [rows * parts, top_k]
  float* out_score;
  int parts;                // > 1: each query's retained blocks split over `parts` jobs, each writing its own top-k
  const int32_t* pages;     // non-NULL: block j of sequence b is page pages[b * nb + j] of the keys ([num_pages, B, d])
  int num_pages;
  int k3d;                  // 1: the key map is 3D (64 elements, rows, 2 panels of 128 bytes): a block of 128
                            //    rows is one load; 0: one 2D load per block and panel
};

struct alignas(16) TokJob {
  int64_t row;
  int64_t orow;            // output row: row * parts + part
  int b, n, nblk, ntiles;
  float qsc;
  uint32_t kmin, kmax, nvalid;     // filled by the scorers for the selector
  alignas(16) float w[64];
  int blk[kTokMaxBlocks];
  int page[kTokMaxBlocks];         // with paged keys: the page of blk[i]
};

__device__ __forceinline__ int64_t tok_job_id(const TokenParams& p, int64_t j) {
  // largest prefixes first; job id = row * parts + part
  return p.rows * p.parts - 1 - (static_cast<int64_t>(blockIdx.x) + j * gridDim.x);
}

template <int DT, int H>
__global__ void __launch_bounds__(kTokThreads, 1) token_tc_kernel(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap, const TokenParams p) {
  using namespace sm100;
  using SelGrp = WarpRange<kTokSelectBase, 32 * kTokSelectWarps, 2>;
  static_assert(kTokAcc % kTokIssuers == 0 && kTokAcc % kTokScoreGroups == 0, "tile ownership");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int row_bytes = p.d * Elem<DT>::bytes;
  const int panels = row_bytes / 128;
  const int panel_elems = 128 / Elem<DT>::bytes;
  const uint32_t q_bytes = H * row_bytes;
  const uint32_t k_bytes = kTokTileM * row_bytes;
  const int blocks_per_tile = kTokTileM / p.B;
  uint8_t* q_buf = smem;                                         // [2][panels][H][128B]
  uint8_t* k_buf = q_buf + 2 * q_bytes;                          // [stages][panels][128][128B]
  uint32_t* cand = reinterpret_cast<uint32_t*>(k_buf + p.stages * k_bytes);   // [2][max_cand]
  TokJob* jobs = reinterpret_cast<TokJob*>(cand + 2 * p.max_cand);            // [kTokJobs]
  SelectSmem* sel = reinterpret_cast<SelectSmem*>(jobs + kTokJobs);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(sel + 1);                     // [kTokMaxBitmapWords]
  uint32_t* bin_key = bitmap + kTokMaxBitmapWords;                             // [kTokBinCap]
  int32_t* bin_pos = reinterpret_cast<int32_t*>(bin_key + kTokBinCap);         // [kTokBinCap]
  uint32_t* bin_count = reinterpret_cast<uint32_t*>(bin_pos + kTokBinCap);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uintptr_t>(bin_count + 1) + 7 & ~uintptr_t(7));
  // Key stage s holding tile g (the CTA's g-th tile) completes on
  // k_full[g % kTokIssuers][s]: consecutive tiles of a stage can go to
  // different issuers, and a barrier waited on by more than one of them could
  // let a parity wait pass on an older phase; per issuer, each barrier's uses
  // are in that issuer's own order.  Both sides keep each barrier's phase as
  // one bit of a register mask.
  uint64_t* k_full = bars;                               // [kTokIssuers][stages]
  uint64_t* k_empty = k_full + kTokIssuers * p.stages;   // [stages]
  uint64_t* q_full = k_empty + p.stages;          // [2]
  uint64_t* q_empty = q_full + 2;                 // [2]
  uint64_t* acc_full = q_empty + 2;               // [kTokAcc]
  uint64_t* acc_empty = acc_full + kTokAcc;       // [kTokAcc]
  uint64_t* job_full = acc_empty + kTokAcc;       // [kTokJobs]
  uint64_t* job_empty = job_full + kTokJobs;      // [kTokJobs]
  uint64_t* cand_full = job_empty + kTokJobs;     // [2]
  uint64_t* cand_empty = cand_full + 2;           // [2]
  uint64_t* drain = cand_empty + 2;                // [kTokIssuers]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + kTokIssuers);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* sel_ok = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTokIssuers * p.stages; ++s) mbar_init(k_full + s, 1);
    for (int s = 0; s < p.stages; ++s) mbar_init(k_empty + s, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1); mbar_init(q_empty + i, kTokIssuers);
      mbar_init(cand_full + i, kTokScorerWarps * kTokScoreGroups); mbar_init(cand_empty + i, 1);
    }
    for (int i = 0; i < kTokAcc; ++i) { mbar_init(acc_full + i, 1); mbar_init(acc_empty + i, kTokScorerWarps); }
    for (int i = 0; i < kTokJobs; ++i) { mbar_init(job_full + i, 1); mbar_init(job_empty + i, 1); }
    for (int i = 0; i < kTokIssuers; ++i) mbar_init(drain + i, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTokAcc * H < 32 ? 32 : kTokAcc * H);
  if (warp == 0 && lane == 0) { tma_prefetch_desc(&qmap); tma_prefetch_desc(&kmap); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int64_t total_jobs = p.rows * p.parts;
  const int64_t njobs = total_jobs > blockIdx.x ? (total_jobs - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ job set-up
    bool ok = true;
    for (int64_t j = 0; j < njobs; ++j) {
      const int slot = static_cast<int>(j % kTokJobs);
      int okl = 1;
      if (lane == 0) okl = mbar_wait(job_empty + slot, static_cast<uint32_t>(((j / kTokJobs) & 1) ^ 1), abort_flag);
      if (!(ok = __shfl_sync(0xffffffffu, okl, 0) != 0)) break;
      TokJob& J = jobs[slot];
      const int64_t jid = tok_job_id(p, j);
      const int64_t row = jid / p.parts;
      const int part = static_cast<int>(jid % p.parts);
      const int b = static_cast<int>(row / p.Q);
      // every global read of the job at once: visibility, block list, weights
      const int n_raw = __ldg(p.n_visible + row);
      constexpr int KW = kTokMaxBlocks / 32;
      int x[KW];
#pragma unroll
      for (int k = 0; k < KW; ++k) {
        const int i = lane + 32 * k;
        x[k] = (32 * k < p.top_m && i < p.top_m) ? __ldg(p.block_idx + row * p.top_m + i) : -1;
      }
      const float w0 = lane < p.H ? __ldg(p.w + row * p.H + lane) : 0.f;
      const float w1 = lane + 32 < p.H ? __ldg(p.w + row * p.H + lane + 32) : 0.f;
      const float qsc = (DT == DT_E4M3 && lane == 0) ? __ldg(p.q_scale + row) : 1.f;
      const int n = max(0, min(n_raw, p.L));
      // retained blocks -> bitmap (repeats collapse, invalid entries dropped),
      // then the set bits are compacted in ascending order
      const int nvis_blocks = min(p.nb, (n + p.B - 1) / p.B);   // blocks holding a visible key
      const int nwords = (nvis_blocks + 31) >> 5;
      for (int wi = lane; wi < nwords; wi += 32) bitmap[wi] = 0u;
      __syncwarp();
#pragma unroll
      for (int k = 0; k < KW; ++k) {
        bool keep = x[k] >= 0 && x[k] < nvis_blocks;
        if (keep && p.pages) {   // a block whose page entry is out of range is dropped and reported
          const int pg = __ldg(p.pages + static_cast<int64_t>(b) * p.nb + x[k]);
          if (pg < 0 || pg >= p.num_pages) {
            keep = false;
            record_status(HISA_ERR_INVALID_ARG);
          }
        }
        if (keep) atomicOr(bitmap + (x[k] >> 5), 1u << (x[k] & 31));
      }
      __syncwarp();
      const int wpl = (nwords + 31) >> 5;                        // words per lane, in order
      int local = 0;
      for (int i = 0; i < wpl; ++i) {
        const int wi = lane * wpl + i;
        if (wi < nwords) local += __popc(bitmap[wi]);
      }
      int incl = local;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const int cnt_all = __shfl_sync(0xffffffffu, incl, 31);
      // this job's share of the blocks (all of them unless the query is split)
      const int lo = static_cast<int>((static_cast<int64_t>(cnt_all) * part) / p.parts);
      const int hi = static_cast<int>((static_cast<int64_t>(cnt_all) * (part + 1)) / p.parts);
      const int cnt = hi - lo;
      int pos = incl - local;
      for (int i = 0; i < wpl; ++i) {
        const int wi = lane * wpl + i;
        if (wi >= nwords) break;
        uint32_t bits = bitmap[wi];
        while (bits) {
          const int bit = __ffs(bits) - 1;
          bits &= bits - 1;
          if (pos >= lo && pos < hi) {
            J.blk[pos - lo] = (wi << 5) + bit;
            if (p.pages) J.page[pos - lo] = __ldg(p.pages + static_cast<int64_t>(b) * p.nb + (wi << 5) + bit);
          }
          ++pos;
        }
      }
      J.w[lane] = w0;
      J.w[lane + 32] = w1;
      if (lane == 0) {
        J.row = row;
        J.orow = jid;
        J.b = b;
        J.n = n;
        J.nblk = cnt;
        J.ntiles = (cnt * p.B + kTokTileM - 1) / kTokTileM;
        J.qsc = qsc;
        J.kmin = 0xFFFFFFFFu;
        J.kmax = 0u;
        J.nvalid = 0u;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(job_full + slot);
    }
  } else if (warp == kTokTmaWarp) {
    // ------------------------------------------------------------ TMA issue
    if (lane == 0) {
      int st = 0, gi = 0;                       // stage, issuer of the next tile
      uint32_t kph = 0, fph = 0;                // k_empty phase; k_full phases, one bit per barrier
      int8_t last_ph[8], last_bar[8];          // per stage: the last full barrier armed and its phase
      for (int i = 0; i < 8; ++i) last_ph[i] = -1;
      int8_t last_qph[2] = {-1, -1};
      bool ok = true;
      for (int64_t j = 0; ok && j < njobs; ++j) {
        const int slot = static_cast<int>(j % kTokJobs);
        if (!(ok = mbar_wait(job_full + slot, static_cast<uint32_t>((j / kTokJobs) & 1), abort_flag))) break;
        const TokJob& J = jobs[slot];
        const int qb = static_cast<int>(j & 1);
        const uint32_t qph = static_cast<uint32_t>((j >> 1) & 1);
        if (!(ok = mbar_wait(q_empty + qb, qph ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(q_full + qb, q_bytes);
        for (int pn = 0; pn < panels; ++pn)
          tma_load_2d(q_buf + qb * q_bytes + pn * (H * 128), &qmap, q_full + qb, pn * panel_elems,
                      static_cast<int>(J.row * p.H));
        last_qph[qb] = static_cast<int8_t>(qph);
        const int kb = J.b * p.L;
        for (int tl = 0; tl < J.ntiles; ++tl) {
          if (!(ok = mbar_wait(k_empty + st, kph ^ 1, abort_flag))) break;
          const int first = tl * blocks_per_tile;
          const int nblk_t = min(blocks_per_tile, J.nblk - first);
          const int kfi = gi * p.stages + st;
          uint64_t* kf = k_full + kfi;
          mbar_arrive_expect_tx(kf, static_cast<uint32_t>(nblk_t * p.B * row_bytes));
          for (int q = 0; q < nblk_t; ++q) {
            const int krow = p.pages ? J.page[first + q] * p.B : kb + J.blk[first + q] * p.B;
            if (p.k3d) {
              // both panels of the block in one instruction: the box is [panel][row][128 B],
              // the layout the panel loads below produce
              tma_load_3d(k_buf + st * k_bytes, &kmap, kf, 0, krow, 0);
            } else {
              for (int pn = 0; pn < panels; ++pn)
                tma_load_2d(k_buf + st * k_bytes + pn * (kTokTileM * 128) + q * p.B * 128, &kmap, kf,
                            pn * panel_elems, krow);
            }
          }
          last_ph[st] = static_cast<int8_t>((fph >> kfi) & 1u);
          last_bar[st] = static_cast<int8_t>(kfi);
          fph ^= 1u << kfi;
          if (++gi == kTokIssuers) gi = 0;
          if (++st == p.stages) { st = 0; kph ^= 1; }
        }
      }
      if (!ok) {   // drain the copies this thread issued before leaving
        for (int i = 0; i < p.stages; ++i)
          if (last_ph[i] >= 0) mbar_drain(k_full + last_bar[i], static_cast<uint32_t>(last_ph[i]));
        for (int i = 0; i < 2; ++i)
          if (last_qph[i] >= 0) mbar_drain(q_full + i, static_cast<uint32_t>(last_qph[i]));
      }
    }
  } else if (warp >= 1 && warp <= kTokIssuers) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      const int me = warp - 1;                        // this issuer takes tiles g with g % kTokIssuers == me
      constexpr uint32_t idesc = instr_desc(kTokTileM, H, DT == DT_BF16 ? 1u : 0u);
      const int ksteps = row_bytes / 32;
      int st = 0, ab = 0, g = 0;
      uint32_t aph = 0, fph = 0;               // fph: phases of this issuer's k_full barriers, one bit per stage
      bool ok = true;
      for (int64_t j = 0; ok && j < njobs; ++j) {
        const int slot = static_cast<int>(j % kTokJobs);
        if (!(ok = mbar_wait(job_full + slot, static_cast<uint32_t>((j / kTokJobs) & 1), abort_flag))) break;
        const int ntiles = jobs[slot].ntiles;
        const int qb = static_cast<int>(j & 1);
        if (!(ok = mbar_wait(q_full + qb, static_cast<uint32_t>((j >> 1) & 1), abort_flag))) break;
        tc_fence_after();
        const uint64_t q_desc = desc_k_sw128(smem_u32(q_buf + qb * q_bytes));
        for (int i = 0; i < ntiles; ++i) {
          if (g == me) {
            if (!(ok = mbar_wait(acc_empty + ab, aph ^ 1, abort_flag))) break;
            if (!(ok = mbar_wait(k_full + me * p.stages + st, (fph >> st) & 1u, abort_flag))) break;
            fph ^= 1u << st;
            tc_fence_after();
            const uint64_t k_desc = desc_k_sw128(smem_u32(k_buf + st * k_bytes));
            const uint32_t d_tmem = tmem_base + ab * H;
            if (ksteps == 8) mma_tile_sw128<DT, 8, kTokTileM, H>(d_tmem, k_desc, q_desc, idesc);
            else mma_tile_sw128<DT, 4, kTokTileM, H>(d_tmem, k_desc, q_desc, idesc);
            mma_commit(k_empty + st);
            mma_commit(acc_full + ab);
          }
          if (++g == kTokIssuers) g = 0;
          if (++st == p.stages) st = 0;
          if (++ab == kTokAcc) { ab = 0; aph ^= 1; }
        }
        if (ok) mma_commit(q_empty + qb);
      }
      mma_commit(drain + me);
      mbar_drain(drain + me, 0);
    }
  } else if (warp >= kTokScorerBase && warp < kTokScorerBase + kTokScorerWarps * kTokScoreGroups) {
    // ------------------------------------------------------------ scorers
    const int grp = (warp - kTokScorerBase) / kTokScorerWarps;   // takes tiles g with g % groups == grp
    const int quarter = warp & 3;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const int bshift = __ffs(p.B) - 1;
    int ab = 0, g = 0;
    uint32_t aph = 0;
    bool ok = true;
    for (int64_t j = 0; ok && j < njobs; ++j) {
      const int slot = static_cast<int>(j % kTokJobs);
      const int cb = static_cast<int>(j & 1);
      int okl = 1;
      if (lane == 0) {
        okl = mbar_wait(job_full + slot, static_cast<uint32_t>((j / kTokJobs) & 1), abort_flag) &&
              mbar_wait(cand_empty + cb, static_cast<uint32_t>(((j >> 1) & 1) ^ 1), abort_flag);
      }
      if (!(ok = __shfl_sync(0xffffffffu, okl, 0) != 0)) break;
      TokJob& J = jobs[slot];
      const int ntiles = J.ntiles;
      uint32_t* cj = cand + cb * p.max_cand;
      uint32_t lo = 0xFFFFFFFFu, hi = 0u, nv = 0u;
      for (int i = 0; i < ntiles; ++i) {
        if (g == grp) {
          if (lane == 0) okl = mbar_wait(acc_full + ab, aph, abort_flag);
          if (!(ok = __shfl_sync(0xffffffffu, okl, 0) != 0)) break;
          tc_fence_after();
          const int c = i * kTokTileM + quarter * 32 + lane;        // candidate position
          const int slot_b = c >> bshift;
          const int s = slot_b < J.nblk ? (J.blk[slot_b] << bshift) + (c & (p.B - 1)) : p.L;
          const bool valid = s < J.n;
          float ksc = 1.f;
          if (DT == DT_E4M3 && valid)
            ksc = __ldg(p.k_scale + (p.pages ? static_cast<int64_t>(J.page[slot_b]) * p.B + (c & (p.B - 1))
                                             : static_cast<int64_t>(J.b) * p.L + s));
          float acc = 0.f;
          if (H >= 32) {
            // 32 columns per TMEM load (32 registers live, not 64), four
            // independent accumulation chains over float4 weight reads
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
            const float4* w4 = reinterpret_cast<const float4*>(J.w);
#pragma unroll
            for (int c0 = 0; c0 < H; c0 += 32) {
              uint32_t v[32];
              tmem_ld32(t_lane + ab * H + c0, v);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float4 wv = w4[c0 / 4 + e];
                a4[0] = fmaf(wv.x, fmaxf(__uint_as_float(v[4 * e + 0]), 0.f), a4[0]);
                a4[1] = fmaf(wv.y, fmaxf(__uint_as_float(v[4 * e + 1]), 0.f), a4[1]);
                a4[2] = fmaf(wv.z, fmaxf(__uint_as_float(v[4 * e + 2]), 0.f), a4[2]);
                a4[3] = fmaf(wv.w, fmaxf(__uint_as_float(v[4 * e + 3]), 0.f), a4[3]);
              }
            }
            acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
          } else {
            uint32_t v[16];
            tmem_ld16(t_lane + ab * H, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) acc = fmaf(J.w[e], fmaxf(__uint_as_float(v[e]), 0.f), acc);
          }
          if (DT == DT_E4M3) acc *= J.qsc * ksc;
          const uint32_t key = valid ? float_key(acc) : 0u;
          cj[c] = key;
          if (valid) { lo = min(lo, key); hi = max(hi, key); ++nv; }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty + ab);
        }
        if (++g == kTokScoreGroups) g = 0;
        if (++ab == kTokAcc) { ab = 0; aph ^= 1; }
      }
      if (!ok) break;
      lo = __reduce_min_sync(0xffffffffu, lo);
      hi = __reduce_max_sync(0xffffffffu, hi);
      nv = __reduce_add_sync(0xffffffffu, nv);
      if (lane == 0 && nv > 0) {
        atomicMin(&J.kmin, lo);
        atomicMax(&J.kmax, hi);
        atomicAdd(&J.nvalid, nv);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(cand_full + cb);
    }
  } else {
    // ------------------------------------------------------------ selector
    const int stid = SelGrp::tid();
    for (int64_t j = 0; j < njobs; ++j) {
      const int slot = static_cast<int>(j % kTokJobs);
      const int cb = static_cast<int>(j & 1);
      if (stid == 0) *sel_ok = mbar_wait(cand_full + cb, static_cast<uint32_t>((j >> 1) & 1), abort_flag) ? 1 : 0;
      SelGrp::sync();
      if (!*sel_ok) break;
      const TokJob& J = jobs[slot];
      const uint32_t* cj = cand + cb * p.max_cand;
      const int ncand = J.ntiles * kTokTileM;
      int32_t* oi = p.out_idx + J.orow * p.top_k;
      float* os = p.out_score ? p.out_score + J.orow * p.top_k : nullptr;
      const int bshift = __ffs(p.B) - 1;
      // indices are staged in shared memory (the selection's histogram space,
      // free once offsets are known) and written out coalesced; with scores
      // requested or k above the staging room they go straight to global
      const bool staged = os == nullptr && p.top_k <= kDigitBins;
      int32_t* stage = reinterpret_cast<int32_t*>(sel->hist);
      auto key_at = [&](int i) { return cj[i]; };
      auto emit = [&](uint32_t slot_out, int i, uint32_t key) {
        const int32_t s_idx = (J.blk[i >> bshift] << bshift) + (i & (p.B - 1));
        if (staged) {
          stage[slot_out] = s_idx;
        } else {
          oi[slot_out] = s_idx;
          if (os) os[slot_out] = key_float(key);
        }
      };
      const uint32_t nv = J.nvalid;
      uint32_t filled = 0;
      if (nv <= static_cast<uint32_t>(p.top_k)) {
        emit_at_least<decltype(key_at), decltype(emit), SelGrp>(key_at, ncand, 1u, emit, *sel);
        filled = nv;
      } else if (scan_topk<decltype(key_at), decltype(emit), SelGrp>(key_at, ncand, static_cast<uint32_t>(p.top_k),
                                                                     emit, *sel, bin_key, bin_pos, kTokBinCap, J.kmin,
                                                                     J.kmax, 1024)) {
        filled = static_cast<uint32_t>(p.top_k);
      } else {
        block_topk_range<decltype(key_at), decltype(emit), SelGrp>(key_at, ncand, static_cast<uint32_t>(p.top_k),
                                                                   emit, *sel, J.kmin, J.kmax, nv);
        filled = static_cast<uint32_t>(p.top_k);
      }
      SelGrp::sync();
      if (staged) {
        if ((p.top_k & 3) == 0) {
          const int4* st4 = reinterpret_cast<const int4*>(stage);
          int4* o4 = reinterpret_cast<int4*>(oi);
          for (int i = stid; i < static_cast<int>(filled) / 4; i += SelGrp::size()) o4[i] = st4[i];
          for (int i = (static_cast<int>(filled) & ~3) + stid; i < static_cast<int>(filled); i += SelGrp::size())
            oi[i] = stage[i];
        } else {
          for (int i = stid; i < static_cast<int>(filled); i += SelGrp::size()) oi[i] = stage[i];
        }
      }
      for (int i = static_cast<int>(filled) + stid; i < p.top_k; i += SelGrp::size()) {
        oi[i] = -1;
        if (os) os[i] = -__int_as_float(0x7f800000);
      }
      SelGrp::sync();
      if (stid == 0) {
        mbar_arrive(cand_empty + cb);
        mbar_arrive(job_empty + slot);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTokAcc * H < 32 ? 32 : kTokAcc * H);
  }
}

inline size_t token_smem_bytes(int row_bytes, int H, int stages, int max_cand) {
  return 1024 + 2 * static_cast<size_t>(H) * row_bytes + static_cast<size_t>(stages) * kTokTileM * row_bytes +
         2 * static_cast<size_t>(max_cand) * 4 + kTokJobs * sizeof(TokJob) + sizeof(SelectSmem) +
         4 * kTokMaxBitmapWords + 8 * kTokBinCap + 4 + 8 +
         8 * ((kTokIssuers + 1) * stages + 4 + 2 * kTokAcc + 2 * kTokJobs + 4 + kTokIssuers) + 16;
}

}  // namespace hisa

// sparse_attn.cuh - attention over each query's selected keys, the consumer of
// the indexer's token-level top-k (HISA abstract: the output keeps the index
// interface that the downstream sparse MLA operator reads).
//
// Latent attention in its absorbed form: every key position holds one row of
// D_QK = 576 features shared by all heads (512 latent + 64 positional), and
// its value is the first D_V = 512 of them.  For a query t with selected set
// S_t (the index row with -1 and repeats dropped),
//     logit[h, j] = scale * q[t, h, :] . kv[s_j, :]
//     o[t, h, :]  = sum_j softmax_j(logit[h, :]) * kv[s_j, :D_V]
//     lse[t, h]   = log sum_j exp(logit[h, j])          (natural log)
// and an empty set gives o = 0, lse = -inf.
//
// One query's 128 heads are the M = 128 rows of every MMA, on a pair of CTAs
// (a cluster of two).  Neither the query (128 x 576 bf16 = 144 KB) nor the
// 512 fp32 accumulator columns of the output fit one SM next to the key
// tiles and the scores, so the pair splits the features 288/288:
//   CTA r  value features 256r .. 256r+255 (four 64-feature panels) and
//          positional features 512+32r .. 512+32r+31 (one 32-feature panel,
//          64-byte swizzle): its part of every logit, and the value columns
//          256r .. 256r+255 of the output
// Each CTA keeps its part of the query in TMEM (the A operand of the logit
// MMA, loaded once per query) and the softmax weights P there too (the A
// operand of the output MMA), so that shared memory holds four key stages
// and two exchange buffers.  Per 64-key tile it computes a partial logit
// tile S_c = q_c . k_c^T (M = 128 heads, N = 64 keys, K = 288) on tcgen05
// into TMEM; the two partial tiles are exchanged through distributed shared
// memory (one buffer per tile parity, so no "buffer free" handshake is
// needed; each tile's exchange is sent before the softmax of the previous
// tile, so it overlaps that work) and summed (the same in both CTAs: fp32
// addition commutes); both run the same online softmax, so each can
// accumulate its half of the output, O_c += P . V_c, with V_c the value
// columns it already holds (B operand read MN-major from the key tile).
// Keys are gathered from their positions by the TMA engine, four rows per
// instruction (tile::gather4 over a one-row box), straight into the swizzled
// layouts the MMA reads.
//
// Warp roles (10 warps):
//   warp 0      TMEM owner, logit MMA issuer (one thread)
//   warp 1      output MMA issuer (one thread)
//   warps 2..5  key gather by TMA: every tile's gather4 operations dealt
//               over the four warps, completing on the tile's stage barrier
//   warps 6..9  softmax: thread = head row; q into TMEM, exchange, online
//               softmax, O rescaling and P (bf16) in TMEM, epilogue
// Every wait is bounded; a timeout sets the CTA's abort flag and the status
// word, and the peer CTA's waits on it then time out too.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace hisa {

constexpr int kAttnHeads = 128;            // M of every MMA: one query's heads
constexpr int kAttnDqk = 576;
constexpr int kAttnDv = 512;
constexpr int kAttnTileN = 64;             // keys per tile
constexpr int kAttnMaxK = 4096;            // longest index row
constexpr int kAttnThreads = 320;
constexpr int kAttnPvWarp = 1;             // warp 0 issues the logit MMAs, warp 1 the output MMAs
constexpr int kAttnGatherBase = 64;        // warps 2..5
constexpr int kAttnGatherWarps = 4;
constexpr int kAttnSoftBase = 192;         // warps 6..9
constexpr int kAttnStages = 4;             // key stages
constexpr int kAttnPer = (kAttnMaxK + kAttnThreads - 1) / kAttnThreads;   // index-row places per thread
constexpr int kAttnHashBits = 13;
constexpr int kAttnHash = 1 << kAttnHashBits;          // dedup slots (2 x kAttnMaxK), in the key stages
constexpr int kAttnPanels = 4;             // 64-feature value panels per CTA
constexpr uint32_t kAttnPanelK = kAttnTileN * 128;     // bytes of one value panel (64 rows x 128 B)
constexpr uint32_t kAttnRopeK = kAttnTileN * 64;       // bytes of the positional half panel (64 rows x 64 B)
constexpr uint32_t kAttnStage = kAttnPanels * kAttnPanelK + kAttnRopeK;
constexpr int kAttnKsteps = kAttnPanels * 4 + 2;       // K = 288 features per CTA, 16 per MMA
constexpr int kAttnGatherOps = 16 * kAttnPanels + 16;  // gather4 operations per tile: 4 key rows each
static_assert(kAttnPer <= 32 && kAttnPer * kAttnThreads >= kAttnMaxK, "one keep bit per place of a thread's run");
static_assert(kAttnHash >= 2 * kAttnMaxK && kAttnHash * 8 <= kAttnStages * kAttnStage, "dedup table fits the stages");
static_assert(kAttnGatherOps % kAttnGatherWarps == 0 && 16 * kAttnPanels % kAttnGatherWarps == 0 &&
                  kAttnGatherOps <= 32 * kAttnGatherWarps, "equal gather shares, one operation per lane");
constexpr uint32_t kAttnTmemS = 0;         // one 64-column logit buffer
constexpr uint32_t kAttnTmemQ = 64;        // the query part: 2 bf16 per column, 144 columns
constexpr uint32_t kAttnTmemP = 208;       // softmax weights of one tile: 64 bf16 = 32 columns
constexpr uint32_t kAttnTmemO = 256;       // 256 output columns
static_assert(kAttnTmemQ + kAttnKsteps * 8 <= kAttnTmemP && kAttnTmemP + 32 <= kAttnTmemO, "TMEM map");
constexpr unsigned kFull = 0xffffffffu;

struct AttnParams {
  int64_t rows;              // batch * Q
  int Q, L, slices;          // slices: heads / 128
  int top_k;
  float scale_log2;          // softmax scale * log2(e)
  const int32_t* idx;        // [rows, top_k]
  const uint16_t* q;         // [rows, heads, 576] bf16
  const uint16_t* kv;        // [batch, L, 576] bf16
  uint16_t* o;               // [rows, heads, 512] bf16
  float* lse;                // [rows, heads]
};

namespace sm100 {

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3; "
      "selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Bounded wait on a barrier completed by the other CTA of the cluster.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      record_status(HISA_ERR_TIMEOUT);
      return false;
    }
  }
}

// Four rows (y0..y3) of a tensor map whose box is one row high, placed in
// shared memory as four consecutive box rows; completion counted on `bar`.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, uint64_t* bar, int x, int y0,
                                            int y1, int y2, int y3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3), "r"(smem_u32(bar))
      : "memory");
}

// A hint to bring the 128-byte line holding `ptr` into L2.
__device__ __forceinline__ void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(ptr)));
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16 bytes into another CTA's shared memory, counted as complete_tx bytes on
// that CTA's mbarrier `remote_bar` when they land (both cluster addresses).
__device__ __forceinline__ void st_async_v4(uint32_t addr, float a, float b, float c, float d, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
               "f"(a), "f"(b), "f"(c), "f"(d), "r"(remote_bar)
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns from registers into TMEM.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns from registers into TMEM.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Shared-memory descriptor of a K-major operand stored by TMA with the
// 64-byte swizzle: rows of 64 bytes (32 bf16), 8-row atoms of 512 bytes
// (stride byte offset 512), layout type 4; version 1 (sm_100).
__device__ __forceinline__ uint64_t desc_k_sw64(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(512 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(4) << 61;
  return d;
}

// Shared-memory descriptor of an MN-major operand stored with the 128-byte
// swizzle: rows of 128 bytes hold 64 consecutive MN elements for one K index,
// 8-row groups along K are `sbo` bytes apart and 64-element groups along MN
// `lbo` bytes apart.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// D[tmem] (+)= A[tmem] * B[smem]^T (bf16), issued by one thread: A is M = 128
// rows in 128 lanes, two consecutive K elements per 32-bit column.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor with the B operand MN-major (bf16, fp32 accumulate).
__host__ __device__ constexpr uint32_t instr_desc_bmn(int M, int N) {
  return instr_desc(M, N, 1u) | (1u << 16);
}

}  // namespace sm100

// 2^x by the SFU's approximate base-2 exponential (ex2.approx, a hardware
// instruction: relative error of a few ulp, 2^-inf = 0); the softmax weights
// it produces are rounded to bf16 before they are used.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

struct AttnSmem {
  uint64_t q_full;
  uint64_t kv_full[kAttnStages], kv_empty[kAttnStages];
  uint64_t s_full, s_empty;
  uint64_t p_full, pv_done;
  uint64_t x_full[2][2];         // partial logits of the peer CTA: [tile parity][key half]
  uint64_t drain[2];             // one per MMA issuer
  uint32_t tmem_base;
  int abort_flag;
  int n_valid;
  int pad;
  int scan[kAttnThreads / 32 + 1];
};

constexpr size_t kAttnSmemBytes = 1024 + kAttnStages * kAttnStage   // key tiles (1 KB for alignment)
                                  + 2 * kAttnHeads * kAttnTileN * 4  // partial logits from the peer, two buffers
                                  + kAttnMaxK * 4                    // the query's deduplicated positions
                                  + sizeof(AttnSmem) + 16;
static_assert(kAttnSmemBytes <= 232448, "dynamic shared memory of one CTA");
inline size_t attn_smem_bytes() { return kAttnSmemBytes; }

__global__ void __launch_bounds__(kAttnThreads, 1) sparse_attn_kernel(const __grid_constant__ CUtensorMap kvmap,
                                                                     const __grid_constant__ CUtensorMap ropemap,
                                                                     const AttnParams p) {
  using namespace sm100;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kv_buf = smem;
  float* x_buf = reinterpret_cast<float*>(kv_buf + kAttnStages * kAttnStage);   // [2 parities][16 pieces][128 rows][4]
  int32_t* sidx = reinterpret_cast<int32_t*>(x_buf + 2 * kAttnHeads * kAttnTileN);
  AttnSmem* sm = reinterpret_cast<AttnSmem*>(sidx + kAttnMaxK);
  volatile int* abort_flag = &sm->abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int64_t item = cluster_id_x();                   // (row, head slice)
  const int64_t row = item / p.slices;
  const int slice = static_cast<int>(item % p.slices);
  const int b = static_cast<int>(row / p.Q);
  const int val0 = 256 * static_cast<int>(rank);          // this CTA's value features: val0 .. val0 + 255
  const int rope0 = kAttnDv + 32 * static_cast<int>(rank); // and positional features rope0 .. rope0 + 31

  if (tid == 0) {
    mbar_init(&sm->q_full, 128);
    for (int i = 0; i < kAttnStages; ++i) {
      mbar_init(&sm->kv_full[i], kAttnGatherWarps);   // one byte-announcing arrive per gather warp
      mbar_init(&sm->kv_empty[i], 1);
    }
    mbar_init(&sm->s_full, 1);
    mbar_init(&sm->s_empty, 128);
    mbar_init(&sm->p_full, 128);
    mbar_init(&sm->pv_done, 1);
    for (int i = 0; i < 2; ++i)
      for (int hf = 0; hf < 2; ++hf)
        mbar_init(&sm->x_full[i][hf], 1);   // local arrive with a half tile's bytes + the peer's st.async bytes
    mbar_init(&sm->drain[0], 1);
    mbar_init(&sm->drain[1], 1);
    sm->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(&sm->tmem_base, 512);
  if (warp == 2 && lane == 0) {
    tma_prefetch_desc(&kvmap);
    tma_prefetch_desc(&ropemap);
  }

  if (warp >= kAttnSoftBase / 32) {
    // this head's part of the query towards L2 while the index row is read
    const uint16_t* qh = p.q + ((row * p.slices + slice) * kAttnHeads + (tid - kAttnSoftBase)) *
                                   static_cast<int64_t>(kAttnDqk);
    for (int c = 0; c < kAttnPanels; ++c) prefetch_l2(qh + val0 + 64 * c);
    prefetch_l2(qh + rope0);
  }

  // ---- the query's positions: -1, out-of-range entries and repeats dropped,
  // compacted in row order.  Each thread takes a contiguous run of the row;
  // a hash table in the (still unused) key stages maps a position to the
  // first place of the row where it occurs, and a place is kept when it is
  // that first place.  The result does not depend on the order of the
  // atomics, so it is the same on every run.
  {
    uint32_t* hkey = reinterpret_cast<uint32_t*>(kv_buf);
    int32_t* hfirst = reinterpret_cast<int32_t*>(kv_buf + kAttnHash * 4);
    const int K = p.top_k;
    const int per = (K + kAttnThreads - 1) / kAttnThreads;   // at most kAttnMaxK / kAttnThreads
    const int lo = min(K, tid * per), hi = min(K, lo + per);
    const int32_t* irow = p.idx + row * K;
    int v[kAttnPer];
#pragma unroll
    for (int u = 0; u < kAttnPer; ++u) {
      int x = lo + u < hi ? __ldg(irow + lo + u) : -1;
      v[u] = x < p.L ? x : -1;                         // negative: not a key
    }
    for (int i = tid; i < kAttnHash / 4; i += kAttnThreads) {
      reinterpret_cast<uint4*>(hkey)[i] = make_uint4(~0u, ~0u, ~0u, ~0u);
      reinterpret_cast<int4*>(hfirst)[i] = make_int4(INT32_MAX, INT32_MAX, INT32_MAX, INT32_MAX);
    }
    __syncthreads();
    int slot[kAttnPer];
#pragma unroll
    for (int u = 0; u < kAttnPer; ++u) {
      slot[u] = -1;
      if (v[u] >= 0) {
        // open addressing; at most kAttnMaxK distinct keys in twice as many slots
        uint32_t hs = (static_cast<uint32_t>(v[u]) * 0x9E3779B1u) >> (32 - kAttnHashBits);
        for (int probe = 0; probe < kAttnHash; ++probe) {
          const uint32_t prev = atomicCAS(&hkey[hs], ~0u, static_cast<uint32_t>(v[u]));
          if (prev == ~0u || prev == static_cast<uint32_t>(v[u])) break;
          hs = (hs + 1) & (kAttnHash - 1);
        }
        atomicMin(&hfirst[hs], lo + u);
        slot[u] = static_cast<int>(hs);
      }
    }
    __syncthreads();
    uint32_t keep = 0;
#pragma unroll
    for (int u = 0; u < kAttnPer; ++u)
      if (slot[u] >= 0 && hfirst[slot[u]] == lo + u) keep |= 1u << u;
    const int cnt = __popc(keep);
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += o;
    }
    if (lane == 31) sm->scan[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w2 = 0; w2 < warp; ++w2) base += sm->scan[w2];
    if (tid == kAttnThreads - 1) sm->n_valid = base + incl;
    int pos = base + incl - cnt;
#pragma unroll
    for (int u = 0; u < kAttnPer; ++u)
      if (keep & (1u << u)) sidx[pos++] = v[u];
  }
  // the table's generic-proxy accesses are ordered before the key gathers
  // (async proxy) that will overwrite it
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  cluster_sync();                                      // the peer's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  const int n_valid = sm->n_valid;
  const int T = (n_valid + kAttnTileN - 1) / kAttnTileN;

  if (warp == 0) {
    // ------------------------------------------------------------ logit MMA issuer
    // S = q_c . k_c^T for tile k as soon as its keys have landed and the
    // softmax has read tile k-1 out of the single logit buffer; the output
    // MMAs come from another thread, so these never queue behind them
    if (lane == 0) {
      constexpr uint32_t id_qk = instr_desc(kAttnHeads, kAttnTileN, 1u);
      bool ok = T == 0 || mbar_wait(&sm->q_full, 0, abort_flag);
      if (ok) tc_fence_after();
      for (int k = 0; ok && k < T; ++k) {
        const int st = k % kAttnStages;
        if (!(ok = mbar_wait(&sm->kv_full[st], static_cast<uint32_t>((k / kAttnStages) & 1), abort_flag))) break;
        if (k >= 1 && !(ok = mbar_wait(&sm->s_empty, static_cast<uint32_t>((k - 1) & 1), abort_flag))) break;
        tc_fence_after();
        const uint32_t base = smem_u32(kv_buf + st * kAttnStage);
        const uint64_t k_desc = desc_k_sw128(base);
#pragma unroll
        for (int ks = 0; ks < 4 * kAttnPanels; ++ks)
          mma_ts(tmem + kAttnTmemS, tmem + kAttnTmemQ + ks * 8,
                 k_desc + static_cast<uint64_t>((ks >> 2) * (kAttnPanelK / 16) + (ks & 3) * 2), id_qk, ks > 0 ? 1u : 0u);
        const uint64_t r_desc = desc_k_sw64(base + kAttnPanels * kAttnPanelK);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          mma_ts(tmem + kAttnTmemS, tmem + kAttnTmemQ + (4 * kAttnPanels + ks) * 8, r_desc + static_cast<uint64_t>(ks * 2),
                 id_qk, 1u);
        mma_commit(&sm->s_full);
      }
      mma_commit(&sm->drain[0]);
      mbar_drain(&sm->drain[0], 0);
    }
  } else if (warp == kAttnPvWarp) {
    // ------------------------------------------------------------ output MMA issuer
    // O_c += P . V_c for tile j once the softmax has written P_j; the tile's
    // key stage is free when this MMA completes
    if (lane == 0) {
      constexpr uint32_t id_pv = instr_desc_bmn(kAttnHeads, 256);
      bool ok = true;
      for (int j = 0; ok && j < T; ++j) {
        const int sj = j % kAttnStages;
        if (!(ok = mbar_wait(&sm->p_full, static_cast<uint32_t>(j & 1), abort_flag))) break;
        tc_fence_after();
        // V: the four 64-feature value panels of the key tile, MN-major
        const uint32_t v0 = smem_u32(kv_buf + sj * kAttnStage);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t vd = desc_mn_sw128(v0 + ks * 16 * 128, kAttnPanelK, 1024);
          mma_ts(tmem + kAttnTmemO, tmem + kAttnTmemP + ks * 8, vd, id_pv, (j > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&sm->kv_empty[sj]);
        mma_commit(&sm->pv_done);
      }
      mma_commit(&sm->drain[1]);
      mbar_drain(&sm->drain[1], 0);
    }
  } else if (warp < kAttnSoftBase / 32) {
    // ------------------------------------------------------------ key gather
    // warps 2..5 share every tile: its gather4 operations (four key rows of
    // one 64-feature value panel, or of the 32 positional features) are dealt
    // round-robin over the warps, one per lane, and each warp announces its
    // own bytes on the stage's barrier
    const int gw = warp - kAttnGatherBase / 32;        // 0..3
    const int kbase = b * p.L;
    constexpr uint32_t my_bytes = (16 * kAttnPanels / kAttnGatherWarps) * 4 * 128 + (16 / kAttnGatherWarps) * 4 * 64;
    static_assert(my_bytes * kAttnGatherWarps == kAttnStage, "gather shares cover the stage");
    int issued = 0;
    for (int i = 0; i < T; ++i) {
      const int st = i % kAttnStages;
      int okl = 1;
      if (lane == 0)
        okl = mbar_wait(&sm->kv_empty[st], static_cast<uint32_t>(((i / kAttnStages) & 1) ^ 1), abort_flag);
      if (__shfl_sync(kFull, okl, 0) == 0) break;
      if (lane == 0) mbar_arrive_expect_tx(&sm->kv_full[st], my_bytes);
      __syncwarp();
      const int x = gw + kAttnGatherWarps * lane;
      if (x < kAttnGatherOps) {
        const bool rope = x >= 16 * kAttnPanels;
        const int g4 = rope ? x - 16 * kAttnPanels : (x & 15);
        int y[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = i * kAttnTileN + 4 * g4 + u;
          y[u] = kbase + sidx[e < n_valid ? e : 0];       // past the last position: any valid row, masked later
        }
        uint8_t* stage = kv_buf + st * kAttnStage;
        const uint32_t dst = rope ? smem_u32(stage + kAttnPanels * kAttnPanelK + g4 * 4 * 64)
                                  : smem_u32(stage + (x >> 4) * kAttnPanelK + g4 * 4 * 128);
        tma_gather4(dst, rope ? &ropemap : &kvmap, &sm->kv_full[st], rope ? rope0 : val0 + 64 * (x >> 4), y[0],
                    y[1], y[2], y[3]);
      }
      ++issued;
    }
    if (lane == 0) {
      // leave only once this warp's copies have landed: the last tile of each stage
      for (int j = max(0, issued - kAttnStages); j < issued; ++j)
        mbar_drain(&sm->kv_full[j % kAttnStages], static_cast<uint32_t>((j / kAttnStages) & 1));
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;                 // head row = TMEM lane
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    constexpr uint32_t kXBytes = kAttnHeads * kAttnTileN * 4;           // one exchange buffer
    const uint32_t peer_x = peer_addr(x_buf + h * 4, peer);            // + buffer * kXBytes + piece * 2 KB
    const uint32_t peer_x_full = peer_addr(&sm->x_full[0][0], peer);   // + (buffer * 2 + half) * 8
    float m = -__int_as_float(0x7f800000), l = 0.f;
    bool ok = true;
    {
      // this head's part of the query into TMEM: the four value panels (32
      // columns each, the next panel's loads in flight while one is stored),
      // then the 32 positional features (16 columns)
      const uint16_t* qh = p.q + ((row * p.slices + slice) * kAttnHeads + h) * static_cast<int64_t>(kAttnDqk);
      const uint4* qg = reinterpret_cast<const uint4*>(qh + val0);
      const uint4* qr = reinterpret_cast<const uint4*>(qh + rope0);
      uint4 rq[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) rq[u] = __ldg(qr + u);
      uint32_t v[32];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint4 x = __ldg(qg + u);
        v[4 * u] = x.x; v[4 * u + 1] = x.y; v[4 * u + 2] = x.z; v[4 * u + 3] = x.w;
      }
#pragma unroll 1
      for (int pn = 0; pn < kAttnPanels; ++pn) {
        uint4 nx[8];
        if (pn + 1 < kAttnPanels) {
#pragma unroll
          for (int u = 0; u < 8; ++u) nx[u] = __ldg(qg + (pn + 1) * 8 + u);
        }
        tmem_st32(t_lane + kAttnTmemQ + pn * 32, v);
        if (pn + 1 < kAttnPanels) {
          tmem_wait_st();                              // v is rewritten below
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            v[4 * u] = nx[u].x; v[4 * u + 1] = nx[u].y; v[4 * u + 2] = nx[u].z; v[4 * u + 3] = nx[u].w;
          }
        }
      }
      uint32_t r16[16];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        r16[4 * u] = rq[u].x; r16[4 * u + 1] = rq[u].y; r16[4 * u + 2] = rq[u].z; r16[4 * u + 3] = rq[u].w;
      }
      tmem_st16(t_lane + kAttnTmemQ + 32 * kAttnPanels, r16);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm->q_full);
    }
    // Every wait below is taken by all lanes and its outcome made
    // warp-uniform: the tcgen05 loads and stores that follow are .sync.aligned.
    //
    // This CTA's partial logits of a tile go to the peer's exchange buffer
    // for the tile's parity as 16 16-byte st.async pieces per thread, which
    // count themselves on the peer's x_full of that parity and key half (each
    // expects half a tile of bytes from a local arrive).  The buffer is
    // piece-major, [piece c][head row h][16 B]: the 32 pieces one warp
    // instruction sends are 512 contiguous bytes (a scattered row-major
    // layout moved about half as many bytes per cycle between the SMs), and
    // the reads are conflict-free.  The partial logits of tile i+1 leave
    // before the softmax of tile i, so the exchange overlaps that work.  A
    // buffer is written again two tiles later: the peer sends tile i+1 after
    // it has received all of my tile i, which each of my threads sends after
    // reading its rows of tile i-1 from the same buffer.
    auto load_send = [&](float (&dst)[64], int tile) -> bool {
      if (!__all_sync(kFull, mbar_wait(&sm->s_full, static_cast<uint32_t>(tile & 1), abort_flag))) return false;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(t_lane + kAttnTmemS, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) dst[j] = __uint_as_float(v[j]);
      tmem_ld32(t_lane + kAttnTmemS + 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) dst[32 + j] = __uint_as_float(v[j]);
      tc_fence_before();
      mbar_arrive(&sm->s_empty);
      const int xb = tile & 1;
      if (h == 0) {
        mbar_arrive_expect_tx(&sm->x_full[xb][0], kXBytes / 2);
        mbar_arrive_expect_tx(&sm->x_full[xb][1], kXBytes / 2);
      }
#pragma unroll
      for (int c = 0; c < 16; ++c)
        st_async_v4(peer_x + xb * kXBytes + c * (kAttnHeads * 16), dst[4 * c], dst[4 * c + 1], dst[4 * c + 2],
                    dst[4 * c + 3], peer_x_full + (xb * 2 + (c >> 3)) * 8);
      return true;
    };
    float s[64], sn[64];
    if (T > 0) ok = load_send(s, 0);
    for (int i = 0; ok && i < T; ++i) {
      // 1. the peer's part of tile i, sent one tile ago
      const int xb = i & 1;
      if (!(ok = __all_sync(kFull, mbar_wait_cluster(&sm->x_full[xb][0], static_cast<uint32_t>((i >> 1) & 1),
                                                     abort_flag) &&
                                       mbar_wait_cluster(&sm->x_full[xb][1], static_cast<uint32_t>((i >> 1) & 1),
                                                         abort_flag))))
        break;
      const float4* x4 = reinterpret_cast<const float4*>(x_buf + xb * (kAttnHeads * kAttnTileN)) + h;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 v = x4[c * kAttnHeads];
        s[4 * c + 0] += v.x; s[4 * c + 1] += v.y; s[4 * c + 2] += v.z; s[4 * c + 3] += v.w;
      }
      // 2. my part of tile i+1 out to the peer
      if (i + 1 < T && !(ok = load_send(sn, i + 1))) break;
      // 3. online softmax of tile i in the log2 domain: logits past the last
      // key are -inf, whose exp2 is 0; maxima and sums in four independent
      // chains.  The reference maximum moves only when the tile's maximum
      // exceeds it by more than 8 (a factor 256): the weights stay below 2^8,
      // the output rows are rescaled rarely, and o = sum p v / sum p is the
      // same for any reference (the natural-log lse adds back the reference
      // that was used)
      const int nk = min(kAttnTileN, n_valid - i * kAttnTileN);
      float mx4[4] = {-__int_as_float(0x7f800000), -__int_as_float(0x7f800000), -__int_as_float(0x7f800000),
                      -__int_as_float(0x7f800000)};
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        s[j] = j < nk ? s[j] * p.scale_log2 : -__int_as_float(0x7f800000);
        mx4[j & 3] = fmaxf(mx4[j & 3], s[j]);
      }
      const float mt = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      const bool move = i == 0 || mt > m + 8.f;
      const float mx = move ? mt : m;
      const float corr = (i == 0) ? 0.f : (move ? fast_exp2(m - mx) : 1.f);
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        s[j] = fast_exp2(s[j] - mx);
        sum4[j & 3] += s[j];
      }
      l = l * corr + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
      m = mx;
      // P and O belong to the previous tile's output MMA until it completes
      if (i >= 1 &&
          !(ok = __all_sync(kFull, mbar_wait(&sm->pv_done, static_cast<uint32_t>((i - 1) & 1), abort_flag))))
        break;
      tc_fence_after();
      // P row (64 keys, bf16 pairs) into TMEM: the A operand of this tile's output MMA
      {
        uint32_t v[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = pack_bf16x2(s[2 * c], s[2 * c + 1]);
        tmem_st32(t_lane + kAttnTmemP, v);
      }
      if (i >= 1) {
        if (__any_sync(kFull, corr != 1.f)) {          // rows whose maximum did not grow scale by 1
#pragma unroll 1
          for (int c0 = 0; c0 < 256; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(t_lane + kAttnTmemO + c0, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * corr);
            tmem_st32(t_lane + kAttnTmemO + c0, v);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm->p_full);
#pragma unroll
      for (int j = 0; j < 64; ++j) s[j] = sn[j];
    }
    // ---- epilogue: O / l in bf16, and lse
    const int64_t orow = (row * p.slices + slice) * kAttnHeads + h;
    uint16_t* od = p.o + orow * kAttnDv + rank * 256;
    const bool have =
        __all_sync(kFull, ok && T > 0 && mbar_wait(&sm->pv_done, static_cast<uint32_t>((T - 1) & 1), abort_flag));
    if (have) {
      tc_fence_after();
      const float inv = 1.f / l;
#pragma unroll 1
      for (int c0 = 0; c0 < 256; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(t_lane + kAttnTmemO + c0, v);
        tmem_wait_ld();
        uint4* dst = reinterpret_cast<uint4*>(od + c0);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * inv, __uint_as_float(v[8 * q4 + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * inv, __uint_as_float(v[8 * q4 + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * inv, __uint_as_float(v[8 * q4 + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * inv, __uint_as_float(v[8 * q4 + 7]) * inv);
          dst[q4] = w;
        }
      }
    } else if (T == 0) {
      uint4* dst = reinterpret_cast<uint4*>(od);
      for (int q4 = 0; q4 < 32; ++q4) dst[q4] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (rank == 0 && (have || T == 0))
      p.lse[orow] = T == 0 ? -__int_as_float(0x7f800000) : (m + log2f(l)) * 0.69314718055994531f;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();                                      // no CTA leaves while its peer may still write to it
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace hisa

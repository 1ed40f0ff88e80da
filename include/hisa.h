/*
 * hisa.h - C ABI of libhisa: the HISA hierarchical lightning indexer and the
 * flat DSA lightning indexer on NVIDIA B200 (sm_100a).
 *
 * What is computed.  "HISA: Efficient Hierarchical Indexing for Fine-Grained
 * Sparse Attention" (arXiv 2603.28458, abstract): the DSA indexer scores every
 * key of a query's prefix and keeps the top-k keys; HISA replaces that flat
 * scan with (1) a coarse stage that scores one pooled key per block and
 * keeps the best blocks, and (2) a refinement stage that runs the original
 * indexer only on the keys of the kept blocks, returning for each query the
 * same kind of k-index set that the downstream sparse attention consumes.  The
 * indexer score used by every entry point is
 *
 *     I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:])
 *
 * and a block is represented by the mean of its keys.  A query t sees keys
 * 0 .. n_visible[t]-1; its current block is c_t = (n_visible[t]-1) / B.  The
 * coarse stage scores only the blocks b < c_t and always keeps c_t.  Ties at
 * the k-th (or m-th) place go to the lower index.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers, 16-byte aligned, dense and
 *    row-major in the layouts given below; the caller owns every buffer,
 *    including the workspace.  The library allocates no memory.
 *  - Work is enqueued on `stream` and runs asynchronously; the return value
 *    reports only host-side validation and launch errors.  On a validation
 *    error nothing is enqueued and the outputs are untouched.
 *  - Kernels that wait on on-chip barriers do so with a bounded spin; if a
 *    wait gives up, the kernel records HISA_ERR_TIMEOUT in a device status
 *    word and exits cleanly.  hisa_get_status() reads (and clears) that word.
 *  - Index outputs are -1 padded.  Without a score output each row's indices
 *    are a set in unspecified order.  With a score output, score[i] belongs
 *    to index[i] and each row is sorted by (score desc, index asc), the
 *    order that defines the top-k, with the -1 / -inf padding last; scored
 *    rows are sorted on chip, so top_k <= 16384 when scores are requested
 *    (HISA_ERR_UNSUPPORTED otherwise).
 *  - dtype HISA_E4M3: q and keys are OFP8 E4M3 codes with one fp32 scale per
 *    query token (over all H*d values) and one per key; the value of a code
 *    is code * scale.  For the other dtypes the scale pointers are ignored
 *    and may be NULL.
 */
#ifndef HISA_H_
#define HISA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HISA_API __attribute__((visibility("default")))
#else
#define HISA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HISA_OK = 0,
  HISA_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size or value   */
  HISA_ERR_UNSUPPORTED = 2,   /* a valid shape this build has no kernel for     */
  HISA_ERR_WORKSPACE = 3,     /* workspace smaller than one unit of work        */
  HISA_ERR_CUDA = 4,          /* a CUDA runtime call failed                     */
  HISA_ERR_TIMEOUT = 5        /* a device-side bounded wait gave up             */
} hisa_status;

typedef enum { HISA_F32 = 0, HISA_BF16 = 1, HISA_E4M3 = 2 } hisa_dtype;

/* Problem shape.  batch independent sequences, each with num_keys keys (L)
 * and num_queries queries (Q); heads H and head_dim d of the indexer; block
 * size B; top_m blocks and top_k tokens kept per query; dtype of q and keys
 * (a hisa_dtype value).  w is always fp32. */
typedef struct {
  int32_t batch;
  int32_t num_keys;
  int32_t num_queries;
  int32_t heads;
  int32_t head_dim;
  int32_t block_size;
  int32_t top_m;
  int32_t top_k;
  int32_t dtype;
} hisa_shape;

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* hisa_stream;

/* op codes for hisa_workspace_size */
enum {
  HISA_OP_BLOCK_SCORE_TOPM = 1,
  HISA_OP_TOKEN_SCORE_TOPK = 2,
  HISA_OP_FLAT_TOPK = 3,
  HISA_OP_FLAT_TOPK_SAMPLED = 4,
  HISA_OP_BLOCK_REFINE_TOPM = 5,
  HISA_OP_INDEXER_FROM_HOST = 6
};

/*
 * Block pooling (HISA coarse stage input; HISA abstract, "pooled block
 * representations").  kpool[b] = mean of keys b*B .. min((b+1)*B, L)-1, the
 * mean taken exactly (fp64 accumulation) and rounded once to the key dtype.
 * For HISA_E4M3 the mean is of the dequantised keys, rounded to fp32, then
 * re-quantised with one scale per block: scale = max|mean| / 448 (1 for an
 * all-zero block), code = E4M3(mean / scale), round to nearest even,
 * saturating.
 *   k            [batch, L, d] in shape->dtype
 *   k_scale      [batch, L] fp32 (E4M3 only)
 *   kpool        [batch, ceil(L/B), d] in shape->dtype          (output)
 *   kpool_scale  [batch, ceil(L/B)] fp32 (E4M3 only)             (output)
 * Uses batch, num_keys, head_dim, block_size, dtype.
 */
HISA_API hisa_status hisa_pool_blocks(const void* k, const float* k_scale, void* kpool,
                             float* kpool_scale, const hisa_shape* shape,
                             hisa_stream stream);

/*
 * Block pooling of a range of blocks: the rows b in [first_block,
 * first_block + block_count) (clipped to ceil(num_keys / B)) of every
 * sequence's kpool (and kpool_scale for E4M3) are written exactly as
 * hisa_pool_blocks writes them; every other row is left untouched.
 * The pages pool keys into blocks once per context (HISA abstract) and do not
 * say how a decoder keeps them; this entry lets it keep the pooled keys as a
 * cache, pooling a block once when its last key arrives, since the coarse
 * stage only scores blocks that are complete (the current block is kept
 * without a score).  Same layouts, ownership and checks as hisa_pool_blocks;
 * first_block < 0 or block_count < 0 is HISA_ERR_INVALID_ARG, an empty range
 * returns HISA_OK without a launch.
 */
HISA_API hisa_status hisa_pool_blocks_range(const void* k, const float* k_scale, void* kpool,
                                            float* kpool_scale, const hisa_shape* shape,
                                            int32_t first_block, int32_t block_count,
                                            hisa_stream stream);

/*
 * Paged keys.  The pages leave the decoder's key storage open; a serving
 * cache keeps each sequence's keys in fixed-size pages that it allocates as
 * the sequence grows.  Here one page holds one HISA block:
 *   k_pages       [num_pages, B, d] in shape->dtype (B = shape->block_size)
 *   k_page_scale  [num_pages, B] fp32 (E4M3 only)
 *   page_table    [batch, ceil(L/B)] int32: block j of sequence b (its keys
 *                 j*B .. j*B+B-1) is page page_table[b * ceil(L/B) + j]
 * L = shape->num_keys is the longest sequence the table covers; pages past a
 * sequence's length are never read.  The results equal those of the
 * contiguous entries on the keys the pages hold.  An entry that is read and
 * lies outside [0, num_pages) is not dereferenced: the block is skipped and
 * the device status word reports HISA_ERR_INVALID_ARG (hisa_get_status).
 *
 * hisa_pool_blocks_paged: hisa_pool_blocks_range over paged keys; block j's
 * mean is over its first min(B, L - j*B) rows.  Same outputs, ownership and
 * checks; page_table must be non-NULL and 4-byte aligned, num_pages >= 1.
 */
HISA_API hisa_status hisa_pool_blocks_paged(const void* k_pages, const float* k_page_scale,
                                            const int32_t* page_table, int32_t num_pages,
                                            void* kpool, float* kpool_scale,
                                            const hisa_shape* shape, int32_t first_block,
                                            int32_t block_count, hisa_stream stream);

/*
 * Key compression ("StreamIndex: Memory-Bounded Compressed Sparse Attention
 * via Streaming Top-k", arXiv 2605.02568, abstract: the indexer runs over keys
 * compressed by a fixed ratio, 4 in V4-Flash).  ck[j] = mean of raw keys
 * j*ratio .. j*ratio+ratio-1, exact mean rounded once to the dtype; a trailing
 * incomplete group is dropped.  dtype HISA_F32 or HISA_BF16.
 *   k_raw [batch, S, d] -> ck [batch, S / ratio, d]
 */
HISA_API hisa_status hisa_compress_keys(const void* k_raw, void* ck, int32_t batch,
                               int32_t num_raw_keys, int32_t head_dim,
                               int32_t ratio, int32_t dtype, hisa_stream stream);

/*
 * Per-row FP8 quantisation of q or keys (the E4M3 variant of the indexer):
 * scale[r] = max_j |x[r,j]| / 448 in fp32 (1 when the row is all zero),
 * codes[r,j] = E4M3(x[r,j] / scale[r]) with the division in fp32, round to
 * nearest even, saturating to +-448.
 *   x      [rows, cols] fp32 (x_dtype HISA_F32) or bf16 (HISA_BF16)
 *   codes  [rows, cols] uint8 (output), scale [rows] fp32 (output)
 * For q use rows = batch*Q, cols = H*d; for keys rows = batch*L, cols = d.
 */
HISA_API hisa_status hisa_quantize_e4m3(const void* x, int32_t x_dtype, int64_t rows,
                               int32_t cols, uint8_t* codes, float* scale,
                               hisa_stream stream);

/*
 * HISA coarse stage (HISA abstract, stage 1): for each query t,
 *   S_b[t,b] = sum_h w[t,h] * ReLU(q[t,h,:] . kpool[b,:])   for b < c_t,
 * then block_idx[t,:] = {c_t} plus the top_m-1 blocks by S_b (ties -> lower
 * b); every block 0..c_t when c_t+1 <= top_m; nothing when n_visible[t]==0.
 *   q          [batch, Q, H, d] in dtype;  q_scale [batch, Q] fp32 (E4M3)
 *   w          [batch, Q, H] fp32
 *   kpool      [batch, ceil(L/B), d] in dtype; kpool_scale [batch, ceil(L/B)]
 *   n_visible  [batch, Q] int32, 0 <= n_visible <= L
 *   block_idx  [batch, Q, top_m] int32 (output), -1 padded, any order
 *   workspace  device scratch of at least
 *              hisa_workspace_size(HISA_OP_BLOCK_SCORE_TOPM) bytes
 */
HISA_API hisa_status hisa_block_score_topm(const void* q, const float* q_scale,
                                  const float* w, const void* kpool,
                                  const float* kpool_scale,
                                  const int32_t* n_visible,
                                  const hisa_shape* shape, int32_t* block_idx,
                                  void* workspace, size_t ws_bytes,
                                  hisa_stream stream);

/*
 * HISA refinement stage (HISA abstract, stage 2): candidates C_t = keys of
 * the blocks in block_idx[t,:] (entries -1 are skipped, repeats count once)
 * that are visible (s < n_visible[t]); topk_idx[t,:] = the top_k of C_t by
 * I[t,s] (ties -> lower s), all of C_t then -1 padding when |C_t| < top_k.
 * Candidate scores stay on chip; nothing of size [Q, H, L] is formed.
 *   k          [batch, L, d] in dtype; k_scale [batch, L] fp32 (E4M3)
 *   block_idx  [batch, Q, top_m] int32, each entry -1 or in [0, ceil(L/B))
 *   topk_idx   [batch, Q, top_k] int32 (output)
 *   topk_score [batch, Q, top_k] fp32 (output, may be NULL; -inf padding)
 * Requires top_m * block_size <= 16384.
 * Workspace: optional.  hisa_workspace_size(HISA_OP_TOKEN_SCORE_TOPK) is
 * nonzero for shapes with few queries (at most half the SM count, as in a
 * decode step); given at least that much (16-byte aligned), each query's
 * blocks are split over several CTAs and their top-k lists merged exactly,
 * so more SMs gather keys.  NULL (or less) runs one CTA per query.  The
 * result is the same either way.
 */
HISA_API hisa_status hisa_token_score_topk(const void* q, const float* q_scale,
                                  const float* w, const void* k,
                                  const float* k_scale,
                                  const int32_t* n_visible,
                                  const int32_t* block_idx,
                                  const hisa_shape* shape, int32_t* topk_idx,
                                  float* topk_score, void* workspace,
                                  size_t ws_bytes, hisa_stream stream);

/*
 * hisa_token_score_topk over paged keys (layout as for
 * hisa_pool_blocks_paged): the TMA tile load of a retained block reads its
 * page.  Same result, outputs and workspace rule as hisa_token_score_topk.
 * Tensor-core shapes only (bf16 or E4M3, head_dim * bytes 128 or 256,
 * H 16, 32 or 64, B 16..128, top_m * B within the on-chip candidate
 * buffers); others return HISA_ERR_UNSUPPORTED.  num_pages * B must fit in
 * int32.
 */
HISA_API hisa_status hisa_token_score_topk_paged(const void* q, const float* q_scale,
                                                 const float* w, const void* k_pages,
                                                 const float* k_page_scale,
                                                 const int32_t* page_table, int32_t num_pages,
                                                 const int32_t* n_visible,
                                                 const int32_t* block_idx,
                                                 const hisa_shape* shape, int32_t* topk_idx,
                                                 float* topk_score, void* workspace,
                                                 size_t ws_bytes, hisa_stream stream);

/*
 * Flat DSA indexer (the comparison path; HISA abstract: the flat scan of
 * every prefix key): topk_idx[t,:] = top_k of {0 .. n_visible[t]-1} by
 * I[t,s], ties -> lower s, -1 padded when n_visible[t] < top_k.
 * Scores go through the workspace as fp32 rows of at most L values (never
 * [Q, H, L]); with less workspace than hisa_workspace_size(HISA_OP_FLAT_TOPK)
 * the queries are processed in chunks that fit.
 * Arguments as for hisa_token_score_topk (block_size and top_m unused).
 */
HISA_API hisa_status dsa_flat_indexer_topk(const void* q, const float* q_scale,
                                  const float* w, const void* k,
                                  const float* k_scale,
                                  const int32_t* n_visible,
                                  const hisa_shape* shape, int32_t* topk_idx,
                                  float* topk_score, void* workspace,
                                  size_t ws_bytes, hisa_stream stream);

/*
 * Three-level indexer, second level ("LongCat Sparse Attention" abstract,
 * Hierarchical Indexing: coarse-to-fine scoring that narrows the candidate
 * set step by step; here HISA's coarse step applied twice).  Super-blocks are
 * runs of `group` blocks (pooled with hisa_pool_blocks at block_size
 * B * group) and superblock_idx [batch, Q, top_m2] is what
 * hisa_block_score_topm returns for them (current super-block forced).  For
 * each query, the fully visible blocks (b < c_t) inside its retained
 * super-blocks are scored with their pooled keys kpool [batch, ceil(L/B), d]
 * (+ kpool_scale for E4M3); block_idx [batch, Q, top_m] receives the current
 * block c_t first, then the top_m-1 best of them by (score desc, block asc),
 * all of them when they fit, -1 padding.  The shape is the indexer's (block
 * size B, top_m m).  Workspace: hisa_workspace_size(HISA_OP_BLOCK_REFINE_TOPM)
 * bytes, 16-byte aligned.  Runs hisa_token_score_topk over the pooled blocks,
 * so its limits apply with block_size = group, top_m = top_m2 and
 * top_k = top_m - 1.
 */
HISA_API hisa_status hisa_block_refine_topm(const void* q, const float* q_scale, const float* w,
                                            const void* kpool, const float* kpool_scale,
                                            const int32_t* n_visible, const int32_t* superblock_idx,
                                            int32_t top_m2, int32_t group, const hisa_shape* shape,
                                            int32_t* block_idx, void* workspace, size_t ws_bytes,
                                            hisa_stream stream);

/*
 * The flat indexer's top-k without score rows, after the sampled-range,
 * write-back-only-promising-candidates scheme of "LITETOPK" (Indexer-TopK
 * abstract): every 16th key (or sparser, so that at most 4096 are sampled) is
 * scored; per query the r-th largest sample score is a threshold at or above
 * which more than k keys lie with overwhelming probability; every key is then
 * scored and only the (position, score) pairs at or above the threshold are
 * written back and selected from.  Queries whose estimate misses (fewer than
 * k pairs, or more than the pair buffer holds) are rescored on CUDA cores.
 * The result is exactly dsa_flat_indexer_topk's; the workspace per query is
 * the sample row plus the pair buffer instead of a full score row.
 * Same arguments, layouts and errors as dsa_flat_indexer_topk; the workspace
 * holds at least hisa_workspace_size(HISA_OP_FLAT_TOPK_SAMPLED) bytes (less
 * runs the queries in chunks).  Tensor-core shapes only (bf16 / E4M3, head_dim
 * x element size of 128 or 256 bytes, H in {16, 32, 64}) whose key count the
 * sample stride divides and whose pair buffer (at most 8192 pairs) is smaller
 * than num_keys; other shapes return HISA_ERR_UNSUPPORTED.
 */
HISA_API hisa_status dsa_flat_indexer_topk_sampled(const void* q, const float* q_scale,
                                          const float* w, const void* k,
                                          const float* k_scale,
                                          const int32_t* n_visible,
                                          const hisa_shape* shape, int32_t* topk_idx,
                                          float* topk_score, void* workspace,
                                          size_t ws_bytes, hisa_stream stream);

/*
 * hisa_block_score_topm without a caller workspace, for callers that cannot
 * allocate device memory when they call the indexer (for example code that
 * runs inside another runtime's memory arena, or a plug-in that is handed only
 * its input and output pointers).  The paper has no counterpart; this is an
 * interface convenience.  Same arguments and results as hisa_block_score_topm
 * minus the workspace.
 *  - The block scores are kept in one 16 MiB array built into the library;
 *    every GPU that loads the library reserves it until the process exits.
 *    Shapes with batch*Q*round_up(ceil(L/B), 4)*4 bytes above 16 MiB return
 *    HISA_ERR_WORKSPACE without launching anything.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *    Each call looks up the array's device address on the current device
 *    (cudaGetSymbolAddress, which allocates nothing); the first call on a
 *    device may load the library's device code there, so make it before any
 *    stream capture.
 *  - All calls share the array and it keeps the last call's contents (nothing
 *    in it needs to start cleared).  Calls that overlap on the GPU, on
 *    different streams or different host threads, race on it: order them.
 */
HISA_API hisa_status hisa_block_score_topm_static(const void* q, const float* q_scale,
                                  const float* w, const void* kpool,
                                  const float* kpool_scale,
                                  const int32_t* n_visible,
                                  const hisa_shape* shape, int32_t* block_idx,
                                  hisa_stream stream);

/*
 * The whole HISA indexer (block pooling, coarse top-m, refinement top-k; HISA
 * abstract, stages 1 and 2) on inputs that live in HOST memory, for callers
 * whose q, keys and weights arrive from the host.  Layouts as for the device
 * entry points, all pointers below HOST pointers:
 *   q          [batch, Q, H, d] in dtype;  q_scale [batch, Q] fp32 (E4M3)
 *   w          [batch, Q, H] fp32
 *   k          [batch, L, d] in dtype;     k_scale [batch, L] fp32 (E4M3)
 *   n_visible  [batch, Q] int32, read by the host during the call
 *   topk_idx   [batch, Q, top_k] int32 (output), -1 padded, any order
 * Page-locked host memory lets the copies overlap the kernels; pageable
 * memory works but serialises them.
 * The work is cut into `pieces` (0 = 16; at most 256) query ranges of one
 * sequence, or ranges of whole sequences, run as a pipeline on three streams
 * of the library's: the host-to-device copy of one piece, the kernels of the
 * previous one and the device-to-host copy of the one before overlap.  A
 * piece copies only the keys its queries see beyond those already copied,
 * and pools only the blocks those keys complete (the coarse stage scores
 * complete blocks only), so the result equals hisa_pool_blocks +
 * hisa_block_score_topm + hisa_token_score_topk on the whole inputs.
 *   workspace  DEVICE memory, 16-byte aligned, of at least
 *              hisa_workspace_size(HISA_OP_INDEXER_FROM_HOST) bytes: the
 *              device copies of every input, the pooled keys, the block and
 *              token indices and the stages' scratch.
 * Ordering: the pipeline starts after the work already enqueued on `stream`,
 * and `stream` waits for the last copy out, so topk_idx is complete once the
 * caller synchronises `stream` (or an event recorded on it after the call).
 * The first call on a device creates the three non-blocking streams and four
 * events it keeps until the process exits (make it before any stream
 * capture); calls are serialised on the host by a lock.  Two calls that share
 * a workspace must be ordered through their streams.
 */
HISA_API hisa_status hisa_indexer_from_host(const void* q, const float* q_scale, const float* w,
                                            const void* k, const float* k_scale,
                                            const int32_t* n_visible, const hisa_shape* shape,
                                            int32_t* topk_idx, int32_t pieces, void* workspace,
                                            size_t ws_bytes, hisa_stream stream);

/*
 * Attention over each query's selected keys: the consumer of the indexer's
 * token-level top-k (HISA abstract: HISA keeps the index interface that the
 * downstream sparse MLA operator reads; the pages give that operator no
 * formula).  Latent attention in absorbed form, one key row per position
 * shared by every head, its first d_v features being the value:
 *     logit[h, j] = scale * q[t, h, :] . kv[s_j, :]
 *     o[t, h, :]  = sum_j softmax_j(logit[h, :]) * kv[s_j, 0 : d_v]
 *     lse[t, h]   = log sum_j exp(logit[h, j])      (natural log)
 * over S_t = the positions in idx[t, :] with -1, out-of-range entries and
 * repeats dropped; an empty S_t gives o = 0 and lse = -inf.
 *   q    [batch, Q, heads, d_qk] bf16 (device)
 *   kv   [batch, L, d_qk] bf16 (device)
 *   idx  [batch, Q, top_k] int32 (device): the indexer's topk_idx
 *   o    [batch, Q, heads, d_v] bf16 (device, output)
 *   lse  [batch, Q, heads] fp32 (device, output)
 * This build takes d_qk = 576, d_v = 512 (512 latent + 64 positional
 * features), heads a multiple of 128 and top_k <= 4096; other shapes return
 * HISA_ERR_UNSUPPORTED.  Each (query, 128-head slice) runs on a cluster of
 * two CTAs; the score tensor [Q, heads, top_k] never leaves the chip.
 */
HISA_API hisa_status hisa_sparse_attention(const void* q, const void* kv, const int32_t* idx,
                                           int32_t batch, int32_t num_queries, int32_t num_keys,
                                           int32_t heads, int32_t d_qk, int32_t d_v, int32_t top_k,
                                           float scale, void* o, float* lse, hisa_stream stream);

/* Workspace bytes that let `op` run on `shape` in one pass (0 if none). */
HISA_API hisa_status hisa_workspace_size(int32_t op, const hisa_shape* shape,
                                size_t* bytes);

/* Synchronises `stream`, then returns and clears the device status word
 * (HISA_OK, or HISA_ERR_TIMEOUT if a bounded wait gave up since the last
 * call); HISA_ERR_CUDA if the synchronisation itself failed. */
HISA_API hisa_status hisa_get_status(hisa_stream stream);

/* Self-test of failure detection: launches one thread that waits, with the
 * same bounded wait the tensor-core kernels use, on a barrier that nothing
 * ever completes; after limit_ns (0 < limit_ns <= 10 s) it gives up and
 * records HISA_ERR_TIMEOUT in the device status word, which the next
 * hisa_get_status() returns (and clears).  Faults nothing: the context stays
 * usable. */
HISA_API hisa_status hisa_selftest_wait_timeout(uint64_t limit_ns, hisa_stream stream);

/* Static description of a status code. */
HISA_API const char* hisa_status_string(hisa_status status);

/* Message of the last validation or CUDA error on the calling thread. */
HISA_API const char* hisa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* HISA_H_ */

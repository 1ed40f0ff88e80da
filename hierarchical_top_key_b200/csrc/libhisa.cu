// libhisa.cu - the C ABI of include/hisa.h: argument validation, workspace
// planning and stream-ordered kernel launches.  Every step of the indexers
// runs in the kernels included below; this file only checks arguments and
// launches them.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <cstdarg>
#include <algorithm>
#include <cmath>
#include <mutex>
#include <vector>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "pool.cuh"
#include "select.cuh"
#include "score_simt.cuh"
#include "score_tc.cuh"
#include "token_tc.cuh"
#include "flat_lite.cuh"
#include "sort.cuh"
#include "sparse_attn.cuh"

using namespace hisa;

namespace {

thread_local char g_last_error[512] = "";

hisa_status fail(hisa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

hisa_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return HISA_OK;
  return fail(HISA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

hisa_status launch_check(const char* what) { return cuda_check(cudaGetLastError(), what); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int elem_bytes(int dt) { return dt == HISA_F32 ? 4 : dt == HISA_BF16 ? 2 : 1; }

constexpr int kMaxCandidates = 16384;   // top_m * block_size held on chip per query
constexpr int kMaxTopM = 256;

hisa_status check_shape(const hisa_shape* s, bool need_blocks) {
  if (!s) return fail(HISA_ERR_INVALID_ARG, "shape is NULL");
  if (s->batch < 1 || s->num_keys < 1 || s->num_queries < 1)
    return fail(HISA_ERR_INVALID_ARG, "batch, num_keys, num_queries must be >= 1");
  if (s->heads < 1 || s->heads > 64) return fail(HISA_ERR_UNSUPPORTED, "heads must be in [1, 64]");
  if (s->head_dim != 64 && s->head_dim != 128) return fail(HISA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (s->dtype != HISA_F32 && s->dtype != HISA_BF16 && s->dtype != HISA_E4M3)
    return fail(HISA_ERR_INVALID_ARG, "unknown dtype %d", s->dtype);
  if (s->top_k < 1) return fail(HISA_ERR_INVALID_ARG, "top_k must be >= 1");
  if (need_blocks) {
    if (s->block_size < 1) return fail(HISA_ERR_INVALID_ARG, "block_size must be >= 1");
    if (s->top_m < 1) return fail(HISA_ERR_INVALID_ARG, "top_m must be >= 1");
  }
  return HISA_OK;
}

int64_t rows_of(const hisa_shape* s) { return static_cast<int64_t>(s->batch) * s->num_queries; }
int64_t pad4(int64_t n) { return (n + 3) / 4 * 4; }
int64_t num_blocks(const hisa_shape* s) { return ceil_div(s->num_keys, s->block_size); }

// ------------------------------------------------------------ dispatch helpers

template <int DT, int HT>
hisa_status launch_score_rows(const hisa_shape* s, const void* q, const float* qsc, const float* w,
                              const void* keys, const float* ksc, const int32_t* nvis, int block_div,
                              int L, int64_t row0, int64_t nrows, float* out, int64_t ld, cudaStream_t st) {
  const int kpc = 2048;
  const size_t smem = SimtTile<DT, HT>::smem_bytes(s->head_dim);
  auto kern = score_rows_simt_kernel<DT, HT>;
  hisa_status e = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  static_cast<int>(smem)), "score_rows attribute");
  if (e != HISA_OK) return e;
  dim3 grid(static_cast<unsigned>(nrows), static_cast<unsigned>(ceil_div(L, kpc)));
  kern<<<grid, kSimtThreads, smem, st>>>(static_cast<const uint8_t*>(q), qsc, w,
                                         static_cast<const uint8_t*>(keys), ksc, nvis, block_div,
                                         s->num_queries, s->heads, s->head_dim, L, row0, out, ld, kpc);
  return launch_check("score_rows_simt_kernel");
}

template <int DT>
hisa_status score_rows_h(const hisa_shape* s, const void* q, const float* qsc, const float* w,
                         const void* keys, const float* ksc, const int32_t* nvis, int block_div, int L,
                         int64_t row0, int64_t nrows, float* out, int64_t ld, cudaStream_t st) {
  if (s->heads <= 4)
    return launch_score_rows<DT, 4>(s, q, qsc, w, keys, ksc, nvis, block_div, L, row0, nrows, out, ld, st);
  if (s->heads <= 16)
    return launch_score_rows<DT, 16>(s, q, qsc, w, keys, ksc, nvis, block_div, L, row0, nrows, out, ld, st);
  return launch_score_rows<DT, 64>(s, q, qsc, w, keys, ksc, nvis, block_div, L, row0, nrows, out, ld, st);
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  }
  return n;
}

// ------------------------------------------------------------ TMA descriptors

PFN_cuTensorMapEncodeTiled_v12000 g_encode_tiled = nullptr;

// A 2D map over [rows, cols] with boxes of box_rows x (128 bytes of columns,
// or box_cols columns), 128-byte swizzle unless another is given.
hisa_status tensor_map_2d(CUtensorMap* map, const void* base, int dtype, uint64_t rows, uint64_t cols,
                          uint32_t box_rows, uint64_t row_stride_elems = 0, uint32_t box_cols = 0,
                          CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  if (!g_encode_tiled) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
      return fail(HISA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const int es = elem_bytes(dtype);
  const CUtensorMapDataType ty = dtype == HISA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {(row_stride_elems ? row_stride_elems : cols) * es};
  cuuint32_t box[2] = {box_cols ? box_cols : static_cast<cuuint32_t>(128 / es), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode_tiled(map, ty, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HISA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return HISA_OK;
}

// A 3D map over [rows, 2 panels of 128 bytes] for 2-panel rows (256 bytes):
// dims {elements per panel, rows, 2}, strides {row bytes, 128 bytes}, boxes of
// box_rows rows x both panels, 128-byte swizzle.  One load of a box fills
// [panel][row][128 B] in shared memory.
hisa_status tensor_map_3d_panels(CUtensorMap* map, const void* base, int dtype, uint64_t rows, uint64_t cols,
                                 uint32_t box_rows) {
  if (!g_encode_tiled) {
    CUtensorMap probe;
    hisa_status e = tensor_map_2d(&probe, base, dtype, rows, cols, 1);   // resolves the entry point
    if (e != HISA_OK) return e;
  }
  const int es = elem_bytes(dtype);
  const uint64_t panel = 128 / es;
  const CUtensorMapDataType ty = dtype == HISA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[3] = {panel, rows, cols / panel};
  cuuint64_t strides[2] = {cols * es, 128};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(panel), box_rows, static_cast<cuuint32_t>(cols / panel)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode_tiled(map, ty, 3, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(HISA_ERR_CUDA, "cuTensorMapEncodeTiled (3D panels) failed (%d)", static_cast<int>(r));
  return HISA_OK;
}

// ------------------------------------------------------------ dense scoring plan

// Tensor-core path: bf16 or E4M3 rows of 128/256 bytes, and H that divides 256
// into whole query groups.
bool dense_tc_ok(const hisa_shape* s) {
  const int rb = s->head_dim * elem_bytes(s->dtype);
  return (s->dtype == HISA_BF16 || s->dtype == HISA_E4M3) && (rb == 128 || rb == 256) &&
         (s->heads == 16 || s->heads == 32 || s->heads == 64);
}

int dense_group(const hisa_shape* s) { return dense_tc_ok(s) ? kDenseN / s->heads : 1; }

struct RowChunk {
  int64_t gg0;
  int ngroups;
  int64_t row0, nrows;
};

// Split the (sequence, query-group) space into chunks whose score rows fit
// in `cap_rows`; every chunk holds whole groups.
hisa_status plan_chunks(const hisa_shape* s, int G, int64_t cap_rows, std::vector<RowChunk>& out) {
  const int64_t gps = ceil_div(s->num_queries, G);
  const int64_t total = gps * s->batch;
  auto row_of = [&](int64_t gg) { return (gg / gps) * s->num_queries + (gg % gps) * G; };
  auto row_end = [&](int64_t gg) {
    return (gg / gps) * s->num_queries + std::min<int64_t>((gg % gps) * G + G, s->num_queries);
  };
  out.clear();
  int64_t gg = 0;
  while (gg < total) {
    const int64_t start = gg, r0 = row_of(gg);
    while (gg < total && row_end(gg) - r0 <= cap_rows && gg - start < (1 << 30)) ++gg;
    if (gg == start) return fail(HISA_ERR_WORKSPACE, "workspace holds fewer score rows than one query group (%d)", G);
    out.push_back({start, static_cast<int>(gg - start), r0, row_end(gg - 1) - r0});
  }
  return HISA_OK;
}

template <int DT, int H>
hisa_status launch_dense_tc(const hisa_shape* s, const CUtensorMap& qmap, const CUtensorMap& kmap, DenseParams p,
                            cudaStream_t st) {
  const int rb = s->head_dim * Elem<DT>::bytes;
  const int tiles_per_group = static_cast<int>(ceil_div(p.L, kDenseTileM));
  const int sms = num_sms();
  if (p.ngroups >= 2 * sms) {
    p.kc_tiles = std::max(tiles_per_group, 1);
  } else {
    p.kc_tiles = static_cast<int>(std::max<int64_t>(2, ceil_div(static_cast<int64_t>(tiles_per_group) * p.ngroups, 4 * sms)));
  }
  p.max_chunks = static_cast<int>(ceil_div(std::max(tiles_per_group, 1), p.kc_tiles));
  if (rb == 256) {
    p.q_bufs = p.kc_tiles > 4 ? 1 : 2;
    p.stages = p.kc_tiles > 4 ? 4 : 2;
  } else {
    p.q_bufs = 2;
    p.stages = 8;
  }
  const size_t smem = dense_smem_bytes(rb, p.stages, p.q_bufs);
  auto kern = dense_score_tc_kernel<DT, H>;
  hisa_status e = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  static_cast<int>(smem)), "dense_score_tc attribute");
  if (e != HISA_OK) return e;
  const int64_t units = static_cast<int64_t>(p.ngroups) * p.max_chunks;
  const int grid = static_cast<int>(std::min<int64_t>(units, sms));
  kern<<<grid, kDenseThreads, smem, st>>>(qmap, kmap, p);
  return launch_check("dense_score_tc_kernel");
}

template <int DT>
hisa_status dense_tc_h(const hisa_shape* s, const CUtensorMap& qm, const CUtensorMap& km, const DenseParams& p,
                       cudaStream_t st) {
  switch (s->heads) {
    case 16: return launch_dense_tc<DT, 16>(s, qm, km, p, st);
    case 32: return launch_dense_tc<DT, 32>(s, qm, km, p, st);
    default: return launch_dense_tc<DT, 64>(s, qm, km, p, st);
  }
}

// Score rows of one chunk: out[(b*Q+t) - row0][s] for the visible keys.
// Tensor-core scoring of one row chunk against every stride-th key (stride >=
// 1), writing score rows (out, ld) or, with `thresh`, compacted pairs.
hisa_status score_rows_tc_mode(const hisa_shape* s, const void* q, const float* qsc, const float* w,
                               const void* keys, const float* ksc, const int32_t* nvis, int stride,
                               const RowChunk& c, float* out, int64_t ld, const uint32_t* thresh, uint2* pairs,
                               uint32_t* counts, int cap, cudaStream_t st) {
  CUtensorMap qm, km;
  const int Lv = s->num_keys / stride;                 // key rows per sequence in the strided view
  hisa_status e = tensor_map_2d(&qm, q, s->dtype, static_cast<uint64_t>(rows_of(s)) * s->heads, s->head_dim, kDenseN);
  if (e != HISA_OK) return e;
  e = tensor_map_2d(&km, keys, s->dtype, static_cast<uint64_t>(s->batch) * Lv, s->head_dim, kDenseTileM,
                    static_cast<uint64_t>(stride) * s->head_dim);
  if (e != HISA_OK) return e;
  DenseParams p{};
  p.Q = s->num_queries; p.H = s->heads; p.d = s->head_dim; p.L = Lv;
  p.G = kDenseN / s->heads;
  p.groups_per_seq = static_cast<int>(ceil_div(s->num_queries, p.G));
  p.block_div = 0;
  p.vis_stride = stride;
  p.gg0 = c.gg0; p.ngroups = c.ngroups; p.row0 = c.row0;
  p.w = w; p.n_visible = nvis; p.q_scale = qsc; p.k_scale = ksc; p.out = out; p.ld = ld; p.minmax = nullptr;
  p.ksc_ld = s->num_keys; p.ksc_step = stride;
  p.thresh = thresh; p.pairs = pairs; p.counts = counts; p.cap = cap;
  return s->dtype == HISA_BF16 ? dense_tc_h<DT_BF16>(s, qm, km, p, st) : dense_tc_h<DT_E4M3>(s, qm, km, p, st);
}

hisa_status score_rows(const hisa_shape* s, const void* q, const float* qsc, const float* w, const void* keys,
                       const float* ksc, const int32_t* nvis, int block_div, int L, const RowChunk& c, float* out,
                       int64_t ld, cudaStream_t st, uint32_t* minmax = nullptr) {
  if (dense_tc_ok(s)) {
    CUtensorMap qm, km;
    hisa_status e = tensor_map_2d(&qm, q, s->dtype, static_cast<uint64_t>(rows_of(s)) * s->heads, s->head_dim, kDenseN);
    if (e != HISA_OK) return e;
    e = tensor_map_2d(&km, keys, s->dtype, static_cast<uint64_t>(s->batch) * L, s->head_dim, kDenseTileM);
    if (e != HISA_OK) return e;
    DenseParams p{};
    p.Q = s->num_queries; p.H = s->heads; p.d = s->head_dim; p.L = L;
    p.G = kDenseN / s->heads;
    p.groups_per_seq = static_cast<int>(ceil_div(s->num_queries, p.G));
    p.block_div = block_div;
    p.gg0 = c.gg0; p.ngroups = c.ngroups; p.row0 = c.row0;
    p.w = w; p.n_visible = nvis; p.q_scale = qsc; p.k_scale = ksc; p.out = out; p.ld = ld; p.minmax = minmax;
    p.ksc_ld = L; p.ksc_step = 1;
    return s->dtype == HISA_BF16 ? dense_tc_h<DT_BF16>(s, qm, km, p, st) : dense_tc_h<DT_E4M3>(s, qm, km, p, st);
  }
  switch (s->dtype) {
    case HISA_F32: return score_rows_h<DT_F32>(s, q, qsc, w, keys, ksc, nvis, block_div, L, c.row0, c.nrows, out, ld, st);
    case HISA_BF16: return score_rows_h<DT_BF16>(s, q, qsc, w, keys, ksc, nvis, block_div, L, c.row0, c.nrows, out, ld, st);
    default: return score_rows_h<DT_E4M3>(s, q, qsc, w, keys, ksc, nvis, block_div, L, c.row0, c.nrows, out, ld, st);
  }
}

template <int DT, int HT>
hisa_status launch_token_simt(const hisa_shape* s, const void* q, const float* qsc, const float* w,
                              const void* k, const float* ksc, const int32_t* nvis, const int32_t* bidx,
                              int32_t* oi, float* os, cudaStream_t st) {
  const size_t smem = SimtTile<DT, HT>::smem_bytes(s->head_dim) +
                      static_cast<size_t>(s->top_m) * s->block_size * sizeof(uint32_t);
  auto kern = token_stage_simt_kernel<DT, HT>;
  hisa_status e = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  static_cast<int>(smem)), "token_stage attribute");
  if (e != HISA_OK) return e;
  kern<<<static_cast<unsigned>(rows_of(s)), kSimtThreads, smem, st>>>(
      static_cast<const uint8_t*>(q), qsc, w, static_cast<const uint8_t*>(k), ksc, nvis, bidx,
      s->num_queries, s->heads, s->head_dim, s->num_keys, s->block_size, s->top_m, s->top_k, oi, os);
  return launch_check("token_stage_simt_kernel");
}

template <int DT>
hisa_status token_simt_h(const hisa_shape* s, const void* q, const float* qsc, const float* w, const void* k,
                         const float* ksc, const int32_t* nvis, const int32_t* bidx, int32_t* oi, float* os,
                         cudaStream_t st) {
  if (s->heads <= 4) return launch_token_simt<DT, 4>(s, q, qsc, w, k, ksc, nvis, bidx, oi, os, st);
  if (s->heads <= 16) return launch_token_simt<DT, 16>(s, q, qsc, w, k, ksc, nvis, bidx, oi, os, st);
  return launch_token_simt<DT, 64>(s, q, qsc, w, k, ksc, nvis, bidx, oi, os, st);
}

constexpr size_t kSmemBudget = 232448;   // 227 KB opt-in dynamic shared memory per CTA
constexpr int kSmemBudgetRows = 200 * 1024;   // shared memory per SM given to resident sorting CTAs

bool token_tc_ok(const hisa_shape* s) {
  const int rb = s->head_dim * elem_bytes(s->dtype);
  if (!((s->dtype == HISA_BF16 || s->dtype == HISA_E4M3) && (rb == 128 || rb == 256) &&
        (s->heads == 16 || s->heads == 32 || s->heads == 64) &&
        (s->block_size == 16 || s->block_size == 32 || s->block_size == 64 || s->block_size == 128) &&
        s->top_m <= kTokMaxBlocks && num_blocks(s) <= 32 * kTokMaxBitmapWords))
    return false;
  // the candidate buffers and two key stages must fit in shared memory; larger
  // m * B go to the CUDA-core kernel
  const int64_t max_cand = ceil_div(static_cast<int64_t>(s->top_m) * s->block_size, kTokTileM) * kTokTileM;
  return token_smem_bytes(rb, s->heads, 2, static_cast<int>(max_cand)) <= kSmemBudget;
}

// Paged keys: block j of sequence b is page table[b * nb + j] of a
// [count, block_size, head_dim] key array (table NULL: keys contiguous).
struct KeyPages {
  const int32_t* table = nullptr;
  int32_t count = 0;
};

template <int DT, int H>
hisa_status launch_token_tc(const hisa_shape* s, const void* q, const float* qsc, const float* w, const void* k,
                            const float* ksc, const int32_t* nvis, const int32_t* bidx, int32_t* oi, float* os,
                            cudaStream_t st, int parts = 1, KeyPages pg = {}) {
  const int rb = s->head_dim * Elem<DT>::bytes;
  TokenParams p{};
  p.rows = rows_of(s);
  p.Q = s->num_queries; p.H = s->heads; p.d = s->head_dim; p.L = s->num_keys; p.B = s->block_size;
  p.top_m = s->top_m; p.top_k = s->top_k;
  p.nb = static_cast<int>(num_blocks(s));
  p.max_cand = static_cast<int>(ceil_div(static_cast<int64_t>(s->top_m) * s->block_size, kTokTileM) * kTokTileM);
  p.parts = parts;
  p.pages = pg.table; p.num_pages = pg.count;
  p.w = w; p.n_visible = nvis; p.block_idx = bidx; p.q_scale = qsc; p.k_scale = ksc; p.out_idx = oi; p.out_score = os;
  if (token_smem_bytes(rb, H, 2, p.max_cand) > kSmemBudget)
    return fail(HISA_ERR_UNSUPPORTED, "top_m * block_size too large for the on-chip candidate buffers");
  // key stages: as many as fit, up to 96 KB of tiles in flight (three bf16
  // tiles of d = 128; a fourth was 3 % slower at 32K keys, measured)
  const int max_stages = std::max(3, static_cast<int>(98304 / (kTokTileM * rb)));
  p.stages = 2;
  while (p.stages < max_stages && token_smem_bytes(rb, H, p.stages + 1, p.max_cand) <= kSmemBudget) ++p.stages;
  const size_t smem = token_smem_bytes(rb, H, p.stages, p.max_cand);
  CUtensorMap qm, km;
  hisa_status e = tensor_map_2d(&qm, q, s->dtype, static_cast<uint64_t>(p.rows) * H, s->head_dim, H);
  if (e != HISA_OK) return e;
  const uint64_t key_rows = pg.table ? static_cast<uint64_t>(pg.count) * s->block_size
                                    : static_cast<uint64_t>(s->batch) * s->num_keys;
  // a 128-key block of 256-byte rows is one load of both panels
  p.k3d = s->block_size == kTokTileM && rb == 256;
  e = p.k3d ? tensor_map_3d_panels(&km, k, s->dtype, key_rows, s->head_dim, s->block_size)
            : tensor_map_2d(&km, k, s->dtype, key_rows, s->head_dim, s->block_size);
  if (e != HISA_OK) return e;
  auto kern = token_tc_kernel<DT, H>;
  e = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)),
                 "token_tc attribute");
  if (e != HISA_OK) return e;
  const int grid = static_cast<int>(std::min<int64_t>(p.rows * parts, num_sms()));
  kern<<<grid, kTokThreads, smem, st>>>(qm, km, p);
  return launch_check("token_tc_kernel");
}

template <int DT>
hisa_status token_tc_h(const hisa_shape* s, const void* q, const float* qsc, const float* w, const void* k,
                       const float* ksc, const int32_t* nvis, const int32_t* bidx, int32_t* oi, float* os,
                       cudaStream_t st, int parts = 1, KeyPages pg = {}) {
  switch (s->heads) {
    case 16: return launch_token_tc<DT, 16>(s, q, qsc, w, k, ksc, nvis, bidx, oi, os, st, parts, pg);
    case 32: return launch_token_tc<DT, 32>(s, q, qsc, w, k, ksc, nvis, bidx, oi, os, st, parts, pg);
    default: return launch_token_tc<DT, 64>(s, q, qsc, w, k, ksc, nvis, bidx, oi, os, st, parts, pg);
  }
}

// Jobs per query of the tensor-core refinement stage: with few queries (a
// decode step) each query's retained blocks are split over several CTAs, whose
// top-k lists are merged exactly afterwards, so that more SMs gather keys.
int token_parts(const hisa_shape* s) {
  const int64_t rows = rows_of(s);
  const int sms = num_sms();
  if (!token_tc_ok(s) || rows * 2 > sms) return 1;
  int parts = static_cast<int>(std::min<int64_t>({4, sms / rows, static_cast<int64_t>(s->top_m)}));
  while (parts > 1 && static_cast<int64_t>(parts) * s->top_k > 8192) --parts;   // merge holds 8192 per row
  return std::max(parts, 1);
}

size_t token_split_bytes(const hisa_shape* s, int parts) {
  return parts > 1 ? static_cast<size_t>(rows_of(s)) * parts * s->top_k * 8 : 0;
}

size_t host_pipe_bytes(const hisa_shape* s);   // device workspace of hisa_indexer_from_host

// ------------------------------------------------------------ flat top-k without score rows

struct LitePlan {
  int stride;        // every stride-th key is sampled
  int r_target;      // the threshold is the r_target-th largest sample score
  int cap;           // pairs kept per query
  int64_t sld;       // sample scores per row (padded)
  int fb_ctas;       // CTAs (scratch rows) of the fallback
  size_t fixed;      // workspace bytes independent of the chunk: counter + fallback scratch
  size_t per_row;    // workspace bytes per row
};

// The sampled-threshold flat path applies to tensor-core shapes whose key
// count the sample stride divides and whose pair buffer would be smaller
// than the visible prefix; r_target and cap put the chance that fewer than k
// or more than cap keys pass the threshold several standard deviations out
// under uniform sampling (a miss only costs the fallback).
bool lite_plan(const hisa_shape* s, LitePlan* lp) {
  if (!dense_tc_ok(s)) return false;
  const int L = s->num_keys, k = s->top_k;
  int stride = 16;
  while (L / stride > 4096) stride *= 2;
  if (L % stride != 0 || L / stride < 1) return false;
  const double kr = static_cast<double>(k) / stride;
  const int r = static_cast<int>(std::ceil(kr + 6.0 * std::sqrt(kr))) + 2;
  int cap = static_cast<int>(std::ceil(r * static_cast<double>(stride) + 8.0 * stride * std::sqrt(static_cast<double>(r))));
  cap = (cap + 63) / 64 * 64;
  if (cap > 8192 || cap >= L) return false;
  lp->stride = stride;
  lp->r_target = r;
  lp->cap = cap;
  lp->sld = pad4(L / stride);
  lp->fb_ctas = std::min(num_sms(), 32);
  lp->fixed = 256 + static_cast<size_t>(lp->fb_ctas) * L * 4 + 16;   // + alignment of the pair buffer
  lp->per_row = static_cast<size_t>(lp->sld) * 4 + 12 + static_cast<size_t>(cap) * 8;
  return true;
}

template <int DT>
hisa_status launch_flat_fallback(const hisa_shape* s, const void* q, const float* qsc, const float* w, const void* k,
                                 const float* ksc, const int32_t* nvis, int64_t row0, const uint32_t* fail_count,
                                 const int32_t* fail_rows, float* scratch, int fb_ctas, int32_t* oi, float* os,
                                 cudaStream_t st) {
  auto run = [&](auto kern, size_t smem) {
    hisa_status e = cuda_check(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    static_cast<int>(smem)), "flat_fallback attribute");
    if (e != HISA_OK) return e;
    kern<<<fb_ctas, kSimtThreads, smem, st>>>(static_cast<const uint8_t*>(q), qsc, w, static_cast<const uint8_t*>(k),
                                              ksc, nvis, row0, s->num_queries, s->heads, s->head_dim, s->num_keys,
                                              s->top_k, fail_count, fail_rows, scratch, oi, os);
    return launch_check("flat_fallback_kernel");
  };
  if (s->heads <= 16) return run(flat_fallback_kernel<DT, 16>, SimtTile<DT, 16>::smem_bytes(s->head_dim));
  return run(flat_fallback_kernel<DT, 64>, SimtTile<DT, 64>::smem_bytes(s->head_dim));
}

hisa_status flat_lite(const hisa_shape* s, const LitePlan& lp, const void* q, const float* qsc, const float* w,
                      const void* k, const float* ksc, const int32_t* nvis, int32_t* oi, float* os, void* workspace,
                      size_t ws_bytes, cudaStream_t st) {
  const int64_t rows = rows_of(s);
  const int64_t cap_rows = static_cast<int64_t>((ws_bytes - lp.fixed) / lp.per_row);
  std::vector<RowChunk> chunks;
  hisa_status e = plan_chunks(s, dense_group(s), std::min<int64_t>(rows, cap_rows), chunks);
  if (e != HISA_OK) return e;
  int64_t R = 0;
  for (const RowChunk& c : chunks) R = std::max(R, c.nrows);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint32_t* fail_count = reinterpret_cast<uint32_t*>(base);
  float* scratch = reinterpret_cast<float*>(base + 256);
  uint8_t* p = base + lp.fixed;
  float* sample = reinterpret_cast<float*>(p);                      p += static_cast<size_t>(R) * lp.sld * 4;
  uint32_t* thresh = reinterpret_cast<uint32_t*>(p);                p += static_cast<size_t>(R) * 4;
  uint32_t* counts = reinterpret_cast<uint32_t*>(p);                p += static_cast<size_t>(R) * 4;
  int32_t* fail_rows = reinterpret_cast<int32_t*>(p);               p += static_cast<size_t>(R) * 4;
  uint2* pairs = reinterpret_cast<uint2*>((reinterpret_cast<uintptr_t>(p) + 7) & ~uintptr_t(7));
  const int sms = num_sms();
  for (const RowChunk& c : chunks) {
    e = cuda_check(cudaMemsetAsync(counts, 0, static_cast<size_t>(c.nrows) * 4, st), "clear pair counts");
    if (e != HISA_OK) return e;
    e = cuda_check(cudaMemsetAsync(fail_count, 0, 4, st), "clear fallback count");
    if (e != HISA_OK) return e;
    e = score_rows_tc_mode(s, q, qsc, w, k, ksc, nvis, lp.stride, c, sample, lp.sld, nullptr, nullptr, nullptr, 0, st);
    if (e != HISA_OK) return e;
    const unsigned tgrid = static_cast<unsigned>(std::min<int64_t>(c.nrows, static_cast<int64_t>(sms) * 16));
    flat_thresh_kernel<32><<<tgrid, 128, 0, st>>>(sample, lp.sld, nvis, c.row0, c.nrows, s->num_keys, lp.stride, lp.cap,
                                                  lp.r_target, thresh);
    e = launch_check("flat_thresh_kernel");
    if (e != HISA_OK) return e;
    e = score_rows_tc_mode(s, q, qsc, w, k, ksc, nvis, 1, c, nullptr, 0, thresh, pairs, counts, lp.cap, st);
    if (e != HISA_OK) return e;
    const unsigned sgrid = static_cast<unsigned>(std::min<int64_t>(c.nrows, static_cast<int64_t>(sms) * 8));
    if (lp.cap <= 256 * 16)
      flat_pairs_select_kernel<16><<<sgrid, 256, 0, st>>>(pairs, counts, lp.cap, nvis, c.row0, c.nrows, s->num_keys,
                                                          s->top_k, oi, os, fail_count, fail_rows);
    else
      flat_pairs_select_kernel<32><<<sgrid, 256, 0, st>>>(pairs, counts, lp.cap, nvis, c.row0, c.nrows, s->num_keys,
                                                          s->top_k, oi, os, fail_count, fail_rows);
    e = launch_check("flat_pairs_select_kernel");
    if (e != HISA_OK) return e;
    e = s->dtype == HISA_BF16
            ? launch_flat_fallback<DT_BF16>(s, q, qsc, w, k, ksc, nvis, c.row0, fail_count, fail_rows, scratch,
                                            lp.fb_ctas, oi, os, st)
            : launch_flat_fallback<DT_E4M3>(s, q, qsc, w, k, ksc, nvis, c.row0, fail_count, fail_rows, scratch,
                                            lp.fb_ctas, oi, os, st);
    if (e != HISA_OK) return e;
  }
  return HISA_OK;
}

hisa_status check_indexer_ptrs(const hisa_shape* s, const void* q, const float* q_scale, const float* w,
                               const void* k, const float* k_scale, const int32_t* n_visible) {
  if (!q || !w || !k || !n_visible) return fail(HISA_ERR_INVALID_ARG, "q, w, keys and n_visible must be non-NULL");
  if (!aligned16(q) || !aligned16(k)) return fail(HISA_ERR_INVALID_ARG, "q and keys must be 16-byte aligned");
  if (!aligned4(w) || !aligned4(n_visible)) return fail(HISA_ERR_INVALID_ARG, "w and n_visible must be 4-byte aligned");
  if (s->dtype == HISA_E4M3 && (!q_scale || !k_scale))
    return fail(HISA_ERR_INVALID_ARG, "E4M3 inputs need q_scale and k_scale");
  return HISA_OK;
}

// Scored outputs are returned sorted by (score desc, index asc); rows longer
// than the on-chip sort are refused up front, before anything is launched.
hisa_status check_scored_rows(const hisa_shape* s, const float* topk_score) {
  if (topk_score && s->top_k > kSortMaxK)
    return fail(HISA_ERR_UNSUPPORTED, "with topk_score, top_k must be <= %d (rows are sorted on chip)", kSortMaxK);
  if (topk_score && !aligned4(topk_score)) return fail(HISA_ERR_INVALID_ARG, "topk_score must be 4-byte aligned");
  return HISA_OK;
}

hisa_status sort_scored_rows(int32_t* idx, float* score, int64_t rows, int k, cudaStream_t st) {
  if (!score || rows == 0) return HISA_OK;
  const int n = sort_pow2(k);
  const int smem = n * static_cast<int>(sizeof(uint64_t));
  hisa_status e = cuda_check(cudaFuncSetAttribute(sort_scored_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  smem), "sort_scored_rows attribute");
  if (e != HISA_OK) return e;
  const int per_sm = std::max(1, std::min(8, static_cast<int>(kSmemBudgetRows / std::max(smem, 1))));
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(rows, static_cast<int64_t>(num_sms()) * per_sm));
  sort_scored_rows_kernel<<<grid, kSortThreads, smem, st>>>(idx, score, rows, k, n);
  return launch_check("sort_scored_rows_kernel");
}

// The refinement stage after argument checks: split queries with the merge,
// the tensor-core kernel, or (contiguous keys only) the CUDA-core kernel.
hisa_status token_score_topk_unsorted(const void* q, const float* q_scale, const float* w, const void* k,
                                      const float* k_scale, const int32_t* n_visible, const int32_t* block_idx,
                                      const hisa_shape* s, int32_t* topk_idx, float* topk_score, void* workspace,
                                      size_t ws_bytes, hisa_stream stream, KeyPages pg);

hisa_status token_score_topk_checked(const void* q, const float* q_scale, const float* w, const void* k,
                                     const float* k_scale, const int32_t* n_visible, const int32_t* block_idx,
                                     const hisa_shape* s, int32_t* topk_idx, float* topk_score, void* workspace,
                                     size_t ws_bytes, hisa_stream stream, KeyPages pg) {
  hisa_status e = token_score_topk_unsorted(q, q_scale, w, k, k_scale, n_visible, block_idx, s, topk_idx, topk_score,
                                            workspace, ws_bytes, stream, pg);
  if (e != HISA_OK) return e;
  return sort_scored_rows(topk_idx, topk_score, rows_of(s), s->top_k, reinterpret_cast<cudaStream_t>(stream));
}

hisa_status token_score_topk_unsorted(const void* q, const float* q_scale, const float* w, const void* k,
                                      const float* k_scale, const int32_t* n_visible, const int32_t* block_idx,
                                      const hisa_shape* s, int32_t* topk_idx, float* topk_score, void* workspace,
                                      size_t ws_bytes, hisa_stream stream, KeyPages pg) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int parts = token_parts(s);
  if (parts > 1 && workspace && aligned16(workspace) && ws_bytes >= token_split_bytes(s, parts)) {
    // split queries: every part's top-k with scores into the workspace, then the exact merge
    const int64_t rows = rows_of(s);
    int32_t* pidx = static_cast<int32_t*>(workspace);
    float* psc = reinterpret_cast<float*>(pidx + rows * parts * s->top_k);
    hisa_status e = s->dtype == HISA_BF16
            ? token_tc_h<DT_BF16>(s, q, q_scale, w, k, k_scale, n_visible, block_idx, pidx, psc, st, parts, pg)
            : token_tc_h<DT_E4M3>(s, q, q_scale, w, k, k_scale, n_visible, block_idx, pidx, psc, st, parts, pg);
    if (e != HISA_OK) return e;
    const int items = parts * s->top_k;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(rows, num_sms() * 4));
    if (items <= 256 * 8)
      merge_parts_kernel<8><<<grid, 256, 0, st>>>(pidx, psc, parts, rows, s->top_k, topk_idx, topk_score);
    else if (items <= 256 * 16)
      merge_parts_kernel<16><<<grid, 256, 0, st>>>(pidx, psc, parts, rows, s->top_k, topk_idx, topk_score);
    else
      merge_parts_kernel<32><<<grid, 256, 0, st>>>(pidx, psc, parts, rows, s->top_k, topk_idx, topk_score);
    return launch_check("merge_parts_kernel");
  }
  if (token_tc_ok(s)) {
    return s->dtype == HISA_BF16
               ? token_tc_h<DT_BF16>(s, q, q_scale, w, k, k_scale, n_visible, block_idx, topk_idx, topk_score, st, 1, pg)
               : token_tc_h<DT_E4M3>(s, q, q_scale, w, k, k_scale, n_visible, block_idx, topk_idx, topk_score, st, 1, pg);
  }
  if (pg.table)
    return fail(HISA_ERR_UNSUPPORTED,
                "paged keys need a tensor-core shape: bf16 or E4M3, head_dim * bytes 128 or 256, H 16/32/64, "
                "B 16..128, top_m * B within the on-chip candidate buffers");
  switch (s->dtype) {
    case HISA_F32: return token_simt_h<DT_F32>(s, q, q_scale, w, k, k_scale, n_visible, block_idx, topk_idx, topk_score, st);
    case HISA_BF16: return token_simt_h<DT_BF16>(s, q, q_scale, w, k, k_scale, n_visible, block_idx, topk_idx, topk_score, st);
    default: return token_simt_h<DT_E4M3>(s, q, q_scale, w, k, k_scale, n_visible, block_idx, topk_idx, topk_score, st);
  }
}


}  // namespace

// Self-test of the bounded-wait path: one thread waits on a barrier that no
// one arrives at; the wait gives up after `limit_ns` and records the timeout.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
    (void)sm100::mbar_wait(&bar, 0, &abort_flag, limit_ns);
  }
}

// =================================================================== C ABI

extern "C" {

const char* hisa_status_string(hisa_status st) {
  switch (st) {
    case HISA_OK: return "HISA_OK";
    case HISA_ERR_INVALID_ARG: return "HISA_ERR_INVALID_ARG: invalid argument";
    case HISA_ERR_UNSUPPORTED: return "HISA_ERR_UNSUPPORTED: shape not supported by this build";
    case HISA_ERR_WORKSPACE: return "HISA_ERR_WORKSPACE: workspace too small";
    case HISA_ERR_CUDA: return "HISA_ERR_CUDA: CUDA runtime error";
    case HISA_ERR_TIMEOUT: return "HISA_ERR_TIMEOUT: a device-side bounded wait gave up";
  }
  return "unknown hisa_status";
}

const char* hisa_last_error(void) { return g_last_error; }

hisa_status hisa_selftest_wait_timeout(uint64_t limit_ns, hisa_stream stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull) return fail(HISA_ERR_INVALID_ARG, "limit_ns must be in (0, 10 s]");
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
  return launch_check("selftest_wait_kernel");
}

hisa_status hisa_get_status(hisa_stream stream) {
  hisa_status e = cuda_check(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)), "stream sync");
  if (e != HISA_OK) return e;
  int v = 0, zero = 0;
  e = cuda_check(cudaMemcpyFromSymbol(&v, g_status, sizeof(int)), "read status word");
  if (e != HISA_OK) return e;
  if (v != 0) {
    e = cuda_check(cudaMemcpyToSymbol(g_status, &zero, sizeof(int)), "clear status word");
    if (e != HISA_OK) return e;
    return fail(static_cast<hisa_status>(v), "device status word reported %d", v);
  }
  return HISA_OK;
}

hisa_status hisa_workspace_size(int32_t op, const hisa_shape* s, size_t* bytes) {
  if (!bytes) return fail(HISA_ERR_INVALID_ARG, "bytes is NULL");
  hisa_status e = check_shape(s, op != HISA_OP_FLAT_TOPK && op != HISA_OP_FLAT_TOPK_SAMPLED);
  if (e != HISA_OK) return e;
  switch (op) {
    case HISA_OP_FLAT_TOPK: *bytes = static_cast<size_t>(rows_of(s) * (pad4(s->num_keys) * 4 + 8)); return HISA_OK;
    case HISA_OP_BLOCK_SCORE_TOPM: *bytes = static_cast<size_t>(rows_of(s) * pad4(num_blocks(s)) * 4); return HISA_OK;
    case HISA_OP_TOKEN_SCORE_TOPK: *bytes = token_split_bytes(s, token_parts(s)); return HISA_OK;
    case HISA_OP_BLOCK_REFINE_TOPM:
      *bytes = static_cast<size_t>(pad4(rows_of(s)) * 4 + rows_of(s) * std::max(s->top_m - 1, 1) * 4);
      return HISA_OK;
    case HISA_OP_INDEXER_FROM_HOST: *bytes = host_pipe_bytes(s); return HISA_OK;
    case HISA_OP_FLAT_TOPK_SAMPLED: {
      LitePlan lp;
      if (!lite_plan(s, &lp)) return fail(HISA_ERR_UNSUPPORTED, "shape not supported by the sampled flat top-k");
      *bytes = lp.fixed + lp.per_row * static_cast<size_t>(rows_of(s));
      return HISA_OK;
    }
  }
  return fail(HISA_ERR_INVALID_ARG, "unknown op %d", op);
}

hisa_status hisa_pool_blocks(const void* k, const float* k_scale, void* kpool, float* kpool_scale,
                             const hisa_shape* s, hisa_stream stream) {
  if (!s) return fail(HISA_ERR_INVALID_ARG, "shape is NULL");
  return hisa_pool_blocks_range(k, k_scale, kpool, kpool_scale, s, 0, static_cast<int32_t>(num_blocks(s)), stream);
}

hisa_status hisa_pool_blocks_range(const void* k, const float* k_scale, void* kpool, float* kpool_scale,
                                   const hisa_shape* s, int32_t first_block, int32_t block_count, hisa_stream stream) {
  if (!s) return fail(HISA_ERR_INVALID_ARG, "shape is NULL");
  if (first_block < 0 || block_count < 0) return fail(HISA_ERR_INVALID_ARG, "first_block and block_count must be >= 0");
  if (s->batch < 1 || s->num_keys < 1 || s->block_size < 1)
    return fail(HISA_ERR_INVALID_ARG, "batch, num_keys, block_size must be >= 1");
  if (s->head_dim != 64 && s->head_dim != 128) return fail(HISA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (!k || !kpool || !aligned16(k) || !aligned16(kpool))
    return fail(HISA_ERR_INVALID_ARG, "k and kpool must be non-NULL and 16-byte aligned");
  if (s->dtype == HISA_E4M3 && (!k_scale || !kpool_scale))
    return fail(HISA_ERR_INVALID_ARG, "E4M3 pooling needs k_scale and kpool_scale");
  const int nb = static_cast<int>(num_blocks(s));
  const int first = std::min(first_block, nb);
  const int count = std::min(block_count, nb - first);
  if (count == 0) return HISA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t threads_total = static_cast<int64_t>(s->batch) * count * (s->head_dim * elem_bytes(s->dtype) / 16);
  const int grid = static_cast<int>(std::min<int64_t>(ceil_div(threads_total, 256), 148 * 64));
  const uint8_t* in = static_cast<const uint8_t*>(k);
  uint8_t* out = static_cast<uint8_t*>(kpool);
  if (s->block_size >= 512) {
    // long groups (super-blocks): one CTA per pooled row, the rows split over its threads
    const int wgrid = static_cast<int>(std::min<int64_t>(static_cast<int64_t>(s->batch) * count, num_sms() * 8));
    switch (s->dtype) {
      case HISA_F32:
        segment_mean_wide_kernel<DT_F32><<<wgrid, 256, 0, st>>>(in, nullptr, out, nullptr, s->batch, s->num_keys, nb,
                                                                s->head_dim, s->block_size, first, count);
        break;
      case HISA_BF16:
        segment_mean_wide_kernel<DT_BF16><<<wgrid, 256, 0, st>>>(in, nullptr, out, nullptr, s->batch, s->num_keys,
                                                                 nb, s->head_dim, s->block_size, first, count);
        break;
      case HISA_E4M3:
        segment_mean_wide_kernel<DT_E4M3><<<wgrid, 256, 0, st>>>(in, k_scale, out, kpool_scale, s->batch,
                                                                 s->num_keys, nb, s->head_dim, s->block_size, first,
                                                                 count);
        break;
      default: return fail(HISA_ERR_INVALID_ARG, "unknown dtype %d", s->dtype);
    }
    return launch_check("segment_mean_wide_kernel");
  }
  switch (s->dtype) {
    case HISA_F32:
      segment_mean_kernel<DT_F32><<<grid, 256, 0, st>>>(in, nullptr, out, nullptr, s->batch, s->num_keys, nb,
                                                        s->head_dim, s->block_size, first, count);
      break;
    case HISA_BF16:
      segment_mean_kernel<DT_BF16><<<grid, 256, 0, st>>>(in, nullptr, out, nullptr, s->batch, s->num_keys, nb,
                                                         s->head_dim, s->block_size, first, count);
      break;
    case HISA_E4M3:
      segment_mean_kernel<DT_E4M3><<<grid, 256, 0, st>>>(in, k_scale, out, kpool_scale, s->batch, s->num_keys,
                                                         nb, s->head_dim, s->block_size, first, count);
      break;
    default: return fail(HISA_ERR_INVALID_ARG, "unknown dtype %d", s->dtype);
  }
  return launch_check("segment_mean_kernel");
}

hisa_status hisa_compress_keys(const void* k_raw, void* ck, int32_t batch, int32_t num_raw_keys,
                               int32_t head_dim, int32_t ratio, int32_t dtype, hisa_stream stream) {
  if (batch < 1 || num_raw_keys < 1 || ratio < 1) return fail(HISA_ERR_INVALID_ARG, "batch, num_raw_keys, ratio must be >= 1");
  if (head_dim != 64 && head_dim != 128) return fail(HISA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (dtype != HISA_F32 && dtype != HISA_BF16) return fail(HISA_ERR_UNSUPPORTED, "compression takes fp32 or bf16 keys");
  if (!k_raw || !ck || !aligned16(k_raw) || !aligned16(ck))
    return fail(HISA_ERR_INVALID_ARG, "k_raw and ck must be non-NULL and 16-byte aligned");
  const int n_out = num_raw_keys / ratio;
  if (n_out == 0) return HISA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t threads_total = static_cast<int64_t>(batch) * n_out * (head_dim * elem_bytes(dtype) / 16);
  const int grid = static_cast<int>(std::min<int64_t>(ceil_div(threads_total, 256), 148 * 64));
  // the input is viewed as n_out * ratio rows per sequence: the dropped tail
  // rows are skipped by giving each sequence its true row count
  const uint8_t* in = static_cast<const uint8_t*>(k_raw);
  uint8_t* out = static_cast<uint8_t*>(ck);
  if (dtype == HISA_F32)
    segment_mean_kernel<DT_F32><<<grid, 256, 0, st>>>(in, nullptr, out, nullptr, batch, num_raw_keys, n_out,
                                                      head_dim, ratio, 0, n_out);
  else
    segment_mean_kernel<DT_BF16><<<grid, 256, 0, st>>>(in, nullptr, out, nullptr, batch, num_raw_keys, n_out,
                                                       head_dim, ratio, 0, n_out);
  return launch_check("segment_mean_kernel (compress)");
}

hisa_status hisa_quantize_e4m3(const void* x, int32_t x_dtype, int64_t rows, int32_t cols, uint8_t* codes,
                               float* scale, hisa_stream stream) {
  if (rows < 0 || cols < 1) return fail(HISA_ERR_INVALID_ARG, "rows must be >= 0 and cols >= 1");
  if (cols % 16 != 0) return fail(HISA_ERR_UNSUPPORTED, "cols must be a multiple of 16");
  if (!x || !codes || !scale || !aligned16(x) || !aligned16(codes) || !aligned4(scale))
    return fail(HISA_ERR_INVALID_ARG, "x/codes must be 16-byte aligned, scale 4-byte aligned, all non-NULL");
  if (rows == 0) return HISA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int grid = static_cast<int>(std::min<int64_t>(ceil_div(rows, 8), 148 * 32));
  const uint8_t* in = static_cast<const uint8_t*>(x);
  if (x_dtype == HISA_F32) quantize_rows_kernel<DT_F32><<<grid, 256, 0, st>>>(in, rows, cols, codes, scale);
  else if (x_dtype == HISA_BF16) quantize_rows_kernel<DT_BF16><<<grid, 256, 0, st>>>(in, rows, cols, codes, scale);
  else return fail(HISA_ERR_UNSUPPORTED, "quantisation input must be fp32 or bf16");
  return launch_check("quantize_rows_kernel");
}

hisa_status hisa_block_score_topm(const void* q, const float* q_scale, const float* w, const void* kpool,
                                  const float* kpool_scale, const int32_t* n_visible, const hisa_shape* s,
                                  int32_t* block_idx, void* workspace, size_t ws_bytes, hisa_stream stream) {
  hisa_status e = check_shape(s, true);
  if (e != HISA_OK) return e;
  e = check_indexer_ptrs(s, q, q_scale, w, kpool, kpool_scale, n_visible);
  if (e != HISA_OK) return e;
  if (!block_idx || !aligned4(block_idx)) return fail(HISA_ERR_INVALID_ARG, "block_idx must be non-NULL, 4-byte aligned");
  const int64_t nb = num_blocks(s);
  const int64_t ld = pad4(nb);
  const int64_t rows = rows_of(s);
  if (!workspace || !aligned16(workspace)) return fail(HISA_ERR_WORKSPACE, "workspace must be non-NULL, 16-byte aligned");
  std::vector<RowChunk> chunks;
  e = plan_chunks(s, dense_group(s), std::min<int64_t>(rows, static_cast<int64_t>(ws_bytes / (ld * 4))), chunks);
  if (e != HISA_OK) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  for (const RowChunk& c : chunks) {
    e = score_rows(s, q, q_scale, w, kpool, kpool_scale, n_visible, s->block_size, static_cast<int>(nb), c, ws, ld, st);
    if (e != HISA_OK) return e;
    const int grid = static_cast<int>(std::min<int64_t>(ceil_div(c.nrows, 8), static_cast<int64_t>(num_sms()) * 8));
    if (nb <= 32 * 8) {
      block_select_warp_kernel<8><<<grid, 256, 0, st>>>(ws, ld, n_visible, c.row0, c.nrows, s->num_keys,
                                                        s->block_size, s->top_m, block_idx);
    } else if (nb <= 32 * 16) {
      block_select_warp_kernel<16><<<grid, 256, 0, st>>>(ws, ld, n_visible, c.row0, c.nrows, s->num_keys,
                                                         s->block_size, s->top_m, block_idx);
    } else if (nb <= 32 * 32) {
      block_select_warp_kernel<32><<<grid, 256, 0, st>>>(ws, ld, n_visible, c.row0, c.nrows, s->num_keys,
                                                         s->block_size, s->top_m, block_idx);
    } else {
      block_select_kernel<<<static_cast<unsigned>(c.nrows), 512, 0, st>>>(ws, ld, n_visible, c.row0, s->num_keys,
                                                                          s->block_size, s->top_m, block_idx);
    }
    e = launch_check("block_select_kernel");
    if (e != HISA_OK) return e;
  }
  return HISA_OK;
}

hisa_status hisa_token_score_topk(const void* q, const float* q_scale, const float* w, const void* k,
                                  const float* k_scale, const int32_t* n_visible, const int32_t* block_idx,
                                  const hisa_shape* s, int32_t* topk_idx, float* topk_score, void* workspace,
                                  size_t ws_bytes, hisa_stream stream) {
  hisa_status e = check_shape(s, true);
  if (e != HISA_OK) return e;
  e = check_indexer_ptrs(s, q, q_scale, w, k, k_scale, n_visible);
  if (e != HISA_OK) return e;
  if (!block_idx || !topk_idx) return fail(HISA_ERR_INVALID_ARG, "block_idx and topk_idx must be non-NULL");
  if (s->top_m > kMaxTopM) return fail(HISA_ERR_UNSUPPORTED, "top_m must be <= %d", kMaxTopM);
  if (static_cast<int64_t>(s->top_m) * s->block_size > kMaxCandidates)
    return fail(HISA_ERR_UNSUPPORTED, "top_m * block_size must be <= %d", kMaxCandidates);
  e = check_scored_rows(s, topk_score);
  if (e != HISA_OK) return e;
  return token_score_topk_checked(q, q_scale, w, k, k_scale, n_visible, block_idx, s, topk_idx, topk_score,
                                  workspace, ws_bytes, stream, KeyPages{});
}

hisa_status hisa_token_score_topk_paged(const void* q, const float* q_scale, const float* w, const void* k_pages,
                                        const float* k_page_scale, const int32_t* page_table, int32_t num_pages,
                                        const int32_t* n_visible, const int32_t* block_idx, const hisa_shape* s,
                                        int32_t* topk_idx, float* topk_score, void* workspace, size_t ws_bytes,
                                        hisa_stream stream) {
  hisa_status e = check_shape(s, true);
  if (e != HISA_OK) return e;
  e = check_indexer_ptrs(s, q, q_scale, w, k_pages, k_page_scale, n_visible);
  if (e != HISA_OK) return e;
  if (!block_idx || !topk_idx) return fail(HISA_ERR_INVALID_ARG, "block_idx and topk_idx must be non-NULL");
  if (!page_table || !aligned4(page_table)) return fail(HISA_ERR_INVALID_ARG, "page_table must be non-NULL and 4-byte aligned");
  if (num_pages < 1) return fail(HISA_ERR_INVALID_ARG, "num_pages must be >= 1");
  if (static_cast<int64_t>(num_pages) * s->block_size > INT32_MAX)
    return fail(HISA_ERR_UNSUPPORTED, "num_pages * block_size must fit in int32");
  if (s->top_m > kMaxTopM) return fail(HISA_ERR_UNSUPPORTED, "top_m must be <= %d", kMaxTopM);
  if (static_cast<int64_t>(s->top_m) * s->block_size > kMaxCandidates)
    return fail(HISA_ERR_UNSUPPORTED, "top_m * block_size must be <= %d", kMaxCandidates);
  e = check_scored_rows(s, topk_score);
  if (e != HISA_OK) return e;
  return token_score_topk_checked(q, q_scale, w, k_pages, k_page_scale, n_visible, block_idx, s, topk_idx,
                                  topk_score, workspace, ws_bytes, stream, KeyPages{page_table, num_pages});
}

hisa_status hisa_pool_blocks_paged(const void* k_pages, const float* k_page_scale, const int32_t* page_table,
                                   int32_t num_pages, void* kpool, float* kpool_scale, const hisa_shape* s,
                                   int32_t first_block, int32_t block_count, hisa_stream stream) {
  if (!s) return fail(HISA_ERR_INVALID_ARG, "shape is NULL");
  if (first_block < 0 || block_count < 0) return fail(HISA_ERR_INVALID_ARG, "first_block and block_count must be >= 0");
  if (s->batch < 1 || s->num_keys < 1 || s->block_size < 1)
    return fail(HISA_ERR_INVALID_ARG, "batch, num_keys, block_size must be >= 1");
  if (s->head_dim != 64 && s->head_dim != 128) return fail(HISA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (!k_pages || !kpool || !aligned16(k_pages) || !aligned16(kpool))
    return fail(HISA_ERR_INVALID_ARG, "k_pages and kpool must be non-NULL and 16-byte aligned");
  if (!page_table || !aligned4(page_table)) return fail(HISA_ERR_INVALID_ARG, "page_table must be non-NULL and 4-byte aligned");
  if (num_pages < 1) return fail(HISA_ERR_INVALID_ARG, "num_pages must be >= 1");
  if (s->dtype == HISA_E4M3 && (!k_page_scale || !kpool_scale))
    return fail(HISA_ERR_INVALID_ARG, "E4M3 pooling needs k_page_scale and kpool_scale");
  const int nb = static_cast<int>(num_blocks(s));
  const int first = std::min(first_block, nb);
  const int count = std::min(block_count, nb - first);
  if (count == 0) return HISA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t threads_total = static_cast<int64_t>(s->batch) * count * (s->head_dim * elem_bytes(s->dtype) / 16);
  const int grid = static_cast<int>(std::min<int64_t>(ceil_div(threads_total, 256), 148 * 64));
  const uint8_t* in = static_cast<const uint8_t*>(k_pages);
  uint8_t* out = static_cast<uint8_t*>(kpool);
  switch (s->dtype) {
    case HISA_F32:
      paged_block_mean_kernel<DT_F32><<<grid, 256, 0, st>>>(in, nullptr, page_table, num_pages, out, nullptr,
                                                            s->batch, s->num_keys, nb, s->head_dim, s->block_size,
                                                            first, count);
      break;
    case HISA_BF16:
      paged_block_mean_kernel<DT_BF16><<<grid, 256, 0, st>>>(in, nullptr, page_table, num_pages, out, nullptr,
                                                             s->batch, s->num_keys, nb, s->head_dim, s->block_size,
                                                             first, count);
      break;
    case HISA_E4M3:
      paged_block_mean_kernel<DT_E4M3><<<grid, 256, 0, st>>>(in, k_page_scale, page_table, num_pages, out,
                                                             kpool_scale, s->batch, s->num_keys, nb, s->head_dim,
                                                             s->block_size, first, count);
      break;
    default: return fail(HISA_ERR_INVALID_ARG, "unknown dtype %d", s->dtype);
  }
  return launch_check("paged_block_mean_kernel");
}

hisa_status hisa_block_refine_topm(const void* q, const float* q_scale, const float* w, const void* kpool,
                                   const float* kpool_scale, const int32_t* n_visible,
                                   const int32_t* superblock_idx, int32_t top_m2, int32_t group,
                                   const hisa_shape* s, int32_t* block_idx, void* workspace, size_t ws_bytes,
                                   hisa_stream stream) {
  hisa_status e = check_shape(s, true);
  if (e != HISA_OK) return e;
  if (group < 1 || top_m2 < 1) return fail(HISA_ERR_INVALID_ARG, "group and top_m2 must be >= 1");
  if (!superblock_idx || !block_idx) return fail(HISA_ERR_INVALID_ARG, "superblock_idx and block_idx must be non-NULL");
  const int64_t nb = num_blocks(s);
  // level two is the refinement stage run over the pooled blocks: "keys" are
  // pooled blocks, its "blocks" are super-blocks of `group` pooled blocks,
  // visibility is the count of fully visible blocks and k is top_m - 1
  hisa_shape s2 = *s;
  s2.num_keys = static_cast<int32_t>(nb);
  s2.block_size = group;
  s2.top_m = top_m2;
  s2.top_k = s->top_m - 1;
  e = check_indexer_ptrs(s, q, q_scale, w, kpool, kpool_scale, n_visible);
  if (e != HISA_OK) return e;
  const int64_t rows = rows_of(s);
  size_t need = 0;
  e = hisa_workspace_size(HISA_OP_BLOCK_REFINE_TOPM, s, &need);
  if (e != HISA_OK) return e;
  if (!workspace || !aligned16(workspace) || ws_bytes < need)
    return fail(HISA_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned)", need);
  int32_t* nvb = static_cast<int32_t*>(workspace);
  int32_t* sel = nvb + pad4(rows);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int grid = static_cast<int>(std::min<int64_t>(ceil_div(rows, 256), 4096));
  visible_blocks_kernel<<<grid, 256, 0, st>>>(n_visible, rows, s->num_keys, s->block_size, nvb);
  e = launch_check("visible_blocks_kernel");
  if (e != HISA_OK) return e;
  if (s->top_m > 1) {
    e = hisa_token_score_topk(q, q_scale, w, kpool, kpool_scale, nvb, superblock_idx, &s2, sel, nullptr, nullptr, 0,
                              stream);
    if (e != HISA_OK) return e;
  }
  assemble_blocks_kernel<<<grid, 256, 0, st>>>(n_visible, s->top_m > 1 ? sel : nullptr, rows, s->num_keys,
                                              s->block_size, s->top_m, block_idx);
  return launch_check("assemble_blocks_kernel");
}

hisa_status dsa_flat_indexer_topk(const void* q, const float* q_scale, const float* w, const void* k,
                                  const float* k_scale, const int32_t* n_visible, const hisa_shape* s,
                                  int32_t* topk_idx, float* topk_score, void* workspace, size_t ws_bytes,
                                  hisa_stream stream) {
  hisa_status e = check_shape(s, false);
  if (e != HISA_OK) return e;
  e = check_indexer_ptrs(s, q, q_scale, w, k, k_scale, n_visible);
  if (e != HISA_OK) return e;
  if (!topk_idx || !aligned4(topk_idx)) return fail(HISA_ERR_INVALID_ARG, "topk_idx must be non-NULL, 4-byte aligned");
  e = check_scored_rows(s, topk_score);
  if (e != HISA_OK) return e;
  const int64_t ld = pad4(s->num_keys);
  const int64_t rows = rows_of(s);
  if (!workspace || !aligned16(workspace)) return fail(HISA_ERR_WORKSPACE, "workspace must be non-NULL, 16-byte aligned");
  // workspace: score rows [chunk][ld] fp32, then (min, max) ordering keys per row
  const int64_t row_bytes = ld * 4 + 8;
  std::vector<RowChunk> chunks;
  e = plan_chunks(s, dense_group(s), std::min<int64_t>(rows, static_cast<int64_t>(ws_bytes / row_bytes)), chunks);
  if (e != HISA_OK) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  int64_t max_rows = 0;
  for (const RowChunk& c : chunks) max_rows = std::max(max_rows, c.nrows);
  uint32_t* minmax = reinterpret_cast<uint32_t*>(ws + max_rows * ld);
  const bool fused_range = dense_tc_ok(s);
  e = cuda_check(cudaFuncSetAttribute(flat_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(sizeof(TwoPassSmem))), "flat_select attribute");
  if (e != HISA_OK) return e;
  for (const RowChunk& c : chunks) {
    if (fused_range) {
      init_minmax_kernel<<<static_cast<unsigned>(std::min<int64_t>(ceil_div(c.nrows, 256), 1024)), 256, 0, st>>>(
          minmax, c.nrows);
      e = launch_check("init_minmax_kernel");
      if (e != HISA_OK) return e;
    }
    e = score_rows(s, q, q_scale, w, k, k_scale, n_visible, 0, s->num_keys, c, ws, ld, st,
                   fused_range ? minmax : nullptr);
    if (e != HISA_OK) return e;
    flat_select_kernel<<<static_cast<unsigned>(c.nrows), 512, sizeof(TwoPassSmem), st>>>(
        ws, ld, fused_range ? minmax : nullptr, n_visible, c.row0, s->num_keys, s->top_k, topk_idx, topk_score);
    e = launch_check("flat_select_kernel");
    if (e != HISA_OK) return e;
  }
  return sort_scored_rows(topk_idx, topk_score, rows, s->top_k, st);
}

hisa_status dsa_flat_indexer_topk_sampled(const void* q, const float* q_scale, const float* w, const void* k,
                                          const float* k_scale, const int32_t* n_visible, const hisa_shape* s,
                                          int32_t* topk_idx, float* topk_score, void* workspace, size_t ws_bytes,
                                          hisa_stream stream) {
  hisa_status e = check_shape(s, false);
  if (e != HISA_OK) return e;
  e = check_indexer_ptrs(s, q, q_scale, w, k, k_scale, n_visible);
  if (e != HISA_OK) return e;
  if (!topk_idx || !aligned4(topk_idx)) return fail(HISA_ERR_INVALID_ARG, "topk_idx must be non-NULL, 4-byte aligned");
  LitePlan lp;
  e = check_scored_rows(s, topk_score);
  if (e != HISA_OK) return e;
  if (!lite_plan(s, &lp))
    return fail(HISA_ERR_UNSUPPORTED, "sampled flat top-k needs a tensor-core shape, num_keys divisible by the "
                                      "sample stride and top_k small enough for the pair buffer");
  if (!workspace || !aligned16(workspace)) return fail(HISA_ERR_WORKSPACE, "workspace must be non-NULL, 16-byte aligned");
  if (ws_bytes < lp.fixed + lp.per_row * dense_group(s))
    return fail(HISA_ERR_WORKSPACE, "workspace holds fewer than one query group (%zu bytes needed)",
                lp.fixed + lp.per_row * dense_group(s));
  e = flat_lite(s, lp, q, q_scale, w, k, k_scale, n_visible, topk_idx, topk_score, workspace, ws_bytes,
                reinterpret_cast<cudaStream_t>(stream));
  if (e != HISA_OK) return e;
  return sort_scored_rows(topk_idx, topk_score, rows_of(s), s->top_k, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// =================================================================== sparse attention

extern "C" {

hisa_status hisa_sparse_attention(const void* q, const void* kv, const int32_t* idx, int32_t batch,
                                  int32_t num_queries, int32_t num_keys, int32_t heads, int32_t d_qk,
                                  int32_t d_v, int32_t top_k, float scale, void* o, float* lse,
                                  hisa_stream stream) {
  if (batch < 1 || num_queries < 1 || num_keys < 1)
    return fail(HISA_ERR_INVALID_ARG, "batch, num_queries and num_keys must be >= 1");
  if (heads < 1 || heads % kAttnHeads != 0)
    return fail(HISA_ERR_UNSUPPORTED, "heads must be a multiple of %d", kAttnHeads);
  if (d_qk != kAttnDqk || d_v != kAttnDv)
    return fail(HISA_ERR_UNSUPPORTED, "d_qk must be %d and d_v %d", kAttnDqk, kAttnDv);
  if (top_k < 1 || top_k > kAttnMaxK) return fail(HISA_ERR_UNSUPPORTED, "top_k must be in [1, %d]", kAttnMaxK);
  if (!std::isfinite(scale)) return fail(HISA_ERR_INVALID_ARG, "scale must be finite");
  if (!q || !kv || !idx || !o || !lse) return fail(HISA_ERR_INVALID_ARG, "q, kv, idx, o and lse must be non-NULL");
  if (!aligned16(q) || !aligned16(kv) || !aligned16(o) || !aligned4(idx) || !aligned4(lse))
    return fail(HISA_ERR_INVALID_ARG, "q, kv and o must be 16-byte aligned, idx and lse 4-byte aligned");
  const int64_t rows = static_cast<int64_t>(batch) * num_queries;
  const int slices = heads / kAttnHeads;
  if (rows * slices * 2 > INT32_MAX) return fail(HISA_ERR_UNSUPPORTED, "too many (query, head slice) pairs");
  if (static_cast<int64_t>(batch) * num_keys > INT32_MAX)
    return fail(HISA_ERR_UNSUPPORTED, "batch * num_keys must fit in int32 (key row coordinates)");
  // one-row boxes for the gathers: 64 value features (128-byte swizzle) and
  // 32 positional features (64-byte swizzle)
  CUtensorMap kvm, ropem;
  hisa_status e = tensor_map_2d(&kvm, kv, HISA_BF16, static_cast<uint64_t>(batch) * num_keys, kAttnDqk, 1);
  if (e != HISA_OK) return e;
  e = tensor_map_2d(&ropem, kv, HISA_BF16, static_cast<uint64_t>(batch) * num_keys, kAttnDqk, 1, 0, 32,
                    CU_TENSOR_MAP_SWIZZLE_64B);
  if (e != HISA_OK) return e;
  const size_t smem = attn_smem_bytes();
  e = cuda_check(cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      static_cast<int>(smem)), "sparse_attn attribute");
  if (e != HISA_OK) return e;
  AttnParams p{};
  p.rows = rows; p.Q = num_queries; p.L = num_keys; p.slices = slices; p.top_k = top_k;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.idx = idx; p.q = static_cast<const uint16_t*>(q); p.kv = static_cast<const uint16_t*>(kv); p.o = static_cast<uint16_t*>(o); p.lse = lse;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(rows * slices * 2));
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cuda_check(cudaLaunchKernelEx(&cfg, sparse_attn_kernel, kvm, ropem, p), "launch sparse_attn_kernel");
  if (e != HISA_OK) return e;
  return launch_check("sparse_attn_kernel");
}

}  // extern "C"

// =================================================================== host buffers
//
// hisa_indexer_from_host: the whole indexer (pool -> coarse top-m -> refine
// top-k) on inputs in host memory, for callers whose q, keys and weights
// arrive from the host.  The work is cut into pieces (query ranges of one
// sequence, or ranges of whole sequences) run as a pipeline on three streams
// of the library's: the copy of piece i+1 in, the kernels of piece i and the
// copy of piece i-1 out overlap.  A piece copies only the keys its queries
// see beyond those earlier pieces copied, and pools only the blocks those
// keys complete (the coarse stage scores complete blocks only).

namespace {

struct HostPipe {
  cudaStream_t in = nullptr, run = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, ready = nullptr, fin = nullptr, last = nullptr;
};

constexpr int kMaxPipeDevices = 64;
std::mutex g_pipe_mu;
HostPipe g_pipe[kMaxPipeDevices];

// The pipeline's streams and events on the current device, created on the
// first call there and kept until the process exits.
hisa_status host_pipe(HostPipe** out) {
  int dev = 0;
  hisa_status e = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (e != HISA_OK) return e;
  if (dev < 0 || dev >= kMaxPipeDevices) return fail(HISA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  HostPipe& p = g_pipe[dev];
  if (!p.in) {
    cudaStream_t* ss[3] = {&p.in, &p.run, &p.out};
    for (cudaStream_t* x : ss) {
      e = cuda_check(cudaStreamCreateWithFlags(x, cudaStreamNonBlocking), "create pipeline stream");
      if (e != HISA_OK) return e;
    }
    cudaEvent_t* es[4] = {&p.start, &p.ready, &p.fin, &p.last};
    for (cudaEvent_t* x : es) {
      e = cuda_check(cudaEventCreateWithFlags(x, cudaEventDisableTiming), "create pipeline event");
      if (e != HISA_OK) return e;
    }
  }
  *out = &p;
  return HISA_OK;
}

constexpr size_t kPipeAlign = 256;

size_t pipe_round(size_t n) { return (n + kPipeAlign - 1) / kPipeAlign * kPipeAlign; }

// Device buffers of the host pipeline, carved from the caller's workspace.
struct PipeBuffers {
  uint8_t *q, *k, *kpool;
  float *w, *q_scale, *k_scale, *kpool_scale;
  int32_t *nv, *blocks, *idx;
  void* coarse;
  size_t coarse_bytes;
  void* split;
  size_t split_bytes;
  size_t total;
};

PipeBuffers pipe_layout(const hisa_shape* s, uint8_t* base) {
  const size_t es = static_cast<size_t>(elem_bytes(s->dtype));
  const size_t rows = static_cast<size_t>(rows_of(s));
  const size_t keys = static_cast<size_t>(s->batch) * s->num_keys;
  const size_t nb = static_cast<size_t>(num_blocks(s));
  const bool e4 = s->dtype == HISA_E4M3;
  PipeBuffers b{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += pipe_round(bytes);
    return p;
  };
  b.q = take(rows * s->heads * s->head_dim * es);
  b.w = reinterpret_cast<float*>(take(rows * s->heads * 4));
  b.nv = reinterpret_cast<int32_t*>(take(rows * 4));
  b.k = take(keys * s->head_dim * es);
  b.kpool = take(static_cast<size_t>(s->batch) * nb * s->head_dim * es);
  b.q_scale = e4 ? reinterpret_cast<float*>(take(rows * 4)) : nullptr;
  b.k_scale = e4 ? reinterpret_cast<float*>(take(keys * 4)) : nullptr;
  b.kpool_scale = e4 ? reinterpret_cast<float*>(take(static_cast<size_t>(s->batch) * nb * 4)) : nullptr;
  b.blocks = reinterpret_cast<int32_t*>(take(rows * s->top_m * 4));
  b.idx = reinterpret_cast<int32_t*>(take(rows * s->top_k * 4));
  b.coarse_bytes = rows * static_cast<size_t>(pad4(static_cast<int64_t>(nb))) * 4;
  b.coarse = take(b.coarse_bytes);
  // split refinement of small pieces: rows * parts <= SM count
  b.split_bytes = static_cast<size_t>(num_sms()) * s->top_k * 8;
  b.split = take(b.split_bytes);
  b.total = off;
  return b;
}

struct Piece {
  int s0, s1, t0, t1;
};

size_t host_pipe_bytes(const hisa_shape* s) { return pipe_layout(s, nullptr).total; }

}  // namespace

extern "C" {

hisa_status hisa_indexer_from_host(const void* q, const float* q_scale, const float* w, const void* k,
                                   const float* k_scale, const int32_t* n_visible, const hisa_shape* s,
                                   int32_t* topk_idx, int32_t pieces, void* workspace, size_t ws_bytes,
                                   hisa_stream stream) {
  hisa_status e = check_shape(s, true);
  if (e != HISA_OK) return e;
  if (!q || !w || !k || !n_visible || !topk_idx)
    return fail(HISA_ERR_INVALID_ARG, "q, w, keys, n_visible and topk_idx must be non-NULL host pointers");
  if (s->dtype == HISA_E4M3 && (!q_scale || !k_scale))
    return fail(HISA_ERR_INVALID_ARG, "E4M3 inputs need q_scale and k_scale");
  if (pieces < 0 || pieces > 256) return fail(HISA_ERR_INVALID_ARG, "pieces must be in [0, 256]");
  if (s->top_m > kMaxTopM) return fail(HISA_ERR_UNSUPPORTED, "top_m must be <= %d", kMaxTopM);
  if (static_cast<int64_t>(s->top_m) * s->block_size > kMaxCandidates)
    return fail(HISA_ERR_UNSUPPORTED, "top_m * block_size must be <= %d", kMaxCandidates);
  const PipeBuffers need = pipe_layout(s, nullptr);
  if (!workspace || !aligned16(workspace) || ws_bytes < need.total)
    return fail(HISA_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned device memory)", need.total);
  const PipeBuffers d = pipe_layout(s, static_cast<uint8_t*>(workspace));
  const int B = s->block_size, L = s->num_keys, Q = s->num_queries, H = s->heads, hd = s->head_dim;
  const int64_t nb = num_blocks(s);
  const size_t es = static_cast<size_t>(elem_bytes(s->dtype));
  const size_t q_row = static_cast<size_t>(H) * hd * es, k_row = static_cast<size_t>(hd) * es;
  const int P = pieces == 0 ? 16 : pieces;
  // pieces: query ranges of a single sequence, or ranges of whole sequences
  std::vector<Piece> plan;
  for (int i = 0; i < P; ++i) {
    Piece pc = s->batch == 1 ? Piece{0, 1, static_cast<int>(static_cast<int64_t>(Q) * i / P),
                                     static_cast<int>(static_cast<int64_t>(Q) * (i + 1) / P)}
                             : Piece{static_cast<int>(static_cast<int64_t>(s->batch) * i / P),
                                     static_cast<int>(static_cast<int64_t>(s->batch) * (i + 1) / P), 0, Q};
    if (pc.s1 > pc.s0 && pc.t1 > pc.t0) plan.push_back(pc);
  }
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe* hp = nullptr;
  e = host_pipe(&hp);
  if (e != HISA_OK) return e;
  cudaStream_t cur = reinterpret_cast<cudaStream_t>(stream);
  const uint8_t* hq = static_cast<const uint8_t*>(q);
  const uint8_t* hk = static_cast<const uint8_t*>(k);
  auto h2d = [&](void* dst, const void* src, size_t bytes) {
    return bytes ? cuda_check(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, hp->in), "copy in") : HISA_OK;
  };
  e = cuda_check(cudaEventRecord(hp->start, cur), "record start");
  if (e != HISA_OK) return e;
  e = cuda_check(cudaStreamWaitEvent(hp->in, hp->start, 0), "wait start");
  if (e != HISA_OK) return e;
  std::vector<int> keys_in(s->batch, 0), pooled(s->batch, 0);
  for (const Piece& pc : plan) {
    const int nseq = pc.s1 - pc.s0, nq = pc.t1 - pc.t0;
    // keys this piece sees beyond the earlier pieces (n_visible read on the host)
    int n_hi = 1;
    for (int b = pc.s0; b < pc.s1; ++b)
      for (int t = pc.t0; t < pc.t1; ++t) n_hi = std::max(n_hi, n_visible[static_cast<int64_t>(b) * Q + t]);
    n_hi = std::min(n_hi, L);
    for (int b = pc.s0; b < pc.s1; ++b) {
      if (n_hi > keys_in[b]) {
        const size_t r0 = static_cast<size_t>(b) * L + keys_in[b];
        const size_t nr = static_cast<size_t>(n_hi - keys_in[b]);
        if ((e = h2d(d.k + r0 * k_row, hk + r0 * k_row, nr * k_row)) != HISA_OK) return e;
        if (d.k_scale && (e = h2d(d.k_scale + r0, k_scale + r0, nr * 4)) != HISA_OK) return e;
        keys_in[b] = n_hi;
      }
    }
    // this piece's rows of q, w, n_visible (and q scales): contiguous in both layouts
    for (int b = pc.s0; b < pc.s1; ++b) {
      const size_t r0 = static_cast<size_t>(b) * Q + pc.t0;
      if ((e = h2d(d.q + r0 * q_row, hq + r0 * q_row, static_cast<size_t>(nq) * q_row)) != HISA_OK) return e;
      if ((e = h2d(d.w + r0 * H, w + r0 * H, static_cast<size_t>(nq) * H * 4)) != HISA_OK) return e;
      if ((e = h2d(d.nv + r0, n_visible + r0, static_cast<size_t>(nq) * 4)) != HISA_OK) return e;
      if (d.q_scale && (e = h2d(d.q_scale + r0, q_scale + r0, static_cast<size_t>(nq) * 4)) != HISA_OK) return e;
    }
    if ((e = cuda_check(cudaEventRecord(hp->ready, hp->in), "record ready")) != HISA_OK) return e;
    if ((e = cuda_check(cudaStreamWaitEvent(hp->run, hp->ready, 0), "wait ready")) != HISA_OK) return e;
    // pool the blocks the new keys complete (every block below the last visible one)
    const int c_hi = (n_hi - 1) / B;
    for (int b = pc.s0; b < pc.s1; ++b) {
      if (c_hi > pooled[b]) {
        hisa_shape one = *s;
        one.batch = 1;
        e = hisa_pool_blocks_range(d.k + static_cast<size_t>(b) * L * k_row,
                                   d.k_scale ? d.k_scale + static_cast<size_t>(b) * L : nullptr,
                                   d.kpool + static_cast<size_t>(b) * nb * k_row,
                                   d.kpool_scale ? d.kpool_scale + static_cast<size_t>(b) * nb : nullptr, &one,
                                   pooled[b], c_hi - pooled[b], reinterpret_cast<hisa_stream>(hp->run));
        if (e != HISA_OK) return e;
        pooled[b] = c_hi;
      }
    }
    hisa_shape ps = *s;
    ps.batch = nseq;
    ps.num_queries = nq;
    // a piece of one sequence is that sequence with only the piece's queries;
    // a piece of whole sequences starts at its first sequence
    const size_t r0 = static_cast<size_t>(pc.s0) * Q + pc.t0;
    const size_t kb = s->batch == 1 ? 0 : static_cast<size_t>(pc.s0);
    const hisa_stream rs = reinterpret_cast<hisa_stream>(hp->run);
    e = hisa_block_score_topm(d.q + r0 * q_row, d.q_scale ? d.q_scale + r0 : nullptr, d.w + r0 * H,
                              d.kpool + kb * nb * k_row, d.kpool_scale ? d.kpool_scale + kb * nb : nullptr,
                              d.nv + r0, &ps, d.blocks + r0 * s->top_m, d.coarse, d.coarse_bytes, rs);
    if (e != HISA_OK) return e;
    e = hisa_token_score_topk(d.q + r0 * q_row, d.q_scale ? d.q_scale + r0 : nullptr, d.w + r0 * H,
                              d.k + kb * L * k_row, d.k_scale ? d.k_scale + kb * L : nullptr, d.nv + r0,
                              d.blocks + r0 * s->top_m, &ps, d.idx + r0 * s->top_k, nullptr, d.split,
                              d.split_bytes, rs);
    if (e != HISA_OK) return e;
    if ((e = cuda_check(cudaEventRecord(hp->fin, hp->run), "record fin")) != HISA_OK) return e;
    if ((e = cuda_check(cudaStreamWaitEvent(hp->out, hp->fin, 0), "wait fin")) != HISA_OK) return e;
    for (int b = pc.s0; b < pc.s1; ++b) {
      const size_t rr = static_cast<size_t>(b) * Q + pc.t0;
      e = cuda_check(cudaMemcpyAsync(topk_idx + rr * s->top_k, d.idx + rr * s->top_k,
                                     static_cast<size_t>(nq) * s->top_k * 4, cudaMemcpyDeviceToHost, hp->out),
                     "copy out");
      if (e != HISA_OK) return e;
    }
  }
  if ((e = cuda_check(cudaEventRecord(hp->last, hp->out), "record last")) != HISA_OK) return e;
  return cuda_check(cudaStreamWaitEvent(cur, hp->last, 0), "wait last");
}

}  // extern "C"

// =================================================================== no-allocation variant
//
// hisa_block_score_topm_static: the coarse stage for callers that cannot
// allocate device memory at call time (code running inside another runtime's
// memory arena, plug-ins handed only input and output pointers, or hosts that
// forbid cudaMalloc on the serving path).  Its block-score rows live in one
// file-scope device array instead of a caller workspace.

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB of fp32 block scores

// Held by every GPU that loads the library, until the process exits.  In host
// code this name is only a host-side handle; its device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) float g_static_block_scores[kStaticScratchBytes / sizeof(float)];

// Device address of the scratch array on the current device.  Looked up on
// every call (the lookup allocates nothing), so an address never outlives the
// context it was taken in, e.g. across a cudaDeviceReset.
hisa_status static_scratch(float** out) {
  void* p = nullptr;
  hisa_status e = cuda_check(cudaGetSymbolAddress(&p, g_static_block_scores), "cudaGetSymbolAddress(block-score scratch)");
  if (e != HISA_OK) return e;
  *out = static_cast<float*>(p);
  return HISA_OK;
}

}  // namespace

extern "C" {

hisa_status hisa_block_score_topm_static(const void* q, const float* q_scale, const float* w, const void* kpool,
                                         const float* kpool_scale, const int32_t* n_visible, const hisa_shape* s,
                                         int32_t* block_idx, hisa_stream stream) {
  hisa_status e = check_shape(s, true);
  if (e != HISA_OK) return e;
  const size_t need = static_cast<size_t>(rows_of(s)) * static_cast<size_t>(pad4(num_blocks(s))) * sizeof(float);
  if (need > kStaticScratchBytes)
    return fail(HISA_ERR_WORKSPACE,
                "block scores need %zu bytes; the built-in scratch holds %zu (use hisa_block_score_topm with a "
                "caller workspace)", need, kStaticScratchBytes);
  float* scratch = nullptr;
  e = static_scratch(&scratch);
  if (e != HISA_OK) return e;
  // every score row the selection reads is written first by the scoring
  // kernel, so nothing in the scratch has to start at zero
  return hisa_block_score_topm(q, q_scale, w, kpool, kpool_scale, n_visible, s, block_idx, scratch,
                               kStaticScratchBytes, stream);
}

}  // extern "C"

"""Python binding of libhisa (include/hisa.h): argument marshalling only.

Every function here checks tensor shapes/dtypes, allocates outputs and the
workspace with torch (the library itself never allocates), and calls the C
entry point of the same name on torch's current CUDA stream.  There is no
fallback: if libhisa.so is missing or fails to load, ``load()`` raises.

Layouts (row-major, contiguous, on the GPU):
  q          [batch, Q, H, d]   float32 / bfloat16 / uint8 (E4M3 codes)
  keys       [batch, L, d]      same dtype as q
  w          [batch, Q, H]      float32
  n_visible  [batch, Q]         int32
  q_scale    [batch, Q]         float32 (E4M3 only);  k_scale [batch, L]
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

HISA_F32, HISA_BF16, HISA_E4M3 = 0, 1, 2
OP_BLOCK, OP_TOKEN, OP_FLAT, OP_FLAT_SAMPLED, OP_BLOCK_REFINE, OP_FROM_HOST = 1, 2, 3, 4, 5, 6
STATUS = {0: "HISA_OK", 1: "HISA_ERR_INVALID_ARG", 2: "HISA_ERR_UNSUPPORTED", 3: "HISA_ERR_WORKSPACE",
          4: "HISA_ERR_CUDA", 5: "HISA_ERR_TIMEOUT"}


class HisaError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {message}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("batch", "num_keys", "num_queries", "heads", "head_dim", "block_size", "top_m", "top_k",
                 "dtype")]


_P = ctypes.c_void_p
_SIGS = {
    "hisa_pool_blocks": [_P, _P, _P, _P, ctypes.POINTER(Shape), _P],
    "hisa_pool_blocks_range": [_P, _P, _P, _P, ctypes.POINTER(Shape), ctypes.c_int32, ctypes.c_int32, _P],
    "hisa_pool_blocks_paged": [_P, _P, _P, ctypes.c_int32, _P, _P, ctypes.POINTER(Shape), ctypes.c_int32,
                               ctypes.c_int32, _P],
    "hisa_compress_keys": [_P, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                           ctypes.c_int32, _P],
    "hisa_quantize_e4m3": [_P, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, _P, _P, _P],
    "hisa_block_score_topm": [_P, _P, _P, _P, _P, _P, ctypes.POINTER(Shape), _P, _P, ctypes.c_size_t, _P],
    "hisa_block_refine_topm": [_P, _P, _P, _P, _P, _P, _P, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(Shape), _P,
                               _P, ctypes.c_size_t, _P],
    "hisa_block_score_topm_static": [_P, _P, _P, _P, _P, _P, ctypes.POINTER(Shape), _P, _P],
    "hisa_token_score_topk": [_P, _P, _P, _P, _P, _P, _P, ctypes.POINTER(Shape), _P, _P, _P, ctypes.c_size_t,
                              _P],
    "hisa_token_score_topk_paged": [_P, _P, _P, _P, _P, _P, ctypes.c_int32, _P, _P, ctypes.POINTER(Shape), _P, _P,
                                    _P, ctypes.c_size_t, _P],
    "dsa_flat_indexer_topk": [_P, _P, _P, _P, _P, _P, ctypes.POINTER(Shape), _P, _P, _P, ctypes.c_size_t, _P],
    "dsa_flat_indexer_topk_sampled": [_P, _P, _P, _P, _P, _P, ctypes.POINTER(Shape), _P, _P, _P, ctypes.c_size_t, _P],
    "hisa_indexer_from_host": [_P, _P, _P, _P, _P, _P, ctypes.POINTER(Shape), _P, ctypes.c_int32, _P,
                               ctypes.c_size_t, _P],
    "hisa_sparse_attention": [_P, _P, _P] + [ctypes.c_int32] * 7 + [ctypes.c_float, _P, _P, _P],
    "hisa_workspace_size": [ctypes.c_int32, ctypes.POINTER(Shape), ctypes.POINTER(ctypes.c_size_t)],
    "hisa_get_status": [_P],
    "hisa_selftest_wait_timeout": [ctypes.c_uint64, _P],
    "hisa_status_string": [ctypes.c_int],
    "hisa_last_error": [],
}
EXPORTS = tuple(_SIGS)

_lib: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return _build.LIB


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libhisa.so (building it first if the sources are newer)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    if path is None:
        path = library_path()
        if not _build.up_to_date():
            _build.build()
    if not os.path.exists(path):
        raise RuntimeError(f"libhisa.so not found at {path}; run `python -m hierarchical_top_key_b200.build`")
    lib = ctypes.CDLL(path)
    for name, args in _SIGS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name in ("hisa_status_string", "hisa_last_error") else ctypes.c_int
    if path == library_path():
        _lib = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        msg = load().hisa_last_error().decode(errors="replace")
        raise HisaError(status, where, msg)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return HISA_F32
    if t.dtype == torch.bfloat16:
        return HISA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return HISA_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t: torch.Tensor, name: str, ndim: int):
    if not t.is_cuda or not t.is_contiguous() or t.dim() != ndim:
        raise ValueError(f"{name} must be a contiguous CUDA tensor with {ndim} dims, got {tuple(t.shape)}")


def make_shape(q: torch.Tensor, k: torch.Tensor, block_size: int = 1, top_m: int = 1, top_k: int = 1) -> Shape:
    _need(q, "q", 4)
    _need(k, "keys", 3)
    b, Q, H, d = q.shape
    if k.shape[0] != b or k.shape[2] != d:
        raise ValueError(f"keys {tuple(k.shape)} do not match q {tuple(q.shape)}")
    if dtype_code(q) != dtype_code(k):
        raise TypeError("q and keys must share a dtype")
    return Shape(b, k.shape[1], Q, H, d, block_size, top_m, top_k, dtype_code(q))


def workspace_size(op: int, shape: Shape) -> int:
    n = ctypes.c_size_t(0)
    _check(load().hisa_workspace_size(op, ctypes.byref(shape), ctypes.byref(n)), "hisa_workspace_size")
    return n.value


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def get_status():
    """Synchronise the current stream and raise if a kernel recorded an error."""
    _check(load().hisa_get_status(_stream()), "hisa_get_status")


# ----------------------------------------------------------------- entry points


def hisa_pool_blocks(k: torch.Tensor, block_size: int, k_scale: Optional[torch.Tensor] = None):
    """Mean-pool each run of block_size keys -> (kpool [batch, nb, d], kpool_scale or None)."""
    _need(k, "keys", 3)
    b, L, d = k.shape
    nb = -(-L // block_size)
    shape = Shape(b, L, 1, 1, d, block_size, 1, 1, dtype_code(k))
    kpool = torch.empty((b, nb, d), dtype=k.dtype, device=k.device)
    kps = torch.empty((b, nb), dtype=torch.float32, device=k.device) if k_scale is not None else None
    _check(load().hisa_pool_blocks(k.data_ptr(), _ptr(k_scale), kpool.data_ptr(), _ptr(kps), ctypes.byref(shape),
                                   _stream()), "hisa_pool_blocks")
    return kpool, kps


def hisa_pool_blocks_range(k: torch.Tensor, block_size: int, first_block: int, block_count: int,
                           kpool: torch.Tensor, k_scale: Optional[torch.Tensor] = None,
                           kpool_scale: Optional[torch.Tensor] = None) -> None:
    """Pool blocks [first_block, first_block + block_count) of every sequence into
    the caller's kpool [batch, nb, d] (and kpool_scale for E4M3) in place."""
    _need(k, "keys", 3)
    b, L, d = k.shape
    nb = -(-L // block_size)
    if tuple(kpool.shape) != (b, nb, d) or kpool.dtype != k.dtype or not kpool.is_contiguous():
        raise ValueError("kpool must be a contiguous [batch, ceil(L/B), d] tensor of the keys' dtype")
    if (k_scale is None) != (kpool_scale is None):
        raise ValueError("k_scale and kpool_scale go together (E4M3 keys)")
    shape = Shape(b, L, 1, 1, d, block_size, 1, 1, dtype_code(k))
    _check(load().hisa_pool_blocks_range(k.data_ptr(), _ptr(k_scale), kpool.data_ptr(), _ptr(kpool_scale),
                                         ctypes.byref(shape), first_block, block_count, _stream()),
           "hisa_pool_blocks_range")


def hisa_compress_keys(k_raw: torch.Tensor, ratio: int) -> torch.Tensor:
    """Mean of each `ratio` consecutive keys (trailing partial group dropped)."""
    _need(k_raw, "k_raw", 3)
    b, S, d = k_raw.shape
    ck = torch.empty((b, S // ratio, d), dtype=k_raw.dtype, device=k_raw.device)
    _check(load().hisa_compress_keys(k_raw.data_ptr(), ck.data_ptr(), b, S, d, ratio, dtype_code(k_raw),
                                     _stream()), "hisa_compress_keys")
    return ck


def hisa_quantize_e4m3(x: torch.Tensor, row_dims: int):
    """E4M3 codes and per-row fp32 scales; rows are the first `row_dims` dims."""
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor")
    rows = 1
    for s in x.shape[:row_dims]:
        rows *= s
    cols = x.numel() // max(rows, 1)
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scale = torch.empty(x.shape[:row_dims], dtype=torch.float32, device=x.device)
    _check(load().hisa_quantize_e4m3(x.data_ptr(), dtype_code(x), rows, cols, codes.data_ptr(), scale.data_ptr(),
                                     _stream()), "hisa_quantize_e4m3")
    return codes, scale


def hisa_block_score_topm(q, w, kpool, n_visible, *, num_keys: int, block_size: int, top_m: int,
                          q_scale=None, kpool_scale=None, workspace: Optional[torch.Tensor] = None):
    """Coarse stage: block_idx [batch, Q, top_m] int32 (-1 padded, any order)."""
    b, Q, H, d = q.shape
    shape = Shape(b, num_keys, Q, H, d, block_size, top_m, 1, dtype_code(q))
    _need(w, "w", 3)
    _need(n_visible, "n_visible", 2)
    out = torch.empty((b, Q, top_m), dtype=torch.int32, device=q.device)
    ws = workspace if workspace is not None else _workspace(workspace_size(OP_BLOCK, shape), q.device)
    _check(load().hisa_block_score_topm(q.data_ptr(), _ptr(q_scale), w.data_ptr(), kpool.data_ptr(),
                                        _ptr(kpool_scale), n_visible.data_ptr(), ctypes.byref(shape),
                                        out.data_ptr(), ws.data_ptr(), ws.numel(), _stream()),
           "hisa_block_score_topm")
    return out


def hisa_block_score_topm_static(q, w, kpool, n_visible, *, num_keys: int, block_size: int, top_m: int,
                                 q_scale=None, kpool_scale=None):
    """Coarse stage using the library's built-in score scratch: no workspace is
    allocated, by torch or by the library (see include/hisa.h for its size
    limit and the rule that calls must not overlap)."""
    b, Q, H, d = q.shape
    shape = Shape(b, num_keys, Q, H, d, block_size, top_m, 1, dtype_code(q))
    _need(w, "w", 3)
    _need(n_visible, "n_visible", 2)
    out = torch.empty((b, Q, top_m), dtype=torch.int32, device=q.device)
    _check(load().hisa_block_score_topm_static(q.data_ptr(), _ptr(q_scale), w.data_ptr(), kpool.data_ptr(),
                                               _ptr(kpool_scale), n_visible.data_ptr(), ctypes.byref(shape),
                                               out.data_ptr(), _stream()), "hisa_block_score_topm_static")
    return out


def _token_workspace(shape, device, workspace):
    """The refinement stage's optional workspace: the caller's, or one sized
    by hisa_workspace_size (None when the shape has no use for one)."""
    need = workspace_size(OP_TOKEN, shape)
    if need == 0:
        return None, 0
    if workspace is not None and workspace.numel() >= need:
        return workspace, workspace.numel()
    return _workspace(need, device), need


def hisa_token_score_topk(q, w, k, n_visible, block_idx, *, block_size: int, top_k: int, q_scale=None,
                          k_scale=None, want_scores: bool = False, workspace: Optional[torch.Tensor] = None):
    """Refinement stage: (topk_idx [batch, Q, top_k] int32, scores or None)."""
    top_m = block_idx.shape[-1]
    shape = make_shape(q, k, block_size, top_m, top_k)
    _need(block_idx, "block_idx", 3)
    b, Q = q.shape[:2]
    idx = torch.empty((b, Q, top_k), dtype=torch.int32, device=q.device)
    sc = torch.empty((b, Q, top_k), dtype=torch.float32, device=q.device) if want_scores else None
    ws, nbytes = _token_workspace(shape, q.device, workspace)
    _check(load().hisa_token_score_topk(q.data_ptr(), _ptr(q_scale), w.data_ptr(), k.data_ptr(), _ptr(k_scale),
                                        n_visible.data_ptr(), block_idx.data_ptr(), ctypes.byref(shape),
                                        idx.data_ptr(), _ptr(sc), _ptr(ws), nbytes, _stream()),
           "hisa_token_score_topk")
    return idx, sc


def _check_pages(k_pages, page_table, block_size: int, batch: int, num_keys: int):
    _need(k_pages, "k_pages", 3)
    if k_pages.shape[1] != block_size:
        raise ValueError(f"k_pages {tuple(k_pages.shape)} must be [num_pages, block_size={block_size}, d]")
    _need(page_table, "page_table", 2)
    nb = -(-num_keys // block_size)
    if page_table.dtype != torch.int32 or tuple(page_table.shape) != (batch, nb):
        raise ValueError(f"page_table must be int32 [batch, ceil(num_keys/B)] = {(batch, nb)}, "
                         f"got {page_table.dtype} {tuple(page_table.shape)}")


def hisa_pool_blocks_paged(k_pages, page_table, *, num_keys: int, first_block: int, block_count: int,
                           kpool: torch.Tensor, k_page_scale: Optional[torch.Tensor] = None,
                           kpool_scale: Optional[torch.Tensor] = None) -> None:
    """hisa_pool_blocks_range over paged keys: k_pages [num_pages, B, d], block j of
    sequence b in page page_table[b, j]; writes kpool [batch, nb, d] rows in place."""
    B = k_pages.shape[1] if k_pages.dim() == 3 else 0
    b = page_table.shape[0] if page_table.dim() == 2 else 0
    _check_pages(k_pages, page_table, B, b, num_keys)
    d = k_pages.shape[2]
    nb = -(-num_keys // B)
    if tuple(kpool.shape) != (b, nb, d) or kpool.dtype != k_pages.dtype or not kpool.is_contiguous():
        raise ValueError("kpool must be a contiguous [batch, ceil(num_keys/B), d] tensor of the keys' dtype")
    if (k_page_scale is None) != (kpool_scale is None):
        raise ValueError("k_page_scale and kpool_scale go together (E4M3 keys)")
    shape = Shape(b, num_keys, 1, 1, d, B, 1, 1, dtype_code(k_pages))
    _check(load().hisa_pool_blocks_paged(k_pages.data_ptr(), _ptr(k_page_scale), page_table.data_ptr(),
                                         k_pages.shape[0], kpool.data_ptr(), _ptr(kpool_scale), ctypes.byref(shape),
                                         first_block, block_count, _stream()), "hisa_pool_blocks_paged")


def hisa_token_score_topk_paged(q, w, k_pages, page_table, n_visible, block_idx, *, num_keys: int, top_k: int,
                                q_scale=None, k_page_scale=None, want_scores: bool = False,
                                workspace: Optional[torch.Tensor] = None):
    """Refinement stage over paged keys (layout as hisa_pool_blocks_paged):
    (topk_idx [batch, Q, top_k] int32, scores or None), equal to
    hisa_token_score_topk on the same keys stored contiguously."""
    _need(q, "q", 4)
    _need(block_idx, "block_idx", 3)
    b, Q, H, d = q.shape
    B = k_pages.shape[1] if k_pages.dim() == 3 else 0
    _check_pages(k_pages, page_table, B, b, num_keys)
    if k_pages.shape[2] != d or dtype_code(k_pages) != dtype_code(q):
        raise ValueError("k_pages must match q in head_dim and dtype")
    shape = Shape(b, num_keys, Q, H, d, B, block_idx.shape[-1], top_k, dtype_code(q))
    idx = torch.empty((b, Q, top_k), dtype=torch.int32, device=q.device)
    sc = torch.empty((b, Q, top_k), dtype=torch.float32, device=q.device) if want_scores else None
    ws, nbytes = _token_workspace(shape, q.device, workspace)
    _check(load().hisa_token_score_topk_paged(q.data_ptr(), _ptr(q_scale), w.data_ptr(), k_pages.data_ptr(),
                                              _ptr(k_page_scale), page_table.data_ptr(), k_pages.shape[0],
                                              n_visible.data_ptr(), block_idx.data_ptr(), ctypes.byref(shape),
                                              idx.data_ptr(), _ptr(sc), _ptr(ws), nbytes, _stream()),
           "hisa_token_score_topk_paged")
    return idx, sc


def dsa_flat_indexer_topk(q, w, k, n_visible, *, top_k: int, q_scale=None, k_scale=None,
                          want_scores: bool = False, workspace: Optional[torch.Tensor] = None):
    """Flat DSA indexer: (topk_idx [batch, Q, top_k] int32, scores or None)."""
    shape = make_shape(q, k, 1, 1, top_k)
    b, Q = q.shape[:2]
    idx = torch.empty((b, Q, top_k), dtype=torch.int32, device=q.device)
    sc = torch.empty((b, Q, top_k), dtype=torch.float32, device=q.device) if want_scores else None
    ws = workspace if workspace is not None else _workspace(workspace_size(OP_FLAT, shape), q.device)
    _check(load().dsa_flat_indexer_topk(q.data_ptr(), _ptr(q_scale), w.data_ptr(), k.data_ptr(), _ptr(k_scale),
                                        n_visible.data_ptr(), ctypes.byref(shape), idx.data_ptr(), _ptr(sc),
                                        ws.data_ptr(), ws.numel(), _stream()), "dsa_flat_indexer_topk")
    return idx, sc


def dsa_flat_indexer_topk_sampled(q, w, k, n_visible, *, top_k: int, q_scale=None, k_scale=None,
                                  want_scores: bool = False, workspace: Optional[torch.Tensor] = None):
    """Flat DSA indexer through the sampled-threshold path (same result, less
    workspace): (topk_idx [batch, Q, top_k] int32, scores or None)."""
    shape = make_shape(q, k, 1, 1, top_k)
    b, Q = q.shape[:2]
    idx = torch.empty((b, Q, top_k), dtype=torch.int32, device=q.device)
    sc = torch.empty((b, Q, top_k), dtype=torch.float32, device=q.device) if want_scores else None
    ws = workspace if workspace is not None else _workspace(workspace_size(OP_FLAT_SAMPLED, shape), q.device)
    _check(load().dsa_flat_indexer_topk_sampled(q.data_ptr(), _ptr(q_scale), w.data_ptr(), k.data_ptr(),
                                                _ptr(k_scale), n_visible.data_ptr(), ctypes.byref(shape),
                                                idx.data_ptr(), _ptr(sc), ws.data_ptr(), ws.numel(), _stream()),
           "dsa_flat_indexer_topk_sampled")
    return idx, sc


def hisa_sparse_attention(q, kv, idx, *, scale: float, d_v: int = 512):
    """Attention over the selected keys (latent KV shared by the heads, value =
    the first d_v features): q [batch, Q, H, d_qk] bf16, kv [batch, L, d_qk]
    bf16, idx [batch, Q, top_k] int32 -> (o [batch, Q, H, d_v] bf16,
    lse [batch, Q, H] fp32)."""
    _need(q, "q", 4)
    _need(kv, "kv", 3)
    _need(idx, "idx", 3)
    b, Q, H, dqk = q.shape
    if kv.shape[0] != b or kv.shape[2] != dqk or idx.shape[:2] != (b, Q) or idx.dtype != torch.int32:
        raise ValueError("kv must be [batch, L, d_qk] and idx int32 [batch, Q, top_k]")
    if q.dtype != torch.bfloat16 or kv.dtype != torch.bfloat16:
        raise TypeError("q and kv must be bfloat16")
    o = torch.empty((b, Q, H, d_v), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((b, Q, H), dtype=torch.float32, device=q.device)
    _check(load().hisa_sparse_attention(q.data_ptr(), kv.data_ptr(), idx.data_ptr(), b, Q, kv.shape[1], H, dqk,
                                        d_v, idx.shape[2], float(scale), o.data_ptr(), lse.data_ptr(), _stream()),
           "hisa_sparse_attention")
    return o, lse


def hisa_block_refine_topm(q, w, kpool, n_visible, superblock_idx, *, num_keys: int, block_size: int, top_m: int,
                           group: int, q_scale=None, kpool_scale=None, workspace: Optional[torch.Tensor] = None):
    """Second level of the three-level indexer: block_idx [batch, Q, top_m] int32
    (current block first, -1 padded) from the retained super-blocks."""
    b, Q, H, d = q.shape
    top_m2 = superblock_idx.shape[-1]
    shape = Shape(b, num_keys, Q, H, d, block_size, top_m, 1, dtype_code(q))
    _need(superblock_idx, "superblock_idx", 3)
    out = torch.empty((b, Q, top_m), dtype=torch.int32, device=q.device)
    ws = workspace if workspace is not None else _workspace(workspace_size(OP_BLOCK_REFINE, shape), q.device)
    _check(load().hisa_block_refine_topm(q.data_ptr(), _ptr(q_scale), w.data_ptr(), kpool.data_ptr(),
                                         _ptr(kpool_scale), n_visible.data_ptr(), superblock_idx.data_ptr(), top_m2,
                                         group, ctypes.byref(shape), out.data_ptr(), ws.data_ptr(), ws.numel(),
                                         _stream()), "hisa_block_refine_topm")
    return out


class HisaIndexer3:
    """Three-level indexer for one layer: pooled super-blocks (top_m2 kept) ->
    blocks inside them (top_m kept) -> tokens (top_k).  Super-blocks are runs
    of `group` blocks."""

    def __init__(self, block_size: int, group: int, top_m2: int, top_m: int, top_k: int):
        self.block_size, self.group, self.top_m2 = block_size, group, top_m2
        self.top_m, self.top_k = top_m, top_k

    def __call__(self, q, w, k, n_visible, q_scale=None, k_scale=None, kpool=None, kpool2=None, return_blocks=False):
        """kpool / kpool2: (pooled keys, scales) of blocks and super-blocks when
        the caller keeps them (a decoder's cache); pooled here otherwise."""
        B, L = self.block_size, k.shape[1]
        kp, kps = kpool if kpool is not None else hisa_pool_blocks(k, B, k_scale)
        kp2, kps2 = kpool2 if kpool2 is not None else hisa_pool_blocks(k, B * self.group, k_scale)
        sb = hisa_block_score_topm(q, w, kp2, n_visible, num_keys=L, block_size=B * self.group, top_m=self.top_m2,
                                   q_scale=q_scale, kpool_scale=kps2)
        blocks = hisa_block_refine_topm(q, w, kp, n_visible, sb, num_keys=L, block_size=B, top_m=self.top_m,
                                        group=self.group, q_scale=q_scale, kpool_scale=kps)
        idx, _ = hisa_token_score_topk(q, w, k, n_visible, blocks, block_size=B, top_k=self.top_k, q_scale=q_scale,
                                       k_scale=k_scale)
        return (idx, sb, blocks) if return_blocks else idx


class HisaIndexer:
    """The whole HISA indexer for one layer: pool -> coarse top-m -> refine top-k.

    Workspaces are allocated once per shape and reused."""

    def __init__(self, block_size: int, top_m: int, top_k: int):
        self.block_size, self.top_m, self.top_k = block_size, top_m, top_k
        self._ws = None
        self._host_ws = None

    def __call__(self, q, w, k, n_visible, q_scale=None, k_scale=None, want_scores=False, return_blocks=False):
        kpool, kps = hisa_pool_blocks(k, self.block_size, k_scale)
        shape = make_shape(q, k, self.block_size, self.top_m, self.top_k)
        need = workspace_size(OP_BLOCK, shape)
        if self._ws is None or self._ws.numel() < need or self._ws.device != q.device:
            self._ws = _workspace(need, q.device)
        blocks = hisa_block_score_topm(q, w, kpool, n_visible, num_keys=k.shape[1], block_size=self.block_size,
                                       top_m=self.top_m, q_scale=q_scale, kpool_scale=kps, workspace=self._ws)
        idx, sc = hisa_token_score_topk(q, w, k, n_visible, blocks, block_size=self.block_size, top_k=self.top_k,
                                        q_scale=q_scale, k_scale=k_scale, want_scores=want_scores)
        return (idx, sc, blocks) if return_blocks else (idx, sc)


    def from_host(self, q: torch.Tensor, w: torch.Tensor, k: torch.Tensor, n_visible: torch.Tensor,
                  out: torch.Tensor, chunks: int = 16, device=None, q_scale: Optional[torch.Tensor] = None,
                  k_scale: Optional[torch.Tensor] = None) -> torch.Tensor:
        """The indexer on inputs in (pinned) host memory, writing the indices into
        the host tensor `out` [batch, Q, top_k] int32, through the C entry point
        hisa_indexer_from_host (copies in, kernels and copies out pipelined over
        `chunks` pieces on the library's streams).  The device workspace is
        allocated here, once per shape, and kept.  Returns `out`; the caller's
        current stream waits for the last copy, so events recorded on it
        bracket the whole call."""
        for t, name, nd in ((q, "q", 4), (w, "w", 3), (k, "keys", 3), (n_visible, "n_visible", 2),
                            (out, "out", 3)):
            if t.is_cuda or not t.is_contiguous() or t.dim() != nd:
                raise ValueError(f"{name} must be a contiguous host tensor with {nd} dims")
        for t, name in ((q_scale, "q_scale"), (k_scale, "k_scale")):
            if t is not None and (t.is_cuda or not t.is_contiguous()):
                raise ValueError(f"{name} must be a contiguous host tensor")
        b, Q, H, d = q.shape
        if tuple(out.shape) != (b, Q, self.top_k) or out.dtype != torch.int32:
            raise ValueError("out must be an int32 [batch, Q, top_k] host tensor")
        if n_visible.dtype != torch.int32 or tuple(n_visible.shape) != (b, Q):
            raise ValueError("n_visible must be int32 [batch, Q]")
        if k.shape[0] != b or k.shape[2] != d or dtype_code(k) != dtype_code(q):
            raise ValueError("keys must be [batch, L, d] in q's dtype")
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        shape = Shape(b, k.shape[1], Q, H, d, self.block_size, self.top_m, self.top_k, dtype_code(q))
        need = workspace_size(OP_FROM_HOST, shape)
        if self._host_ws is None or self._host_ws.numel() < need or self._host_ws.device != dev:
            self._host_ws = _workspace(need, dev)
        with torch.cuda.device(dev):
            _check(load().hisa_indexer_from_host(q.data_ptr(), _ptr(q_scale), w.data_ptr(), k.data_ptr(),
                                                 _ptr(k_scale), n_visible.data_ptr(), ctypes.byref(shape),
                                                 out.data_ptr(), chunks, self._host_ws.data_ptr(),
                                                 self._host_ws.numel(), torch.cuda.current_stream(dev).cuda_stream),
                   "hisa_indexer_from_host")
        return out


def to_device_inputs(inputs, device="cuda", fp8: bool = False, compress: bool = True):
    """Upload one synthetic draw (``synthetic.Inputs``) in its storage dtype.

    Returns a dict with q, w, k (compressed by the workload's ratio through the
    library when `compress`), n_visible, and for fp8 the E4M3 codes/scales
    produced by the library's quantiser."""
    wl = inputs.workload
    tdt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    q = torch.from_numpy(inputs.q).to(device=device).to(tdt).contiguous()
    k = torch.from_numpy(inputs.keys).to(device=device).to(tdt).contiguous()
    w = torch.from_numpy(inputs.w).to(device=device).contiguous()
    nv = torch.from_numpy(inputs.n_visible).to(device=device).contiguous()
    if compress and wl.compress_ratio > 1:
        k = hisa_compress_keys(k, wl.compress_ratio)
    out = dict(q=q, w=w, k=k, n_visible=nv, q_scale=None, k_scale=None)
    if fp8:
        b, Q, H, d = q.shape
        qc, qs = hisa_quantize_e4m3(q, 2)
        kc, ks = hisa_quantize_e4m3(k, 2)
        out.update(q=qc, k=kc, q_scale=qs, k_scale=ks)
    return out

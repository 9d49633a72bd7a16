"""Thin ctypes binding of libdsa (include/dsa.h).

Each function keeps the C name without the ``dsa_`` prefix, takes torch tensors that
already live on the current CUDA device, checks their dtype/shape (argument
marshalling), and passes raw pointers plus the current stream to the library.  Every
step of the computation runs in the library's CUDA kernels; there is no fallback.
Workspaces are allocated here from PyTorch's caching allocator, the only device memory
this module creates.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

REGION, G, DI, HI, HQ, D, PAGE = 8, 4, 256, 16, 64, 192, 64
MAX_TOPK = 2048
Q_FP8 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")
_lib = None
_lock = threading.Lock()

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE = range(6)


class DsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libdsa status {status}: {msg}")
        self.status = status


_VP, _I32P, _I64P, _F32P, _U8P = (ctypes.c_void_p,) * 5
_SIG = {
    "dsa_version": (ctypes.c_int, []),
    "dsa_last_error": (ctypes.c_char_p, []),
    "dsa_get_last_error": (ctypes.c_size_t, [ctypes.c_char_p, ctypes.c_size_t]),
    "dsa_check_device": (ctypes.c_int, [_VP]),
    "dsa_compress_regions": (ctypes.c_int, [_VP, ctypes.c_int64, ctypes.c_int64, _I64P, _I64P, ctypes.c_int,
                                            _U8P, _F32P, ctypes.c_int64, _VP]),
    "dsa_indexer_workspace_size": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int64]),
    "dsa_indexer_scores": (ctypes.c_int, [_VP, _F32P, _I32P, _I32P, ctypes.c_int, _U8P, _F32P, ctypes.c_int64,
                                          _I64P, ctypes.c_int, _F32P, ctypes.c_int64, ctypes.c_uint32, _VP,
                                          ctypes.c_size_t, _VP]),
    "dsa_topk_workspace_size": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int64, ctypes.c_int]),
    "dsa_topk_regions": (ctypes.c_int, [_F32P, ctypes.c_int64, _I32P, ctypes.c_int, ctypes.c_int, _I32P, _I32P,
                                        _VP, ctypes.c_size_t, _VP]),
    "dsa_topk_regions_noalloc": (ctypes.c_int, [_F32P, ctypes.c_int64, _I32P, ctypes.c_int, ctypes.c_int, _I32P,
                                                _I32P, _VP]),
    "dsa_decode_select_workspace_size": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int64, ctypes.c_int]),
    "dsa_window_decode_launches": (ctypes.c_int, [ctypes.c_int, ctypes.c_int]),
    "dsa_decode_select": (ctypes.c_int, [_VP, _F32P, _I32P, _I32P, ctypes.c_int, _U8P, _F32P, ctypes.c_int64,
                                         _I64P, ctypes.c_int, _F32P, ctypes.c_int64, ctypes.c_uint32, ctypes.c_int,
                                         _I32P, _I32P, _VP, ctypes.c_size_t, _VP]),
    "dsa_copy": (ctypes.c_int, [_VP, _VP, ctypes.c_size_t, _VP]),
    "dsa_compress_regions_groups": (ctypes.c_int, [_VP, ctypes.c_int64, ctypes.c_int64, _I64P, _I64P, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_int, _U8P, _F32P, ctypes.c_int64, _VP]),
    "dsa_decode_select_groups": (ctypes.c_int, [_VP, _F32P, _I32P, _I32P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                _U8P, _F32P, ctypes.c_int64, _I64P, ctypes.c_int, _F32P,
                                                ctypes.c_int64, ctypes.c_uint32, ctypes.c_int, _I32P, _I32P, _VP,
                                                ctypes.c_size_t, _VP]),
    "dsa_attn_groups_workspace_size": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "dsa_sparse_attn_decode_groups": (ctypes.c_int, [_VP, _VP, _VP, ctypes.c_int64, _I32P, ctypes.c_int, _I32P,
                                                     ctypes.c_int, ctypes.c_int, ctypes.c_int, _I32P, _I32P,
                                                     ctypes.c_int, _VP, _F32P, _VP, ctypes.c_size_t, _VP]),
    "dsa_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_int64, _VP]),
    "dsa_attn_workspace_size": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int]),
    "dsa_sparse_attn_decode": (ctypes.c_int, [_VP, _VP, _VP, ctypes.c_int64, _I32P, ctypes.c_int, _I32P,
                                              ctypes.c_int, _I32P, _I32P, ctypes.c_int, _VP, _F32P, _VP,
                                              ctypes.c_size_t, _VP]),
    "dsa_sparse_attn_prefill": (ctypes.c_int, [_VP, _VP, _VP, ctypes.c_int64, _I32P, ctypes.c_int, ctypes.c_int,
                                               _I32P, _I32P, ctypes.c_int, _I32P, _I32P, ctypes.c_int, _VP, _F32P,
                                               _VP, ctypes.c_size_t, _VP]),
    "dsa_kv_append": (ctypes.c_int, [_VP, _VP, ctypes.c_int64, _I32P, ctypes.c_int, ctypes.c_int, _I32P, _I32P,
                                     ctypes.c_int, _VP, _VP, _VP]),
    "dsa_window_attn_workspace_size": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int]),
    "dsa_indexer_frontend": (ctypes.c_int, [_VP, ctypes.c_int, ctypes.c_int, _VP, _VP, _VP, _I32P, _VP, _VP, _F32P,
                                            _VP]),
    "dsa_window_attn": (ctypes.c_int, [_VP, _VP, _VP, ctypes.c_int64, _I32P, ctypes.c_int, ctypes.c_int, _I32P,
                                       _I32P, ctypes.c_int, ctypes.c_int, _VP, _F32P, _VP, ctypes.c_size_t, _VP]),
    "dsa_window_decode": (ctypes.c_int, [_VP, _VP, ctypes.c_int64, _I32P, ctypes.c_int, ctypes.c_int, _I32P, _I32P,
                                         ctypes.c_int, _VP, _VP, _VP, ctypes.c_int, _VP, _F32P, _VP,
                                         ctypes.c_size_t, _VP]),
}


def lib() -> ctypes.CDLL:
    """Loads libdsa.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with "
                                  "`python -m sparse_long_context_dsa_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIG.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def exported_symbols():
    return list(_SIG)


def _check(status: int):
    if status != OK:
        raise DsaError(status, lib().dsa_last_error().decode(errors="replace"))


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _need(t, dtype, shape=None, name="tensor"):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device)


def version() -> int:
    return int(lib().dsa_version())


def check_device():
    """Synchronises the current stream and raises if a kernel flagged an error."""
    _check(lib().dsa_check_device(_stream()))


def compress_regions(index_k, src_row, dst_slot, summaries, scales):
    """index_k bf16 [rows][4][256] (or [rows][stride] with stride >= 1024); src_row,
    dst_slot int64 [n]; summaries uint8 [4][n_slots][256]; scales fp32 [4][n_slots]."""
    _need(index_k, torch.bfloat16, name="index_k")
    _need(src_row, torch.int64, name="src_row")
    _need(dst_slot, torch.int64, (src_row.numel(),), "dst_slot")
    _need(summaries, torch.uint8, name="summaries")
    n_slots = summaries.shape[1]
    if summaries.dim() != 3 or summaries.shape[0] != G or summaries.shape[2] != DI:
        raise ValueError("summaries must be [4][n_slots][256]")
    _need(scales, torch.float32, (G, n_slots), "scales")
    row_stride = index_k[0].numel() if index_k.shape[0] else G * DI
    _check(lib().dsa_compress_regions(_p(index_k), row_stride, index_k.shape[0], _p(src_row), _p(dst_slot),
                                      src_row.numel(), _p(summaries), _p(scales), n_slots, _stream()))


def indexer_scores(index_q, gate, q_req, q_pos, summaries, scales, sum_base, scores, flags=0):
    """Fills scores fp32 [nq][4][ld] for r < q_pos//8 (other entries untouched)."""
    nq = index_q.shape[0]
    _need(index_q, torch.bfloat16, (nq, HI, DI), "index_q")
    _need(gate, torch.float32, (nq, HI), "gate")
    _need(q_req, torch.int32, (nq,), "q_req")
    _need(q_pos, torch.int32, (nq,), "q_pos")
    _need(summaries, torch.uint8, name="summaries")
    n_slots = summaries.shape[1]
    _need(scales, torch.float32, (G, n_slots), "scales")
    _need(sum_base, torch.int64, name="sum_base")
    _need(scores, torch.float32, name="scores")
    if scores.dim() != 3 or scores.shape[0] != nq or scores.shape[1] != G:
        raise ValueError("scores must be [nq][4][ld]")
    ld = scores.shape[2]
    nbytes = lib().dsa_indexer_workspace_size(nq, ld)
    ws = _workspace(nbytes, scores.device)
    _check(lib().dsa_indexer_scores(_p(index_q), _p(gate), _p(q_req), _p(q_pos), nq, _p(summaries), _p(scales),
                                    n_slots, _p(sum_base), sum_base.numel(), _p(scores), ld, flags, _p(ws),
                                    nbytes, _stream()))


def decode_select(index_q, gate, q_req, q_pos, summaries, scales, sum_base, scores, k, flags=0, sel_idx=None,
                  sel_count=None):
    """dsa_decode_select: the indexer scores into `scores` [nq][4][ld] and the top-k selection
    in one call.  Returns (sel_idx, sel_count) as topk_regions does."""
    nq = index_q.shape[0]
    _need(index_q, torch.bfloat16, (nq, HI, DI), "index_q")
    _need(gate, torch.float32, (nq, HI), "gate")
    _need(q_req, torch.int32, (nq,), "q_req")
    _need(q_pos, torch.int32, (nq,), "q_pos")
    _need(summaries, torch.uint8, name="summaries")
    n_slots = summaries.shape[1]
    _need(scales, torch.float32, (G, n_slots), "scales")
    _need(sum_base, torch.int64, name="sum_base")
    _need(scores, torch.float32, name="scores")
    if scores.dim() != 3 or scores.shape[0] != nq or scores.shape[1] != G:
        raise ValueError("scores must be [nq][4][ld]")
    ld = scores.shape[2]
    if sel_idx is None:
        sel_idx = torch.empty((nq, G, k), dtype=torch.int32, device=scores.device)
    if sel_count is None:
        sel_count = torch.empty((nq, G), dtype=torch.int32, device=scores.device)
    _need(sel_idx, torch.int32, (nq, G, k), "sel_idx")
    _need(sel_count, torch.int32, (nq, G), "sel_count")
    nbytes = lib().dsa_decode_select_workspace_size(nq, ld, k)
    ws = _workspace(nbytes, scores.device)
    _check(lib().dsa_decode_select(_p(index_q), _p(gate), _p(q_req), _p(q_pos), nq, _p(summaries), _p(scales), n_slots,
                                   _p(sum_base), sum_base.numel(), _p(scores), ld, flags, k, _p(sel_idx),
                                   _p(sel_count), _p(ws), nbytes, _stream()))
    return sel_idx, sel_count


def topk_regions(scores, q_pos, k, sel_idx=None, sel_count=None):
    """Returns (sel_idx int32 [nq][4][k], sel_count int32 [nq][4])."""
    _need(scores, torch.float32, name="scores")
    nq, g, ld = scores.shape
    if g != G:
        raise ValueError("scores must be [nq][4][ld]")
    _need(q_pos, torch.int32, (nq,), "q_pos")
    if sel_idx is None:
        sel_idx = torch.empty((nq, G, k), dtype=torch.int32, device=scores.device)
    if sel_count is None:
        sel_count = torch.empty((nq, G), dtype=torch.int32, device=scores.device)
    _need(sel_idx, torch.int32, (nq, G, k), "sel_idx")
    _need(sel_count, torch.int32, (nq, G), "sel_count")
    nbytes = lib().dsa_topk_workspace_size(nq, ld, k)
    ws = _workspace(nbytes, scores.device)
    _check(lib().dsa_topk_regions(_p(scores), ld, _p(q_pos), nq, k, _p(sel_idx), _p(sel_count), _p(ws), nbytes,
                                  _stream()))
    return sel_idx, sel_count


def topk_regions_noalloc(scores, q_pos, k, sel_idx, sel_count):
    """dsa_topk_regions_noalloc: the same selection with no device allocation at all, for
    callers that cannot allocate (outputs must be passed in; scratch is the library's
    static per-GPU buffer, so overlapping calls on one GPU race)."""
    _need(scores, torch.float32, name="scores")
    nq, g, ld = scores.shape
    if g != G:
        raise ValueError("scores must be [nq][4][ld]")
    _need(q_pos, torch.int32, (nq,), "q_pos")
    _need(sel_idx, torch.int32, (nq, G, k), "sel_idx")
    _need(sel_count, torch.int32, (nq, G), "sel_count")
    _check(lib().dsa_topk_regions_noalloc(_p(scores), ld, _p(q_pos), nq, k, _p(sel_idx), _p(sel_count), _stream()))
    return sel_idx, sel_count


def _group_range(g0, ng):
    if ng not in (1, 2, 4) or g0 < 0 or g0 + ng > G:
        raise ValueError("groups g0 .. g0 + ng - 1 must be 1, 2 or 4 consecutive groups of 0 .. 3")


def compress_regions_groups(index_k, src_row, dst_slot, summaries, scales, g0):
    """dsa_compress_regions_groups: groups g0 .. g0 + ng - 1 of index_k bf16 [rows][4][256]
    into a shard's pool summaries uint8 [ng][n_slots][256], scales fp32 [ng][n_slots]."""
    _need(index_k, torch.bfloat16, name="index_k")
    _need(src_row, torch.int64, name="src_row")
    _need(dst_slot, torch.int64, (src_row.numel(),), "dst_slot")
    _need(summaries, torch.uint8, name="summaries")
    ng, n_slots = summaries.shape[0], summaries.shape[1]
    _group_range(g0, ng)
    _need(scales, torch.float32, (ng, n_slots), "scales")
    row_stride = index_k[0].numel() if index_k.shape[0] else G * DI
    _check(lib().dsa_compress_regions_groups(_p(index_k), row_stride, index_k.shape[0], _p(src_row), _p(dst_slot),
                                             src_row.numel(), g0, ng, _p(summaries), _p(scales), n_slots, _stream()))


def decode_select_groups(index_q, gate, q_req, q_pos, summaries, scales, sum_base, scores, k, g0, flags=0,
                         sel_idx=None, sel_count=None):
    """dsa_decode_select_groups: scores [nq][ng][ld] and selection [nq][ng][k] of the shard
    holding groups g0 .. g0 + ng - 1 (ng = summaries.shape[0])."""
    nq = index_q.shape[0]
    _need(index_q, torch.bfloat16, (nq, HI, DI), "index_q")
    _need(gate, torch.float32, (nq, HI), "gate")
    _need(q_req, torch.int32, (nq,), "q_req")
    _need(q_pos, torch.int32, (nq,), "q_pos")
    _need(summaries, torch.uint8, name="summaries")
    ng, n_slots = summaries.shape[0], summaries.shape[1]
    _group_range(g0, ng)
    _need(scales, torch.float32, (ng, n_slots), "scales")
    _need(sum_base, torch.int64, name="sum_base")
    _need(scores, torch.float32, name="scores")
    if scores.dim() != 3 or scores.shape[0] != nq or scores.shape[1] != ng:
        raise ValueError("scores must be [nq][ng][ld]")
    ld = scores.shape[2]
    if sel_idx is None:
        sel_idx = torch.empty((nq, ng, k), dtype=torch.int32, device=scores.device)
    if sel_count is None:
        sel_count = torch.empty((nq, ng), dtype=torch.int32, device=scores.device)
    _need(sel_idx, torch.int32, (nq, ng, k), "sel_idx")
    _need(sel_count, torch.int32, (nq, ng), "sel_count")
    nbytes = lib().dsa_decode_select_workspace_size(nq, ld, k)
    ws = _workspace(nbytes, scores.device)
    _check(lib().dsa_decode_select_groups(_p(index_q), _p(gate), _p(q_req), _p(q_pos), nq, g0, ng, _p(summaries),
                                          _p(scales), n_slots, _p(sum_base), sum_base.numel(), _p(scores), ld, flags,
                                          k, _p(sel_idx), _p(sel_count), _p(ws), nbytes, _stream()))
    return sel_idx, sel_count


def sparse_attn_decode_groups(q, k_cache, v_cache, block_table, q_pos, sel_idx, sel_count, g0, out=None, lse=None):
    """dsa_sparse_attn_decode_groups: the shard's caches [n_pages][ng][64][192] and selection
    [B][ng][k]; returns out bf16 [B][16 ng][192] (the heads of groups g0 .. g0 + ng - 1)."""
    nq = q.shape[0]
    _need(q, torch.bfloat16, (nq, HQ, D), "q")
    _need(k_cache, torch.bfloat16, name="k_cache")
    ng = k_cache.shape[1]
    _group_range(g0, ng)
    if k_cache.dim() != 4 or tuple(k_cache.shape[2:]) != (PAGE, D):
        raise ValueError("k_cache must be [n_pages][ng][64][192]")
    _need(v_cache, torch.bfloat16, tuple(k_cache.shape), "v_cache")
    _need(block_table, torch.int32, name="block_table")
    _need(q_pos, torch.int32, (nq,), "q_pos")
    k = sel_idx.shape[-1]
    _need(sel_idx, torch.int32, (nq, ng, k), "sel_idx")
    _need(sel_count, torch.int32, (nq, ng), "sel_count")
    hq = 16 * ng
    if out is None:
        out = torch.empty((nq, hq, D), dtype=torch.bfloat16, device=q.device)
    _need(out, torch.bfloat16, (nq, hq, D), "out")
    if lse is not None:
        _need(lse, torch.float32, (nq, hq), "lse")
    nbytes = lib().dsa_attn_groups_workspace_size(nq, k, ng)
    ws = _workspace(nbytes, q.device)
    _check(lib().dsa_sparse_attn_decode_groups(_p(q), _p(k_cache), _p(v_cache), k_cache.shape[0], _p(block_table),
                                               block_table.shape[1], _p(q_pos), nq, g0, ng, _p(sel_idx),
                                               _p(sel_count), k, _p(out), _p(lse), _p(ws), nbytes, _stream()))
    return out


def selftest_wait_timeout(limit_cycles: int):
    """dsa_selftest_wait_timeout: one kernel whose mbarrier wait nothing completes gives up
    after limit_cycles and sets the timeout bit (read it with check_device)."""
    _check(lib().dsa_selftest_wait_timeout(int(limit_cycles), _stream()))


def copy(dst, src):
    """dsa_copy: copies src into dst (same byte size) with a kernel on the current stream;
    either may be a CUDA tensor or a pinned CPU tensor (reached by the GPU directly)."""
    for t, n in ((dst, "dst"), (src, "src")):
        if not (t.is_cuda or t.is_pinned()):
            raise ValueError(f"{n} must be a CUDA tensor or pinned host memory")
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    nbytes = dst.numel() * dst.element_size()
    if src.numel() * src.element_size() != nbytes:
        raise ValueError("dst and src differ in size")
    _check(lib().dsa_copy(_p(dst), _p(src), nbytes, _stream()))
    return dst


def _attn_args(q, k_cache, v_cache, block_table, q_pos, sel_idx, sel_count, out, lse):
    nq = q.shape[0]
    _need(q, torch.bfloat16, (nq, HQ, D), "q")
    _need(k_cache, torch.bfloat16, name="k_cache")
    if k_cache.dim() != 4 or tuple(k_cache.shape[1:]) != (G, PAGE, D):
        raise ValueError("k_cache must be [n_pages][4][64][192]")
    _need(v_cache, torch.bfloat16, tuple(k_cache.shape), "v_cache")
    _need(block_table, torch.int32, name="block_table")
    _need(q_pos, torch.int32, (nq,), "q_pos")
    k = sel_idx.shape[-1]
    _need(sel_idx, torch.int32, (nq, G, k), "sel_idx")
    _need(sel_count, torch.int32, (nq, G), "sel_count")
    if out is None:
        out = torch.empty((nq, HQ, D), dtype=torch.bfloat16, device=q.device)
    _need(out, torch.bfloat16, (nq, HQ, D), "out")
    if lse is not None:
        _need(lse, torch.float32, (nq, HQ), "lse")
    return nq, k, out


def sparse_attn_decode(q, k_cache, v_cache, block_table, q_pos, sel_idx, sel_count, out=None, lse=None):
    """One query per request (request b = row b of block_table).  Returns out bf16 [B][64][192]."""
    nq, k, out = _attn_args(q, k_cache, v_cache, block_table, q_pos, sel_idx, sel_count, out, lse)
    nbytes = lib().dsa_attn_workspace_size(nq, k)
    ws = _workspace(nbytes, q.device)
    _check(lib().dsa_sparse_attn_decode(_p(q), _p(k_cache), _p(v_cache), k_cache.shape[0], _p(block_table),
                                        block_table.shape[1], _p(q_pos), nq, _p(sel_idx), _p(sel_count), k,
                                        _p(out), _p(lse), _p(ws), nbytes, _stream()))
    return out


def sparse_attn_prefill(q, k_cache, v_cache, block_table, q_req, q_pos, sel_idx, sel_count, out=None, lse=None):
    """Queries of several requests (q_req selects the block_table row).  Returns out."""
    nq, k, out = _attn_args(q, k_cache, v_cache, block_table, q_pos, sel_idx, sel_count, out, lse)
    _need(q_req, torch.int32, (nq,), "q_req")
    nbytes = lib().dsa_attn_workspace_size(nq, k)
    ws = _workspace(nbytes, q.device)
    _check(lib().dsa_sparse_attn_prefill(_p(q), _p(k_cache), _p(v_cache), k_cache.shape[0], _p(block_table),
                                         block_table.shape[1], block_table.shape[0], _p(q_req), _p(q_pos), nq,
                                         _p(sel_idx), _p(sel_count), k, _p(out), _p(lse), _p(ws), nbytes,
                                         _stream()))
    return out


def _cache_args(k_cache, v_cache, block_table):
    _need(k_cache, torch.bfloat16, name="k_cache")
    if k_cache.dim() != 4 or tuple(k_cache.shape[1:]) != (G, PAGE, D):
        raise ValueError("k_cache must be [n_pages][4][64][192]")
    _need(v_cache, torch.bfloat16, tuple(k_cache.shape), "v_cache")
    _need(block_table, torch.int32, name="block_table")
    if block_table.dim() != 2:
        raise ValueError("block_table must be [n_req][max_pages]")


def kv_append(k_cache, v_cache, block_table, q_pos, new_k, new_v, q_req=None):
    """Writes token i's K and V rows (new_k, new_v bf16 [n][4][192]) to the slot of position
    q_pos[i] of request q_req[i] (or i).  With a cyclic block table: the window ring buffer."""
    _cache_args(k_cache, v_cache, block_table)
    n = q_pos.shape[0]
    _need(q_pos, torch.int32, (n,), "q_pos")
    _need(new_k, torch.bfloat16, (n, G, D), "new_k")
    _need(new_v, torch.bfloat16, (n, G, D), "new_v")
    if q_req is not None:
        _need(q_req, torch.int32, (n,), "q_req")
    _check(lib().dsa_kv_append(_p(k_cache), _p(v_cache), k_cache.shape[0], _p(block_table), block_table.shape[1],
                               block_table.shape[0], _p(q_req), _p(q_pos), n, _p(new_k), _p(new_v), _stream()))


def window_attn(q, k_cache, v_cache, block_table, q_pos, window=512, q_req=None, out=None, lse=None):
    """GQA of each query over its last `window` tokens (positions max(0, p-window+1) .. p of
    request q_req[i], or i), read through the block table.  Returns out bf16 [nq][64][192]."""
    nq = q.shape[0]
    _need(q, torch.bfloat16, (nq, HQ, D), "q")
    _cache_args(k_cache, v_cache, block_table)
    _need(q_pos, torch.int32, (nq,), "q_pos")
    if q_req is not None:
        _need(q_req, torch.int32, (nq,), "q_req")
    if out is None:
        out = torch.empty((nq, HQ, D), dtype=torch.bfloat16, device=q.device)
    _need(out, torch.bfloat16, (nq, HQ, D), "out")
    if lse is not None:
        _need(lse, torch.float32, (nq, HQ), "lse")
    nbytes = lib().dsa_window_attn_workspace_size(nq, window)
    ws = _workspace(nbytes, q.device)
    _check(lib().dsa_window_attn(_p(q), _p(k_cache), _p(v_cache), k_cache.shape[0], _p(block_table),
                                 block_table.shape[1], block_table.shape[0], _p(q_req), _p(q_pos), nq, int(window),
                                 _p(out), _p(lse), _p(ws), nbytes, _stream()))
    return out


def window_decode(q, k_cache, v_cache, block_table, q_pos, new_k, new_v, window=512, q_req=None, out=None,
                  lse=None):
    """One window-layer decode step: kv_append(new_k, new_v at q_pos), then window_attn over the
    window ending at the appended token (one launch where the clustered kernel serves it).
    The queries must be distinct requests.  Returns out bf16 [nq][64][192]."""
    nq = q.shape[0]
    _need(q, torch.bfloat16, (nq, HQ, D), "q")
    _cache_args(k_cache, v_cache, block_table)
    _need(q_pos, torch.int32, (nq,), "q_pos")
    _need(new_k, torch.bfloat16, (nq, G, D), "new_k")
    _need(new_v, torch.bfloat16, (nq, G, D), "new_v")
    if q_req is not None:
        _need(q_req, torch.int32, (nq,), "q_req")
    if out is None:
        out = torch.empty((nq, HQ, D), dtype=torch.bfloat16, device=q.device)
    _need(out, torch.bfloat16, (nq, HQ, D), "out")
    if lse is not None:
        _need(lse, torch.float32, (nq, HQ), "lse")
    nbytes = lib().dsa_window_attn_workspace_size(nq, window)
    ws = _workspace(nbytes, q.device)
    _check(lib().dsa_window_decode(_p(k_cache), _p(v_cache), k_cache.shape[0], _p(block_table), block_table.shape[1],
                                   block_table.shape[0], _p(q_req), _p(q_pos), nq, _p(new_k), _p(new_v), _p(q),
                                   int(window), _p(out), _p(lse), _p(ws), nbytes, _stream()))
    return out


FRONTEND_ROWS = HI * DI + G * DI + HI      # weight rows: 16 q heads x 256, 4 k groups x 256, 16 gates


def indexer_frontend(hidden, w, gamma_q, gamma_k, pos, index_q=None, index_k=None, z=None):
    """Hidden states bf16 [T][hid] -> (index_q bf16 [T][16][256], index_k bf16 [T][4][256],
    z fp32 [T][16]): projection by w bf16 [5136][hid], per-head RMSNorm with gamma_q / gamma_k,
    partial RoPE at positions pos int32 [T], sigmoid gates."""
    T, hid = hidden.shape
    _need(hidden, torch.bfloat16, (T, hid), "hidden")
    _need(w, torch.bfloat16, (FRONTEND_ROWS, hid), "w")
    _need(gamma_q, torch.bfloat16, (DI,), "gamma_q")
    _need(gamma_k, torch.bfloat16, (DI,), "gamma_k")
    _need(pos, torch.int32, (T,), "pos")
    dev = hidden.device
    if index_q is None:
        index_q = torch.empty((T, HI, DI), dtype=torch.bfloat16, device=dev)
    if index_k is None:
        index_k = torch.empty((T, G, DI), dtype=torch.bfloat16, device=dev)
    if z is None:
        z = torch.empty((T, HI), dtype=torch.float32, device=dev)
    _need(index_q, torch.bfloat16, (T, HI, DI), "index_q")
    _need(index_k, torch.bfloat16, (T, G, DI), "index_k")
    _need(z, torch.float32, (T, HI), "z")
    _check(lib().dsa_indexer_frontend(_p(hidden), hid, T, _p(w), _p(gamma_q), _p(gamma_k), _p(pos), _p(index_q),
                                      _p(index_k), _p(z), _stream()))
    return index_q, index_k, z

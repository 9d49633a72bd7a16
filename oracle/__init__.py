"""CPU oracle for DSA region-sparse GQA (test infrastructure).

Only the test-suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The CUDA library never does, and this package imports
nothing from it: the two share no code.  The arithmetic lives in ``oracle.c``
(plain C, double precision, one function per step of the method); this module
only compiles it with gcc and marshals numpy arrays.

Functions mirror the library's C-ABI calls:
  compress_regions   A1  region compression          (summary = e4m3 mean of 8 tokens)
  indexer_scores     A2  16-head indexer score        sum_h z_h ReLU(q_h . s)/16
  topk_regions       A3  own region + top-(k-1)       ties -> lower index
  sparse_attention   A4  exact GQA over the selection softmax(q K^T / sqrt(192)) V
  window_attention       the window layers: the same over the last `window` tokens
  indexer_frontend       hidden state -> index_q, index_k (RMSNorm, partial RoPE), gates
plus the number-format helpers the pins use (bf16 and OCP E4M3 codecs).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

REGION, G, DI, HI, HQ, D, PAGE = 8, 4, 256, 16, 64, 192, 64
Q_FP8 = 1

CFLAGS = ["-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp",
          "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _P(t):
    return ctypes.POINTER(t)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            L.oracle_bf16_to_f64.restype = ctypes.c_double
            L.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
            L.oracle_f64_to_bf16.restype = ctypes.c_uint16
            L.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
            L.oracle_e4m3_to_f64.restype = ctypes.c_double
            L.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
            L.oracle_f32_to_e4m3.restype = ctypes.c_uint8
            L.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
            L.oracle_compress_regions.restype = None
            L.oracle_compress_regions.argtypes = [
                _P(ctypes.c_uint16), ctypes.c_int64, _P(ctypes.c_int64), _P(ctypes.c_int64),
                ctypes.c_int, ctypes.c_int64, _P(ctypes.c_uint8), _P(ctypes.c_float)]
            L.oracle_indexer_scores.restype = None
            L.oracle_indexer_scores.argtypes = [
                _P(ctypes.c_uint16), _P(ctypes.c_float), _P(ctypes.c_int32), _P(ctypes.c_int32),
                ctypes.c_int, _P(ctypes.c_uint8), _P(ctypes.c_float), _P(ctypes.c_int64),
                ctypes.c_int64, _P(ctypes.c_float), ctypes.c_int64, ctypes.c_uint32]
            L.oracle_topk_regions.restype = None
            L.oracle_topk_regions.argtypes = [
                _P(ctypes.c_float), ctypes.c_int64, _P(ctypes.c_int32), ctypes.c_int, ctypes.c_int,
                _P(ctypes.c_int32), _P(ctypes.c_int32)]
            L.oracle_sparse_attention.restype = None
            L.oracle_sparse_attention.argtypes = [
                _P(ctypes.c_uint16), _P(ctypes.c_uint16), _P(ctypes.c_uint16),
                _P(ctypes.c_int32), ctypes.c_int, _P(ctypes.c_int32), _P(ctypes.c_int32),
                ctypes.c_int, _P(ctypes.c_int32), _P(ctypes.c_int32), ctypes.c_int,
                _P(ctypes.c_uint16), _P(ctypes.c_float), _P(ctypes.c_double)]
            L.oracle_window_attention.restype = None
            L.oracle_window_attention.argtypes = [
                _P(ctypes.c_uint16), _P(ctypes.c_uint16), _P(ctypes.c_uint16),
                _P(ctypes.c_int32), ctypes.c_int, _P(ctypes.c_int32), _P(ctypes.c_int32),
                ctypes.c_int, ctypes.c_int, _P(ctypes.c_uint16), _P(ctypes.c_float), _P(ctypes.c_double)]
            L.oracle_indexer_frontend.restype = None
            L.oracle_indexer_frontend.argtypes = [
                _P(ctypes.c_uint16), _P(ctypes.c_uint16), _P(ctypes.c_uint16), _P(ctypes.c_uint16),
                _P(ctypes.c_int32), ctypes.c_int, ctypes.c_int, _P(ctypes.c_uint16), _P(ctypes.c_uint16),
                _P(ctypes.c_float)]
            L.oracle_set_threads.restype = None
            L.oracle_set_threads.argtypes = [ctypes.c_int]
            L.oracle_get_threads.restype = ctypes.c_int
            L.oracle_get_threads.argtypes = []
            _lib = L
    return _lib


def _arr(a, dtype):
    """C-contiguous numpy view of `a` with the exact dtype (no value conversion)."""
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def _ptr(a, ct):
    return a.ctypes.data_as(_P(ct))


# ---------------------------------------------------------------- formats

def bf16_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).ravel()
    L = lib()
    return np.array([L.oracle_bf16_to_f64(int(x)) for x in b], dtype=np.float64)


def f64_to_bf16(x) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_f64_to_bf16(float(v)) for v in np.asarray(x, np.float64).ravel()],
                    dtype=np.uint16)


def e4m3_to_f64(codes) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_e4m3_to_f64(int(c)) for c in np.asarray(codes, np.uint8).ravel()],
                    dtype=np.float64)


def f32_to_e4m3(x) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_f32_to_e4m3(float(v)) for v in np.asarray(x, np.float32).ravel()],
                    dtype=np.uint8)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


# ---------------------------------------------------------------- A1..A4

def compress_regions(index_k_bits, src_row, dst_slot, n_slots, summaries=None, scales=None):
    """index_k_bits: uint16 [tokens][4][256] (bf16 bit patterns, rows may be a 2-D
    [tokens][row_stride] view).  Returns the group-major pool (summaries uint8
    [4][n_slots][256], scales float32 [4][n_slots]); untouched slots stay as passed
    (zeros by default)."""
    k = _arr(index_k_bits, np.uint16)
    row_stride = int(np.prod(k.shape[1:]))
    src = _arr(np.asarray(src_row, np.int64), np.int64)
    dst = _arr(np.asarray(dst_slot, np.int64), np.int64)
    n = int(src.shape[0])
    if n and (src.min() < 0 or src.max() + REGION > k.shape[0]):
        raise ValueError("src_row out of range")
    if n and (dst.min() < 0 or dst.max() >= n_slots):
        raise ValueError("dst_slot out of range")
    S = np.zeros((G, n_slots, DI), np.uint8) if summaries is None else _arr(summaries, np.uint8)
    C = np.zeros((G, n_slots), np.float32) if scales is None else _arr(scales, np.float32)
    if S.shape != (G, n_slots, DI) or C.shape != (G, n_slots):
        raise ValueError("pool shape must be [4][n_slots][256] / [4][n_slots]")
    lib().oracle_compress_regions(_ptr(k, ctypes.c_uint16), row_stride, _ptr(src, ctypes.c_int64),
                                  _ptr(dst, ctypes.c_int64), n, int(n_slots), _ptr(S, ctypes.c_uint8),
                                  _ptr(C, ctypes.c_float))
    return S, C


def indexer_scores(index_q_bits, gate, q_req, q_pos, summaries, scales, sum_base, ld=None,
                   flags=0, fill=np.nan):
    """Returns float32 [nq][4][ld]; entries r >= q_pos//8 hold `fill`."""
    q = _arr(index_q_bits, np.uint16)
    nq = int(q.shape[0])
    z = _arr(np.asarray(gate, np.float32), np.float32)
    qr = _arr(np.asarray(q_req, np.int32), np.int32)
    qp = _arr(np.asarray(q_pos, np.int32), np.int32)
    S = _arr(summaries, np.uint8)
    C = _arr(scales, np.float32)
    base = _arr(np.asarray(sum_base, np.int64), np.int64)
    if S.ndim != 3 or S.shape[0] != G or S.shape[2] != DI or C.shape != S.shape[:2]:
        raise ValueError("pool shape must be [4][n_slots][256] / [4][n_slots]")
    n_slots = int(S.shape[1])
    own = qp // REGION
    if ld is None:
        ld = max(1, int(own.max()) if nq else 1)
    if nq and int(own.max()) > ld:
        raise ValueError("ld smaller than the largest own-region index")
    for i in range(nq):
        if own[i] > 0 and base[qr[i]] + own[i] > n_slots:
            raise ValueError("summary slots out of range")
    out = np.full((nq, G, ld), fill, np.float32)
    lib().oracle_indexer_scores(_ptr(q, ctypes.c_uint16), _ptr(z, ctypes.c_float),
                                _ptr(qr, ctypes.c_int32), _ptr(qp, ctypes.c_int32), nq,
                                _ptr(S, ctypes.c_uint8), _ptr(C, ctypes.c_float),
                                _ptr(base, ctypes.c_int64), n_slots, _ptr(out, ctypes.c_float),
                                int(ld), int(flags))
    return out


def topk_regions(scores, q_pos, k):
    """scores float32 [nq][4][ld] -> (sel_idx int32 [nq][4][k], sel_count int32 [nq][4])."""
    s = _arr(scores, np.float32)
    nq, g, ld = s.shape
    assert g == G
    qp = _arr(np.asarray(q_pos, np.int32), np.int32)
    if nq and int((qp // REGION).max()) > ld:
        raise ValueError("ld smaller than the largest own-region index")
    if k < 1:
        raise ValueError("k must be >= 1")
    idx = np.empty((nq, G, k), np.int32)
    cnt = np.empty((nq, G), np.int32)
    lib().oracle_topk_regions(_ptr(s, ctypes.c_float), int(ld), _ptr(qp, ctypes.c_int32), nq, int(k),
                              _ptr(idx, ctypes.c_int32), _ptr(cnt, ctypes.c_int32))
    return idx, cnt


def sparse_attention(q_bits, k_cache_bits, v_cache_bits, block_table, q_req, q_pos, sel_idx,
                     sel_count, want_f64=False):
    """q uint16 [nq][64][192]; caches uint16 [pages][4][64][192]; block_table int32
    [B][max_pages]; sel_idx int32 [nq][4][k].  Returns (out bf16 bits [nq][64][192],
    lse float32 [nq][64][, out float64])."""
    q = _arr(q_bits, np.uint16)
    kc = _arr(k_cache_bits, np.uint16)
    vc = _arr(v_cache_bits, np.uint16)
    bt = _arr(np.asarray(block_table, np.int32), np.int32)
    qr = _arr(np.asarray(q_req, np.int32), np.int32)
    qp = _arr(np.asarray(q_pos, np.int32), np.int32)
    si = _arr(np.asarray(sel_idx, np.int32), np.int32)
    sc = _arr(np.asarray(sel_count, np.int32), np.int32)
    nq = int(q.shape[0])
    k = int(si.shape[-1])
    max_pages = int(bt.shape[1])
    n_pages = int(kc.shape[0])
    for i in range(nq):
        for g in range(G):
            sel = si[i, g, : sc[i, g]]
            if sel.size:
                toks = (sel.astype(np.int64) * REGION)
                toks = np.concatenate([toks + u for u in range(REGION)])
                toks = toks[toks <= qp[i]]
                if toks.size and int(toks.max()) // PAGE >= max_pages:
                    raise ValueError("selected token beyond the block table")
                pages = bt[qr[i], np.unique(toks // PAGE)] if toks.size else np.array([], np.int32)
                if pages.size and (pages.min() < 0 or pages.max() >= n_pages):
                    raise ValueError("page index out of range")
    out = np.empty((nq, HQ, D), np.uint16)
    lse = np.empty((nq, HQ), np.float32)
    o64 = np.empty((nq, HQ, D), np.float64) if want_f64 else None
    lib().oracle_sparse_attention(
        _ptr(q, ctypes.c_uint16), _ptr(kc, ctypes.c_uint16), _ptr(vc, ctypes.c_uint16),
        _ptr(bt, ctypes.c_int32), max_pages, _ptr(qr, ctypes.c_int32), _ptr(qp, ctypes.c_int32),
        nq, _ptr(si, ctypes.c_int32), _ptr(sc, ctypes.c_int32), k, _ptr(out, ctypes.c_uint16),
        _ptr(lse, ctypes.c_float), _ptr(o64, ctypes.c_double) if want_f64 else None)
    if want_f64:
        return out, lse, o64
    return out, lse


def window_attention(q_bits, k_cache_bits, v_cache_bits, block_table, q_req, q_pos, window=512,
                     want_f64=False):
    """Sliding-window GQA of the window layers ([P1] §滑窗注意力; [P2] §第一招: the last 512
    tokens, kept in a ring buffer): query i attends tokens max(0, p - window + 1) .. p of its
    request through the block table.  q uint16 [nq][64][192]; caches uint16
    [pages][4][64][192]; block_table int32 [B][max_pages].  Returns (out bf16 bits
    [nq][64][192], lse float32 [nq][64][, out float64])."""
    q = _arr(q_bits, np.uint16)
    kc = _arr(k_cache_bits, np.uint16)
    vc = _arr(v_cache_bits, np.uint16)
    bt = _arr(np.asarray(block_table, np.int32), np.int32)
    qr = _arr(np.asarray(q_req, np.int32), np.int32)
    qp = _arr(np.asarray(q_pos, np.int32), np.int32)
    if window < 1:
        raise ValueError("window must be >= 1")
    nq = int(q.shape[0])
    max_pages = int(bt.shape[1])
    n_pages = int(kc.shape[0])
    for i in range(nq):
        p = int(qp[i])
        if p < 0:
            continue
        lo = max(0, p - window + 1)
        if p // PAGE >= max_pages:
            raise ValueError("window token beyond the block table")
        pages = bt[qr[i], lo // PAGE: p // PAGE + 1]
        if pages.min() < 0 or pages.max() >= n_pages:
            raise ValueError("page index out of range")
    out = np.empty((nq, HQ, D), np.uint16)
    lse = np.empty((nq, HQ), np.float32)
    o64 = np.empty((nq, HQ, D), np.float64) if want_f64 else None
    lib().oracle_window_attention(
        _ptr(q, ctypes.c_uint16), _ptr(kc, ctypes.c_uint16), _ptr(vc, ctypes.c_uint16),
        _ptr(bt, ctypes.c_int32), max_pages, _ptr(qr, ctypes.c_int32), _ptr(qp, ctypes.c_int32),
        nq, int(window), _ptr(out, ctypes.c_uint16), _ptr(lse, ctypes.c_float),
        _ptr(o64, ctypes.c_double) if want_f64 else None)
    if want_f64:
        return out, lse, o64
    return out, lse


FRONTEND_ROWS = HI * DI + G * DI + HI          # 5,136 projection rows: q heads, k groups, gates


def indexer_frontend(hidden_bits, w_bits, gamma_q_bits, gamma_k_bits, pos):
    """Indexer front end ([P2] §索引器打分: index_q / index_k / index_z projected from the
    hidden state, normalised, RoPE on part of the dimensions).  hidden uint16 (bf16 bits)
    [T][hid]; w uint16 [5136][hid] (rows: 16 x 256 q, 4 x 256 k, 16 gates); gamma_q/gamma_k
    uint16 [256]; pos int32 [T].  Returns (index_q bf16 bits [T][16][256], index_k bf16 bits
    [T][4][256], z float32 [T][16])."""
    h = _arr(hidden_bits, np.uint16)
    w = _arr(w_bits, np.uint16)
    gq = _arr(gamma_q_bits, np.uint16)
    gk = _arr(gamma_k_bits, np.uint16)
    p = _arr(np.asarray(pos, np.int32), np.int32)
    T, hid = int(h.shape[0]), int(h.shape[1])
    if w.shape != (FRONTEND_ROWS, hid) or gq.shape != (DI,) or gk.shape != (DI,) or p.shape != (T,):
        raise ValueError("shapes: hidden [T][hid], w [5136][hid], gammas [256], pos [T]")
    iq = np.empty((T, HI, DI), np.uint16)
    ik = np.empty((T, G, DI), np.uint16)
    z = np.empty((T, HI), np.float32)
    lib().oracle_indexer_frontend(_ptr(h, ctypes.c_uint16), _ptr(w, ctypes.c_uint16), _ptr(gq, ctypes.c_uint16),
                                  _ptr(gk, ctypes.c_uint16), _ptr(p, ctypes.c_int32), T, hid,
                                  _ptr(iq, ctypes.c_uint16), _ptr(ik, ctypes.c_uint16), _ptr(z, ctypes.c_float))
    return iq, ik, z

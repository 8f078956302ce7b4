"""Oracle: a plain, slow CPU definition of the CSA2 decode step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``csa2_fp4_sparse_b200``) never does, and the two
share no code.

The arithmetic lives in ``oracle.c`` (double precision on dequantised values,
see the header there for the definitions and the pages' passages they follow);
this module only marshals numpy arrays and composes the per-query steps in the
order the pages give:

* Full layer (dbyun.net article 10794, section "KV Cache 成为这一代架构改造的核心",
  the paragraphs on the three layer modes and on the hierarchical indexer):
  score every visible position, keep the best ``P`` blocks of 8 positions as the
  candidate pool, then the best ``K`` positions of that pool.
* Reindex layer (same passage): rescore only the Full layer's pool with the
  layer's own indexer query, keep the best ``K``.
* Reuse layer (same passage): attention only, over the index list of the
  nearest preceding Full/Reindex layer.
* Sliding-window attention (prism.simon-ai.net article 7901, the SWA section:
  window of the last 128 tokens; page 1: SWA KV stays FP8) merged with the
  sparse attention as one softmax over the concatenated key sets.

Readings of the pages where they are silent: a query at position p sees
positions 0..p; block ties and position ties go to the lower id; every Reindex
layer rescores the Full layer's pool; the Full layer attends with its own top-K.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_U8 = ctypes.POINTER(ctypes.c_uint8)
_F = ctypes.POINTER(ctypes.c_float)
_I64 = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (plain C11, OpenMP, no FMA contraction)."""
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
            "-fno-fast-math", "-Wall", "-o", _LIB_PATH, src, "-lm",
        ])
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode_nonneg.restype = ctypes.c_uint8
        L.orc_e4m3_encode_nonneg.argtypes = [ctypes.c_double]
        L.orc_e2m1_value.restype = ctypes.c_double
        L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        L.orc_quantize_fp4.restype = ctypes.c_int64
        L.orc_quantize_fp4.argtypes = [_F, ctypes.c_int64, ctypes.c_int, _U8, _U8]
        L.orc_dequant_fp4.restype = None
        L.orc_dequant_fp4.argtypes = [_U8, _U8, ctypes.c_int64, ctypes.c_int, _D]
        L.orc_index_scores_fp4.restype = None
        L.orc_index_scores_fp4.argtypes = [_D, _D, ctypes.c_int, ctypes.c_int, _U8, _U8, ctypes.c_int64, _D]
        L.orc_topk.restype = ctypes.c_int64
        L.orc_topk.argtypes = [_D, _I64, ctypes.c_int64, ctypes.c_int64, _I64]
        L.orc_block_scores.restype = ctypes.c_int64
        L.orc_block_scores.argtypes = [_D, ctypes.c_int64, ctypes.c_int, _D]
        L.orc_attend.restype = None
        L.orc_attend.argtypes = [_D, ctypes.c_int, ctypes.c_int, _D, ctypes.c_int64, ctypes.c_double, _D, _D]
        _lib = L
    return _lib


def _p(a, t):
    return a.ctypes.data_as(t)


# ---------------------------------------------------------------------------
# formats

def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(code)


def e4m3_encode(v: float) -> int:
    """nearest non-negative finite E4M3 code (ties to even, saturating)"""
    return lib().orc_e4m3_encode_nonneg(float(v))


def e2m1_value(nib: int) -> float:
    return lib().orc_e2m1_value(nib)


def quantize_fp4(x: np.ndarray):
    """x [n][d] float32 -> (codes [n][d/2] u8, scales [n][d/32] u8, n_nonfinite_groups)"""
    x = np.ascontiguousarray(x, dtype=np.float32)
    n, d = x.shape
    assert d % 32 == 0
    codes = np.zeros((n, d // 2), np.uint8)
    scales = np.zeros((n, d // 32), np.uint8)
    bad = lib().orc_quantize_fp4(_p(x, _F), n, d, _p(codes, _U8), _p(scales, _U8))
    return codes, scales, int(bad)


def dequant_fp4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    n = codes.shape[0]
    d = codes.shape[1] * 2
    out = np.zeros((n, d), np.float64)
    lib().orc_dequant_fp4(_p(codes, _U8), _p(scales, _U8), n, d, _p(out, _D))
    return out


def e4m3_decode_array(codes: np.ndarray) -> np.ndarray:
    table = np.array([e4m3_value(c) for c in range(256)], np.float64)
    return table[np.asarray(codes, np.uint8)]


# ---------------------------------------------------------------------------
# per-query steps

def index_scores(q: np.ndarray, w: np.ndarray, kcodes: np.ndarray, kscales: np.ndarray) -> np.ndarray:
    """s_t = sum_h w_h * max(0, q_h . k_t) for every row t of the FP4 key rows.

    q: [H][d] dequantised indexer query (double), w: [H]."""
    q = np.ascontiguousarray(q, np.float64)
    w = np.ascontiguousarray(w, np.float64)
    kcodes = np.ascontiguousarray(kcodes, np.uint8)
    kscales = np.ascontiguousarray(kscales, np.uint8)
    H, d = q.shape
    n = kcodes.shape[0]
    s = np.zeros(n, np.float64)
    lib().orc_index_scores_fp4(_p(q, _D), _p(w, _D), H, d, _p(kcodes, _U8), _p(kscales, _U8), n, _p(s, _D))
    return s


def topk(score: np.ndarray, ids: np.ndarray, k: int) -> np.ndarray:
    """the k best ids by (score desc, id asc), returned ascending"""
    score = np.ascontiguousarray(score, np.float64)
    ids = np.ascontiguousarray(ids, np.int64)
    out = np.zeros(max(k, 1), np.int64)
    m = lib().orc_topk(_p(score, _D), _p(ids, _I64), len(score), k, _p(out, _I64))
    return out[:m].copy()


def block_scores(s: np.ndarray, p: int, blk: int = 8) -> np.ndarray:
    s = np.ascontiguousarray(s, np.float64)
    nb = (p + 1 + blk - 1) // blk
    bs = np.zeros(max(nb, 1), np.float64)
    m = lib().orc_block_scores(_p(s, _D), p, blk, _p(bs, _D))
    return bs[:m].copy()


def attend(q: np.ndarray, v: np.ndarray, scale: float):
    """softmax(scale * q v^T) v per head; q [H][D], v [n][D]; returns (out [H][D], lse [H])"""
    q = np.ascontiguousarray(q, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    H, D = q.shape
    n = v.shape[0]
    out = np.zeros((H, D), np.float64)
    lse = np.zeros(H, np.float64)
    lib().orc_attend(_p(q, _D), H, D, _p(v, _D), n, scale, _p(out, _D), _p(lse, _D))
    return out, lse


@dataclass
class FullResult:
    scores: np.ndarray        # s_t, t = 0..p
    block_scores: np.ndarray  # B_j, j = 0..nb-1
    pool: np.ndarray          # selected block ids, ascending
    idx: np.ndarray           # selected positions, ascending


def pool_positions(pool_blocks: np.ndarray, p: int, blk: int = 8) -> np.ndarray:
    """visible positions of the pool blocks (ascending)"""
    if len(pool_blocks) == 0:
        return np.zeros(0, np.int64)
    pos = (np.asarray(pool_blocks, np.int64)[:, None] * blk + np.arange(blk)[None, :]).reshape(-1)
    return pos[pos <= p]


def full_select(q: np.ndarray, w: np.ndarray, kcodes: np.ndarray, kscales: np.ndarray, p: int,
                P: int, K: int, blk: int = 8) -> FullResult:
    """Full mode over the visible rows 0..p of the indexer K (rows indexed by position)."""
    s = index_scores(q, w, kcodes[: p + 1], kscales[: p + 1])
    bs = block_scores(s, p, blk)
    pool = topk(bs, np.arange(len(bs), dtype=np.int64), P)
    pos = pool_positions(pool, p, blk)
    idx = topk(s[pos], pos, K)
    return FullResult(s, bs, pool, idx)


def reindex_select(q: np.ndarray, w: np.ndarray, kcodes: np.ndarray, kscales: np.ndarray, p: int,
                   pool: np.ndarray, K: int, blk: int = 8):
    """Reindex mode: rescore the pool positions with (q, w); returns (idx, scores over pool positions, positions)."""
    pos = pool_positions(pool, p, blk)
    s = index_scores(q, w, kcodes[pos], kscales[pos])
    return topk(s, pos, K), s, pos


def attend_rows(qmain: np.ndarray, kv_rows: np.ndarray, swa_rows: np.ndarray | None, scale: float):
    """Attention of one query token over the gathered Main KV rows, optionally
    concatenated with the sliding-window rows (one softmax over both sets)."""
    v = kv_rows if swa_rows is None or len(swa_rows) == 0 else np.concatenate([kv_rows, swa_rows], 0)
    return attend(qmain, v, scale)

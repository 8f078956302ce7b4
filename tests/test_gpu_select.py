"""The two selections (block top-P pool, pool top-K positions) on planted
scores, exact.

With one indexer head, weight 1 and a one-hot FP4 query (1.0 on channel 0),
the score of position t is exactly the dequantised channel 0 of its key,
e2m1(code_t) * e4m3(scale_t) (ReLU of a non-negative value), so the planted
key bytes fix every score exactly and the selections can be compared with the
oracle's exhaustive top-k id for id: ties at the k-th score take the lowest
ids.  The patterns cover a single CTA per group, groups split over several
CTAs, heavy ties, all-equal scores and a structured pattern (high scores on
an evenly spaced grid of blocks)."""
import ctypes

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _C():
    import csa2_fp4_sparse_b200 as C
    return C


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _run(code, scale, P, K):
    """code, scale: per-position channel-0 E2M1 code (1..7 or 0) and E4M3
    scale byte of one sequence of L = len(code) positions, one query token at
    the last position.  Returns (pool, idx) from csa2_index_full and the exact
    position scores."""
    C = _C()
    L = len(code)
    dI = 64
    rows = (L + 7) // 8 * 8  # the indexer cache holds a multiple of 8 rows at d_I = 64
    codes = np.zeros((rows, dI // 2), np.uint8)
    codes[:L, 0] = np.asarray(code, np.uint8) & 7
    scales = np.zeros((rows, dI // 32), np.uint8)
    scales[:L, 0] = np.asarray(scale, np.uint8)
    val = np.array([E2M1[c & 7] for c in code], np.float64) * np.array([oracle.e4m3_value(int(s)) for s in scale])
    dev = "cuda"
    kc_t = torch.from_numpy(codes).to(dev)
    ks_t = torch.from_numpy(scales).to(dev)
    seq_len = torch.tensor([L], dtype=torch.int32, device=dev)
    tok_start = torch.tensor([0, 1], dtype=torch.int32, device=dev)
    tok_seq = torch.tensor([0], dtype=torch.int32, device=dev)
    tok_pos = torch.tensor([L - 1], dtype=torch.int32, device=dev)
    seq_base = torch.tensor([0], dtype=torch.int64, device=dev)
    qb = C.csa2_query_batch(1, 1, L, 1, seq_len.data_ptr(), tok_start.data_ptr(), tok_seq.data_ptr(),
                            tok_pos.data_ptr())
    kc = C.csa2_fp4_cache(kc_t.data_ptr(), ks_t.data_ptr(), rows, dI, 0, None, 0, seq_base.data_ptr())
    qcodes = torch.zeros(1, dI // 2, dtype=torch.uint8, device=dev)
    qcodes[0, 0] = 0x2  # element 0 = 1.0
    qscales = torch.zeros(1, dI // 32, dtype=torch.uint8, device=dev)
    qscales[0, 0] = 0x38  # E4M3 1.0
    w = torch.ones(1, dtype=torch.float32, device=dev)
    nb = ctypes.c_size_t(0)
    C.check(C.csa2_index_workspace_size(ctypes.byref(qb), 1, dI, P, K, ctypes.byref(nb)))
    ws = torch.empty(nb.value, dtype=torch.uint8, device=dev)
    pool = torch.full((1, P), -7, dtype=torch.int32, device=dev)
    pool_n = torch.zeros(1, dtype=torch.int32, device=dev)
    idx = torch.full((1, K), -7, dtype=torch.int32, device=dev)
    idx_n = torch.zeros(1, dtype=torch.int32, device=dev)
    C.check(C.csa2_index_full(ctypes.byref(qb), qcodes.data_ptr(), qscales.data_ptr(), w.data_ptr(), 1,
                              ctypes.byref(kc), P, K, pool.data_ptr(), pool_n.data_ptr(), idx.data_ptr(),
                              idx_n.data_ptr(), None, ws.data_ptr(), ws.numel(), _stream()))
    st = C.csa2_get_status(_stream())
    assert st == 0, (st, C.csa2_last_error())
    pl, pn = pool[0].cpu().numpy(), int(pool_n[0])
    ix, xn = idx[0].cpu().numpy(), int(idx_n[0])
    assert np.all(pl[pn:] == -1) and np.all(ix[xn:] == -1)
    return pl[:pn].astype(np.int64), ix[:xn].astype(np.int64), val


def _expect(val, P, K):
    L = len(val)
    bs = oracle.block_scores(val, L - 1)
    pool = oracle.topk(bs, np.arange(len(bs)), P)
    pos = oracle.pool_positions(pool, L - 1)
    idx = oracle.topk(val[pos], pos, K)
    return pool, idx


def _check(code, scale, P=2048, K=512):
    pool, idx, val = _run(code, scale, P, K)
    epool, eidx = _expect(val, P, K)
    assert np.array_equal(pool, epool), f"pool differs at {np.flatnonzero(pool[:len(epool)] != epool[:len(pool)])[:5]}"
    assert np.array_equal(idx, eidx), f"idx differs at {np.flatnonzero(idx[:len(eidx)] != eidx[:len(idx)])[:5]}"


@pytest.mark.parametrize("nb", [3000, 40000, 131072])
def test_random_with_heavy_ties(nb):
    """few distinct score levels: the k-th score is shared by many ids"""
    rng = np.random.default_rng(nb)
    L = nb * 8
    code = rng.integers(1, 8, L)
    scale = rng.integers(0x30, 0x34, L)  # 4 scales x 7 codes: under 28 levels
    _check(code, scale)


@pytest.mark.parametrize("nb", [5000, 40000])
def test_distinct_scores_with_needles(nb):
    rng = np.random.default_rng(7 + nb)
    L = nb * 8
    code = rng.integers(1, 8, L)
    scale = rng.integers(0x20, 0x58, L)
    needles = rng.choice(nb, 64, replace=False)
    for b in needles:
        scale[b * 8:(b + 1) * 8] = 0x70
    _check(code, scale)


@pytest.mark.parametrize("nb", [300, 40000])
def test_all_scores_equal(nb):
    L = nb * 8
    _check(np.full(L, 2), np.full(L, 0x38))


def test_evenly_spaced_high_blocks():
    """4096 high blocks on an evenly spaced grid over 40000 (more than P), in
    eight score levels, over a flat background"""
    nb, ns = 40000, 4096
    L = nb * 8
    code = np.full(L, 1)
    scale = np.full(L, 0x30)
    for i in range(ns):
        b = ((2 * i + 1) * nb) // (2 * ns)
        scale[b * 8:(b + 1) * 8] = 0x50 + (i % 8)
    _check(code, scale)


def test_pool_smaller_than_p_and_k():
    """fewer blocks than P and fewer positions than K: everything is taken"""
    rng = np.random.default_rng(3)
    L = 100 * 8 + 5
    _check(rng.integers(0, 8, L), rng.integers(0x30, 0x40, L), P=2048, K=2048)

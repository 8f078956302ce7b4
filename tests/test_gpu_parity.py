"""GPU-vs-oracle parity through the C ABI (libcsa2.so)."""
import ctypes
import math

import numpy as np
import pytest

import oracle
from tests.harness import OracleView, check_token, grade_attention, grade_set

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _C():
    import csa2_fp4_sparse_b200 as C
    return C


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _status():
    return _C().csa2_get_status(_stream())


# ---------------------------------------------------------------- quantiser

def _special_rows(rng, n, d):
    x = rng.standard_normal((n, d)).astype(np.float32)
    x *= np.exp(rng.uniform(-12, 10, (n, 1))).astype(np.float32)
    # rounding boundaries of the E2M1 grid for random E4M3 scales
    for r in range(0, n, 3):
        sc = oracle.e4m3_value(int(rng.integers(1, 0x7F)))
        mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float64) * sc
        vals = np.concatenate([mids, np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
                               np.nextafter(mids.astype(np.float32), np.float32(0))]).astype(np.float32)
        row = np.resize(vals, d).astype(np.float32)
        row[::32] = np.float32(6 * sc)
        row[1::5] *= -1
        x[r] = row
    x[1] = 0.0
    x[2] = -0.0
    x[4, :32] = np.float32(1e-5)
    x[5, :32] = np.float32(448 * 6 * 3)  # saturating scale
    return x


@pytest.mark.parametrize("d", [32, 64, 128, 512])
def test_quantize_bitexact(d):
    C = _C()
    rng = np.random.default_rng(d)
    x = _special_rows(rng, 3000, d)
    xd = torch.from_numpy(x).cuda()
    codes = torch.zeros(3000, d // 2, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(3000, d // 32, dtype=torch.uint8, device="cuda")
    C.check(C.csa2_quantize_fp4(xd.data_ptr(), 3000, d, None, codes.data_ptr(), scales.data_ptr(), _stream()))
    assert _status() == 0
    rc, rs, bad = oracle.quantize_fp4(x)
    assert bad == 0
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy(), rs)


def test_quantize_slot_mapping_and_nonfinite():
    C = _C()
    rng = np.random.default_rng(5)
    x = rng.standard_normal((100, 128)).astype(np.float32)
    x[7, 40] = np.inf
    slot = rng.permutation(200)[:100].astype(np.int64)
    codes = torch.full((200, 64), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((200, 4), 0xAB, dtype=torch.uint8, device="cuda")
    xd = torch.from_numpy(x).cuda()  # kept alive until the kernel has run
    sd = torch.from_numpy(slot).cuda()
    C.check(C.csa2_quantize_fp4(xd.data_ptr(), 100, 128, sd.data_ptr(), codes.data_ptr(), scales.data_ptr(),
                                _stream()))
    assert _status() == C.CSA2_ERR_NONFINITE
    assert _status() == 0  # cleared
    rc, rs, bad = oracle.quantize_fp4(x)
    assert bad == 1
    gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
    ok = np.ones(100, bool)
    ok[7] = False
    assert np.array_equal(gc[slot[ok]], rc[ok]) and np.array_equal(gs[slot[ok]], rs[ok])
    assert np.all(gc[slot[7], 16:32] == 0) and gs[slot[7], 1] == 0  # the bad group is zeroed
    untouched = np.setdiff1d(np.arange(200), slot)
    assert np.all(gc[untouched] == 0xAB)


def test_selftest_timeout_status():
    C = _C()
    C.check(C.csa2_selftest_wait_timeout(2_000_000, _stream()))
    assert _status() == C.CSA2_ERR_TIMEOUT
    assert _status() == 0
    x = torch.ones(4, 32, device="cuda")  # the context is still usable
    assert float(x.sum()) == 128.0


# ---------------------------------------------------------------- decode stack

def _run_stack(cfg, append=True):
    from synth.gpu import DeviceWorkload
    from synth.workloads import make_workload
    C = _C()
    w = make_workload(cfg)
    dw = DeviceWorkload(w)
    dw.fill_caches(include_new=not append)
    desc = dw.stack_desc(append=append)
    ws = dw.stack_workspace(desc)
    C.check(C.csa2_decode_stack(ctypes.byref(desc), ws.data_ptr(), ws.numel(), _stream()))
    assert _status() == 0, C.csa2_last_error()
    return w, dw


def _gpu_view(w, dw, tok):
    out = {"pool": dw.pool_out[tok].cpu().numpy(), "idx": {}, "out": {}}
    out["pool_n"] = int((out["pool"] >= 0).sum())
    for l, m in enumerate(w.modes):
        if m in "FR":
            out["idx"][l] = dw.idx_out[l][tok].cpu().numpy()
        out["out"][l] = dw.out[l][tok].float().cpu().numpy()
    return out


def _check_all(w, dw, toks):
    swaps = 0
    for tok in toks:
        st = check_token(OracleView(w), tok, _gpu_view(w, dw, tok))
        swaps += st["swaps"]
    return swaps


def _small(i, **kw):
    from synth.workloads import CONFIGS
    return CONFIGS[i].with_(**kw)


def test_stack_config1_full_size():
    from synth.workloads import CONFIGS
    w, dw = _run_stack(CONFIGS[1])
    _check_all(w, dw, range(w.T))


@pytest.mark.parametrize("i", [2, 3, 4, 5, 6])
def test_stack_full_size_sampled(i):
    """The full-size workloads the benchmark times (same kernels and grids),
    graded on sampled query tokens: the first, the last and two seeded picks,
    every layer of each."""
    from synth.workloads import CONFIGS
    w, dw = _run_stack(CONFIGS[i])
    rng = np.random.default_rng(100 + i)
    toks = sorted(set([0, w.T - 1] + rng.choice(w.T, size=min(2, w.T), replace=False).tolist()))
    _check_all(w, dw, toks)


@pytest.mark.parametrize("case", [
    dict(i=2, B=2, lengths=("fixed", 5000)),
    dict(i=2, B=3, lengths=("list", [8, 9, 1000])),                        # tiny contexts, partial blocks
    dict(i=2, B=2, lengths=("list", [100, 17000]), n_needles=4),           # K > visible, pool < nblocks
    dict(i=3, B=4, lengths=("uniform8", 2000, 20000)),                     # paged, permuted pages
    dict(i=4, B=2, lengths=("fixed", 20000)),                              # outliers, needles
    dict(i=5, B=6, lengths=("loguniform", 60, 30000)),                     # SWA + W in 1..6, window truncated
    dict(i=5, B=3, lengths=("list", [7, 200, 5000]), out_dtype="f32"),     # SWA, fp32 output graded strictly
])
def test_stack_small_variants(case):
    case = dict(case)
    i = case.pop("i")
    w, dw = _run_stack(_small(i, **case))
    _check_all(w, dw, range(w.T))


def test_stack_all_zero_keys_ties():
    """every key zero: all scores tie at 0; selections must take the lowest ids"""
    from synth.gpu import DeviceWorkload
    from synth.workloads import make_workload
    C = _C()
    cfg = _small(2, B=1, lengths=("fixed", 3000), n_reindex=1, n_reuse=1, n_needles=0)
    w = make_workload(cfg)
    dw = DeviceWorkload(w)
    desc = dw.stack_desc(append=False)  # caches stay all-zero
    ws = dw.stack_workspace(desc)
    C.check(C.csa2_decode_stack(ctypes.byref(desc), ws.data_ptr(), ws.numel(), _stream()))
    assert _status() == 0
    nb = (3000 + 7) // 8
    pool = dw.pool_out[0].cpu().numpy()
    assert list(pool[:nb]) == list(range(nb))  # nb <= P: every block
    idx = dw.idx_out[0][0].cpu().numpy()
    assert list(idx) == list(range(cfg.K))
    # attention over zero rows: output 0
    assert float(dw.out[0].float().abs().max()) == 0.0


def test_individual_entry_points_match_stack():
    """csa2_index_full / csa2_index_reindex / csa2_attend_reuse called one by one"""
    from synth.gpu import DeviceWorkload
    from synth.workloads import make_workload
    C = _C()
    cfg = _small(2, B=2, lengths=("fixed", 9000), n_reindex=1, n_reuse=1)
    w = make_workload(cfg)
    dw = DeviceWorkload(w)
    dw.fill_caches(include_new=True)
    qb = dw.batch()
    kc = dw.cache("kidx")
    kv = dw.cache("kv")
    T, c = w.T, cfg
    qcodes = torch.zeros(T * c.H_I, c.d_I // 2, dtype=torch.uint8, device="cuda")
    qscales = torch.zeros(T * c.H_I, c.d_I // 32, dtype=torch.uint8, device="cuda")
    nb = ctypes.c_size_t(0)
    C.check(C.csa2_index_workspace_size(ctypes.byref(qb), c.H_I, c.d_I, c.P, c.K, ctypes.byref(nb)))
    ws = torch.empty(nb.value, dtype=torch.uint8, device="cuda")
    pool = torch.zeros(T, c.P, dtype=torch.int32, device="cuda")
    pool_n = torch.zeros(T, dtype=torch.int32, device="cuda")
    idx = torch.zeros(T, c.K, dtype=torch.int32, device="cuda")
    idx_n = torch.zeros(T, dtype=torch.int32, device="cuda")
    nbk = (int(w.lens.max()) + 7) // 8
    bscore = torch.zeros(T, nbk, dtype=torch.float32, device="cuda")
    ov = OracleView(w)
    for l, m in enumerate(w.modes):
        if m == "U":
            continue
        C.check(C.csa2_quantize_fp4(dw.iq[l].data_ptr(), T * c.H_I, c.d_I, None, qcodes.data_ptr(),
                                    qscales.data_ptr(), _stream()))
        if m == "F":
            C.check(C.csa2_index_full(ctypes.byref(qb), qcodes.data_ptr(), qscales.data_ptr(), dw.iw[l].data_ptr(),
                                      c.H_I, ctypes.byref(kc), c.P, c.K, pool.data_ptr(), pool_n.data_ptr(),
                                      idx.data_ptr(), idx_n.data_ptr(), bscore.data_ptr(), ws.data_ptr(),
                                      ws.numel(), _stream()))
        else:
            C.check(C.csa2_index_reindex(ctypes.byref(qb), qcodes.data_ptr(), qscales.data_ptr(),
                                         dw.iw[l].data_ptr(), c.H_I, ctypes.byref(kc), pool.data_ptr(),
                                         pool_n.data_ptr(), c.P, c.K, idx.data_ptr(), idx_n.data_ptr(),
                                         ws.data_ptr(), ws.numel(), _stream()))
        assert _status() == 0
        for tok in range(T):
            b, p = int(w.tok_seq[tok]), int(w.tok_pos[tok])
            kcod, ksc = ov.kidx_rows(b, p + 1)
            q, wh = ov.iq(l, tok)
            n = int(idx_n[tok])
            g = idx[tok].cpu().numpy()
            assert np.all(g[n:] == -1)
            pl = pool[tok].cpu().numpy()[: int(pool_n[tok])]
            if m == "F":
                s = oracle.index_scores(q, wh, kcod, ksc)
                bs = oracle.block_scores(s, p)
                np.testing.assert_allclose(bscore[tok].cpu().numpy()[: len(bs)], bs, rtol=2e-6, atol=1e-6)
                grade_set(pl, np.arange(len(bs)), bs, c.P, "pool")
            pos = oracle.pool_positions(pl, p)
            grade_set(g[:n], pos, oracle.index_scores(q, wh, kcod[pos], ksc[pos]), c.K, f"layer {l}")
        # attention through csa2_attend_reuse on this selection
        out = torch.zeros(T, c.Hq, c.D, dtype=torch.float32, device="cuda")
        lse = torch.zeros(T, c.Hq, dtype=torch.float32, device="cuda")
        na = ctypes.c_size_t(0)
        C.check(C.csa2_attend_workspace_size(ctypes.byref(qb), c.Hq, c.D, c.K, 0, ctypes.byref(na)))
        wsa = torch.empty(na.value, dtype=torch.uint8, device="cuda")
        C.check(C.csa2_attend_reuse(ctypes.byref(qb), dw.q[l].data_ptr(), C.CSA2_BF16, c.Hq, ctypes.byref(kv),
                                    idx.data_ptr(), idx_n.data_ptr(), c.K, None, 0.0, out.data_ptr(), C.CSA2_F32,
                                    lse.data_ptr(), wsa.data_ptr(), wsa.numel(), _stream()))
        assert _status() == 0
        for tok in range(T):
            b = int(w.tok_seq[tok])
            g = idx[tok].cpu().numpy()
            g = g[g >= 0]
            ref, rlse = oracle.attend(w.qmain_f64(l, tok), ov.kv_rows(b, g), 1 / math.sqrt(c.D))
            grade_attention(out[tok].cpu().numpy(), ref, "f32", "attend")
            np.testing.assert_allclose(lse[tok].cpu().numpy(), rlse, rtol=1e-5, atol=1e-5)


def test_stack_attend_wait_event():
    """Main queries uploaded on a second stream: with attend_wait_event the
    stack's attention waits for them and gives the outputs of the plain call"""
    from synth.gpu import DeviceWorkload
    from synth.workloads import make_workload
    C = _C()
    cfg = _small(2, B=2, lengths=("fixed", 6000), n_reindex=1, n_reuse=2)
    w = make_workload(cfg)
    dw = DeviceWorkload(w)
    dw.fill_caches(include_new=True)
    desc = dw.stack_desc(append=False)
    ws = dw.stack_workspace(desc)
    C.check(C.csa2_decode_stack(ctypes.byref(desc), ws.data_ptr(), ws.numel(), _stream()))
    assert _status() == 0
    ref = dw.out_all.clone()
    h_q = dw.inputs_main_q.cpu().pin_memory()
    dw.inputs_main_q.zero_()
    dw.out_all.zero_()
    s2 = torch.cuda.Stream()
    ready = torch.cuda.Event()
    torch.cuda.synchronize()
    with torch.cuda.stream(s2):
        torch.cuda._sleep(2_000_000)  # the copy lands well after the indexer kernels were queued
        dw.inputs_main_q.copy_(h_q, non_blocking=True)
        ready.record(s2)
    desc.attend_wait_event = ready.cuda_event
    C.check(C.csa2_decode_stack(ctypes.byref(desc), ws.data_ptr(), ws.numel(), _stream()))
    assert _status() == 0
    torch.cuda.synchronize()
    assert torch.equal(dw.out_all, ref)


_OVERLAP_CHILD = r"""
import ctypes, hashlib, sys
sys.path.insert(0, sys.argv[1])
import torch
import csa2_fp4_sparse_b200 as C
from synth.gpu import DeviceWorkload
from synth.workloads import CONFIGS
cfg = CONFIGS[int(sys.argv[2])].with_(B=int(sys.argv[3]), lengths=("fixed", int(sys.argv[4])))
from synth.workloads import make_workload
w = make_workload(cfg)
dw = DeviceWorkload(w)
dw.fill_caches(include_new=False)
desc = dw.stack_desc(append=True, copies=False)
ws = dw.stack_workspace(desc)
sp = torch.cuda.current_stream().cuda_stream
for _ in range(4):  # back to back: each step's first kernel follows the last one's attention
    C.check(C.csa2_decode_stack(ctypes.byref(desc), ws.data_ptr(), ws.numel(), sp))
torch.cuda.synchronize()
assert C.csa2_get_status(sp) == 0
print(hashlib.sha256(dw.out_all.cpu().view(torch.uint8).numpy().tobytes()).hexdigest())
"""


@pytest.mark.parametrize("i,B,L", [(2, 3, 9000), (4, 2, 40000), (5, 6, 3000)])
def test_stack_overlapped_launches_bit_identical(i, B, L):
    """Decode steps with no overlapped launch (CSA2_OVERLAP=0), the default
    set and every kernel kind overlapped (31) give bit-identical outputs"""
    import os
    import subprocess
    import sys
    root = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))
    digests = {}
    for mask in ("0", None, "31"):
        env = dict(os.environ)
        env.pop("CSA2_OVERLAP", None)
        if mask is not None:
            env["CSA2_OVERLAP"] = mask
        r = subprocess.run([sys.executable, "-c", _OVERLAP_CHILD, root, str(i), str(B), str(L)], env=env,
                           capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        digests[mask] = r.stdout.strip().splitlines()[-1]
    assert len(set(digests.values())) == 1, digests

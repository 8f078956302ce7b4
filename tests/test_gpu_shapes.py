"""GPU-vs-oracle parity for every shape class the C ABI accepts beyond the
benchmark workloads: long runs of query tokens per sequence (speculative
verify, chunked prefill), 32 query heads, fp32 queries and outputs, and the
full-size million-token and SWA workloads graded with fp32 outputs (the
strict tolerance: max |d| <= 2e-3, sum|d| / sum|ref| <= 1e-3)."""
import ctypes

import numpy as np
import pytest

from tests.harness import OracleView, check_token

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _C():
    import csa2_fp4_sparse_b200 as C
    return C


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _run(cfg, append=True):
    from synth.gpu import DeviceWorkload
    from synth.workloads import make_workload
    C = _C()
    w = make_workload(cfg)
    dw = DeviceWorkload(w)
    dw.fill_caches(include_new=not append)
    desc = dw.stack_desc(append=append)
    ws = dw.stack_workspace(desc)
    C.check(C.csa2_decode_stack(ctypes.byref(desc), ws.data_ptr(), ws.numel(), _stream()))
    st = C.csa2_get_status(_stream())
    assert st == 0, (st, C.csa2_last_error())
    return w, dw


def _grade(w, dw, toks):
    ov = OracleView(w)
    for tok in toks:
        g = {"pool": dw.pool_out[tok].cpu().numpy(), "idx": {}, "out": {}}
        g["pool_n"] = int((g["pool"] >= 0).sum())
        for l, m in enumerate(w.modes):
            if m in "FR":
                g["idx"][l] = dw.idx_out[l][tok].cpu().numpy()
            g["out"][l] = dw.out[l][tok].float().cpu().numpy()
        check_token(ov, tok, g)


def _cfg(i, **kw):
    from synth.workloads import CONFIGS
    return CONFIGS[i].with_(**kw)


@pytest.mark.parametrize("case", [
    # more than 8 query tokens per sequence: the scan takes each sequence's
    # tokens in chunks of 8 (one pass over the keys per chunk)
    dict(B=3, lengths=("list", [3000, 20000, 700]), widths=("list", [9, 12, 16])),
    dict(B=2, lengths=("list", [6000, 90]), widths=("list", [64, 17]), out_dtype="f32"),  # chunked prefill
])
def test_long_token_runs(case):
    w, dw = _run(_cfg(2, n_reindex=1, n_reuse=1, n_needles=4, **case))
    assert int(w.widths.max()) > 8
    _grade(w, dw, range(w.T))


@pytest.mark.parametrize("case", [
    dict(i=2, B=3, lengths=("list", [5000, 300, 12000]), Hq=32),
    dict(i=2, B=2, lengths=("list", [5000, 9000]), Hq=32, out_dtype="f32"),
    dict(i=5, B=4, lengths=("loguniform", 60, 20000), Hq=32, out_dtype="f32"),           # with SWA
    dict(i=1, Hq=32),                                                                     # D = 128, fp32 q and out
    dict(i=1, Hq=64),
    dict(i=2, B=2, lengths=("list", [4000, 7000]), Hq=32, q_dtype="f32", out_dtype="f32"),  # D*Hq = 16384
])
def test_attention_head_counts_and_dtypes(case):
    case = dict(case)
    i = case.pop("i")
    w, dw = _run(_cfg(i, n_reindex=1, n_reuse=1, **case))
    _grade(w, dw, range(w.T))


def test_full_size_ctx1m_fp32_out():
    """4 x 1M context, the benchmark's shapes and launch configuration, fp32
    output graded strictly on every query token and layer"""
    w, dw = _run(_cfg(4, out_dtype="f32"))
    _grade(w, dw, range(w.T))


def test_full_size_swa_verify_fp32_out():
    """64 sequences with 1-6 query tokens each and the FP8 window, fp32 output:
    for every width 1..6 the first and last token of one sequence of that
    width, plus seeded picks (16 tokens at least)"""
    w, dw = _run(_cfg(5, out_dtype="f32"))
    toks = set()
    for W in range(1, 7):
        seqs = np.flatnonzero(w.widths == W)
        if len(seqs):
            b = int(seqs[0])
            toks.update([int(w.tok_start[b]), int(w.tok_start[b + 1]) - 1])
    rng = np.random.default_rng(55)
    while len(toks) < 16:
        toks.add(int(rng.integers(0, w.T)))
    _grade(w, dw, sorted(toks))


def test_query_beyond_fp16_range_is_reported():
    """The attention MMAs take the query in fp16; a bf16 query at or beyond
    65520 has no fp16 form and is reported as CSA2_ERR_RANGE"""
    from synth.gpu import DeviceWorkload
    from synth.workloads import make_workload
    C = _C()
    cfg = _cfg(2, B=1, lengths=("fixed", 2000), n_reindex=0, n_reuse=0)
    w = make_workload(cfg)
    dw = DeviceWorkload(w)
    dw.fill_caches(include_new=True)
    desc = dw.stack_desc(append=False)
    ws = dw.stack_workspace(desc)
    dw.q[0][0, 3, 17] = 70000.0
    C.check(C.csa2_decode_stack(ctypes.byref(desc), ws.data_ptr(), ws.numel(), _stream()))
    assert C.csa2_get_status(_stream()) == C.CSA2_ERR_RANGE
    assert C.csa2_get_status(_stream()) == 0
    dw.q[0][0, 3, 17] = 1.0
    C.check(C.csa2_decode_stack(ctypes.byref(desc), ws.data_ptr(), ws.numel(), _stream()))
    assert C.csa2_get_status(_stream()) == 0

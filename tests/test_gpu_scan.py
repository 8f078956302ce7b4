"""The Full-layer scan (block scores) against the oracle, on the tensor-core
path: dense, paged, d_I = 64 and 128, several query tokens per sequence."""
import ctypes

import numpy as np
import pytest

import oracle
from tests.harness import OracleView

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _scan(cfg):
    import csa2_fp4_sparse_b200 as C
    from synth.gpu import DeviceWorkload
    from synth.workloads import make_workload
    w = make_workload(cfg)
    dw = DeviceWorkload(w)
    dw.fill_caches(include_new=True)
    T, c = w.T, cfg
    sp = torch.cuda.current_stream().cuda_stream
    qc = torch.zeros(T * c.H_I, c.d_I // 2, dtype=torch.uint8, device="cuda")
    qs = torch.zeros(T * c.H_I, c.d_I // 32, dtype=torch.uint8, device="cuda")
    C.check(C.csa2_quantize_fp4(dw.iq[0].data_ptr(), T * c.H_I, c.d_I, None, qc.data_ptr(), qs.data_ptr(), sp))
    qb = dw.batch()
    kc = dw.cache("kidx")
    nb = ctypes.c_size_t(0)
    C.check(C.csa2_index_workspace_size(ctypes.byref(qb), c.H_I, c.d_I, c.P, c.K, ctypes.byref(nb)))
    ws = torch.empty(nb.value, dtype=torch.uint8, device="cuda")
    ld = (int(w.lens.max()) + 7) // 8
    bs = torch.full((T, ld), float("nan"), dtype=torch.float32, device="cuda")
    pool = torch.zeros(T, c.P, dtype=torch.int32, device="cuda")
    pool_n = torch.zeros(T, dtype=torch.int32, device="cuda")
    idx = torch.zeros(T, c.K, dtype=torch.int32, device="cuda")
    idx_n = torch.zeros(T, dtype=torch.int32, device="cuda")
    C.check(C.csa2_index_full(ctypes.byref(qb), qc.data_ptr(), qs.data_ptr(), dw.iw[0].data_ptr(), c.H_I,
                              ctypes.byref(kc), c.P, c.K, pool.data_ptr(), pool_n.data_ptr(), idx.data_ptr(),
                              idx_n.data_ptr(), bs.data_ptr(), ws.data_ptr(), ws.numel(), sp))
    st = C.csa2_get_status(sp)
    assert st == 0, f"status {st}"
    return w, bs.cpu().numpy()


@pytest.mark.parametrize("case", [
    dict(i=2, B=2, lengths=("list", [300, 5000])),
    dict(i=1, lengths=("fixed", 3000)),                                   # d_I = 64, 16 heads
    dict(i=3, B=3, lengths=("list", [64, 1000, 7000])),                   # paged
    dict(i=5, B=4, lengths=("list", [9, 130, 1111, 4321]), widths=("list", [3, 6, 1, 8])),
])
def test_block_scores_vs_oracle(case):
    from synth.workloads import CONFIGS
    case = dict(case)
    cfg = CONFIGS[case.pop("i")].with_(**case)
    w, bs = _scan(cfg)
    ov = OracleView(w)
    worst = 0.0
    for tok in range(w.T):
        b, p = int(w.tok_seq[tok]), int(w.tok_pos[tok])
        kc, ks = ov.kidx_rows(b, p + 1)
        q, wh = ov.iq(0, tok)
        ref = oracle.block_scores(oracle.index_scores(q, wh, kc, ks), p)
        got = bs[tok, : len(ref)].astype(np.float64)
        assert np.all(np.isfinite(got)), f"tok {tok}: unwritten block scores"
        err = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-3 * np.abs(ref).max())
        worst = max(worst, float(err.max()))
    print(f"max relative block-score error {worst:.3e}")
    assert worst <= 1e-5

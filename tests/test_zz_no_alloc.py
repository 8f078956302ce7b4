"""csa2_index_reindex_noalloc: the Reindex call for callers that cannot
allocate device memory (its scratch is a fixed device array inside the
library).  Checked through the C ABI against csa2_index_reindex, which takes a
caller workspace, on two calls in a row with different queries; collected
last so that a failure here comes after every other test has run."""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def test_noalloc_reindex_matches_workspace_reindex():
    import csa2_fp4_sparse_b200 as C
    from synth.gpu import DeviceWorkload
    from synth.workloads import CONFIGS, make_workload

    cfg = CONFIGS[2].with_(B=3, lengths=("list", [700, 9000, 20000]), widths=("list", [1, 2, 1]), n_reindex=2,
                           n_reuse=0)
    w = make_workload(cfg)
    dw = DeviceWorkload(w)
    dw.fill_caches(include_new=True)
    T, c = w.T, cfg
    sp = torch.cuda.current_stream().cuda_stream
    qb = dw.batch()
    kc = dw.cache("kidx")
    nb = ctypes.c_size_t(0)
    C.check(C.csa2_index_workspace_size(ctypes.byref(qb), c.H_I, c.d_I, c.P, c.K, ctypes.byref(nb)))
    ws = torch.empty(nb.value, dtype=torch.uint8, device="cuda")

    def quant(layer):
        qc = torch.zeros(T * c.H_I, c.d_I // 2, dtype=torch.uint8, device="cuda")
        qs = torch.zeros(T * c.H_I, c.d_I // 32, dtype=torch.uint8, device="cuda")
        C.check(C.csa2_quantize_fp4(dw.iq[layer].data_ptr(), T * c.H_I, c.d_I, None, qc.data_ptr(), qs.data_ptr(),
                                    sp))
        return qc, qs

    def out():
        return (torch.full((T, c.K), -7, dtype=torch.int32, device="cuda"),
                torch.full((T,), -7, dtype=torch.int32, device="cuda"))

    # the Full layer's pool, shared by the Reindex layers
    q0c, q0s = quant(0)
    pool = torch.zeros(T, c.P, dtype=torch.int32, device="cuda")
    pool_n = torch.zeros(T, dtype=torch.int32, device="cuda")
    fi, fn = out()
    C.check(C.csa2_index_full(ctypes.byref(qb), q0c.data_ptr(), q0s.data_ptr(), dw.iw[0].data_ptr(), c.H_I,
                              ctypes.byref(kc), c.P, c.K, pool.data_ptr(), pool_n.data_ptr(), fi.data_ptr(),
                              fn.data_ptr(), None, ws.data_ptr(), ws.numel(), sp))
    layers = [l for l, m in enumerate(w.modes) if m == "R"]
    assert len(layers) == 2
    results = []
    for l in layers:  # two calls in a row, different queries, one shared scratch array
        qc, qs = quant(l)
        ri, rn = out()
        C.check(C.csa2_index_reindex(ctypes.byref(qb), qc.data_ptr(), qs.data_ptr(), dw.iw[l].data_ptr(), c.H_I,
                                     ctypes.byref(kc), pool.data_ptr(), pool_n.data_ptr(), c.P, c.K, ri.data_ptr(),
                                     rn.data_ptr(), ws.data_ptr(), ws.numel(), sp))
        ni, nn = out()
        C.check(C.csa2_index_reindex_noalloc(ctypes.byref(qb), qc.data_ptr(), qs.data_ptr(), dw.iw[l].data_ptr(),
                                             c.H_I, ctypes.byref(kc), pool.data_ptr(), pool_n.data_ptr(), c.P, c.K,
                                             ni.data_ptr(), nn.data_ptr(), sp))
        assert C.csa2_get_status(sp) == 0
        # same kernels on the same inputs: identical selections (inside any tolerance)
        assert torch.equal(rn, nn), (rn, nn)
        assert torch.equal(ri, ni)
        assert int(nn.min()) > 0
        results.append(ni.cpu().numpy())
    assert not np.array_equal(results[0], results[1])  # the second call did not reuse the first's scores

    # sizes beyond the fixed scratch are refused before anything is launched
    big = C.csa2_query_batch(qb.n_seq, 70, qb.max_seq_len, qb.max_q_per_seq, qb.seq_len, qb.tok_start, qb.tok_seq,
                             qb.tok_pos)
    ni, nn = out()
    rc = C.csa2_index_reindex_noalloc(ctypes.byref(big), q0c.data_ptr(), q0s.data_ptr(), dw.iw[0].data_ptr(),
                                      c.H_I, ctypes.byref(kc), pool.data_ptr(), pool_n.data_ptr(), c.P, c.K,
                                      ni.data_ptr(), nn.data_ptr(), sp)
    assert rc == C.CSA2_ERR_WORKSPACE
    assert "fixed scratch" in C.csa2_last_error()

"""The largest pool and index list the C ABI accepts (P = 4096 blocks, K = 2048
positions) through the whole stack, every query token checked against the
oracle; contexts long enough that both the pool and the index list are full."""
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def test_stack_max_pool_and_k():
    from tests.test_gpu_parity import _check_all, _run_stack, _small

    cfg = _small(2, B=2, P=4096, K=2048, lengths=("list", [40000, 70000]), widths=("list", [2, 1]),
                 n_reindex=1, n_reuse=1)
    w, dw = _run_stack(cfg)
    for l, m in enumerate(w.modes):
        if m in "FR":
            assert int((dw.idx_out[l] >= 0).sum(dim=1).min()) == 2048  # full index lists
    assert int((dw.pool_out >= 0).sum(dim=1).min()) == 4096           # full pools
    _check_all(w, dw, range(w.T))

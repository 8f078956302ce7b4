"""Context-parallel decode step on one GPU: the ranks of a G-way split of the
positions run one after the other in this process (their caches are separate
slices), the all-gathers are emulated by stacking the ranks' buffers, and the
result must equal the single-GPU stack: the pool and every selector's index
list exactly, and every layer's output within the oracle's tolerance."""
import ctypes

import numpy as np
import pytest

from tests.harness import OracleView, check_token

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _C():
    import csa2_fp4_sparse_b200 as C
    return C


def _ranges(L, G, align=64):
    cuts = [0] + [min(L, (L * r // G) // align * align) for r in range(1, G)] + [L]
    return [(cuts[r], cuts[r + 1]) for r in range(G)]


def _rank_state(w, dw, lo, hi, cp, C):
    """rank-local caches (rows lo..hi-1 of every sequence), batch and layers"""
    c = w.cfg
    B = w.B
    dev = dw.kidx_codes.device
    lens = w.lens.astype(np.int64)
    loc_len = np.clip(np.minimum(lens, hi) - lo, 0, None)
    padded = (loc_len + 127) // 128 * 128
    base = np.concatenate([[0], np.cumsum(padded)[:-1]]).astype(np.int64)
    n_rows = max(int(padded.sum()), 128)
    st = {}
    for name, (codes, scales) in {"kidx": (dw.kidx_codes, dw.kidx_scales), "kv": (dw.kv_codes, dw.kv_scales)}.items():
        lc = torch.zeros(n_rows, codes.shape[1], dtype=torch.uint8, device=dev)
        ls = torch.zeros(n_rows, scales.shape[1], dtype=torch.uint8, device=dev)
        for b in range(B):
            n = int(loc_len[b])
            if n:
                src = int(w.seq_base[b]) + lo
                lc[base[b]:base[b] + n] = codes[src:src + n]
                ls[base[b]:base[b] + n] = scales[src:src + n]
        st[name] = (lc, ls)
    tok_pos = w.tok_pos.astype(np.int64)
    lp = np.where(tok_pos < lo, -1, np.minimum(tok_pos - lo, loc_len[w.tok_seq] - 1)).astype(np.int32)
    t = {
        "seq_len": torch.from_numpy(loc_len.astype(np.int32)).to(dev),
        "tok_start": torch.from_numpy(w.tok_start.astype(np.int32)).to(dev),
        "tok_seq": torch.from_numpy(w.tok_seq.astype(np.int32)).to(dev),
        "tok_pos": torch.from_numpy(lp).to(dev),
        "base": torch.from_numpy(base).to(dev),
    }
    st["t"] = t
    qb = C.csa2_query_batch(B, w.T, max(int(loc_len.max()), 1), int(w.widths.max()), t["seq_len"].data_ptr(),
                            t["tok_start"].data_ptr(), t["tok_seq"].data_ptr(), t["tok_pos"].data_ptr())
    kc = C.csa2_fp4_cache(st["kidx"][0].data_ptr(), st["kidx"][1].data_ptr(), n_rows, c.d_I, 0, None, 0,
                          t["base"].data_ptr())
    kv = C.csa2_fp4_cache(st["kv"][0].data_ptr(), st["kv"][1].data_ptr(), n_rows, c.D, 0, None, 0,
                          t["base"].data_ptr())
    odt = torch.float32 if c.out_dtype == "f32" else torch.bfloat16
    outs = {l: torch.zeros(w.T, c.Hq, c.D, dtype=odt, device=dev) for l in range(len(w.modes))}
    layers = cp.StackLayers(list(w.modes), dict(dw.iq), dict(dw.iw), dict(dw.q), outs)
    return st, qb, kc, kv, layers, max(int(loc_len.max()), 1)


@pytest.mark.parametrize("G", [2, 3])
def test_context_parallel_equals_single_gpu(G):
    from csa2_fp4_sparse_b200 import cp
    from synth.gpu import DeviceWorkload
    from synth.workloads import CONFIGS, make_workload
    C = _C()
    cfg = CONFIGS[4].with_(B=2, lengths=("list", [40000, 23000]), n_reindex=1, n_reuse=2, n_needles=8,
                           out_dtype="f32")
    w = make_workload(cfg)
    dw = DeviceWorkload(w)
    dw.fill_caches(include_new=True)
    sp = torch.cuda.current_stream().cuda_stream
    desc = dw.stack_desc(append=False)
    ws = dw.stack_workspace(desc)
    C.check(C.csa2_decode_stack(ctypes.byref(desc), ws.data_ptr(), ws.numel(), sp))
    assert C.csa2_get_status(sp) == 0
    c = cfg
    L = int(w.lens.max())
    ranks, keep = [], []
    for r, (lo, hi) in enumerate(_ranges(L, G)):
        st, qb, kc, kv, layers, mx = _rank_state(w, dw, lo, hi, cp, C)
        keep.append((st, layers))
        ranks.append(cp.CPRank(cp.Slice(r, G, lo, hi), qb, kc, kv, layers, c.H_I, c.d_I, c.P, c.K, c.Hq, c.D,
                               C.CSA2_BF16, C.CSA2_F32, (mx + 7) // 8, sp, torch))

    def gather(per_rank):  # emulated all-gather: stack the ranks' buffers
        return [torch.stack([x[i] for x in per_rank]) for i in range(len(per_rank[0]))]

    g = gather([rk.phase_a() for rk in ranks])
    g = gather([rk.phase_b(*g) for rk in ranks])
    g = gather([rk.phase_c(g[0]) for rk in ranks])
    for rk in ranks:
        rk.phase_d(*g)
    assert C.csa2_get_status(sp) == 0
    rk = ranks[0]
    # the pool and every selector's list: exactly the single-GPU ones
    assert torch.equal(rk.pool, dw.pool_out), "pool"
    for i, l in enumerate(rk.L.selectors):
        assert torch.equal(rk.idx[i], dw.idx_out[l]), f"selector layer {l}"
    # every layer's output, graded against the oracle on the CP run's selections
    ov = OracleView(w)
    for tok in range(w.T):
        gv = {"pool": rk.pool[tok].cpu().numpy(), "idx": {}, "out": {}}
        gv["pool_n"] = int((gv["pool"] >= 0).sum())
        for i, l in enumerate(rk.L.selectors):
            gv["idx"][l] = rk.idx[i][tok].cpu().numpy()
        for l in range(len(w.modes)):
            gv["out"][l] = rk.L.out[l][tok].float().cpu().numpy()
        check_token(ov, tok, gv)
    # every rank merged the same outputs
    for other in ranks[1:]:
        for l in range(len(w.modes)):
            assert torch.equal(other.L.out[l], rk.L.out[l])

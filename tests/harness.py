"""Parity harness: oracle views of a workload and the grading rules.

Grading (the workload's stated tolerances):
  * FP4 codes and scales: bit-exact.
  * index sets (pool blocks, top-K positions): same size, no duplicates, every
    selected id visible, and every selected id scores at least
    tau - 1e-5 * max(|tau|, 1e-30) under the oracle, tau being the oracle's
    k-th best score -- i.e. exact except for swaps across a gap below 1e-5
    relative.
  * attention (fp32 out): max |d| <= 2e-3 and sum|d| / sum|ref| <= 1e-3;
    (bf16 out): the same tolerances with the output's own rounding taken out:
    max |d| <= 2e-3 + half a bf16 ulp of the value, and
    sum|gpu - bf16(ref)| / sum|ref| <= 1e-3 (bf16 rounding alone is ~1e-3
    relative on average, so comparing with the unrounded oracle would grade
    the format, not the kernel).
Downstream steps are graded on the GPU's upstream choice (Reindex on the GPU's
pool, attention on the GPU's index list), so one near-tie never cascades.
"""
from __future__ import annotations

import math

import numpy as np

import oracle
from synth import bf16_bits_to_f32
from synth.workloads import BLOCK, Workload

SET_RTOL = 1e-5
ATT_MAX_ABS = 2e-3
ATT_MEAN_REL = 1e-3


class OracleView:
    """Oracle-side inputs of one workload, regenerated on the host from the
    same seeds and quantised by the oracle itself."""

    def __init__(self, w: Workload):
        self.w = w
        self._kidx = {}

    def kidx_rows(self, b: int, n: int):
        """FP4 indexer keys of positions 0..n-1 of sequence b (oracle-quantised)"""
        key = (b, n)
        if key not in self._kidx:
            self._kidx.clear()
            x = self.w.kidx.rows_f32(b, 0, n)
            c, s, bad = oracle.quantize_fp4(x)
            assert bad == 0
            self._kidx[key] = (c, s)
        return self._kidx[key]

    def kv_rows(self, b: int, pos: np.ndarray) -> np.ndarray:
        x = self.w.kv.select_rows_f32(b, np.asarray(pos, np.int64))
        c, s, bad = oracle.quantize_fp4(x)
        assert bad == 0
        return oracle.dequant_fp4(c, s)

    def iq(self, layer: int, tok: int):
        c = self.w.cfg
        x = self.w.iq_f32(layer, tok).reshape(c.H_I, c.d_I)
        qc, qs, _ = oracle.quantize_fp4(x)
        return oracle.dequant_fp4(qc, qs), self.w.iw_f32(layer, tok).astype(np.float64)

    def swa_rows(self, layer: int, tok: int) -> np.ndarray:
        codes, scale = self.w.swa_rows_e4m3(layer, tok)
        return oracle.e4m3_decode_array(codes) * scale.astype(np.float64)[:, None]


def grade_set(gpu_ids, cand_ids, cand_scores, k, what=""):
    """gpu_ids: the GPU's selection; cand_ids/cand_scores: every candidate with
    its oracle score; k: requested count."""
    gpu_ids = np.asarray(gpu_ids, np.int64)
    cand_ids = np.asarray(cand_ids, np.int64)
    cand_scores = np.asarray(cand_scores, np.float64)
    ref = oracle.topk(cand_scores, cand_ids, k)
    assert len(gpu_ids) == len(ref), f"{what}: size {len(gpu_ids)} != oracle {len(ref)}"
    assert len(np.unique(gpu_ids)) == len(gpu_ids), f"{what}: duplicates"
    assert np.all(np.diff(gpu_ids) > 0), f"{what}: not ascending"
    score_of = dict(zip(cand_ids.tolist(), cand_scores.tolist()))
    missing = [a for a in gpu_ids.tolist() if a not in score_of]
    assert not missing, f"{what}: ids outside the candidates: {missing[:5]}"
    if len(ref) == 0:
        return 0
    tau = min(score_of[r] for r in ref.tolist())
    floor = tau - SET_RTOL * max(abs(tau), 1e-30)
    bad = [a for a in gpu_ids.tolist() if score_of[a] < floor]
    assert not bad, f"{what}: {len(bad)} ids below the k-th score {tau} (e.g. {bad[:3]})"
    return int(np.sum(~np.isin(gpu_ids, ref)))  # near-tie swaps (informational)


def bf16_round(x: np.ndarray) -> np.ndarray:
    f = np.asarray(x, np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return bf16_bits_to_f32(u.astype(np.uint16))


def grade_attention(gpu, ref, out_dtype, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    if out_dtype == "f32":
        d = np.abs(gpu - ref)
        mx = float(d.max())
        mrel = float(d.sum() / max(np.abs(ref).sum(), 1e-30))
        assert mx <= ATT_MAX_ABS, f"{what}: max abs {mx}"
        assert mrel <= ATT_MEAN_REL, f"{what}: mean rel {mrel}"
        return mx, mrel
    r16 = bf16_round(ref).astype(np.float64)
    e = np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126)))
    half_ulp = 2.0 ** (e - 8)
    d = np.abs(gpu - ref)
    bad = d > ATT_MAX_ABS + half_ulp
    if bad.any():
        i = np.flatnonzero(bad.reshape(-1))[:4]
        raise AssertionError(f"{what}: {int(bad.sum())} outputs beyond 2e-3 + half ulp: gpu {gpu.reshape(-1)[i]} "
                             f"ref {ref.reshape(-1)[i]}")
    mrel = float(np.abs(gpu - r16).sum() / max(np.abs(ref).sum(), 1e-30))
    assert mrel <= ATT_MEAN_REL, f"{what}: mean rel vs bf16(ref) {mrel}"
    return float(d.max()), mrel


def selector_of(modes, layer):
    for l in range(layer, -1, -1):
        if modes[l] in "FR":
            return l
    raise ValueError("no selector")


def check_token(ov: OracleView, tok: int, gpu: dict, layers=None, check_pool=True):
    """Grade one query token of a decode-stack run.

    gpu: {"pool": [P], "pool_n": int, "idx": {sel_layer: [K] ids (-1 padded)},
          "out": {layer: [Hq][D]}} (numpy)."""
    w = ov.w
    c = w.cfg
    b, p = int(w.tok_seq[tok]), int(w.tok_pos[tok])
    kc, ks = ov.kidx_rows(b, p + 1)
    stats = {"swaps": 0, "att": []}
    pool = np.asarray(gpu["pool"][: gpu["pool_n"]], np.int64)
    # Full layer: pool over the block scores of the whole visible context
    q0, w0 = ov.iq(0, tok)
    s_all = oracle.index_scores(q0, w0, kc, ks)
    if check_pool:
        bs = oracle.block_scores(s_all, p, BLOCK)
        stats["swaps"] += grade_set(pool, np.arange(len(bs)), bs, c.P, f"tok{tok} pool")
    pos = oracle.pool_positions(pool, p, BLOCK)
    layers = range(len(w.modes)) if layers is None else layers
    for l in layers:
        m = w.modes[l]
        if m in "FR":
            if m == "F":
                sc = s_all[pos]
            else:
                ql, wl = ov.iq(l, tok)
                sc = oracle.index_scores(ql, wl, kc[pos], ks[pos])
            g = np.asarray(gpu["idx"][l], np.int64)
            g = g[g >= 0]
            stats["swaps"] += grade_set(g, pos, sc, c.K, f"tok{tok} layer{l} idx")
    for l in layers:
        if l not in gpu["out"]:
            continue
        sel = selector_of(w.modes, l)
        g = np.asarray(gpu["idx"][sel], np.int64)
        g = g[g >= 0]
        kvr = ov.kv_rows(b, g)
        sw = ov.swa_rows(l, tok) if c.swa else None
        ref, _ = oracle.attend_rows(w.qmain_f64(l, tok), kvr, sw, 1.0 / math.sqrt(c.D))
        stats["att"].append(grade_attention(gpu["out"][l], ref, c.out_dtype, f"tok{tok} layer{l} out"))
    return stats

"""Decode-step workloads: shapes, seeded metadata and input tensors.

Five configurations follow the workload descriptions of the CSA2 decode step
(tiny, medium, ragged/paged, million-token, SWA + speculative verify), plus
small variants used by the parity tests.  Host-only metadata (lengths, query
widths, page tables, needle blocks, outlier channels) is drawn here with
numpy's seeded generator; element values come from the counter-based
generator in ``csa2_synth.h`` so that host and device agree bit for bit.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np

from . import (KIND_NORMAL, KIND_UNIFORM, S_IQ, S_IW, S_KIDX, S_KV, S_QMAIN, S_SWA, TensorSpec,
               bf16_bits_to_f32)

BLOCK = 8  # positions per indexer block (the pages' 8-position blocks)


@dataclass
class Config:
    name: str
    seed: int
    B: int
    H_I: int
    d_I: int
    P: int
    K: int
    Hq: int
    D: int
    n_reindex: int
    n_reuse: int
    q_dtype: str = "bf16"          # main query dtype: "f32" | "bf16"
    out_dtype: str = "bf16"        # attention output dtype: "f32" | "bf16"
    lengths: tuple = ("fixed", 8192)  # ("fixed", L) | ("uniform8", lo, hi) | ("loguniform", lo, hi) | ("list", [..])
    widths: tuple = ("fixed", 1)      # ("fixed", W) | ("uniform", lo, hi) | ("list", [..])
    paged: bool = False
    page_size: int = 64
    swa: bool = False
    window: int = 128
    swa_cap: int = 136
    n_needles: int = 0
    outliers: bool = False         # t(3) in 1% of channels (1/128 indexer, 5/512 main)
    needle_shift: float = 2.0

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


CONFIGS = {
    1: Config("tiny", 1, B=1, H_I=16, d_I=64, P=256, K=128, Hq=16, D=128, n_reindex=1, n_reuse=1,
              q_dtype="f32", out_dtype="f32", lengths=("fixed", 8192), n_needles=8),
    2: Config("medium", 2, B=8, H_I=64, d_I=128, P=2048, K=512, Hq=64, D=512, n_reindex=2, n_reuse=8,
              lengths=("fixed", 65536), n_needles=32),
    3: Config("ragged_paged", 3, B=32, H_I=64, d_I=128, P=2048, K=512, Hq=64, D=512, n_reindex=3,
              n_reuse=16, lengths=("uniform8", 16384, 262144), paged=True, page_size=64, n_needles=32),
    4: Config("ctx1m", 4, B=4, H_I=64, d_I=128, P=2048, K=512, Hq=64, D=512, n_reindex=3, n_reuse=16,
              lengths=("fixed", 1048576), n_needles=64, outliers=True),
    5: Config("swa_verify", 5, B=64, H_I=64, d_I=128, P=2048, K=512, Hq=64, D=512, n_reindex=3,
              n_reuse=16, lengths=("loguniform", 4096, 524288), widths=("uniform", 1, 6), swa=True,
              n_needles=32),
    # chunked prefill: a 256-token chunk appended to each of two 128K
    # contexts; every chunk token selects its own pool and top-K
    6: Config("chunked_prefill", 6, B=2, H_I=64, d_I=128, P=2048, K=512, Hq=64, D=512, n_reindex=3,
              n_reuse=16, lengths=("fixed", 131072), widths=("fixed", 256), n_needles=32),
}


def layer_modes(n_reindex: int, n_reuse: int) -> list:
    """Layer order: one Full layer, then the Reindex layers, with the Reuse
    layers spread as evenly as possible after each selector (earlier groups
    take the remainder)."""
    groups = 1 + n_reindex
    base, rem = divmod(n_reuse, groups)
    modes = []
    for g in range(groups):
        modes.append("F" if g == 0 else "R")
        modes += ["U"] * (base + (1 if g < rem else 0))
    return modes


def _draw_lengths(cfg: Config, rng) -> np.ndarray:
    kind = cfg.lengths[0]
    if kind == "fixed":
        return np.full(cfg.B, int(cfg.lengths[1]), np.int64)
    if kind == "list":
        return np.asarray(cfg.lengths[1], np.int64)
    if kind == "uniform8":
        lo, hi = cfg.lengths[1], cfg.lengths[2]
        return (rng.integers(lo // 8, hi // 8 + 1, size=cfg.B) * 8).astype(np.int64)
    if kind == "loguniform":
        lo, hi = cfg.lengths[1], cfg.lengths[2]
        return np.floor(np.exp(rng.uniform(math.log(lo), math.log(hi), size=cfg.B))).astype(np.int64)
    raise ValueError(kind)


def _draw_widths(cfg: Config, rng) -> np.ndarray:
    kind = cfg.widths[0]
    if kind == "fixed":
        return np.full(cfg.B, int(cfg.widths[1]), np.int64)
    if kind == "list":
        return np.asarray(cfg.widths[1], np.int64)
    if kind == "uniform":
        return rng.integers(cfg.widths[1], cfg.widths[2] + 1, size=cfg.B).astype(np.int64)
    raise ValueError(kind)


@dataclass
class Workload:
    cfg: Config
    lens: np.ndarray                  # [B] cached positions per sequence (incl. the W new ones)
    widths: np.ndarray                # [B] query tokens per sequence
    tok_start: np.ndarray             # [B+1]
    tok_seq: np.ndarray               # [T]
    tok_pos: np.ndarray               # [T] position p of each query token
    modes: list
    seq_base: np.ndarray | None       # [B] first physical row (unpaged)
    page_table: np.ndarray | None     # [B][max_pages] physical page ids (paged)
    n_rows: int                       # physical rows of each cache
    kidx: TensorSpec = None
    kv: TensorSpec = None
    iq: dict = field(default_factory=dict)     # layer -> spec (selector layers)
    iw: dict = field(default_factory=dict)
    qmain: dict = field(default_factory=dict)  # layer -> spec
    swa: dict = field(default_factory=dict)    # layer -> spec

    @property
    def T(self) -> int:
        return int(self.tok_start[-1])

    @property
    def B(self) -> int:
        return len(self.lens)

    def physical_rows(self, b: int, pos: np.ndarray) -> np.ndarray:
        pos = np.asarray(pos, np.int64)
        if self.page_table is None:
            return self.seq_base[b] + pos
        ps = self.cfg.page_size
        return self.page_table[b][pos // ps].astype(np.int64) * ps + pos % ps

    # --- host views used by the CPU reference checks ------------------------------
    def iq_f32(self, layer: int, tok: int) -> np.ndarray:
        c = self.cfg
        return self.iq[layer].rows_f32(0, tok, 1).reshape(c.H_I, c.d_I)

    def iw_f32(self, layer: int, tok: int) -> np.ndarray:
        return self.iw[layer].rows_f32(0, tok, 1).reshape(-1)

    def qmain_f64(self, layer: int, tok: int) -> np.ndarray:
        c = self.cfg
        if c.q_dtype == "f32":
            q = self.qmain[layer].rows_f32(0, tok, 1)
        else:
            q = bf16_bits_to_f32(self.qmain[layer].rows_bf16_bits(0, tok, 1))
        return q.reshape(c.Hq, c.D).astype(np.float64)

    def swa_rows_e4m3(self, layer: int, tok: int):
        """FP8 sliding-window rows (codes, per-row scale) of a query token, positions max(0,p-w+1)..p"""
        b, p = int(self.tok_seq[tok]), int(self.tok_pos[tok])
        lo = max(0, p - self.cfg.window + 1)
        return self.swa[layer].rows_e4m3(b, lo, p - lo + 1)


def make_workload(cfg: Config) -> Workload:
    rng = np.random.default_rng(cfg.seed * 7919 + 17)
    lens = _draw_lengths(cfg, rng)
    widths = _draw_widths(cfg, rng)
    assert len(lens) == cfg.B and len(widths) == cfg.B
    assert np.all(widths >= 1) and np.all(lens >= widths)
    tok_start = np.concatenate([[0], np.cumsum(widths)]).astype(np.int64)
    T = int(tok_start[-1])
    tok_seq = np.repeat(np.arange(cfg.B), widths).astype(np.int64)
    tok_pos = np.concatenate([np.arange(L - W, L) for L, W in zip(lens, widths)]).astype(np.int64)
    modes = layer_modes(cfg.n_reindex, cfg.n_reuse)

    # physical layout of the caches
    if cfg.paged:
        ps = cfg.page_size
        npages = (lens + ps - 1) // ps
        total = int(npages.sum())
        perm = rng.permutation(total).astype(np.int32)
        max_pages = int(npages.max())
        page_table = np.zeros((cfg.B, max_pages), np.int32)
        o = 0
        for b in range(cfg.B):
            page_table[b, : npages[b]] = perm[o: o + npages[b]]
            o += npages[b]
        seq_base, n_rows = None, total * ps
    else:
        padded = (lens + 127) // 128 * 128
        seq_base = np.concatenate([[0], np.cumsum(padded)[:-1]]).astype(np.int64)
        page_table, n_rows = None, int(padded.sum())

    w = Workload(cfg, lens, widths, tok_start, tok_seq, tok_pos, modes, seq_base, page_table, n_rows)

    sd = cfg.seed
    for l, m in enumerate(modes):
        if m in "FR":
            w.iq[l] = TensorSpec(sd, S_IQ + l, cfg.H_I * cfg.d_I)
            w.iw[l] = TensorSpec(sd, S_IW + l, cfg.H_I, kind=KIND_UNIFORM)
        w.qmain[l] = TensorSpec(sd, S_QMAIN + l, cfg.Hq * cfg.D)
        if cfg.swa:
            w.swa[l] = TensorSpec(sd, S_SWA + l, cfg.D)

    # outlier channels (t(3) in about 1% of the channels)
    out_i = out_m = None
    if cfg.outliers:
        out_i = np.zeros(cfg.d_I, np.uint8)
        out_i[rng.choice(cfg.d_I, max(1, round(cfg.d_I / 100)), replace=False)] = 1
        out_m = np.zeros(cfg.D, np.uint8)
        out_m[rng.choice(cfg.D, max(1, round(cfg.D / 100)), replace=False)] = 1

    # needle blocks: distinct full history blocks, visible to every query of the sequence
    nblk = blk_dir_i = blk_dir_m = None
    n = cfg.n_needles
    if n > 0:
        nblk = np.zeros((cfg.B, n), np.int32)
        blk_dir_i = np.zeros((cfg.B, cfg.d_I), np.float32)
        blk_dir_m = np.zeros((cfg.B, cfg.D), np.float32)
        for b in range(cfg.B):
            full_hist = int((lens[b] - widths[b]) // BLOCK)
            k = min(n, full_hist)
            ch = np.sort(rng.choice(full_hist, k, replace=False)) if k > 0 else np.zeros(0, np.int64)
            row = np.full(n, -1, np.int32)
            row[:k] = ch
            nblk[b] = row
            t0 = int(tok_start[b])
            # direction of the Full layer's weighted indexer query of the first token
            q = w.iq[0].rows_f32(0, t0, 1).reshape(cfg.H_I, cfg.d_I).astype(np.float64)
            wh = w.iw[0].rows_f32(0, t0, 1).reshape(-1).astype(np.float64)
            u = (wh[:, None] * q).sum(0)
            blk_dir_i[b] = (u / max(np.linalg.norm(u), 1e-30)).astype(np.float32)
            qm = w.qmain_f64(0, t0).sum(0)
            blk_dir_m[b] = (qm / max(np.linalg.norm(qm), 1e-30)).astype(np.float32)

    w.kidx = TensorSpec(sd, S_KIDX, cfg.d_I, outlier=out_i, needle_blk=nblk, needle_dir=blk_dir_i,
                        needle_shift=cfg.needle_shift, needle_block=BLOCK)
    w.kv = TensorSpec(sd, S_KV, cfg.D, outlier=out_m, needle_blk=nblk, needle_dir=blk_dir_m,
                      needle_shift=cfg.needle_shift, needle_block=BLOCK)
    return w


def algorithmic_bytes(w: Workload) -> dict:
    """Bytes the method must move per decode step (scan, pool rescoring,
    attention gathers, sliding window, append) -- the roofline numerators."""
    c = w.cfg
    ki_row = c.d_I // 2 + c.d_I // 32
    kv_row = c.D // 2 + c.D // 32
    scan_pos = int(sum(int(p) + 1 for p in _scan_extent(w)))
    n_sel = sum(1 for m in w.modes if m in "FR")
    pool_pos = np.minimum(((w.tok_pos + 1 + BLOCK - 1) // BLOCK), c.P) * BLOCK
    pool_pos = np.minimum(pool_pos, w.tok_pos + 1)
    rescore = int(pool_pos.sum()) * ki_row * n_sel
    sel = np.minimum(w.tok_pos + 1, c.K)
    attn = int(sel.sum()) * kv_row * len(w.modes)
    swa = 0
    if c.swa:
        win = np.minimum(w.tok_pos + 1, c.window)
        swa = int(win.sum()) * (c.D + 4) * len(w.modes)
    return {"scan": scan_pos * ki_row, "rescore": rescore, "attend": attn, "swa": swa,
            "total": scan_pos * ki_row + rescore + attn + swa}


def _scan_extent(w: Workload):
    """last visible position per sequence (the scan reads each key once per sequence)"""
    return [int(w.lens[b]) - 1 for b in range(w.B)]

"""Context-parallel decode step: one long sequence's positions over G ranks.

Rank r holds positions [lo_r, hi_r) of every sequence (ascending ranges,
lo_r a multiple of 8) in its own FP4 caches.  A step runs in four phases, each
ending in an all-gather of small buffers over the process group (NCCL over
NVLink between GPUs):

  A  Full scan of the slice (csa2_index_full with its block scores) and the
     slice's best P blocks as (score, global block id)     -> gather [G][T][P]
  B  merge into the global pool (csa2_cp_merge), keep the pool's own blocks
     (csa2_cp_localize, aligned) and rescore their positions for every
     selector layer (csa2_cp_pool_scores)                 -> gather [G][S][T][8P]
  C  each selector's best K positions of the global pool (csa2_cp_select_positions);
     per layer, attention over this rank's selected rows (csa2_cp_localize,
     compact; csa2_attend_reuse with fp32 output and log-sum-exp)
                                                           -> gather [G][L][T][Hq][D], [G][L][T][Hq]
  D  log-sum-exp merge of every layer's parts (csa2_cp_attend_merge)

The selections are exactly the single-GPU ones (the global top-k lies in the
union of the slices' top-k); attention is the same softmax, merged.  This
module only orders the library's calls and the collective exchanges: every
step of the computation runs in the CUDA kernels of libcsa2.so.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field

from . import _lib as C


@dataclass
class Slice:
    """This rank's part of the sequences: positions [lo, hi) of each."""
    rank: int
    world: int
    lo: int
    hi: int


@dataclass
class StackLayers:
    """The stack's layers as the library sees them (modes and per-layer device tensors)."""
    modes: list                      # "F" / "R" / "U" per layer
    iq: dict                         # selector layer -> indexer query [T][H_I][d_I] fp32
    iw: dict                         # selector layer -> head weights [T][H_I] fp32
    q: dict                          # layer -> main query [T][Hq][D]
    out: dict                        # layer -> output [T][Hq][D]
    selectors: list = field(default_factory=list)

    def __post_init__(self):
        self.selectors = [l for l, m in enumerate(self.modes) if m in "FR"]

    def selector_of(self, layer: int) -> int:
        return max(s for s in self.selectors if s <= layer)


class CPRank:
    """The state and calls of one rank of a context-parallel step.  `batch` is
    the rank's csa2_query_batch (query positions relative to the slice),
    `k_idx` / `kv` its csa2_fp4_cache slices; dims and shapes as in the
    single-GPU stack.  Tensors are allocated with `torch` on the rank's device."""

    def __init__(self, sl: Slice, batch, k_idx, kv, layers: StackLayers, H_I: int, d_I: int, P: int, K: int,
                 Hq: int, D: int, q_dtype: int, out_dtype: int, max_blocks: int, stream, torch):
        self.sl, self.batch, self.k_idx, self.kv, self.L = sl, batch, k_idx, kv, layers
        self.H_I, self.d_I, self.P, self.K, self.Hq, self.D = H_I, d_I, P, K, Hq, D
        self.q_dtype, self.out_dtype = q_dtype, out_dtype
        self.stream = stream
        self.torch = torch
        dev = torch.device("cuda", torch.cuda.current_device())
        T = batch.n_tok
        self.T = T
        S = len(layers.selectors)
        self.S = S
        u8, i32, f32 = torch.uint8, torch.int32, torch.float32
        self.qc = torch.zeros(S, T * H_I, d_I // 2, dtype=u8, device=dev)
        self.qs = torch.zeros(S, T * H_I, d_I // 32, dtype=u8, device=dev)
        self.ld = max_blocks
        self.bs = torch.zeros(T, max_blocks, dtype=f32, device=dev)
        self.pool_loc = torch.zeros(T, P, dtype=i32, device=dev)
        self.pool_n_loc = torch.zeros(T, dtype=i32, device=dev)
        self.idx_loc = torch.zeros(T, K, dtype=i32, device=dev)
        self.idx_n_loc = torch.zeros(T, dtype=i32, device=dev)
        self.cand_score = torch.zeros(T, P, dtype=f32, device=dev)
        self.cand_id = torch.zeros(T, P, dtype=i32, device=dev)
        self.pool = torch.zeros(T, P, dtype=i32, device=dev)
        self.pool_n = torch.zeros(T, dtype=i32, device=dev)
        self.pool_al = torch.zeros(T, P, dtype=i32, device=dev)
        self.pool_al_n = torch.zeros(T, dtype=i32, device=dev)
        self.pscores = torch.zeros(S, T, P * 8, dtype=f32, device=dev)
        self.idx = torch.zeros(S, T, K, dtype=i32, device=dev)
        self.idx_n = torch.zeros(S, T, dtype=i32, device=dev)
        n_layers = len(layers.modes)
        self.o_part = torch.zeros(n_layers, T, Hq, D, dtype=f32, device=dev)
        self.lse_part = torch.zeros(n_layers, T, Hq, dtype=f32, device=dev)
        self.att_idx = torch.zeros(T, K, dtype=i32, device=dev)
        self.att_n = torch.zeros(T, dtype=i32, device=dev)
        nb = ctypes.c_size_t(0)
        C.check(C.csa2_index_workspace_size(ctypes.byref(batch), H_I, d_I, P, K, ctypes.byref(nb)))
        self.ws_index = torch.empty(nb.value, dtype=u8, device=dev)
        C.check(C.csa2_attend_workspace_size(ctypes.byref(batch), Hq, D, K, 0, ctypes.byref(nb)))
        self.ws_attend = torch.empty(nb.value, dtype=u8, device=dev)

    # ---------------------------------------------------------------- phases
    def phase_a(self):
        """quantise the selectors' queries; Full scan of the slice; its pool as candidates"""
        L, T, sp = self.L, self.T, self.stream
        for i, l in enumerate(L.selectors):
            C.check(C.csa2_quantize_fp4(L.iq[l].data_ptr(), T * self.H_I, self.d_I, None, self.qc[i].data_ptr(),
                                        self.qs[i].data_ptr(), sp))
        f = L.selectors[0]
        C.check(C.csa2_index_full(ctypes.byref(self.batch), self.qc[0].data_ptr(), self.qs[0].data_ptr(),
                                  L.iw[f].data_ptr(), self.H_I, ctypes.byref(self.k_idx), self.P, self.K,
                                  self.pool_loc.data_ptr(), self.pool_n_loc.data_ptr(), self.idx_loc.data_ptr(),
                                  self.idx_n_loc.data_ptr(), self.bs.data_ptr(), self.ws_index.data_ptr(),
                                  self.ws_index.numel(), sp))
        C.check(C.csa2_cp_candidates(self.bs.data_ptr(), self.ld, self.pool_loc.data_ptr(), T, self.P, 1,
                                     self.sl.lo // 8, self.cand_score.data_ptr(), self.cand_id.data_ptr(), sp))
        return [self.cand_score, self.cand_id]

    def phase_b(self, g_score, g_id):
        """global pool; this rank's pool positions rescored for every selector"""
        T, sp = self.T, self.stream
        G = self.sl.world
        C.check(C.csa2_cp_merge(g_score.data_ptr(), g_id.data_ptr(), G, T, self.P, self.P, self.pool.data_ptr(),
                                self.pool_n.data_ptr(), sp))
        C.check(C.csa2_cp_localize(self.pool.data_ptr(), self.pool_n.data_ptr(), T, self.P, self.sl.lo // 8,
                                   (self.sl.hi + 7) // 8, 0, self.pool_al.data_ptr(), self.pool_al_n.data_ptr(), sp))
        ws = (ctypes.c_void_p * self.S)(*[self.L.iw[l].data_ptr() for l in self.L.selectors])
        C.check(C.csa2_cp_pool_scores(ctypes.byref(self.batch), self.qc.data_ptr(), self.qs.data_ptr(), ws, self.S,
                                      self.H_I, ctypes.byref(self.k_idx), self.pool_al.data_ptr(),
                                      self.pool_al_n.data_ptr(), self.P, self.pscores.data_ptr(), sp))
        return [self.pscores]

    def phase_c(self, g_pscores, swa_of=None, softmax_scale: float = 0.0):
        """every selector's top-K of the global pool; each layer's attention
        over this rank's selected rows (fp32 parts with log-sum-exp)"""
        T, sp, L = self.T, self.stream, self.L
        G = self.sl.world
        C.check(C.csa2_cp_select_positions(g_pscores.data_ptr(), G, self.S, T, self.pool.data_ptr(),
                                           self.pool_n.data_ptr(), self.P, self.K, self.idx.data_ptr(),
                                           self.idx_n.data_ptr(), sp))
        for l in range(len(L.modes)):
            s = L.selectors.index(L.selector_of(l))
            C.check(C.csa2_cp_localize(self.idx[s].data_ptr(), self.idx_n[s].data_ptr(), T, self.K, self.sl.lo,
                                       self.sl.hi, 1, self.att_idx.data_ptr(), self.att_n.data_ptr(), sp))
            swa = swa_of(l) if swa_of else None
            C.check(C.csa2_attend_reuse(ctypes.byref(self.batch), L.q[l].data_ptr(), self.q_dtype, self.Hq,
                                        ctypes.byref(self.kv), self.att_idx.data_ptr(), self.att_n.data_ptr(),
                                        self.K, ctypes.byref(swa) if swa is not None else None, softmax_scale,
                                        self.o_part[l].data_ptr(), C.CSA2_F32, self.lse_part[l].data_ptr(),
                                        self.ws_attend.data_ptr(), self.ws_attend.numel(), sp))
        return [self.o_part, self.lse_part]

    def phase_d(self, g_o, g_lse):
        """every layer's output: the log-sum-exp merge of the ranks' parts
        (part of rank g for layer l at g_o[g][l], g_lse[g][l])"""
        T, sp = self.T, self.stream
        G = self.sl.world
        n_layers = len(self.L.modes)
        o_stride = n_layers * T * self.Hq * self.D
        lse_stride = n_layers * T * self.Hq
        for l in range(n_layers):
            C.check(C.csa2_cp_attend_merge(g_o[0, l].data_ptr(), g_lse[0, l].data_ptr(), G, o_stride, lse_stride, T,
                                           self.Hq, self.D, self.L.out[l].data_ptr(), self.out_dtype, None, sp))


def run_step(rank: CPRank, all_gather, swa_of=None, softmax_scale: float = 0.0):
    """One context-parallel decode step of this rank.  all_gather(list of
    tensors) -> list of tensors with a leading rank dimension (every rank
    calls it at the same points, in the same order)."""
    a = rank.phase_a()
    g = all_gather(a)
    b = rank.phase_b(*g)
    g = all_gather(b)
    c = rank.phase_c(g[0], swa_of, softmax_scale)
    g = all_gather(c)
    rank.phase_d(*g)


def torch_all_gather(group=None):
    """all_gather over a torch.distributed process group: tensors gathered
    into one buffer with a leading rank dimension each"""
    import torch
    import torch.distributed as dist

    def gather(tensors):
        out = []
        world = dist.get_world_size(group)
        for t in tensors:
            # the ranks' tensors concatenated along the first dimension, seen
            # with a leading rank dimension
            buf = torch.empty((world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
            dist.all_gather_into_tensor(buf, t.contiguous(), group=group)
            out.append(buf.view((world,) + tuple(t.shape)))
        return out

    return gather

"""Materialise a workload on the GPU for the tests and the benchmark.

Buffers are torch tensors (device memory only); their contents come from the
device generator (bit-identical to the host one), and the FP4 caches are
filled through the library's public quantiser, the same call a user makes to
fill a cache.  Nothing here computes any part of the decode step.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

import csa2_fp4_sparse_b200 as C

from .workloads import Workload


def _i32(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(dev)


def _i64(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, np.int64)).to(dev)


class DeviceWorkload:
    def __init__(self, w: Workload, device: str = "cuda", chunk_rows: int = 1 << 16):
        self.w = w
        self.dev = torch.device(device)
        self.chunk_rows = chunk_rows
        c = w.cfg
        dev = self.dev
        self.stream = torch.cuda.current_stream(dev).cuda_stream
        # batch
        self.seq_len = _i32(w.lens, dev)
        self.tok_start = _i32(w.tok_start, dev)
        self.tok_seq = _i32(w.tok_seq, dev)
        self.tok_pos = _i32(w.tok_pos, dev)
        # caches
        n = w.n_rows
        self.kidx_codes = torch.zeros(n, c.d_I // 2, dtype=torch.uint8, device=dev)
        self.kidx_scales = torch.zeros(n, c.d_I // 32, dtype=torch.uint8, device=dev)
        self.kv_codes = torch.zeros(n, c.D // 2, dtype=torch.uint8, device=dev)
        self.kv_scales = torch.zeros(n, c.D // 32, dtype=torch.uint8, device=dev)
        self.page_table = None if w.page_table is None else _i32(w.page_table, dev)
        self.seq_base = None if w.seq_base is None else _i64(w.seq_base, dev)
        # per-layer inputs
        T = w.T
        self.iq, self.iw, self.q, self.out, self.lse, self.idx_out = {}, {}, {}, {}, {}, {}
        self.swa_codes, self.swa_scale = {}, {}
        qdt = torch.float32 if c.q_dtype == "f32" else torch.bfloat16
        odt = torch.float32 if c.out_dtype == "f32" else torch.bfloat16
        # every per-step input in one contiguous device buffer: first what the
        # indexer needs (queries and head weights of every selector, the new
        # tokens), then the Main queries of every layer (read only by
        # attention); every layer's output in one tensor.  A step's host copies
        # are then one transfer each way, or two in, the second overlapping the
        # indexer kernels
        n_fr = sum(1 for m in w.modes if m in "FR")
        qsz = 4 if qdt == torch.float32 else 2
        parts = [T * c.H_I * c.d_I * 4, T * c.H_I * 4] * n_fr + [T * c.d_I * 4, T * c.D * 4] + [
            T * c.Hq * c.D * qsz] * len(w.modes)
        self.inputs_packed = torch.empty(sum((n + 255) // 256 * 256 for n in parts), dtype=torch.uint8, device=dev)
        self._in_off = 0

        def take(shape, dtype):
            n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
            t = self.inputs_packed[self._in_off:self._in_off + n].view(dtype).view(*shape)
            self._in_off += (n + 255) // 256 * 256
            return t

        for l, m in enumerate(w.modes):
            if m in "FR":
                self.iq[l] = take((T, c.H_I, c.d_I), torch.float32)
                self.iw[l] = take((T, c.H_I), torch.float32)
        # this step's new tokens (appended by the decode step)
        self.new_kidx = take((T, c.d_I), torch.float32)
        self.new_kv = take((T, c.D), torch.float32)
        self.inputs_index = self.inputs_packed[:self._in_off]
        for l in range(len(w.modes)):
            self.q[l] = take((T, c.Hq, c.D), qdt)
        self.inputs_main_q = self.inputs_packed[self.inputs_index.numel():]
        assert self._in_off == self.inputs_packed.numel()
        self.out_all = torch.zeros(len(w.modes), T, c.Hq, c.D, dtype=odt, device=dev)
        for l, m in enumerate(w.modes):
            if m in "FR":
                w.iq[l].dev_rows_f32(0, 0, T, self.iq[l].data_ptr(), self.stream)
                w.iw[l].dev_rows_f32(0, 0, T, self.iw[l].data_ptr(), self.stream)
                self.idx_out[l] = torch.full((T, c.K), -2, dtype=torch.int32, device=dev)
            if c.q_dtype == "f32":
                w.qmain[l].dev_rows_f32(0, 0, T, self.q[l].data_ptr(), self.stream)
            else:
                w.qmain[l].dev_rows_bf16(0, 0, T, self.q[l].data_ptr(), self.stream)
            self.out[l] = self.out_all[l]
            self.lse[l] = torch.zeros(T, c.Hq, dtype=torch.float32, device=dev)
            if c.swa:
                cap = c.swa_cap
                self.swa_codes[l] = torch.zeros(w.B * cap, c.D, dtype=torch.uint8, device=dev)
                self.swa_scale[l] = torch.ones(w.B * cap, dtype=torch.float32, device=dev)
                st = w.swa[l].device(dev)
                for b in range(w.B):
                    L = int(w.lens[b])
                    lo = max(0, L - cap)
                    w.swa[l].dev_rows_e4m3(b, lo, L - lo, cap, self.swa_codes[l][b * cap:].data_ptr(),
                                           self.swa_scale[l][b * cap:].data_ptr(), self.stream, st=st)
        self.pool_out = torch.full((T, c.P), -2, dtype=torch.int32, device=dev)
        sk, sv = w.kidx.device(dev), w.kv.device(dev)
        for b in range(w.B):
            t0, t1 = int(w.tok_start[b]), int(w.tok_start[b + 1])
            L = int(w.lens[b])
            w.kidx.dev_rows_f32(b, L - (t1 - t0), t1 - t0, self.new_kidx[t0:].data_ptr(), self.stream, st=sk)
            w.kv.dev_rows_f32(b, L - (t1 - t0), t1 - t0, self.new_kv[t0:].data_ptr(), self.stream, st=sv)
        slots = np.concatenate([w.physical_rows(b, w.tok_pos[w.tok_start[b]:w.tok_start[b + 1]])
                                for b in range(w.B)])
        self.new_slot = _i64(slots, dev)
        self._keep = []

    # ------------------------------------------------------------------ fill
    def fill_caches(self, include_new: bool = False):
        """Quantise the history positions 0..L-W-1 (or 0..L-1) of every
        sequence into the FP4 caches through csa2_quantize_fp4."""
        w, c, dev = self.w, self.w.cfg, self.dev
        sk, sv = w.kidx.device(dev), w.kv.device(dev)
        ch = self.chunk_rows
        buf_k = torch.empty(ch, c.d_I, dtype=torch.float32, device=dev)
        buf_v = torch.empty(ch, c.D, dtype=torch.float32, device=dev)
        for b in range(w.B):
            L = int(w.lens[b]) if include_new else int(w.lens[b] - w.widths[b])
            for p0 in range(0, L, ch):
                n = min(ch, L - p0)
                w.kidx.dev_rows_f32(b, p0, n, buf_k.data_ptr(), self.stream, st=sk)
                w.kv.dev_rows_f32(b, p0, n, buf_v.data_ptr(), self.stream, st=sv)
                if w.page_table is None:
                    r0 = int(w.seq_base[b]) + p0
                    for buf, d, codes, scales in ((buf_k, c.d_I, self.kidx_codes, self.kidx_scales),
                                                  (buf_v, c.D, self.kv_codes, self.kv_scales)):
                        C.check(C.csa2_quantize_fp4(buf.data_ptr(), n, d, None, codes[r0:].data_ptr(),
                                                    scales[r0:].data_ptr(), self.stream))
                else:
                    slot = _i64(w.physical_rows(b, np.arange(p0, p0 + n)), dev)
                    for buf, d, codes, scales in ((buf_k, c.d_I, self.kidx_codes, self.kidx_scales),
                                                  (buf_v, c.D, self.kv_codes, self.kv_scales)):
                        C.check(C.csa2_quantize_fp4(buf.data_ptr(), n, d, slot.data_ptr(), codes.data_ptr(),
                                                    scales.data_ptr(), self.stream))
                    torch.cuda.current_stream(dev).synchronize()  # slot buffer lifetime
        torch.cuda.current_stream(dev).synchronize()

    # ------------------------------------------------------------- descriptors
    def batch(self) -> C.csa2_query_batch:
        w = self.w
        return C.csa2_query_batch(w.B, w.T, int(w.lens.max()), int(w.widths.max()), self.seq_len.data_ptr(),
                                  self.tok_start.data_ptr(), self.tok_seq.data_ptr(), self.tok_pos.data_ptr())

    def cache(self, which: str) -> C.csa2_fp4_cache:
        w = self.w
        codes, scales, dim = ((self.kidx_codes, self.kidx_scales, w.cfg.d_I) if which == "kidx"
                              else (self.kv_codes, self.kv_scales, w.cfg.D))
        if self.page_table is None:
            return C.csa2_fp4_cache(codes.data_ptr(), scales.data_ptr(), w.n_rows, dim, 0, None, 0,
                                    self.seq_base.data_ptr())
        return C.csa2_fp4_cache(codes.data_ptr(), scales.data_ptr(), w.n_rows, dim, w.cfg.page_size,
                                self.page_table.data_ptr(), self.page_table.shape[1], None)

    def swa_desc(self, layer: int):
        c = self.w.cfg
        if not c.swa:
            return None
        return C.csa2_swa_desc(self.swa_codes[layer].data_ptr(), self.swa_scale[layer].data_ptr(), c.swa_cap,
                               c.window, c.D)

    def stack_desc(self, append: bool = True, copies: bool = True) -> C.csa2_stack_desc:
        w, c = self.w, self.w.cfg
        n = len(w.modes)
        layers = (C.csa2_layer_desc * n)()
        swas = []
        for l, m in enumerate(w.modes):
            L = layers[l]
            L.mode = {"F": C.CSA2_MODE_FULL, "R": C.CSA2_MODE_REINDEX, "U": C.CSA2_MODE_REUSE}[m]
            if m in "FR":
                L.iq = self.iq[l].data_ptr()
                L.iw = self.iw[l].data_ptr()
                if copies:
                    L.idx_out = self.idx_out[l].data_ptr()
            if m == "F" and copies:
                L.pool_out = self.pool_out.data_ptr()
            L.q = self.q[l].data_ptr()
            L.out = self.out[l].data_ptr()
            L.lse = self.lse[l].data_ptr()
            sd = self.swa_desc(l)
            if sd is not None:
                swas.append(sd)
                L.swa = ctypes.pointer(sd)
        d = C.csa2_stack_desc()
        d.qb = self.batch()
        d.k_idx = self.cache("kidx")
        d.kv = self.cache("kv")
        d.H_I, d.P, d.K, d.Hq = c.H_I, c.P, c.K, c.Hq
        d.q_dtype = C.CSA2_F32 if c.q_dtype == "f32" else C.CSA2_BF16
        d.out_dtype = C.CSA2_F32 if c.out_dtype == "f32" else C.CSA2_BF16
        d.softmax_scale = 0.0
        if append:
            d.new_k_idx = self.new_kidx.data_ptr()
            d.new_kv = self.new_kv.data_ptr()
            d.new_slot_k_idx = self.new_slot.data_ptr()
            d.new_slot_kv = self.new_slot.data_ptr()
        d.n_layers = n
        d.layers = layers
        self._keep = [layers, swas]
        return d

    def stack_workspace(self, desc) -> torch.Tensor:
        nb = ctypes.c_size_t(0)
        C.check(C.csa2_stack_workspace_size(ctypes.byref(desc), ctypes.byref(nb)))
        return torch.empty(nb.value, dtype=torch.uint8, device=self.dev)

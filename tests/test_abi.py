"""The C ABI: the library loads, exports every entry point declared in
include/csa2.h, and rejects bad arguments on the host (no GPU needed)."""
import ctypes
import os
import re

import pytest

import csa2_fp4_sparse_b200 as C

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "csa2.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(csa2_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported_and_bound():
    lib = ctypes.CDLL(C._lib.LIB_PATH)
    names = _declared()
    assert "csa2_decode_stack" in names and len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
        assert n in C.EXPORTED, n


def test_version_and_error_string():
    assert C.csa2_version() >= 100
    assert isinstance(C.csa2_last_error(), str)


def _batch(**kw):
    b = C.csa2_query_batch(1, 1, 100, 1, 8, 8, 8, 8)
    for k, v in kw.items():
        setattr(b, k, v)
    return b


def test_quantize_rejects_bad_shapes():
    assert C.csa2_quantize_fp4(16, 10, 48, None, 16, 16, None) == C.CSA2_ERR_UNSUPPORTED
    assert "dim" in C.csa2_last_error()
    assert C.csa2_quantize_fp4(16, -1, 64, None, 16, 16, None) == C.CSA2_ERR_INVALID_ARG
    assert C.csa2_quantize_fp4(None, 10, 64, None, 16, 16, None) == C.CSA2_ERR_INVALID_ARG
    assert C.csa2_quantize_fp4(8, 10, 64, None, 16, 16, None) == C.CSA2_ERR_INVALID_ARG  # misaligned x


def test_index_rejects_bad_arguments():
    kc = C.csa2_fp4_cache(16, 16, 100, 128, 0, None, 0, 16)
    b = _batch()
    args = lambda qb, H, kc_, P, K, ws_bytes=1 << 30: C.csa2_index_full(  # noqa: E731
        ctypes.byref(qb) if qb is not None else None, 256, 256, 256, H, ctypes.byref(kc_), P, K, 256, 256, 256,
        256, None, 256, ws_bytes, None)
    assert args(None, 64, kc, 2048, 512) == C.CSA2_ERR_INVALID_ARG
    assert args(_batch(n_tok=0), 64, kc, 2048, 512) == C.CSA2_ERR_INVALID_ARG
    assert args(b, 65, kc, 2048, 512) == C.CSA2_ERR_UNSUPPORTED
    assert args(b, 64, kc, 16, 512) == C.CSA2_ERR_UNSUPPORTED  # K > 8P
    assert args(b, 64, C.csa2_fp4_cache(16, 16, 100, 96, 0, None, 0, 16), 2048, 512) == C.CSA2_ERR_UNSUPPORTED
    assert args(b, 64, C.csa2_fp4_cache(16, 16, 100, 128, 32, 16, 4, None), 2048, 512) == C.CSA2_ERR_UNSUPPORTED
    assert args(b, 64, C.csa2_fp4_cache(16, 16, 100, 128, 0, None, 0, None), 2048, 512) == C.CSA2_ERR_INVALID_ARG
    assert args(b, 64, kc, 2048, 512, ws_bytes=10) == C.CSA2_ERR_WORKSPACE


def test_workspace_size_queries():
    b = _batch(n_tok=4, max_seq_len=1 << 20)
    n = ctypes.c_size_t(0)
    assert C.csa2_index_workspace_size(ctypes.byref(b), 64, 128, 2048, 512, ctypes.byref(n)) == 0
    assert n.value >= 4 * (1 << 17) * 4 + 4 * 16384 * 4
    assert C.csa2_attend_workspace_size(ctypes.byref(b), 64, 512, 512, 1, ctypes.byref(n)) == 0
    assert n.value > 0


def test_attend_rejects_bad_swa():
    kv = C.csa2_fp4_cache(16, 16, 100, 512, 0, None, 0, 16)
    b = _batch(max_q_per_seq=4)
    sw = C.csa2_swa_desc(16, 16, 128, 128, 512)  # cap < window + W - 1
    rc = C.csa2_attend_reuse(ctypes.byref(b), 256, C.CSA2_BF16, 64, ctypes.byref(kv), 256, 256, 512,
                             ctypes.byref(sw), 0.0, 256, C.CSA2_BF16, None, 256, 1 << 30, None)
    assert rc == C.CSA2_ERR_INVALID_ARG
    rc = C.csa2_attend_reuse(ctypes.byref(b), 256, C.CSA2_BF16, 48, ctypes.byref(kv), 256, 256, 512, None, 0.0,
                             256, C.CSA2_BF16, None, 256, 1 << 30, None)
    assert rc == C.CSA2_ERR_UNSUPPORTED


def test_stack_rejects_non_full_first_layer():
    layers = (C.csa2_layer_desc * 1)()
    layers[0].mode = C.CSA2_MODE_REUSE
    d = C.csa2_stack_desc()
    d.qb = _batch()
    d.n_layers = 1
    d.layers = layers
    assert C.csa2_decode_stack(ctypes.byref(d), 256, 1 << 30, None) == C.CSA2_ERR_INVALID_ARG
    assert "FULL" in C.csa2_last_error()


def test_product_package_does_not_import_oracle():
    """The product package and the shared input generators never name the
    oracle (so they cannot import, link or call it)."""
    for sub in ("csa2_fp4_sparse_b200", "synth", "include"):
        for dirpath, _, files in os.walk(os.path.join(ROOT, sub)):
            for f in files:
                if f.endswith((".py", ".cu", ".cuh", ".h", ".c")):
                    txt = open(os.path.join(dirpath, f), encoding="utf-8").read()
                    assert "oracle" not in txt.lower(), os.path.join(dirpath, f)


def test_struct_layouts_match_header(tmp_path):
    """The ctypes mirrors have the header's sizes and field offsets (a plain C
    program built with gcc against include/csa2.h prints them)."""
    import shutil
    import subprocess

    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    structs = {name: getattr(C._lib, name) for name in
               ("csa2_query_batch", "csa2_fp4_cache", "csa2_swa_desc", "csa2_layer_desc", "csa2_stack_desc",
                "csa2_kernel_stat")}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "csa2.h"', "int main(void) {"]
    for name, cls in structs.items():
        lines.append(f'  printf("{name} sizeof %zu\\n", sizeof({name}));')
        for f in cls._fields_:
            lines.append(f'  printf("{name} {f[0]} %zu\\n", offsetof({name}, {f[0]}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    out = subprocess.check_output([str(exe)], text=True).split("\n")
    got = {(a, b): int(c) for a, b, c in (l.split() for l in out if l)}
    for name, cls in structs.items():
        assert got[(name, "sizeof")] == ctypes.sizeof(cls), name
        for f in cls._fields_:
            assert got[(name, f[0])] == getattr(cls, f[0]).offset, (name, f[0])


def test_paged_cache_must_cover_the_batch():
    """A paged cache whose table rows cover fewer positions than the batch's
    longest sequence is refused before any launch (the kernels index the page
    table without a bound)."""
    b = _batch(max_seq_len=1000)
    short = C.csa2_fp4_cache(16, 16, 1 << 20, 128, 64, 16, 15, None)   # 15 * 64 = 960 < 1000
    enough = C.csa2_fp4_cache(16, 16, 1 << 20, 128, 64, 16, 16, None)  # 1024
    full = lambda kc: C.csa2_index_full(ctypes.byref(b), 256, 256, 256, 64, ctypes.byref(kc), 2048, 512, 256,  # noqa: E731
                                        256, 256, 256, None, 256, 1 << 30, None)
    assert full(short) == C.CSA2_ERR_INVALID_ARG
    assert "max_pages" in C.csa2_last_error()
    reindex = lambda kc: C.csa2_index_reindex(ctypes.byref(b), 256, 256, 256, 64, ctypes.byref(kc), 256, 256,  # noqa: E731
                                              2048, 512, 256, 256, 256, 1 << 30, None)
    assert reindex(short) == C.CSA2_ERR_INVALID_ARG
    kv_short = C.csa2_fp4_cache(16, 16, 1 << 20, 512, 64, 16, 15, None)
    rc = C.csa2_attend_reuse(ctypes.byref(b), 256, C.CSA2_BF16, 64, ctypes.byref(kv_short), 256, 256, 512, None,
                             0.0, 256, C.CSA2_BF16, None, 256, 1 << 30, None)
    assert rc == C.CSA2_ERR_INVALID_ARG
    # the covering table passes the table check: with a too-small workspace
    # the call stops at the workspace check instead (nothing is launched)
    rc = C.csa2_index_full(ctypes.byref(b), 256, 256, 256, 64, ctypes.byref(enough), 2048, 512, 256, 256, 256, 256,
                           None, 256, 10, None)
    assert rc == C.CSA2_ERR_WORKSPACE


def test_attend_shapes():
    """Hq in {16, 32, 64}, D in {128, 512}; fp32 queries need D * Hq <= 16384"""
    b = _batch()
    call = lambda Hq, D, qdt: C.csa2_attend_reuse(  # noqa: E731
        ctypes.byref(b), 256, qdt, Hq, ctypes.byref(C.csa2_fp4_cache(16, 16, 100, D, 0, None, 0, 16)), 256, 256,
        512, None, 0.0, 256, C.CSA2_BF16, None, 256, 10, None)
    for Hq in (16, 32, 64):
        for D in (128, 512):
            for qdt in (C.CSA2_BF16, C.CSA2_F32):
                rc = call(Hq, D, qdt)
                if qdt == C.CSA2_F32 and D * Hq > 16384:
                    assert rc == C.CSA2_ERR_UNSUPPORTED, (Hq, D)
                    assert "fp32" in C.csa2_last_error()
                else:  # accepted shape: only the (deliberately tiny) workspace is refused
                    assert rc == C.CSA2_ERR_WORKSPACE, (Hq, D, qdt, C.csa2_last_error())
    assert call(48, 512, C.CSA2_BF16) == C.CSA2_ERR_UNSUPPORTED
    assert call(64, 256, C.CSA2_BF16) == C.CSA2_ERR_UNSUPPORTED

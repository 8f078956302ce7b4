"""The synthetic input generator: determinism, distributions, and host/device identity."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from synth import workloads as W


def test_normal_moments_and_determinism():
    t = synth.TensorSpec(123, synth.S_KIDX, 128)
    a = t.rows_f32(3, 1000, 2000)
    b = t.rows_f32(3, 1000, 2000)
    assert np.array_equal(a, b)
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1) < 0.01
    assert np.abs(a).max() <= 6.0
    # random access: a sub-range equals the slice
    assert np.array_equal(t.rows_f32(3, 1500, 10), a[500:510])
    assert np.array_equal(t.select_rows_f32(3, np.array([1000, 2999, 1500])), a[[0, 1999, 500]])


def test_streams_differ():
    a = synth.TensorSpec(1, synth.S_KIDX, 64).rows_f32(0, 0, 4)
    b = synth.TensorSpec(1, synth.S_KV, 64).rows_f32(0, 0, 4)
    c = synth.TensorSpec(2, synth.S_KIDX, 64).rows_f32(0, 0, 4)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)


def test_bf16_rounding_matches_torch():
    t = synth.TensorSpec(5, synth.S_QMAIN, 512)
    f = t.rows_f32(0, 0, 64)
    bits = t.rows_bf16_bits(0, 0, 64)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)


def test_e4m3_code_matches_torch():
    L = synth.host_lib()
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-448, 448, 5000), rng.standard_normal(5000) * 0.01,
                        [0.0, -0.0, 448.0, -448.0, 2.0**-10, 3 * 2.0**-10, 240.0, 248.0]]).astype(np.float32)
    got = np.array([L.syn_host_e4m3_code(float(x)) for x in v], np.uint8)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_outliers_and_needles():
    cfg = W.CONFIGS[1].with_(lengths=("fixed", 4096), outliers=True)
    w = W.make_workload(cfg)
    rows = w.kidx.rows_f32(0, 0, 4096)
    ch = np.nonzero(w.kidx.outlier)[0]
    assert len(ch) == 1
    blk = w.kidx.needle_blk[0]
    assert len(set(blk.tolist())) == len(blk) and np.all(blk * 8 + 7 < 4096 - 1)
    # needle keys are shifted by 2*dir relative to the same draw without the shift
    plain = synth.TensorSpec(w.kidx.seed, w.kidx.stream, w.kidx.dim, outlier=w.kidx.outlier).rows_f32(0, 0, 4096)
    d = rows - plain
    j = int(blk[0])
    np.testing.assert_allclose(d[8 * j: 8 * j + 8], np.repeat(2 * w.kidx.needle_dir[0][None], 8, 0), atol=1e-6)
    mask = np.ones(4096, bool)
    for b in blk:
        mask[8 * b: 8 * b + 8] = False
    assert np.all(d[mask] == 0)


def test_layer_order_reading():
    assert W.layer_modes(1, 1) == ["F", "U", "R"]
    assert W.layer_modes(2, 8) == list("FUUURUUURUU")
    assert W.layer_modes(3, 16) == list("FUUUURUUUURUUUURUUUU")


@pytest.mark.gpu
def test_host_device_identity():
    cfg = W.CONFIGS[4].with_(lengths=("fixed", 8192), B=2)
    w = W.make_workload(cfg)
    s = torch.cuda.current_stream().cuda_stream
    for spec, rows in [(w.kidx, 4096), (w.kv, 1024)]:
        out = torch.empty(rows, spec.dim, dtype=torch.float32, device="cuda")
        spec.dev_rows_f32(1, 100, rows, out.data_ptr(), s)
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy(), spec.rows_f32(1, 100, rows))
    q = w.qmain[0]
    ob = torch.empty(3, q.dim, dtype=torch.int16, device="cuda")
    q.dev_rows_bf16(0, 0, 3, ob.data_ptr(), s)
    torch.cuda.synchronize()
    assert np.array_equal(ob.cpu().numpy().view(np.uint16), q.rows_bf16_bits(0, 0, 3))
    sw = synth.TensorSpec(5, synth.S_SWA, 512)
    codes = torch.zeros(136, 512, dtype=torch.uint8, device="cuda")
    scale = torch.zeros(136, dtype=torch.float32, device="cuda")
    sw.dev_rows_e4m3(2, 1000, 130, 136, codes.data_ptr(), scale.data_ptr(), s)
    torch.cuda.synchronize()
    hc, hs = sw.rows_e4m3(2, 1000, 130, ring=136)
    slots = np.arange(1000, 1130) % 136  # slots the 130 positions land in
    assert np.array_equal(codes.cpu().numpy()[slots], hc[slots])
    assert np.array_equal(scale.cpu().numpy()[slots], hs[slots])

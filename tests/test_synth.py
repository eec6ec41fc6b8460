"""The shared seeded input generator: published Philox answers and distribution shape."""
import numpy as np

import synth
from synth.philox import _cos_sin_turn, _ln_unit, philox4x32_10


def test_philox_known_answers():
    # Known-answer vectors of Philox4x32-10 published with the Random123 library.
    cases = [
        ((0, 0, 0, 0, 0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
        ((0xFFFFFFFF,) * 6, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
        ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344, 0xA4093822, 0x299F31D0),
         (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
    ]
    for args, want in cases:
        got = tuple(int(x) for x in philox4x32_10(*args))
        assert got == want


def test_series_match_libm():
    rng = np.random.default_rng(0)
    u = rng.random(200000) + 1e-15
    assert np.abs(_ln_unit(u) - np.log(u)).max() < 1e-14
    a = rng.random(200000)
    c, s = _cos_sin_turn(a)
    assert np.abs(c - np.cos(2 * np.pi * a)).max() < 1e-14
    assert np.abs(s - np.sin(2 * np.pi * a)).max() < 1e-14


def test_normal_moments():
    z = synth.normals(7, 0, 1, np.arange(1 << 20, dtype=np.uint64))
    assert abs(z.mean()) < 5e-3
    assert abs(z.std() - 1.0) < 5e-3
    assert abs((z ** 4).mean() - 3.0) < 0.05


def test_student_t_tails():
    from synth.philox import student_t3
    t = student_t3(3, 0, 1, np.arange(1 << 18, dtype=np.uint64))
    # t(3): P(|t| > 5.841) = 0.01 (two-sided 99% quantile)
    frac = np.mean(np.abs(t) > 5.841)
    assert 0.008 < frac < 0.012


def test_workload_shapes_and_channels():
    w = synth.workload("llama7b_layer_32k")
    sc = synth.heavy_channel_scale(w)
    assert sc.shape == (32, 128)
    assert (np.sum(sc == 10.0, axis=1) == 6).all()
    w4 = synth.workload("llama3_8b_gqa_128k")
    assert (synth.student_t_channels(w4).sum(axis=1) == 8).all()
    # random access agrees with the full tensor
    ws = synth.workload("tiny_single_head")
    K = synth.gen_k(ws)
    t = np.array([0, 5, 2047])
    assert np.array_equal(synth.gen_k(ws, 0, 0, t[:, None], 0, np.arange(128)[None, :]),
                          K[0, t, 0])
    V = synth.gen_v(w, 0, 0, np.arange(4)[:, None, None], np.arange(32)[None, :, None],
                    np.arange(128)[None, None, :])
    assert V.dtype == np.float16 and V.shape == (4, 32, 128)

"""The seeded input generators: formats, distributions and determinism."""
import numpy as np

import mova_inputs as MI


def test_bf16_fast_path_matches_rne():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100_000).astype(np.float32),
                        np.array([1.0, -2.5, 1.00390625, 1.01171875, 3.0e38, 1e-40], np.float32)])
    assert (MI._f32_to_bf16_bits_fast(a) == MI.f32_to_bf16_bits(a)).all()
    # ties to even: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> 1
    assert MI.f32_to_bf16_bits(np.array([1.00390625], np.float32))[0] == 0x3F80
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6 -> even (1 + 2^-6)
    assert MI.f32_to_bf16_bits(np.array([1.01171875], np.float32))[0] == 0x3F82


def test_layer_determinism_and_stats():
    a = MI.make_layer(3, 0, E=4, n=64, d=256)
    b = MI.make_layer(3, 0, E=4, n=64, d=256)
    c = MI.make_layer(3, 1, E=4, n=64, d=256)
    assert (a.Wv == b.Wv).all() and (a.Wr == b.Wr).all()
    assert not (a.Wv == c.Wv).all()
    assert a.Wv.dtype == np.uint16 and a.Wv.shape == (4, 64, 256)
    wv = (a.Wv.astype(np.uint32) << 16).view(np.float32)
    assert abs(wv.std() - 1 / 16) < 0.01 * 1 / 16 * 10
    assert abs(a.Wr.std() - 0.02) < 0.002
    assert a.Wr.dtype == np.float32 and a.br.dtype == np.float32


def test_zipf_bias():
    br = MI.zipf_bias()
    p = np.exp(br.astype(np.float64) / 2.0)
    np.testing.assert_allclose(p.sum(), 1.0, rtol=1e-6)
    np.testing.assert_allclose(p[0] / p[1], 2.0 ** 1.2, rtol=1e-5)
    assert (np.diff(br) < 0).all()


def test_given_routing():
    b = MI.make_batch(500, 0, dtype="bf16", mode="given")
    assert b.idx.dtype == np.int8 and b.w.dtype == np.float16
    assert b.idx.shape == (500, 4)
    for row in b.idx:
        assert len(set(row.tolist())) == 4
    assert (b.idx >= 0).all() and (b.idx < 64).all()
    np.testing.assert_allclose(b.w.astype(np.float64).sum(axis=1), 2.5, rtol=2e-3)
    assert (b.w > 0).all()


def test_workload_table():
    assert MI.WORKLOADS["decode"]["T"] == 8
    assert MI.WORKLOADS["prefill"]["T"] == 4096
    assert MI.WORKLOADS["skewed"]["T"] == 16384
    assert MI.WORKLOADS["given"]["T"] == 32768
    assert MI.N_OUT == 8 * 128 and MI.D_MODEL == 2560 and MI.N_EXPERTS == 64

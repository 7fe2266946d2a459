"""Seeded input generators: published test vector, determinism, value statistics."""
import numpy as np

from synth import configs, gen, workloads


def test_splitmix64_published_vector():
    # First five outputs of SplitMix64 seeded with 1234567 (the reference
    # implementation's published test values).
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    assert gen.splitmix64(1234567, np.arange(5)).tolist() == want


def test_table_rows_are_counter_based():
    full = gen.table_bf16(0, 3, 50, 16, 0.02)
    rows = gen.table_rows_bf16(0, 3, [49, 7, 7], 16, 0.02)
    np.testing.assert_array_equal(rows, full[[49, 7, 7]])
    other = gen.table_bf16(0, 4, 50, 16, 0.02)
    assert (other != full).mean() > 0.9


def test_table_statistics():
    v = gen.bf16_bits_to_f32(gen.table_bf16(1, 0, 512, 512, 0.02)).astype(np.float64)
    assert abs(v.mean()) < 2e-4
    assert abs(v.std() - 0.02) < 2e-4
    w = gen.table_f32(1, gen.TAG_W, 256, 256, 0.25)
    assert abs(w.std() - 0.25) < 3e-3


def test_bf16_rounding_is_rne():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -8 + 2 ** -20], np.float32)
    b = gen.f32_to_bf16_bits(x)
    np.testing.assert_array_equal(gen.bf16_bits_to_f32(b),
                                  np.array([1.0, 1.0, 1.0 + 4 * 2 ** -8, -2.5, 1.0 + 2 ** -7], np.float32))


def test_zipf_tokens_shape_and_skew():
    t = gen.zipf_tokens(0, 20000, 131072)
    assert t.dtype == np.int32 and t.min() >= 0 and t.max() < 131072
    assert (t == 0).mean() > 0.05            # rank 1 carries ~ 1/zeta-ish mass
    np.testing.assert_array_equal(t, gen.zipf_tokens(0, 20000, 131072))


def test_workloads():
    toks, off = workloads.prefill_tokens(configs.PREFILL_D2048)
    assert len(toks) == 32768 and off.tolist() == list(range(0, 32769, 4096))
    toks, off = workloads.prefill_tokens(configs.PREFILL_D4096_VARLEN)
    lens = np.diff(off)
    assert off[-1] == 65536 and len(lens) == 16 and lens[0] == 1 and lens[1] == 3 and lens.min() >= 1
    ds = workloads.DecodeStream(configs.SPEC_DECODE)
    a = ds.accept_lengths(3)
    assert a.min() >= 0 and a.max() <= 4 and len(a) == 256
    assert len(ds.step_tokens(0)) == 1280
    ids, poff = ds.prompts()
    assert np.diff(poff).max() <= 16 and len(ids) == poff[-1]


def test_config_sizes():
    c = configs.PREFILL_D2048
    assert c.V_nk == (2162717, 2162737, 2162747, 2162803) and c.d == 512 and c.S == 4
    c = configs.FULL_SCALE
    assert c.V_nk[0] == 7274513 and abs(c.table_bytes() / 1e9 - 59.6) < 0.1
    for c in configs.CONFIGS:
        for v in c.V_nk:
            assert configs.is_prime(v)
        if c.V0 == 131072:
            # away from integer multiples of V0 (collision rule)
            for v in c.V_nk:
                frac = (v / c.V0) % 1.0
                assert 0.25 < frac < 0.75

"""The seeded input generator: deterministic, counter-based, with the stated distributions."""
import numpy as np

import synth


def test_deterministic_and_counter_based():
    a = synth.normal(7, 2, (1000,), 1.0, "f32")
    b = synth.normal(7, 2, (1000,), 1.0, "f32")
    np.testing.assert_array_equal(a, b)
    # any sub-range equals the slice of the full draw
    c = synth.normal(7, 2, (300,), 1.0, "f32", offset=333)
    np.testing.assert_array_equal(c, a[333:633])
    # streams and seeds are independent
    assert not np.array_equal(a, synth.normal(7, 3, (1000,), 1.0, "f32"))
    assert not np.array_equal(a, synth.normal(8, 2, (1000,), 1.0, "f32"))


def test_normal_moments():
    a = synth.normal(1, 0, (1 << 20,), 0.5, "f32").astype(np.float64)
    assert abs(a.mean()) < 3e-3
    assert abs(a.std() - 0.5) < 3e-3
    assert abs(((a / 0.5) ** 4).mean() - 3.0) < 0.05


def test_bf16_is_round_to_nearest_even_of_f32():
    f = synth.normal(3, 1, (100000,), 1.0, "f32")
    b = synth.normal(3, 1, (100000,), 1.0, "bf16")
    np.testing.assert_array_equal(b, synth.f32_to_bf16(f))
    back = synth.bf16_to_f32(b)
    assert np.all(np.abs(back - f) <= np.abs(f) * 2.0 ** -8)
    # ties go to even
    t = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8], np.float32)
    np.testing.assert_array_equal(synth.bf16_to_f32(synth.f32_to_bf16(t)), [1.0, 1.0 + 2 ** -6])


def test_uniform_int_and_ternary():
    L = synth.uniform_int(1004, synth.STREAM_LEN, 10000, 1000, 32768)
    assert L.min() >= 1000 and L.max() <= 32768
    assert abs(L.mean() - (1000 + 32768) / 2) < 400
    t = synth.ternary(5, 0, (100000,), 0.25, "f32")
    assert set(np.unique(t)) <= {-1.0, 0.0, 1.0}
    assert abs((t != 0).mean() - 0.25) < 0.01


def test_workload_table():
    w = synth.WORKLOADS
    assert [w[n].seed for n in ("tiny_f32", "prefill_8k", "prefill_128k", "varlen_16", "decode_256")] == \
        [1001, 1002, 1003, 1004, 1005]
    assert w["prefill_128k"].T == 131072 and w["prefill_128k"].H == 64 and w["prefill_128k"].D == 128
    lens = synth.varlen_lengths(w["varlen_16"])
    assert len(lens) == 16 and lens.min() >= 1000 and lens.max() <= 32768
    mixed = w["mixed_256"]
    ml = synth.mixed_lengths(mixed)
    assert (ml == 1).sum() == 256 and (ml == 4096).sum() == 2 and len(ml) == 258 and mixed.seed == 1006
    assert w["backward_128k"].seed == 1007 and w["backward_8k"].seed == 1008 and w["backward_8k"].T == 8192
    assert w["znorm_128k"].seed == 1009 and w["znorm_128k"].qk_shift == 1.0
    assert w["chunk_state_128k"].seed == 1010 and w["chunk_state_128k"].kind == "chunk_state"
    assert w["train_128k"].seed == 1011 and w["train_128k"].kind == "train"
    assert w["prefill_128k_h8"].seed == 1012 and w["prefill_128k_h8"].H == 8
    a = synth.normal(7, 0, (1000,), 0.5, "bf16")
    b = synth.shifted(a, 1.0)
    assert b.dtype == np.uint16 and np.allclose(synth.bf16_to_f32(b), synth.bf16_to_f32(a) + 1.0, atol=2 ** -7)

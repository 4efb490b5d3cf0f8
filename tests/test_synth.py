"""Host-side checks of the seeded input generator (no GPU)."""
import numpy as np

import synth


def test_splitmix64_reference_sequence():
    # SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) started from state
    # 1234567: the widely published first five outputs.
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    assert [int(v) for v in synth.words(1234567, 0, 5)] == want


def test_streams_are_counter_based():
    key = synth.stream_key(3, 1, synth.W13_CODES, 7)
    full = synth.random_bytes(key, 1000)
    assert np.array_equal(full[333:777], synth.random_bytes(key, 444, 333))
    c = synth.expert_codes(3, 1, 7, "w13", 64, 256)
    part = synth.expert_codes(3, 1, 7, "w13", 64, 256, row0=10, nrows=5)
    assert np.array_equal(c[10:15], part)


def test_value_ranges_and_moments():
    sc = synth.expert_scales(0, 0, 0, "w13", 1536, 2560)
    assert sc.min() == synth.SCALE_LO and sc.max() == synth.SCALE_HI
    codes = synth.expert_codes(0, 0, 0, "w13", 1536, 2560)
    nib = np.concatenate([codes & 0xF, codes >> 4]).ravel()
    hist = np.bincount(nib, minlength=16) / nib.size
    assert np.all(np.abs(hist - 1 / 16) < 2e-3)
    x = synth.bf16_bits_to_f64(synth.hidden_states(0, 0, 64, 2560)).ravel()
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    w = synth.bf16_bits_to_f64(synth.router_weight(0, 0, 64, 2560)).ravel()
    assert abs(w.std() - 0.02) < 0.0005


def test_zipf_bias_is_a_permutation_of_ranks():
    b = synth.zipf_router_bias(0, 0, 512)
    r = np.rint(np.exp(-b.astype(np.float64) / 1.1)).astype(int)
    assert sorted(r.tolist()) == list(range(1, 513))

"""Host-side logic of the GPU converter's binding (no GPU): the fit sample
the binding draws is the oracle converter's sample."""

import numpy as np

import oracle as O
import synth
from w4a8_codebook_quantized_rotate_b200 import binding as B


def test_fit_sample_positions_pick_the_oracle_sample():
    n, k, cap = 40, 512, 1000
    w = synth.weights(n, k, synth.rng_for(50, 0, "weight"))
    w[3] = 0.0
    w[5, : k // 2] = 0.0
    ref = O.convert_weight(w, sample_cap=cap)
    live = np.repeat((ref["s_rel"] & 0x7F) != 0, 16, axis=1) & (ref["s_ch"] > 0)[:, None]
    pos = B.fit_sample_positions(ref["s_rel"], ref["s_ch"], cap, 42)
    expected = np.random.Generator(np.random.PCG64(42)).choice(ref["v"][live], size=cap, replace=False)
    assert pos.dtype == np.int64 and pos.size == cap
    assert np.array_equal(ref["v"].ravel()[pos], expected)
    assert live.ravel()[pos].all()


def test_fit_sample_positions_whole_pool_below_cap():
    n, k = 8, 256
    w = synth.weights(n, k, synth.rng_for(51, 0, "weight"))
    ref = O.convert_weight(w)
    assert B.fit_sample_positions(ref["s_rel"], ref["s_ch"], n * k, 42) is None

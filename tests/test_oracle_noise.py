"""Pins of the oracle's noisy-gate draws (oracle/moe_oracle.py, Philox4x64-10
+ Box-Muller), none of them by re-running the oracle's own formulas:

* Philox4x64-10 against NumPy's independent implementation
  (numpy.random.Philox, which advances its counter before each block);
* the normals' distribution (mean, variance, the one-sigma mass, no
  correlation between neighbouring experts or tokens);
* closed forms: W_noise = 0 gives z * ln 2; softplus at 0, far right, far left;
* token_base: a block of the batch draws what the whole batch draws there.
"""
import math

import numpy as np
import pytest

from oracle import moe_oracle as O


@pytest.mark.parametrize("key", [(0, 0), (1, 2), (0xDEADBEEF, 7), (2 ** 64 - 1, 2 ** 63 + 5)])
@pytest.mark.parametrize("counter", [(0, 0, 0, 0), (5, 9, 0, 1), (2 ** 64 - 3, 1, 2, 3)])
def test_philox_matches_numpy(key, counter):
    bg = np.random.Philox(key=np.array(key, dtype=np.uint64),
                          counter=np.array(counter, dtype=np.uint64))
    raw = bg.random_raw(12)
    mask = 2 ** 64 - 1
    for b in range(3):
        # NumPy adds 1 to the 256-bit counter (carrying across words) before each block
        c = (sum(int(v) << (64 * i) for i, v in enumerate(counter)) + 1 + b) % 2 ** 256
        ctr = tuple((c >> (64 * i)) & mask for i in range(4))
        assert O.philox4x64(ctr, key) == tuple(int(v) for v in raw[4 * b:4 * b + 4])


def test_normals_are_standard_normal_and_independent():
    z = np.array([[O.gate_normal(123, 4, t, e) for e in range(8)] for t in range(3000)])
    flat = z.ravel()
    assert abs(flat.mean()) < 0.03
    assert abs(flat.var() - 1.0) < 0.04
    assert abs(np.mean(np.abs(flat) < 1.0) - 0.6827) < 0.01
    assert abs(np.corrcoef(z[:, 0], z[:, 1])[0, 1]) < 0.05
    assert abs(np.corrcoef(z[:-1, 3], z[1:, 3])[0, 1]) < 0.05
    # seed and offset change the draws
    assert O.gate_normal(123, 4, 7, 2) != O.gate_normal(124, 4, 7, 2)
    assert O.gate_normal(123, 4, 7, 2) != O.gate_normal(123, 5, 7, 2)


def test_softplus_closed_forms():
    assert O.softplus(np.array([0.0]))[0] == pytest.approx(math.log(2.0), rel=1e-15)
    assert O.softplus(np.array([50.0]))[0] == pytest.approx(50.0, rel=1e-15)
    assert O.softplus(np.array([-50.0]))[0] == pytest.approx(math.exp(-50.0), rel=1e-12)
    assert np.isfinite(O.softplus(np.array([1000.0, -1000.0]))).all()


def test_zero_noise_weights_give_z_ln2():
    T, d, E = 20, 16, 6
    rng = np.random.default_rng(0)
    x = rng.standard_normal((T, d)).astype(np.float32)
    n = O.gate_noise(x, np.zeros((d, E), np.float32), "f32", seed=9, offset=1)
    ref = np.array([[O.gate_normal(9, 1, t, e) * math.log(2.0) for e in range(E)]
                    for t in range(T)]).astype(np.float32)
    assert np.array_equal(n, ref)


def test_token_base_draws_the_batch_noise():
    T, d, E = 30, 8, 4
    rng = np.random.default_rng(1)
    x = rng.standard_normal((T, d)).astype(np.float32)
    W = (rng.standard_normal((d, E)) / math.sqrt(d)).astype(np.float32)
    whole = O.gate_noise(x, W, "f32", seed=3, offset=0)
    part = O.gate_noise(x[12:], W, "f32", seed=3, offset=0, token_base=12)
    assert np.array_equal(part, whole[12:])

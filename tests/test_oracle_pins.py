"""The float64 oracle against what the pages and plain mathematics fix (CPU only)."""
import glob
import json
import os

import numpy as np
import pytest

from tests import oracle_pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin, oracle_mod):
    pin(oracle_mod)


@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(GOLDEN, "*.json"))),
                         ids=os.path.basename)
def test_golden(path, oracle_mod):
    g = json.load(open(path))
    s, i, f = g["shape"], g["inputs"], g["flags"]
    Bsz, L, Dm, N = s["batch"], s["seqlen"], s["dim"], s["dstate"]
    f32 = lambda k, shape: np.asarray(i[k], dtype=np.float32).reshape(shape)
    y, h = oracle_mod.scan(f32("x", (Bsz, L, Dm)), f32("dt", (Bsz, L, Dm)), f32("A", (Dm, N)),
                           f32("B", (Bsz, L, N)), f32("C", (Bsz, L, N)), D=f32("D", (Dm,)),
                           dt_bias=f32("dt_bias", (Dm,)),
                           h0=f32("h0", (Bsz, Dm, N)) if "h0" in i else None,
                           delta_softplus=f["delta_softplus"], exact_zoh=f["exact_zoh"])
    tol = g["tolerance"]
    np.testing.assert_allclose(y.reshape(-1), g["expected"]["y"], rtol=tol, atol=tol)
    np.testing.assert_allclose(h.reshape(-1), g["expected"]["h_last"], rtol=tol, atol=tol)


def test_threads_do_not_change_results(oracle_mod):
    rng = np.random.default_rng(0)
    Bsz, L, Dm, N = 3, 40, 7, 5
    x, dt, z = (rng.standard_normal((Bsz, L, Dm)).astype(np.float32) for _ in range(3))
    Bm, Cm = (rng.standard_normal((Bsz, L, N)).astype(np.float32) for _ in range(2))
    A = -rng.uniform(0.1, 2, (Dm, N)).astype(np.float32)
    y1, h1 = oracle_mod.scan(x, dt, A, Bm, Cm, z=z, nthreads=1)
    y4, h4 = oracle_mod.scan(x, dt, A, Bm, Cm, z=z, nthreads=4)
    assert np.array_equal(y1, y4) and np.array_equal(h1, h4)


def test_rejects_bad_arguments(oracle_mod):
    x = np.zeros((1, 4, 2), np.float32)
    with pytest.raises(ValueError):
        oracle_mod.scan(x, x, np.zeros((2, 3), np.float32), np.zeros((1, 4, 2), np.float32),
                        np.zeros((1, 4, 3), np.float32))

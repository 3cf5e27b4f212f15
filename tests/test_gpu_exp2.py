"""The prefill kernels' FMA-pipe exponential (exp2_fma2: Cody-Waite range
reduction to x = n + f with f in [-1/2, 1/2], a cubic minimax polynomial for
2^f, 2^n added to the exponent field), held to its stated bound against
2^x in fp64. The differential kernel evaluates a quarter of its
exponentials with it, so a regression there would otherwise only show as a
small loss of accuracy inside the attention parity bar."""
import numpy as np
import pytest
import torch

import differential_attention_swa_b200 as swa

pytestmark = pytest.mark.gpu

REL_BOUND = 1.02e-4  # on [-125, 8]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from differential_attention_swa_b200 import build

    build.build()
    swa.library()


def evaluate(x: np.ndarray) -> np.ndarray:
    y = swa.debug_exp2(torch.from_numpy(x.astype(np.float32)).cuda())
    assert swa.last_device_error() == swa.OK
    return y.cpu().numpy()


def test_relative_error_bound_on_the_kernel_range():
    # a dense sweep (about 2^22 points) plus every half-integer and its
    # float neighbours, where the range reduction switches n
    dense = np.linspace(-125.0, 8.0, 1 << 22, dtype=np.float64).astype(np.float32)
    half = (np.arange(-250, 17) * 0.5).astype(np.float32)
    edges = np.concatenate([half, np.nextafter(half, np.float32(-np.inf)), np.nextafter(half, np.float32(np.inf))])
    x = np.concatenate([dense, edges[(edges >= -125.0) & (edges <= 8.0)]])
    y = evaluate(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(y - want) / want
    assert np.isfinite(y).all()
    assert rel.max() <= REL_BOUND, f"max relative error {rel.max():.3e} at x = {x[rel.argmax()]!r}"
    # integers come out exact: f = 0 and the polynomial's constant term is 1
    ints = np.arange(-125, 9).astype(np.float32)
    assert np.array_equal(evaluate(ints).astype(np.float64), np.exp2(ints.astype(np.float64)))


def test_clamp_to_zero_and_no_nan_below_the_range():
    x = np.concatenate([np.linspace(-130.0, -127.0, 4097, dtype=np.float32),
                        np.array([-127.0, -128.0, -1e30, -np.inf, np.finfo(np.float32).min], dtype=np.float32)])
    y = evaluate(x)
    assert (y == 0.0).all(), f"nonzero output at x = {x[y != 0][:4]}"
    assert not np.signbit(y).any()


def test_between_the_clamp_and_the_bound_stays_tiny_and_finite():
    # [-127, -125]: results near the bottom of the normal range; the relative
    # bound does not hold there, but the error stays below 2^-125
    x = np.linspace(-127.0, -125.0, 8193, dtype=np.float32)
    y = evaluate(x).astype(np.float64)
    assert np.isfinite(y).all() and (y >= 0).all()
    assert np.abs(y - np.exp2(x.astype(np.float64))).max() <= 2.0 ** -125


def test_odd_length_and_pairs_agree():
    """The kernel works on pairs; an odd tail and either lane of a pair give
    the same value for the same input."""
    x = np.random.default_rng(3).uniform(-40, 8, 1001).astype(np.float32)
    y = evaluate(x)
    y_rev = evaluate(x[::-1].copy())[::-1]
    assert np.array_equal(y, y_rev)

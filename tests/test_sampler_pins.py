"""Pins of the sampler oracle against what the pages fix: the DDPM forward process
x_t = sqrt(abar_t) x0 + sqrt(1 - abar_t) eps ("Sora / DiT", training-objective bullet)
and the rectified-flow path x_t = t x1 + (1 - t) x0 ("GOKU", §2.3)."""
import numpy as np
import pytest

from oracle import sampler as SM

RNG = np.random.default_rng(7)
SHAPE = (2, 4, 6, 5)


def noisy(x0, eps, a):
    return np.sqrt(a) * x0 + np.sqrt(1.0 - a) * eps


@pytest.mark.parametrize("a,b", [(0.02, 0.3), (0.3, 0.31), (0.5, 0.9), (0.9, 0.5), (0.7, 1.0)])
def test_ddim_step_lands_on_the_forward_process_point(a, b):
    x0, eps = RNG.standard_normal(SHAPE), RNG.standard_normal(SHAPE)
    got = SM.ddim_step(noisy(x0, eps, a), eps, a, b)
    assert np.allclose(got, noisy(x0, eps, b), rtol=1e-12, atol=1e-12)


def test_ddim_step_special_levels():
    x0, eps = RNG.standard_normal(SHAPE), RNG.standard_normal(SHAPE)
    xt = noisy(x0, eps, 0.25)
    assert np.allclose(SM.ddim_step(xt, eps, 0.25, 1.0), x0, rtol=0, atol=1e-13)      # abar = 1: clean
    assert np.allclose(SM.ddim_step(xt, eps, 0.25, 0.25), xt, rtol=0, atol=1e-13)     # same level: identity


@pytest.mark.parametrize("t,tn", [(0.0, 0.25), (0.1, 0.9), (0.6, 1.0), (0.8, 0.3)])
def test_euler_step_follows_the_straight_path(t, tn):
    x0, x1 = RNG.standard_normal(SHAPE), RNG.standard_normal(SHAPE)
    xt = t * x1 + (1.0 - t) * x0
    got = SM.euler_step(xt, x1 - x0, t, tn)          # the path's velocity is x1 - x0
    assert np.allclose(got, tn * x1 + (1.0 - tn) * x0, rtol=1e-12, atol=1e-12)


def test_step_reads_the_first_C_channels_of_a_learned_sigma_head():
    x = RNG.standard_normal(SHAPE)
    eps = RNG.standard_normal(SHAPE)
    out = np.concatenate([eps, 100.0 * RNG.standard_normal(SHAPE)], axis=1)   # [eps | Sigma]
    assert np.array_equal(SM.step(SM.DDIM, x, out, 0.4, 0.6), SM.ddim_step(x, eps, 0.4, 0.6))
    assert np.array_equal(SM.step(SM.EULER, x, out, 0.4, 0.6), SM.euler_step(x, eps, 0.4, 0.6))


def test_loop_with_an_exact_model_reaches_the_data():
    x0, eps = RNG.standard_normal(SHAPE), RNG.standard_normal(SHAPE)
    levels = [0.05, 0.2, 0.45, 0.8, 1.0]
    exact_eps = lambda x, t: eps                     # the noise that generated x_T
    got = SM.sample(SM.DDIM, exact_eps, noisy(x0, eps, levels[0]), [999, 750, 500, 250], levels)
    assert np.allclose(got, x0, rtol=0, atol=1e-12)
    x1 = RNG.standard_normal(SHAPE)
    times = [0.0, 0.3, 0.55, 1.0]
    got = SM.sample(SM.EULER, lambda x, t: x1 - x0, x0, times[:-1], times)
    assert np.allclose(got, x1, rtol=0, atol=1e-12)


def test_loop_feeds_the_scheduled_timestep_to_the_model():
    seen = []
    SM.sample(SM.EULER, lambda x, t: (seen.append(t), np.zeros_like(x))[1], np.zeros(SHAPE), [0.1, 0.5], [0.1, 0.5, 1.0])
    assert seen == [0.1, 0.5]


# planted mistakes: each plausible slip in the step must fail one of the pins above
def _pin_ddim(fn):
    x0, eps = RNG.standard_normal(SHAPE), RNG.standard_normal(SHAPE)
    return np.allclose(fn(noisy(x0, eps, 0.3), eps, 0.3, 0.7), noisy(x0, eps, 0.7), rtol=1e-9, atol=1e-9)


@pytest.mark.parametrize("bad", [
    lambda x, e, a, b: np.sqrt(1 - b) * ((x - np.sqrt(1 - a) * e) / np.sqrt(a)) + np.sqrt(b) * e,   # swapped roots
    lambda x, e, a, b: np.sqrt(b) * ((x - np.sqrt(a) * e) / np.sqrt(1 - a)) + np.sqrt(1 - b) * e,   # x0 from the wrong root
    lambda x, e, a, b: np.sqrt(b) * ((x - (1 - a) * e) / np.sqrt(a)) + np.sqrt(1 - b) * e,          # missing sqrt
    lambda x, e, a, b: np.sqrt(a) * ((x - np.sqrt(1 - b) * e) / np.sqrt(b)) + np.sqrt(1 - a) * e,   # levels swapped
])
def test_planted_ddim_mistakes_are_caught(bad):
    assert _pin_ddim(SM.ddim_step)
    assert not _pin_ddim(bad)


def test_planted_euler_mistake_is_caught():
    x0, x1 = RNG.standard_normal(SHAPE), RNG.standard_normal(SHAPE)
    xt = 0.3 * x1 + 0.7 * x0
    wrong = xt + (0.3 - 0.8) * (x1 - x0)                       # step direction reversed
    assert np.allclose(SM.euler_step(xt, x1 - x0, 0.3, 0.8), 0.8 * x1 + 0.2 * x0)
    assert not np.allclose(wrong, 0.8 * x1 + 0.2 * x0)

"""Oracle pins for the flow-matching elementwise step (SkyReels-V4 digest,
step 4): the endpoints and the midpoint of the interpolation, the target's
independence of t, and closed forms of the loss."""
import numpy as np

import oracle as O


def _r(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_flow_noise_endpoints_and_midpoint():
    z0, eps = _r((3, 5, 7), 1), _r((3, 5, 7), 2)
    zt, u = O.flow_noise(z0, eps, [1.0, 0.0, 0.5])
    assert np.array_equal(zt[0], z0[0])            # t = 1: the clean latent
    assert np.array_equal(zt[1], eps[1])           # t = 0: pure noise
    assert np.allclose(zt[2], 0.5 * (z0[2] + eps[2]))
    assert np.array_equal(u, z0 - eps)             # the target does not depend on t
    # z_t moves along u: d z_t / d t = z_0 - eps
    a, _ = O.flow_noise(z0, eps, [0.3, 0.3, 0.3])
    b, _ = O.flow_noise(z0, eps, [0.7, 0.7, 0.7])
    assert np.allclose((b - a) / 0.4, u)


def test_flow_loss_closed_forms():
    z0, eps = _r((2, 4, 6), 3), _r((2, 4, 6), 4)
    _, u = O.flow_noise(z0, eps, [0.2, 0.9])
    assert np.array_equal(O.flow_loss(u, z0, eps), np.zeros(2))   # perfect prediction
    c = np.array([0.5, -2.0]).reshape(2, 1, 1)
    # a constant offset c on every one of the 24 values: loss = 24 c^2
    assert np.allclose(O.flow_loss(u + c, z0, eps), 24 * c.ravel() ** 2)
    # predicting zero: the loss is the squared norm of the target
    assert np.allclose(O.flow_loss(np.zeros_like(u), z0, eps), (u.reshape(2, -1) ** 2).sum(1))

"""Pins of the optimizer oracle (oracle/optim.py) against mathematics and an
independent implementation, CPU only.

- Polar Express: one step with a tuple (a, b, c) must map every singular
  value s to a s + b s^3 + c s^5 and keep the singular vectors (checked
  against numpy's SVD, with the two tuples the page prints); the textbook
  cubic Newton-Schulz tuple (1.5, -0.5, 0) repeated converges to the polar
  factor U V^T; the result is invariant to a positive scale of the update and
  a wide update gives the transpose of the tall result.
- AdamW: agrees with torch.optim.AdamW (a separate implementation of the
  published algorithm) over several steps, and its first step without weight
  decay is lr * g / (|g| + eps) in closed form.
"""
import numpy as np
import pytest
import torch

from oracle import optim as oo

PAGE_TUPLES = [(8.156, -22.483, 15.879), (4.043, -2.809, 0.500)]


def _svd_map(G, a, b, c, eps=1e-7):
    X = G / (np.linalg.norm(G) + eps)
    U, s, Vt = np.linalg.svd(X, full_matrices=False)
    return U @ np.diag(a * s + b * s ** 3 + c * s ** 5) @ Vt


@pytest.mark.parametrize("shape", [(12, 7), (9, 9), (40, 16)])
@pytest.mark.parametrize("abc", PAGE_TUPLES)
def test_one_step_maps_singular_values_by_the_odd_polynomial(shape, abc):
    G = np.random.default_rng(1).standard_normal(shape)
    out = oo.polar_express(G, [abc])
    assert np.allclose(out, _svd_map(G, *abc), rtol=0, atol=1e-10)


def test_two_page_steps_compose():
    G = np.random.default_rng(2).standard_normal((20, 11))
    X = G / (np.linalg.norm(G) + 1e-7)
    U, s, Vt = np.linalg.svd(X, full_matrices=False)
    for a, b, c in PAGE_TUPLES:
        s = a * s + b * s ** 3 + c * s ** 5
    assert np.allclose(oo.polar_express(G, PAGE_TUPLES), U @ np.diag(s) @ Vt, atol=1e-9)
    # ns_steps selects the first tuples only
    assert np.allclose(oo.polar_express(G, PAGE_TUPLES, ns_steps=1), oo.polar_express(G, PAGE_TUPLES[:1]))


def test_cubic_newton_schulz_converges_to_polar_factor():
    G = np.random.default_rng(3).standard_normal((24, 10))
    U, _, Vt = np.linalg.svd(G, full_matrices=False)
    out = oo.polar_express(G, [(1.5, -0.5, 0.0)] * 60)
    assert np.allclose(out, U @ Vt, atol=1e-8)


def test_scale_invariance_and_wide_transpose():
    G = np.random.default_rng(4).standard_normal((8, 30))
    ref = oo.polar_express(G, PAGE_TUPLES)
    # exact up to the 1e-7 guard added to the norm, which the first steps amplify (a ~ 8)
    assert np.allclose(oo.polar_express(7.5 * G, PAGE_TUPLES), ref, atol=1e-7)
    assert np.allclose(oo.polar_express(G.T, PAGE_TUPLES), ref.T, atol=1e-12)
    assert ref.shape == G.shape


def test_adamw_matches_torch_over_steps():
    rng = np.random.default_rng(5)
    p0 = rng.standard_normal((6, 5))
    grads = [rng.standard_normal((6, 5)) for _ in range(5)]
    hp = dict(lr=3e-3, betas=(0.8, 0.95), eps=1e-10, weight_decay=0.1)
    tp = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([tp], **hp)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p, m, v = oo.adamw_step(p, g, m, v, t, hp["lr"], hp["betas"][0], hp["betas"][1], hp["eps"],
                                hp["weight_decay"])
    assert np.allclose(p, tp.detach().numpy(), rtol=1e-12, atol=1e-14)


def test_adamw_first_step_closed_form():
    g = np.array([3.0, -0.5, 2e-3, 0.0])
    p, m, v = oo.adamw_step(np.ones(4), g, np.zeros(4), np.zeros(4), 1, lr=0.01, eps=1e-8)
    assert np.allclose(p, 1.0 - 0.01 * g / (np.abs(g) + 1e-8), rtol=0, atol=1e-15)


def test_param_groups_follow_the_table():
    for name in ("wte", "w_lm", "ve_table", "smear_lambda", "backout_lambda", "resid_lambda", "x0_lambda"):
        assert oo.param_group(name) == "adamw"
    for name in ("w_qkv", "w_o", "w_fc", "w_proj", "w_ve_gate", "w_smear_gate"):
        assert oo.param_group(name) == "muon"

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


# ------------------------------------------------ Polar Express coefficients
def _chain_intervals(coeffs, lo=1e-3, hi=1.0, n=200001):
    """Image interval of [lo, hi] under each successive odd quintic."""
    out = []
    for a, b, c in coeffs:
        x = np.linspace(lo, hi, n)
        p = a * x + b * x ** 3 + c * x ** 5
        out.append((lo, hi, float(p.min()), float(p.max()), float(np.max(np.abs(1 - p)))))
        lo, hi = float(p.min()), float(p.max())
    return out


def _minimax_error(lo, hi, iters=80):
    """Smallest max|1 - p| over odd quintics p on [lo, hi] (Remez exchange on the
    four alternation points lo < x2 < x3 < hi), an independent computation."""
    xs = np.array([lo, lo + (hi - lo) / 3, lo + 2 * (hi - lo) / 3, hi])
    sg = np.array([-1.0, 1.0, -1.0, 1.0])
    E = None
    for _ in range(iters):
        a, b, c, E = np.linalg.solve(np.stack([xs, xs ** 3, xs ** 5, -sg], 1), np.ones(4))
        r = np.roots([5 * c, 0, 3 * b, 0, a])
        r = np.sort(np.real(r[(np.abs(np.imag(r)) < 1e-12) & (np.real(r) > lo) & (np.real(r) < hi)]))
        if len(r) != 2:
            break
        xs = np.array([lo, r[0], r[1], hi])
    return abs(E)


def test_coefficients_start_with_the_printed_tuples():
    for got, printed in zip(oo.POLAR_EXPRESS_COEFFS[:2], PAGE_TUPLES):
        assert np.allclose(got, printed, rtol=0, atol=1e-3)
    assert len(oo.POLAR_EXPRESS_COEFFS) == 5  # "5 itérations"


def test_coefficients_follow_the_greedy_minimax_construction():
    # each tuple approximates 1 on the image interval of the previous steps
    # (starting from [1e-3, 1]) as well as the best odd quintic does, to 2 %
    # (the published tuples carry a small safety margin over the plain minimax),
    # so its image is centred on 1 (lo + hi = 2) and the error shrinks
    chain = _chain_intervals(oo.POLAR_EXPRESS_COEFFS)
    errs = []
    for lo, hi, plo, phi, err in chain:
        assert err <= 1.02 * _minimax_error(lo, hi)
        assert abs(plo + phi - 2.0) < 0.01
        errs.append(err)
    assert all(e1 < e0 for e0, e1 in zip(errs, errs[1:]))
    _, _, plo, phi, _ = chain[-1]
    assert 0.85 < plo and phi < 1.15        # five steps bring [1e-3, 1] near 1


# ------------------------------------------------------- Muon and NorMuon
def test_muon_nesterov_momentum_closed_form():
    g = np.random.default_rng(3).standard_normal((4, 3))
    u1, b1 = oo.muon_momentum(g, np.zeros_like(g), 0.9)
    assert np.allclose(b1, g) and np.allclose(u1, 1.9 * g)
    u2, b2 = oo.muon_momentum(g, b1, 0.9)
    assert np.allclose(b2, 1.9 * g) and np.allclose(u2, g + 0.9 * 1.9 * g)


def test_normuon_keeps_the_norm_and_equalises_rows():
    rng = np.random.default_rng(4)
    o = rng.standard_normal((6, 10)) * rng.uniform(0.1, 3.0, (6, 1))   # rows of unequal scale
    upd, v = oo.normuon_scale(o, np.zeros(6), beta2=0.0)
    assert np.isclose(np.linalg.norm(upd), np.linalg.norm(o), rtol=1e-12)
    assert np.allclose(v, np.mean(o * o, axis=1))
    rms = np.sqrt(np.mean(upd * upd, axis=1))          # beta2 = 0: every row gets the same RMS
    assert np.allclose(rms, rms[0], rtol=1e-12)
    # with history, rows are normalised by the EMA, not by the current step only
    upd2, v2 = oo.normuon_scale(o, np.full(6, 4.0), beta2=0.5)
    assert np.allclose(v2, 0.5 * 4.0 + 0.5 * np.mean(o * o, axis=1))
    assert np.isclose(np.linalg.norm(upd2), np.linalg.norm(o), rtol=1e-12)
    assert np.allclose(upd2 / o, (upd2 / o)[:, :1])    # one scale per row


def test_muon_step_on_an_orthogonal_gradient():
    # a gradient with orthonormal columns times a scale: the normalised update
    # has every singular value 1/sqrt(k); the polynomial chain maps it to one
    # common value s_out, so the orthogonalised update is s_out * sqrt(k) * Q;
    # NorMuon with beta2 = 0 then gives every row the RMS of the whole update
    rng = np.random.default_rng(5)
    Q, _ = np.linalg.qr(rng.standard_normal((12, 4)))
    G = 3.0 * Q
    W = rng.standard_normal((12, 4))
    s = 0.5                                                 # 1/sqrt(4)
    for a, b, c in oo.POLAR_EXPRESS_COEFFS:
        s = a * s + b * s ** 3 + c * s ** 5
    O = s * Q                                               # polar factor scaled by the chain's value
    Wn, buf, v = oo.muon_step(W, G, np.zeros_like(G), np.zeros(12), lr=0.1, mu=0.0, beta2=0.0,
                              weight_decay=0.5)
    row = np.sqrt(np.mean(O * O, axis=1))
    expect = O / row[:, None] * np.linalg.norm(O) / np.sqrt(O.size)
    assert np.allclose(Wn, W * (1 - 0.1 * 0.5) - 0.1 * expect, rtol=0, atol=1e-6)
    assert np.allclose(buf, G)

"""Central finite differences in fp64 pin every hand-derived gradient of the
oracle (block and whole stack, fp64 and FP8-off).  CPU only."""
import numpy as np
import pytest

from oracle import model as om
from test_oracle_pins import tiny_cfg, tiny_weights

EPS = 1e-5


def _check(f, get, set_, analytic, rng, n=6, name=""):
    """Compare analytic grads with central differences at n random coordinates."""
    base = np.array(get(), dtype=np.float64)
    flat_an = np.asarray(analytic, dtype=np.float64).reshape(-1)
    scale = np.max(np.abs(flat_an)) + 1e-300
    coords = rng.choice(base.size, size=min(n, base.size), replace=False) if base.ndim else [None]
    for ci in coords:
        def at(delta):
            t = base.copy()
            if ci is None:
                t = base + delta
            else:
                t.reshape(-1)[ci] += delta
            set_(t)
            return f()
        fd = (at(EPS) - at(-EPS)) / (2 * EPS)
        set_(base)
        an = flat_an[0] if ci is None else flat_an[ci]
        assert abs(fd - an) <= 1e-6 * scale + 1e-7 * abs(an), (name, ci, fd, an, scale)


@pytest.mark.parametrize("layer", [0, 1, 2])
def test_block_gradients_fd(layer):
    rng = np.random.default_rng(11 + layer)
    c = tiny_cfg()
    w = tiny_weights(c, rng)
    lw = w["layers"][layer]
    x, x0, dy = (rng.standard_normal((2, 10, 32)) for _ in range(3))
    idx = rng.integers(0, c["vocab"], (2, 10))
    state = {"x": x, "x0": x0}

    def f():
        y, _ = om.block_forward(c, lw, state["x"], state["x0"], idx, layer)
        return float(np.sum(y * dy))

    _, cache = om.block_forward(c, lw, x, x0, idx, layer)
    dx, dx0, g = om.block_backward(c, lw, cache, dy, idx, layer)
    _check(f, lambda: state["x"], lambda t: state.__setitem__("x", t), dx, rng, name="x")
    _check(f, lambda: state["x0"], lambda t: state.__setitem__("x0", t), dx0, rng, name="x0")
    for name, gv in g.items():
        if name.startswith("_"):
            continue
        _check(f, lambda n=name: lw[n], lambda t, n=name: lw.__setitem__(n, t), gv, rng, name=name)


def test_stack_gradients_fd():
    rng = np.random.default_rng(5)
    c = tiny_cfg()
    w = tiny_weights(c, rng)
    idx = rng.integers(0, c["vocab"], (2, 10))
    tg = rng.integers(0, c["vocab"], (2, 10))

    def f():
        loss, _ = om.stack_forward(c, w, idx, tg)
        return loss

    _, cache = om.stack_forward(c, w, idx, tg)
    g = om.stack_backward(c, w, cache, idx)
    for name in ("wte", "w_lm", "w_smear_gate", "smear_lambda", "backout_lambda"):
        _check(f, lambda n=name: w[n], lambda t, n=name: w.__setitem__(n, t), g[name], rng, name=name)
    for i, lw in enumerate(w["layers"]):
        for name, gv in g["layers"][i].items():
            if name.startswith("_"):
                continue
            _check(f, lambda n=name, lw=lw: lw[n], lambda t, n=name, lw=lw: lw.__setitem__(n, t),
                   gv, rng, n=4, name=f"L{i}.{name}")


def test_stack_gradients_fd_backout_at_layer0_and_mha():
    rng = np.random.default_rng(9)
    c = tiny_cfg(n_kv_head=4, backout_layer=0, window=[-1, 1, -1], has_ve=[0, 1, 0])
    w = tiny_weights(c, rng)
    idx = rng.integers(0, c["vocab"], (2, 10))
    tg = rng.integers(0, c["vocab"], (2, 10))

    def f():
        return om.stack_forward(c, w, idx, tg)[0]

    _, cache = om.stack_forward(c, w, idx, tg)
    g = om.stack_backward(c, w, cache, idx)
    for name in ("wte", "backout_lambda", "smear_lambda"):
        _check(f, lambda n=name: w[n], lambda t, n=name: w.__setitem__(n, t), g[name], rng, name=name)
    lw = w["layers"][1]
    for name in ("w_qkv", "ve_table", "w_ve_gate", "x0_lambda"):
        _check(f, lambda n=name: lw[n], lambda t, n=name: lw.__setitem__(n, t),
               g["layers"][1][name], rng, name=name)

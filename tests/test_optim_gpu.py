"""Optimizer-step kernels through the C ABI against the fp64 oracle
(oracle/optim.py): AdamW (fp32, 1e-5) and the Polar Express
orthogonalisation on the tensor-core GEMM (bf16 operands and stores, 2e-2)."""
import numpy as np
import pytest
import torch

from helpers import TOL, relerr
from oracle import optim as oo

pytestmark = pytest.mark.gpu

PAGE_TUPLES = [(8.156, -22.483, 15.879), (4.043, -2.809, 0.500)]


@pytest.mark.parametrize("n", [4096, 4099, 1])
def test_adamw_step_matches_oracle(cuda_lib, n):
    gb = cuda_lib
    rng = np.random.default_rng(11)
    p0 = rng.standard_normal(n).astype(np.float32)
    hp = dict(lr=2e-3, beta1=0.8, beta2=0.95, eps=1e-10, weight_decay=0.05)
    p, m, v = (torch.tensor(x, device="cuda") for x in (p0, np.zeros(n, np.float32), np.zeros(n, np.float32)))
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    rp, rm, rv = p0.astype(np.float64), np.zeros(n), np.zeros(n)
    for t in range(1, 4):
        g = rng.standard_normal(n).astype(np.float32)
        gb.gptb_adamw_step(p, torch.tensor(g, device="cuda"), m, v, pb, n, hp["lr"], hp["beta1"], hp["beta2"],
                           hp["eps"], hp["weight_decay"], t)
        rp, rm, rv = oo.adamw_step(rp, g, rm, rv, t, hp["lr"], hp["beta1"], hp["beta2"], hp["eps"],
                                   hp["weight_decay"])
    torch.cuda.synchronize()
    assert relerr(p.double().cpu().numpy() - p0, rp - p0) <= TOL["f32"] * 10  # the update itself, to 1e-4
    assert relerr(p.double().cpu().numpy(), rp) <= TOL["f32"]
    assert relerr(m.double().cpu().numpy(), rm) <= TOL["f32"]
    assert relerr(v.double().cpu().numpy(), rv) <= TOL["f32"]
    # the bf16 copy is the round-to-nearest of the fp32 result
    assert torch.equal(pb, p.bfloat16())


@pytest.mark.parametrize("shape", [(256, 128), (192, 192), (128, 384), (1536, 6144)])
def test_polar_express_matches_oracle(cuda_lib, shape):
    gb = cuda_lib
    m, n = shape
    g = torch.Generator().manual_seed(5)
    G = (torch.randn(m, n, generator=g) * 0.02).bfloat16()
    out = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(gb.gptb_polar_express_workspace_bytes(m, n, len(PAGE_TUPLES)), dtype=torch.uint8,
                     device="cuda")
    gb.gptb_polar_express(G.cuda(), out, m, n, PAGE_TUPLES, ws)
    torch.cuda.synchronize()
    assert gb.gptb_device_error() == 0
    ref = oo.polar_express(G.double().numpy(), PAGE_TUPLES)
    # bf16 stores of X, A and B in each step: a float model of that rounding gives 6e-3 for these sizes
    assert relerr(out.double().cpu().numpy(), ref) <= TOL["bf16"]


def test_polar_express_single_step_singular_values(cuda_lib):
    """One step maps singular values by a s + b s^3 + c s^5 (property, any size)."""
    gb = cuda_lib
    m, n = 512, 256
    g = torch.Generator().manual_seed(9)
    G = (torch.randn(m, n, generator=g)).bfloat16()
    out = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(gb.gptb_polar_express_workspace_bytes(m, n, 1), dtype=torch.uint8, device="cuda")
    a, b, c = PAGE_TUPLES[1]
    gb.gptb_polar_express(G.cuda(), out, m, n, [(a, b, c)], ws)
    torch.cuda.synchronize()
    X = G.double().numpy()
    s = np.linalg.svd(X / np.linalg.norm(X), compute_uv=False)
    want = np.sort(np.abs(a * s + b * s ** 3 + c * s ** 5))[::-1]
    got = np.linalg.svd(out.double().cpu().numpy(), compute_uv=False)
    assert np.max(np.abs(got - want)) / want.max() <= TOL["bf16"]


@pytest.mark.parametrize("shape", [(256, 128), (128, 384), (768, 768)])
def test_muon_step_matches_oracle(cuda_lib, shape):
    """Two Muon steps (momentum, the five Polar Express tuples, NorMuon, decay)
    against oracle.optim.muon_step: the weight update, the momentum buffer and
    the second moment (bf16 orthogonalisation: 2e-2; fp32 momentum: 1e-5)."""
    gb = cuda_lib
    m, n = shape
    rng = np.random.default_rng(m + n)
    w0 = rng.standard_normal((m, n)).astype(np.float32) * 0.02
    hp = dict(lr=0.02, mu=0.95, beta2=0.95, weight_decay=0.1)
    w = torch.tensor(w0, device="cuda")
    buf = torch.zeros(m, n, device="cuda")
    v = torch.zeros(m, device="cuda")
    wb = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(gb.gptb_muon_workspace_bytes(m, n, 5), dtype=torch.uint8, device="cuda")
    rw, rbuf, rv = w0.astype(np.float64), np.zeros((m, n)), np.zeros(m)
    for _ in range(2):
        g = rng.standard_normal((m, n)).astype(np.float32)
        gb.gptb_muon_step(w, wb, torch.tensor(g, device="cuda"), buf, v, m, n, oo.POLAR_EXPRESS_COEFFS, hp["lr"],
                          hp["mu"], hp["beta2"], hp["weight_decay"], ws)
        rw, rbuf, rv = oo.muon_step(rw, g, rbuf, rv, hp["lr"], hp["mu"], hp["beta2"], hp["weight_decay"])
    torch.cuda.synchronize()
    assert gb.gptb_device_error() == 0
    got = w.double().cpu().numpy()
    assert relerr(got - w0, rw - w0) <= TOL["bf16"]
    assert relerr(buf.double().cpu().numpy(), rbuf) <= TOL["f32"]
    assert relerr(v.double().cpu().numpy(), rv) <= TOL["bf16"]
    assert torch.equal(wb, w.bfloat16())


def test_muon_step_rejects_bad_shapes(cuda_lib):
    gb = cuda_lib
    t = torch.zeros(64, device="cuda")
    with pytest.raises(gb.GPTBError) as e:
        gb.gptb_muon_step(t, None, t, t, t, 12, 8, oo.POLAR_EXPRESS_COEFFS, 0.1, 0.9, 0.9, 0.0, t)
    assert e.value.code == gb.ERR_INVALID_ARG


@pytest.mark.parametrize("shape,count", [((256, 128), 3), ((128, 384), 2), ((768, 768), 4)])
def test_muon_step_batched_matches_oracle(cuda_lib, shape, count):
    """gptb_muon_step_batched on `count` same-shape matrices (every Polar
    Express product one batched GEMM) against oracle.optim.muon_step per
    matrix, with the tolerances of the single-matrix test, and against
    gptb_muon_step on the same inputs (the same products in the same order per
    tile; only the float sums of the norms may add in another order)."""
    gb = cuda_lib
    m, n = shape
    rng = np.random.default_rng(7 * m + n + count)
    hp = dict(lr=0.02, mu=0.95, beta2=0.95, weight_decay=0.1)
    w0 = [rng.standard_normal((m, n)).astype(np.float32) * 0.02 for _ in range(count)]
    gs = [[rng.standard_normal((m, n)).astype(np.float32) for _ in range(count)] for _ in range(2)]
    ws = [torch.tensor(x, device="cuda") for x in w0]
    bufs = [torch.zeros(m, n, device="cuda") for _ in range(count)]
    vs = [torch.zeros(m, device="cuda") for _ in range(count)]
    wbs = [torch.empty(m, n, dtype=torch.bfloat16, device="cuda") for _ in range(count)]
    work = torch.empty(gb.gptb_muon_batched_workspace_bytes(count, m, n, 5), dtype=torch.uint8, device="cuda")
    # the same steps one matrix at a time
    ws1 = [torch.tensor(x, device="cuda") for x in w0]
    bufs1 = [torch.zeros(m, n, device="cuda") for _ in range(count)]
    vs1 = [torch.zeros(m, device="cuda") for _ in range(count)]
    work1 = torch.empty(gb.gptb_muon_workspace_bytes(m, n, 5), dtype=torch.uint8, device="cuda")
    for step in range(2):
        gt = [torch.tensor(x, device="cuda") for x in gs[step]]
        gb.gptb_muon_step_batched(ws, wbs, gt, bufs, vs, m, n, oo.POLAR_EXPRESS_COEFFS, hp["lr"], hp["mu"],
                                  hp["beta2"], hp["weight_decay"], work)
        for i in range(count):
            gb.gptb_muon_step(ws1[i], None, gt[i], bufs1[i], vs1[i], m, n, oo.POLAR_EXPRESS_COEFFS, hp["lr"],
                              hp["mu"], hp["beta2"], hp["weight_decay"], work1)
    torch.cuda.synchronize()
    assert gb.gptb_device_error() == 0
    for i in range(count):
        rw, rbuf, rv = w0[i].astype(np.float64), np.zeros((m, n)), np.zeros(m)
        for step in range(2):
            rw, rbuf, rv = oo.muon_step(rw, gs[step][i], rbuf, rv, hp["lr"], hp["mu"], hp["beta2"],
                                        hp["weight_decay"])
        got = ws[i].double().cpu().numpy()
        assert relerr(got - w0[i], rw - w0[i]) <= TOL["bf16"], i
        assert relerr(bufs[i].double().cpu().numpy(), rbuf) <= TOL["f32"], i
        assert relerr(vs[i].double().cpu().numpy(), rv) <= TOL["bf16"], i
        assert torch.equal(wbs[i], ws[i].bfloat16())
        one = ws1[i].double().cpu().numpy()
        assert relerr(got - w0[i], one - w0[i]) <= 1e-3, i


def test_muon_step_batched_rejects_bad_count(cuda_lib):
    gb = cuda_lib
    t = torch.zeros(64, 64, device="cuda")
    with pytest.raises(gb.GPTBError) as e:
        gb.gptb_muon_step_batched([t] * 65, [None] * 65, [t] * 65, [t] * 65, [t] * 65, 64, 64,
                                  oo.POLAR_EXPRESS_COEFFS, 0.1, 0.9, 0.9, 0.0, t)
    assert e.value.code == gb.ERR_INVALID_ARG

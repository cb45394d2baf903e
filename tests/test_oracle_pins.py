"""Pins for the fp64 oracle: closed forms, invariants, special cases and
independent torch CPU library routines.  CPU only.

Each check is chosen so that a plausible slip in the oracle (dropped term,
wrong sign, wrong index, transposed operand) fails at least one of them; the
planted-mistake tests at the bottom demonstrate that for a few such slips.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import model as om
from oracle import fp8 as of

RNG = np.random.default_rng(7)


def rnd(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


# ---------------------------------------------------------------- e4m3 -------

def test_e4m3_all_codes_are_fixed_points():
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    finite = codes[np.isfinite(codes)]
    assert finite.size == 254
    np.testing.assert_array_equal(of.e4m3_round(finite), finite)


def test_e4m3_midpoints_and_random_match_torch():
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    pos = np.unique(codes[np.isfinite(codes) & (codes >= 0)])
    mids = (pos[1:] + pos[:-1]) / 2                    # exact ties: round to even
    x = np.concatenate([mids, -mids, RNG.uniform(-460, 460, 20000),
                        RNG.standard_normal(20000) * 1e-2])
    ref = torch.from_numpy(x).float().to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(of.e4m3_round(x), ref)


def test_e4m3_saturates():
    np.testing.assert_array_equal(of.e4m3_round(np.array([470.0, 1e6, -500.0])),
                                  [448.0, 448.0, -448.0])


def test_fp8_matmul_exact_on_representable_operands():
    # operands already on the e4m3 grid with amax 448 have scale 1: exact product
    a = of.e4m3_round(RNG.uniform(-448, 448, (5, 7)))
    b = of.e4m3_round(RNG.uniform(-448, 448, (7, 3)))
    a[0, 0], b[0, 0] = 448.0, 448.0
    np.testing.assert_allclose(of.fp8_matmul(a, b), a @ b, rtol=0, atol=0)


def test_fp8_matmul_closed_forms_at_non_unit_scales():
    # 1x1: the single element is its own amax, so it maps to 448 exactly and back
    np.testing.assert_allclose(of.fp8_matmul(np.array([[3.0]]), np.array([[5.0]])), [[15.0]], rtol=2e-7)
    # 2x2 by hand: amax(a) = 2, scale 224; 0.3 * 224 = 67.2 lies between the e4m3
    # neighbours 64 and 72 (spacing 8 in [64, 128)) and rounds to 64, i.e. 2/7;
    # 1*224, 0.5*224 and 2*224 are on the grid.  b = [[1, 3], [2, 0.75]] has
    # amax 3, scale 448/3: 1 -> 149.33 -> 144 (spacing 16 in [128, 256)), i.e.
    # 144*3/448 = 27/28; 2 -> 298.67 -> 288, i.e. 27/14; 3 -> 448 exactly;
    # 0.75 -> 112 exactly.
    # (the scale 448/3 is not an fp32 value: the dequantised values carry its
    # fp32 rounding, a relative 2^-24 at most)
    a = np.array([[1.0, 0.3], [0.5, 2.0]])
    b = np.array([[1.0, 3.0], [2.0, 0.75]])
    qa = np.array([[1.0, 2.0 / 7.0], [0.5, 2.0]])
    qb = np.array([[27.0 / 28.0, 3.0], [27.0 / 14.0, 0.75]])
    np.testing.assert_allclose(of.fp8_matmul(a, b), qa @ qb, rtol=2e-7, atol=0)
    q, s = of.quantize_e4m3(a)
    assert s == 224.0
    np.testing.assert_array_equal(q, [[224.0, 64.0], [112.0, 448.0]])
    q, _ = of.quantize_e4m3(b)
    np.testing.assert_array_equal(q, [[144.0, 448.0], [288.0, 112.0]])


def test_fp8_matmul_power_of_two_scaling_is_exact():
    # scaling an operand by 2^k scales its amax by 2^k and its scale by 2^-k:
    # the codes are unchanged and the product scales by exactly 2^k
    a, b = rnd(6, 9), rnd(9, 4, scale=0.03)
    base = of.fp8_matmul(a, b)
    for k, m in ((3, 0), (-5, 2), (7, -9)):
        np.testing.assert_array_equal(of.fp8_matmul(a * 2.0 ** k, b * 2.0 ** m), base * 2.0 ** (k + m))


def test_fp8_matmul_error_bound_and_torch_casts():
    # per element: |fp8(a) fp8(b) - ab| <= sum_k |a||b| ((1+u)^2 - 1) + subnormal terms,
    # u = 2^-4 the unit roundoff of e4m3 (3 mantissa bits); codes below 2^-6 carry an
    # absolute error of at most 2^-10 before rescaling
    a, b = rnd(12, 40), rnd(40, 7, scale=5.0)
    a[3, 4] = 1e-5  # lands in the subnormal range after scaling
    sa, sb = 448.0 / np.max(np.abs(a)), 448.0 / np.max(np.abs(b))
    u = 2.0 ** -4
    ea = np.abs(a) * u + 2.0 ** -10 / sa
    eb = np.abs(b) * u + 2.0 ** -10 / sb
    bound = np.abs(a) @ eb + ea @ np.abs(b) + ea @ eb
    err = np.abs(of.fp8_matmul(a, b) - a @ b)
    assert np.all(err <= bound * (1 + 1e-6))
    # the same product from torch's own e4m3 casts of the scaled fp32 operands
    np.testing.assert_allclose(of.fp8_matmul(a, b), _torch_fp8_product(a, b, torch.float8_e4m3fn, 448.0),
                               rtol=1e-13, atol=0)


def _fp32_scale(t, qmax):
    """qmax / amax as one fp32 division (torch)."""
    return torch.tensor(qmax, dtype=torch.float32) / torch.from_numpy(np.asarray(t)).float().abs().max()


def _torch_fp8_product(a, b, a_dtype, a_qmax):
    """a @ b from torch's float8 casts of the fp32 products value * fp32 scale
    (a in a_dtype, b in e4m3), accumulated and rescaled in fp64."""
    sa, sb = _fp32_scale(a, a_qmax), _fp32_scale(b, 448.0)
    qa = (torch.from_numpy(a).float() * sa).to(a_dtype).double()
    qb = (torch.from_numpy(b).float() * sb).to(torch.float8_e4m3fn).double()
    return ((qa @ qb) / (float(sa) * float(sb))).numpy()


def test_bf16_round_matches_torch():
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    codes = bits.double().numpy()
    finite = codes[np.isfinite(codes)]
    np.testing.assert_array_equal(of.bf16_round(finite), finite)
    pos = np.unique(finite[finite > 0])
    mids = (pos[1:] + pos[:-1]) / 2                     # exact ties: round to even
    x = np.concatenate([mids, -mids, RNG.standard_normal(20000) * 3.0, RNG.standard_normal(2000) * 1e-39])
    ref = torch.from_numpy(x).float().to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(of.bf16_round(x), ref)
    assert np.isinf(of.bf16_round(np.array([3.4e38]))[0])


def test_fp8_block_product_quantises_bf16_tensors():
    # the FP8 product of the model acts on bf16 tensors: x = 0.265625 + 2^-12
    # rounds to 0.265625 in bf16 (spacing 2^-9 in [0.25, 0.5)); with amax 1.75
    # the scale is 256, so the bf16 value maps to 68, the e4m3 tie between 64
    # and 72, which goes to 64 (even).  Unrounded, 68.0625 would go to 72.
    a = np.array([[1.75, 0.265625 + 2.0 ** -12]])
    ones = np.array([[1.0], [1.0]])
    np.testing.assert_array_equal(om._mm(a, ones, True), [[1.75 + 64.0 / 256.0]])
    np.testing.assert_array_equal(of.fp8_matmul(a, ones), [[1.75 + 72.0 / 256.0]])


# ------------------------------------------------------------- RMSNorm -------

def test_rmsnorm_matches_torch_and_unit_rms():
    x = rnd(3, 5, 16)
    y, r = om.rmsnorm(x, 1e-6)
    ref = F.rms_norm(torch.from_numpy(x), (16,), eps=1e-6).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, -1)), 1.0, rtol=1e-5)


def test_rmsnorm_backward_matches_torch_autograd():
    x = torch.from_numpy(rnd(4, 16)).requires_grad_()
    dy = rnd(4, 16)
    F.rms_norm(x, (16,), eps=1e-6).backward(torch.from_numpy(dy))
    y, r = om.rmsnorm(x.detach().numpy(), 1e-6)
    np.testing.assert_allclose(om.rmsnorm_backward(dy, y, r), x.grad.numpy(), rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- RoPE -------

def test_rope_head_dim_2_is_textbook_rotation_by_t_radians():
    # hd=2: one pair, frequency base^0 = 1, so position t rotates by t radians
    T = 7
    cos, sin = om.rope_tables(T, 2, 10000.0)
    x = np.zeros((1, T, 1, 2))
    x[..., 0] = 1.0
    y = om.rope(x, cos, sin)
    t = np.arange(T)
    np.testing.assert_allclose(y[0, :, 0, 0], np.cos(t), atol=1e-15)
    np.testing.assert_allclose(y[0, :, 0, 1], np.sin(t), atol=1e-15)


def test_rope_frequencies_and_pairing():
    # pair j couples channels j and j + hd/2 and turns at base^(-2j/hd) rad/pos
    hd, T, base = 8, 5, 10000.0
    cos, sin = om.rope_tables(T, hd, base)
    for j in range(hd // 2):
        x = np.zeros((1, T, 1, hd))
        x[..., j] = 1.0
        y = om.rope(x, cos, sin)
        ang = np.arange(T) * base ** (-2.0 * j / hd)
        np.testing.assert_allclose(y[0, :, 0, j], np.cos(ang), atol=1e-15)
        np.testing.assert_allclose(y[0, :, 0, j + hd // 2], np.sin(ang), atol=1e-15)
        others = [i for i in range(hd) if i not in (j, j + hd // 2)]
        assert np.all(y[0, :, 0, others] == 0)


def test_rope_invariants():
    hd, T = 16, 9
    cos, sin = om.rope_tables(T, hd, 10000.0)
    x = rnd(2, T, 3, hd)
    y = om.rope(x, cos, sin)
    half = hd // 2
    np.testing.assert_allclose(x[..., :half] ** 2 + x[..., half:] ** 2,
                               y[..., :half] ** 2 + y[..., half:] ** 2, rtol=1e-12)
    np.testing.assert_allclose(y[:, 0], x[:, 0], atol=0)            # t = 0: identity
    # relative position: <R_t q, R_s k> depends only on t - s
    q, k = rnd(hd), rnd(hd)
    Q = om.rope(np.broadcast_to(q, (1, T, 1, hd)).copy(), cos, sin)[0, :, 0]
    K = om.rope(np.broadcast_to(k, (1, T, 1, hd)).copy(), cos, sin)[0, :, 0]
    np.testing.assert_allclose(Q[5] @ K[2], Q[3] @ K[0], rtol=1e-10)
    # backward is the inverse rotation
    np.testing.assert_allclose(om.rope_backward(y, cos, sin), x, atol=1e-12)


# ----------------------------------------------------------- attention -------

def _sdpa_ref(q, k, v, window):
    B, T, H, hd = q.shape
    G = H // k.shape[2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = j <= i
    if window >= 0:
        mask &= (i - j) <= window
    return qt, kt, vt, mask


@pytest.mark.parametrize("H,Hk,window", [(4, 4, -1), (4, 2, 3), (6, 2, 0), (4, 1, 5)])
def test_attention_matches_torch_sdpa(H, Hk, window):
    B, T, hd = 2, 11, 8
    q, k, v = rnd(B, T, H, hd), rnd(B, T, Hk, hd), rnd(B, T, Hk, hd)
    o, lse = om.attention_forward(q, k, v, window)
    qt, kt, vt, mask = _sdpa_ref(q, k, v, window)
    ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-12)
    s = (qt @ kt.transpose(-1, -2)) / math.sqrt(hd)
    lse_ref = torch.logsumexp(s.masked_fill(~mask, -float("inf")), dim=-1).numpy()
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12)


@pytest.mark.parametrize("H,Hk,window", [(4, 2, -1), (4, 2, 2), (3, 1, 4)])
def test_attention_backward_matches_torch_autograd(H, Hk, window):
    B, T, hd = 2, 9, 8
    q, k, v, do = rnd(B, T, H, hd), rnd(B, T, Hk, hd), rnd(B, T, Hk, hd), rnd(B, T, H, hd)
    qt = torch.from_numpy(q).requires_grad_()
    kt = torch.from_numpy(k).requires_grad_()
    vt = torch.from_numpy(v).requires_grad_()
    G = H // Hk
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = (j <= i) & (((i - j) <= window) if window >= 0 else torch.ones(T, T, dtype=torch.bool))
    out = F.scaled_dot_product_attention(
        qt.permute(0, 2, 1, 3), kt.permute(0, 2, 1, 3).repeat_interleave(G, 1),
        vt.permute(0, 2, 1, 3).repeat_interleave(G, 1), attn_mask=mask).permute(0, 2, 1, 3)
    out.backward(torch.from_numpy(do))
    dq, dk, dv = om.attention_backward(q, k, v, do, window)
    for a, b in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
        np.testing.assert_allclose(a, b.numpy(), rtol=1e-9, atol=1e-11)


def test_attention_invariants():
    B, T, H, hd = 1, 10, 2, 4
    q, k, v = rnd(B, T, H, hd), rnd(B, T, H, hd), rnd(B, T, H, hd)
    full, _ = om.attention_forward(q, k, v, -1)
    wide, _ = om.attention_forward(q, k, v, T - 1)                  # window >= T-1
    np.testing.assert_array_equal(full, wide)
    self_only, _ = om.attention_forward(q, k, v, 0)                 # W=0: o[t] = v[t]
    np.testing.assert_allclose(self_only, v, atol=1e-15)
    ones, _ = om.attention_forward(q, k, np.ones_like(v), 3)        # rows sum to one
    np.testing.assert_allclose(ones, 1.0, rtol=1e-14)
    # GQA with duplicated kv heads equals MHA on the repeated heads
    k1, v1 = rnd(B, T, 1, hd), rnd(B, T, 1, hd)
    gqa, _ = om.attention_forward(q, k1, v1, -1)
    mha, _ = om.attention_forward(q, np.repeat(k1, 2, 2), np.repeat(v1, 2, 2), -1)
    np.testing.assert_allclose(gqa, mha, atol=1e-15)


# ------------------------------------------------------------ lm head --------

def test_xent_closed_form_and_torch():
    n, d, V = 6, 4, 10
    loss, dh, dw = om.lm_head_xent(np.zeros((n, d)), rnd(V, d), RNG.integers(0, V, n))
    assert loss == pytest.approx(math.log(V), abs=1e-14)            # zero logits
    h, w, y = rnd(2, 3, d), rnd(V, d), RNG.integers(0, V, (2, 3))
    ht = torch.from_numpy(h).requires_grad_()
    wt = torch.from_numpy(w).requires_grad_()
    lt = F.cross_entropy((ht @ wt.T).reshape(-1, V), torch.from_numpy(y).reshape(-1).long())
    lt.backward()
    loss, dh, dw = om.lm_head_xent(h, w, y)
    assert loss == pytest.approx(lt.item(), rel=1e-13)
    np.testing.assert_allclose(dh, ht.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(dw, wt.grad.numpy(), rtol=1e-10, atol=1e-14)


# ------------------------------------------------------------- smear ---------

def test_smear_two_token_closed_form():
    # x[1] += lam * sigmoid(x[1,:C].w) * x[0];  x[0] unchanged
    x = np.array([[[1.0, 2.0, 3.0], [0.5, -1.0, 4.0]]])
    w = np.array([0.3, -0.2])
    lam = 0.7
    y, _ = om.smear_forward(x, w, lam)
    z = 0.5 * 0.3 + (-1.0) * (-0.2)
    gate = lam / (1 + math.exp(-z))
    np.testing.assert_allclose(y[0, 0], x[0, 0], atol=0)
    np.testing.assert_allclose(y[0, 1], x[0, 1] + gate * x[0, 0], rtol=1e-15)
    y0, _ = om.smear_forward(x, w, 0.0)                              # lambda 0: no-op
    np.testing.assert_array_equal(y0, x)


# ------------------------------------------------------------- block ---------

def tiny_cfg(**kw):
    c = dict(B=2, T=10, d=32, n_head=4, n_kv_head=2, head_dim=8, mlp_hidden=64,
             vocab=23, n_layer=3, window=[3, -1, 2], has_ve=[1, 0, 1], ve_gate_ch=5,
             smear_ch=4, backout_layer=1, rope_base=10000.0, norm_eps=1e-6,
             dtype="f64", lm_head=True)
    c.update(kw)
    return c


def tiny_weights(c, rng=None, scale=0.3):
    rng = rng or np.random.default_rng(3)
    d, H, Hk, hd, Fh, V = c["d"], c["n_head"], c["n_kv_head"], c["head_dim"], c["mlp_hidden"], c["vocab"]
    w = {"layers": []}
    for i in range(c["n_layer"]):
        lw = dict(w_qkv=rng.standard_normal(((H + 2 * Hk) * hd, d)) * scale,
                  w_o=rng.standard_normal((d, H * hd)) * scale,
                  w_fc=rng.standard_normal((Fh, d)) * scale,
                  w_proj=rng.standard_normal((d, Fh)) * scale,
                  resid_lambda=rng.uniform(0.5, 1.5), x0_lambda=rng.uniform(-0.5, 0.5))
        if c["has_ve"][i]:
            lw["w_ve_gate"] = rng.standard_normal((Hk, c["ve_gate_ch"])) * 0.5
            lw["ve_table"] = rng.standard_normal((V, Hk * hd))
        w["layers"].append(lw)
    w["wte"] = rng.standard_normal((V, d))
    w["w_lm"] = rng.standard_normal((V, d)) * scale
    w["w_smear_gate"] = rng.standard_normal(c["smear_ch"])
    w["smear_lambda"] = 0.6
    w["backout_lambda"] = 0.4
    return w


def torch_block(c, lw, x, x0, idx, layer):
    """Independent library-built block: F.rms_norm, F.linear, SDPA, torch.sigmoid."""
    B, T, d = x.shape
    H, Hk, hd = c["n_head"], c["n_kv_head"], c["head_dim"]
    eps = c["norm_eps"]
    xm = lw["resid_lambda"] * x + lw["x0_lambda"] * x0
    h = F.rms_norm(xm, (d,), eps=eps)
    qkv = F.linear(h, lw["w_qkv"])
    q, k, v = qkv.split([H * hd, Hk * hd, Hk * hd], dim=-1)
    q, k, v = q.view(B, T, H, hd), k.view(B, T, Hk, hd), v.view(B, T, Hk, hd)
    if c["has_ve"][layer]:
        ve = F.embedding(idx.long(), lw["ve_table"]).view(B, T, Hk, hd)
        gate = 3 * torch.sigmoid(F.linear(h[..., :c["ve_gate_ch"]], lw["w_ve_gate"]))
        v = v + gate.unsqueeze(-1) * ve
    q, k = F.rms_norm(q, (hd,), eps=eps), F.rms_norm(k, (hd,), eps=eps)
    # rotation of the split halves by +t * base^(-2j/hd), built from torch.polar
    j = torch.arange(hd // 2, dtype=torch.float64)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * c["rope_base"] ** (-2 * j / hd)
    rot = torch.polar(torch.ones_like(ang), ang)[None, :, None, :]

    def rope_t(t):
        zc = torch.complex(t[..., : hd // 2], t[..., hd // 2:]) * rot
        return torch.cat([zc.real, zc.imag], dim=-1)

    q, k = rope_t(q), rope_t(k)
    G = H // Hk
    i = torch.arange(T)[:, None]
    jj = torch.arange(T)[None, :]
    W = c["window"][layer]
    mask = (jj <= i) & (((i - jj) <= W) if W >= 0 else torch.ones(T, T, dtype=torch.bool))
    o = F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2).repeat_interleave(G, 1),
                                       v.transpose(1, 2).repeat_interleave(G, 1), attn_mask=mask)
    o = o.transpose(1, 2).reshape(B, T, H * hd)
    x1 = xm + F.linear(o, lw["w_o"])
    u = F.linear(F.rms_norm(x1, (d,), eps=eps), lw["w_fc"])
    return x1 + F.linear(F.relu(u).square(), lw["w_proj"])


def _tw(lw):
    out = {}
    for k_, v_ in lw.items():
        out[k_] = torch.tensor(v_, dtype=torch.float64, requires_grad=True) if np.ndim(v_) == 0 \
            else torch.from_numpy(np.array(v_)).requires_grad_()
    return out


@pytest.mark.parametrize("layer", [0, 1, 2])
def test_block_matches_torch_library_build(layer):
    c = tiny_cfg()
    w = tiny_weights(c)
    lw = w["layers"][layer]
    x, x0, dy = rnd(2, 10, 32), rnd(2, 10, 32), rnd(2, 10, 32)
    idx = RNG.integers(0, c["vocab"], (2, 10))
    y, cache = om.block_forward(c, lw, x, x0, idx, layer)
    dx, dx0, g = om.block_backward(c, lw, cache, dy, idx, layer)
    tl = _tw(lw)
    xt = torch.from_numpy(x).requires_grad_()
    x0t = torch.from_numpy(x0).requires_grad_()
    yt = torch_block(c, tl, xt, x0t, torch.from_numpy(idx), layer)
    np.testing.assert_allclose(y, yt.detach().numpy(), rtol=1e-10, atol=1e-10)
    yt.backward(torch.from_numpy(dy))
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-8, atol=1e-10)
    np.testing.assert_allclose(dx0, x0t.grad.numpy(), rtol=1e-8, atol=1e-10)
    for name, gv in g.items():
        if name.startswith("_"):
            continue
        np.testing.assert_allclose(gv, tl[name].grad.numpy(), rtol=1e-8, atol=1e-10, err_msg=name)


def test_block_special_cases():
    c = tiny_cfg()
    w = tiny_weights(c)
    x, x0 = rnd(2, 10, 32), rnd(2, 10, 32)
    idx = RNG.integers(0, c["vocab"], (2, 10))
    # lambdas (1, 0): the plain pre-norm block, independent of x0
    lw = dict(w["layers"][1], resid_lambda=1.0, x0_lambda=0.0)
    y1, _ = om.block_forward(c, lw, x, x0, idx, 1)
    y2, _ = om.block_forward(c, lw, x, rnd(2, 10, 32), idx, 1)
    np.testing.assert_array_equal(y1, y2)
    # VE gate with zero weights is exactly 3*sigmoid(0) = 1.5
    lw = dict(w["layers"][0], w_ve_gate=np.zeros_like(w["layers"][0]["w_ve_gate"]))
    _, cache = om.block_forward(c, lw, x, x0, idx, 0)
    np.testing.assert_array_equal(cache["gate"], 1.5)
    H, Hk, hd = 4, 2, 8
    qkv = cache["h"] @ lw["w_qkv"].T
    v_raw = qkv[..., (H + Hk) * hd:].reshape(2, 10, Hk, hd)
    np.testing.assert_allclose(cache["v"] - v_raw, 1.5 * cache["ve"], atol=1e-12)
    # an all-zero VE table leaves v (and the block) as a no-VE block
    lw = dict(w["layers"][0], ve_table=np.zeros_like(w["layers"][0]["ve_table"]))
    ya, _ = om.block_forward(c, lw, x, x0, idx, 0)
    yb, _ = om.block_forward(dict(c, has_ve=[0, 0, 1]), lw, x, x0, idx, 0)
    np.testing.assert_allclose(ya, yb, atol=1e-13)


def test_relu_squared_closed_form():
    c = tiny_cfg()
    w = tiny_weights(c)
    x, x0 = rnd(2, 10, 32), rnd(2, 10, 32)
    idx = RNG.integers(0, c["vocab"], (2, 10))
    _, cache = om.block_forward(c, w["layers"][1], x, x0, idx, 1)
    u = cache["u"]
    np.testing.assert_array_equal(cache["act"], np.where(u > 0, u * u, 0.0))


def test_stack_backout_and_smear_switches():
    c = tiny_cfg()
    w = tiny_weights(c)
    idx = RNG.integers(0, c["vocab"], (2, 10))
    tg = RNG.integers(0, c["vocab"], (2, 10))
    w0 = dict(w, backout_lambda=0.0)
    l_a, _ = om.stack_forward(c, w0, idx, tg)
    l_b, _ = om.stack_forward(dict(c, backout_layer=-1), w0, idx, tg)
    assert l_a == l_b
    w1 = dict(w, smear_lambda=0.0)
    l_c, _ = om.stack_forward(c, w1, idx, tg)
    l_d, _ = om.stack_forward(dict(c, smear_ch=0), w1, idx, tg)
    assert l_c == l_d


# ---------------------------------------------------------------- e5m2 -------
def test_e5m2_all_codes_are_fixed_points():
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).double().numpy()
    finite = codes[np.isfinite(codes)]
    np.testing.assert_array_equal(of.e5m2_round(finite), finite)


def test_e5m2_midpoints_and_random_match_torch():
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).double().numpy()
    grid = np.unique(codes[np.isfinite(codes)])
    mids = (grid[:-1] + grid[1:]) / 2.0              # exact ties: round half to even
    x = np.concatenate([mids, RNG.uniform(-57344, 57344, 20000), RNG.standard_normal(20000) * 1e-3])
    ref = torch.from_numpy(x).to(torch.float8_e5m2).double().numpy()
    np.testing.assert_array_equal(of.e5m2_round(x), ref)


def test_e5m2_saturates_and_mixed_matmul():
    np.testing.assert_array_equal(of.e5m2_round(np.array([60000.0, 1e9, -70000.0])),
                                  np.array([57344.0, 57344.0, -57344.0]))
    # operands on their grids with amax at the format maxima have scale 1: the product is exact
    g = of.e5m2_round(RNG.uniform(-57344, 57344, (4, 6)))
    g[0, 0] = 57344.0
    w = of.e4m3_round(RNG.uniform(-448, 448, (6, 3)))
    w[0, 0] = 448.0
    np.testing.assert_allclose(of.fp8_matmul_grad(g, w), g @ w, rtol=0, atol=0)


# ------------------------------------------------- FP8 variants (NEXT rows) --
def test_fp8_matmul_grad_at_non_unit_scales():
    # 1x1: each operand is its own amax and maps to the format maximum exactly
    np.testing.assert_allclose(of.fp8_matmul_grad(np.array([[0.3]]), np.array([[7.0]])), [[2.1]], rtol=2e-7)
    # exact power-of-two scaling, as for e4m3
    g, w = rnd(5, 8), rnd(8, 3, scale=0.1)
    base = of.fp8_matmul_grad(g, w)
    np.testing.assert_array_equal(of.fp8_matmul_grad(g * 2.0 ** -7, w * 8.0), base * 2.0 ** -4)
    # error bound: e5m2 has unit roundoff 2^-3, e4m3 2^-4 (subnormals absolute)
    sg, sw = 57344.0 / np.max(np.abs(g)), 448.0 / np.max(np.abs(w))
    eg = np.abs(g) * 2.0 ** -3 + 2.0 ** -17 / sg
    ew = np.abs(w) * 2.0 ** -4 + 2.0 ** -10 / sw
    bound = np.abs(g) @ ew + eg @ np.abs(w) + eg @ ew
    assert np.all(np.abs(base - g @ w) <= bound * (1 + 1e-6))
    # against torch's own e5m2 / e4m3 casts of the scaled fp32 operands
    np.testing.assert_allclose(base, _torch_fp8_product(g, w, torch.float8_e5m2, 57344.0), rtol=1e-13, atol=0)


def test_fp8_e5m2_mode_quantises_only_gradient_operands():
    # 0.65 with amax 1: e4m3 scale 448 -> 291.2 -> 288 (spacing 32 in [256, 512));
    # e5m2 scale 57344 -> 37273.6 -> 40960 (spacing 8192 in [32768, 65536))
    a = np.array([[1.0, 0.65]])
    ones = np.array([[1.0], [1.0]])
    np.testing.assert_allclose(om._mm(a, ones, True, grad=True), [[1.0 + 288.0 / 448.0]], rtol=1e-15)
    np.testing.assert_allclose(om._mm(a, ones, "e5m2", grad=True), [[1.0 + 40960.0 / 57344.0]], rtol=1e-15)
    np.testing.assert_allclose(om._mm(a, ones, "e5m2", grad=False), [[1.0 + 288.0 / 448.0]], rtol=1e-15)


@pytest.mark.parametrize("mode", [True, "e5m2"])
def test_fp8_lm_head_matches_torch_casts_and_bound(mode):
    rng = np.random.default_rng(21)
    n, d, V = 12, 16, 40
    h = of.bf16_round(rng.standard_normal((n, d)))
    w = of.bf16_round(rng.standard_normal((V, d)) * 0.3)
    y = rng.integers(0, V, n)
    loss, dh, dw = om.lm_head_xent(h, w, y, fp8=mode)
    # the same steps from torch: e4m3 casts of h and W with their amax scales,
    # fp64 softmax of the dequantised product, dz = (softmax - onehot)/n cast
    # to bf16 and then to the gradient format with the fixed scale qmax * n
    th, tw = torch.from_numpy(h).float(), torch.from_numpy(w).float()
    sh, sw = _fp32_scale(h, 448.0), _fp32_scale(w, 448.0)
    qh = (th * sh).to(torch.float8_e4m3fn).double()
    qw = (tw * sw).to(torch.float8_e4m3fn).double()
    z = (qh @ qw.T) / (float(sh) * float(sw))
    lse = torch.logsumexp(z, 1)
    assert abs(loss - float(torch.mean(lse - z[torch.arange(n), torch.from_numpy(y)]))) < 1e-12
    dz = torch.softmax(z, 1)
    dz[torch.arange(n), torch.from_numpy(y)] -= 1.0
    dz = (dz / n).to(torch.bfloat16).double()
    assert float(dz.abs().max()) <= 1.0 / n
    fdt, qmax = (torch.float8_e5m2, 57344.0) if mode == "e5m2" else (torch.float8_e4m3fn, 448.0)
    sdz = torch.tensor(qmax, dtype=torch.float32) / (torch.tensor(1.0, dtype=torch.float32) / n)  # fp32, 1/n bound
    qdz = (dz.float() * sdz).to(fdt).double()
    sdz, sh, sw = float(sdz), float(sh), float(sw)
    np.testing.assert_allclose(dh, ((qdz @ qw) / (sdz * sw)).numpy(), rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(dw, ((qdz.T @ qh) / (sdz * sh)).numpy(), rtol=1e-12, atol=1e-18)
    # and close to the exact head (FP8 rounding only)
    l0, dh0, dw0 = om.lm_head_xent(h, w, y)
    assert abs(loss - l0) < 0.05 * abs(l0)

"""fp64 reference of the GPT block stack, forward and hand-derived backward.

TEST INFRASTRUCTURE ONLY (see the package docstring for the sources [AP-*]
and the readings taken where the pages are silent).

Shapes: activations are [B, T, ...] row-major; weights follow nn.Linear,
[out, in], and every projection is y = x @ W^T (the Linear of [AP-lin]).
All arithmetic is float64.  ``fp8=True`` replaces every product of the four
block GEMMs (qkv, attention output, MLP fc, MLP proj) -- forward, input
gradient and weight gradient -- by its per-tensor e4m3 emulation from
``fp8.py``.  Reading of [AP-lin] ("most layers" become FP8 linears with
per-tensor scaling; the model's activations are bf16, the Linear casting its
weight to the activation dtype): an FP8 linear quantises the bf16 tensors it
is given, so each operand is first rounded to bf16 and then scaled by
448/amax and rounded to e4m3; the products accumulate exactly and are
rescaled.  The small gate linears stay exact.

Variants (NEXT rows of the same reading): ``fp8="e5m2"`` quantises the
gradient operand of the input-gradient and weight-gradient products to e5m2
(scale 57344/amax) instead of e4m3; a config with ``fp8_lm_head`` also runs
the lm_head products in FP8: the logits from e4m3 casts of hf and W_lm, and
the two gradient products from the logits gradient dz, whose entries
(softmax - onehot)/n lie in [-1/n, 1/n], quantised with the per-tensor
scale that bound fixes (448 n, or 57344 n for e5m2, formed in fp32 as
qmax / fp32(1/n)), so that splitting the rows into chunks does not change
the product.  Without ``fp8_lm_head`` the
lm_head stays exact.
"""
from __future__ import annotations

import numpy as np

from .fp8 import (E4M3_MAX, E5M2_MAX, bf16_round, bound_scale, fp8_matmul, fp8_matmul_grad, quantize_e4m3,
                  quantize_fixed)


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def _mm(a, b, fp8, grad=False):
    """Plain matrix product of 2-D operands.  FP8: the e4m3 product of the
    operands as bf16 tensors (each rounded to bf16, then quantised per
    tensor), accumulated exactly; with fp8 == "e5m2" a gradient operand a
    (grad=True) is quantised to e5m2 instead."""
    if not fp8:
        return a @ b
    if grad and fp8 == "e5m2":
        return fp8_matmul_grad(bf16_round(a), bf16_round(b))
    return fp8_matmul(bf16_round(a), bf16_round(b))


def _linear(x, w, fp8=False):
    """y = x @ w^T over the last axis of x ([AP-lin])."""
    lead = x.shape[:-1]
    y = _mm(x.reshape(-1, x.shape[-1]), w.T, fp8)
    return y.reshape(*lead, w.shape[0])


def _linear_dgrad(dy, w, fp8=False):
    """Input gradient of y = x @ w^T: dx = dy @ w."""
    lead = dy.shape[:-1]
    dx = _mm(dy.reshape(-1, dy.shape[-1]), w, fp8, grad=True)
    return dx.reshape(*lead, w.shape[1])


def _linear_wgrad(dy, x, fp8=False):
    """Weight gradient of y = x @ w^T: dw = dy^T @ x, summed over tokens."""
    return _mm(dy.reshape(-1, dy.shape[-1]).T, x.reshape(-1, x.shape[-1]), fp8, grad=True)


# ---------------------------------------------------------------------------
# RMSNorm (parameter-free; reading: pre-norm before attention, MLP, lm_head;
# the same norm over each head is the QK normalisation of [AP-feat])
# ---------------------------------------------------------------------------

def rmsnorm(x, eps):
    """y = x / sqrt(mean(x^2) + eps) over the last axis; returns (y, rstd)."""
    x = _f64(x)
    rstd = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * rstd, rstd


def rmsnorm_backward(dy, y, rstd):
    """dx for y = x*rstd(x):  dx = rstd * (dy - y * mean(dy * y))."""
    return rstd * (dy - y * np.mean(dy * y, axis=-1, keepdims=True))


# ---------------------------------------------------------------------------
# Rotary embedding ([AP-feat] "RoPE: relative positional encoding, no learned
# position embeddings").  Reading: split-half pairs (j, j + hd/2), angle
# t * base^(-2j/hd), positions 0..T-1 within each row, rotation by +angle.
# ---------------------------------------------------------------------------

def rope_tables(T, hd, base):
    j = np.arange(hd // 2, dtype=np.float64)
    inv_freq = base ** (-2.0 * j / hd)
    ang = np.arange(T, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang), np.sin(ang)


def rope(x, cos, sin):
    """Rotate x [B, T, heads, hd] pairwise by the per-position angles."""
    half = x.shape[-1] // 2
    c, s = cos[None, :, None, :], sin[None, :, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def rope_backward(dy, cos, sin):
    """Transpose (= inverse) rotation applied to the gradient."""
    half = dy.shape[-1] // 2
    c, s = cos[None, :, None, :], sin[None, :, None, :]
    d1, d2 = dy[..., :half], dy[..., half:]
    return np.concatenate([d1 * c + d2 * s, -d1 * s + d2 * c], axis=-1)


# ---------------------------------------------------------------------------
# Causal grouped-query attention with a sliding window ([AP-feat], [AP-fa]).
# Key j is visible from query t iff j <= t and (window < 0 or t - j <= window).
# ---------------------------------------------------------------------------

def visible_mask(T, window):
    t = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    m = j <= t
    if window is not None and window >= 0:
        m = m & ((t - j) <= window)
    return m


def attention_forward(q, k, v, window):
    """q [B,T,H,hd], k/v [B,T,Hkv,hd] -> o [B,T,H,hd], lse [B,H,T]."""
    B, T, H, hd = q.shape
    Hk = k.shape[2]
    G = H // Hk
    scale = 1.0 / np.sqrt(hd)
    mask = visible_mask(T, window)
    o = np.zeros((B, T, H, hd))
    lse = np.zeros((B, H, T))
    for b in range(B):
        for h in range(H):
            kv = h // G
            s = (q[b, :, h, :] @ k[b, :, kv, :].T) * scale
            s = np.where(mask, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            z = e.sum(axis=1, keepdims=True)
            o[b, :, h, :] = (e / z) @ v[b, :, kv, :]
            lse[b, h, :] = (m + np.log(z))[:, 0]
    return o, lse


def attention_backward(q, k, v, do, window):
    """Gradients of o = softmax(q k^T / sqrt(hd) + mask) v w.r.t. q, k, v."""
    B, T, H, hd = q.shape
    Hk = k.shape[2]
    G = H // Hk
    scale = 1.0 / np.sqrt(hd)
    mask = visible_mask(T, window)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            kv = h // G
            s = np.where(mask, (q[b, :, h, :] @ k[b, :, kv, :].T) * scale, -np.inf)
            e = np.exp(s - s.max(axis=1, keepdims=True))
            p = e / e.sum(axis=1, keepdims=True)
            dv[b, :, kv, :] += p.T @ do[b, :, h, :]
            dp = do[b, :, h, :] @ v[b, :, kv, :].T
            ds = p * (dp - np.sum(dp * p, axis=1, keepdims=True))
            dq[b, :, h, :] = (ds @ k[b, :, kv, :]) * scale
            dk[b, :, kv, :] += (ds.T @ q[b, :, h, :]) * scale
    return dq, dk, dv


# ---------------------------------------------------------------------------
# One transformer block
# ---------------------------------------------------------------------------

def block_forward(c, lw, x, x0, idx, layer, fp8=False):
    """One block: lambda mix, attention with QK-norm/RoPE/VE, ReLU^2 MLP.

    xm  = resid_lambda * x + x0_lambda * x0                      [AP-mix]
    h   = rmsnorm(xm);  q,k,v = split(h @ Wqkv^T)
    v  += 3*sigmoid(h[..., :C] @ Wg^T)[..., None] * VE[idx]     [AP-ve]
    q,k = rope(rmsnorm_per_head(q,k))                           [AP-feat]
    x1  = xm + attn(q,k,v) @ Wo^T
    x2  = x1 + relu(rmsnorm(x1) @ Wfc^T)^2 @ Wproj^T            [AP-feat]
    Returns (x2, cache).
    """
    B, T, d = x.shape
    H, Hk, hd, eps = c["n_head"], c["n_kv_head"], c["head_dim"], c["norm_eps"]
    x, x0 = _f64(x), _f64(x0)
    a, b = float(lw["resid_lambda"]), float(lw["x0_lambda"])
    xm = a * x + b * x0
    h, r1 = rmsnorm(xm, eps)
    qkv = _linear(h, _f64(lw["w_qkv"]), fp8)
    q = qkv[..., : H * hd].reshape(B, T, H, hd)
    k = qkv[..., H * hd:(H + Hk) * hd].reshape(B, T, Hk, hd)
    v = qkv[..., (H + Hk) * hd:].reshape(B, T, Hk, hd)
    cache = dict(x=x, x0=x0, xm=xm, h=h, r1=r1)
    if c["has_ve"][layer]:
        C = c["ve_gate_ch"]
        ve = _f64(lw["ve_table"])[np.asarray(idx)].reshape(B, T, Hk, hd)
        z = _linear(h[..., :C], _f64(lw["w_ve_gate"]))       # [B,T,Hk]
        sg = _sigmoid(z)
        gate = 3.0 * sg
        v = v + gate[..., None] * ve
        cache.update(ve=ve, sg=sg, gate=gate)
    qn, rq = rmsnorm(q, eps)
    kn, rk = rmsnorm(k, eps)
    cos, sin = rope_tables(T, hd, c["rope_base"])
    qr, kr = rope(qn, cos, sin), rope(kn, cos, sin)
    o, lse = attention_forward(qr, kr, v, c["window"][layer])
    o2 = o.reshape(B, T, H * hd)
    x1 = xm + _linear(o2, _f64(lw["w_o"]), fp8)
    h2, r2 = rmsnorm(x1, eps)
    u = _linear(h2, _f64(lw["w_fc"]), fp8)
    act = np.maximum(u, 0.0) ** 2
    x2 = x1 + _linear(act, _f64(lw["w_proj"]), fp8)
    cache.update(q=q, k=k, v=v, qn=qn, kn=kn, rq=rq, rk=rk, qr=qr, kr=kr,
                 o=o2, lse=lse, x1=x1, h2=h2, r2=r2, u=u, act=act, cos=cos, sin=sin)
    return x2, cache


def block_backward(c, lw, cache, dx2, idx, layer, fp8=False):
    """Backward of ``block_forward`` given dL/dx2.

    Returns (dx, dx0, grads) with grads keys w_qkv, w_o, w_fc, w_proj,
    resid_lambda, x0_lambda and, on value-embedding layers, w_ve_gate and
    ve_table (dense [V, Hkv*hd], the scatter-add of the per-token grads).
    """
    B, T, d = dx2.shape
    H, Hk, hd = c["n_head"], c["n_kv_head"], c["head_dim"]
    dx2 = _f64(dx2)
    g = {}
    # MLP
    g["w_proj"] = _linear_wgrad(dx2, cache["act"], fp8)
    dact = _linear_dgrad(dx2, _f64(lw["w_proj"]), fp8)
    du = dact * 2.0 * np.maximum(cache["u"], 0.0)
    g["w_fc"] = _linear_wgrad(du, cache["h2"], fp8)
    dh2 = _linear_dgrad(du, _f64(lw["w_fc"]), fp8)
    dx1 = dx2 + rmsnorm_backward(dh2, cache["h2"], cache["r2"])
    # attention output projection
    g["w_o"] = _linear_wgrad(dx1, cache["o"], fp8)
    do = _linear_dgrad(dx1, _f64(lw["w_o"]), fp8).reshape(B, T, H, hd)
    dxm = dx1.copy()
    dqr, dkr, dv = attention_backward(cache["qr"], cache["kr"], cache["v"], do,
                                      c["window"][layer])
    dqn = rope_backward(dqr, cache["cos"], cache["sin"])
    dkn = rope_backward(dkr, cache["cos"], cache["sin"])
    dq = rmsnorm_backward(dqn, cache["qn"], cache["rq"])
    dk = rmsnorm_backward(dkn, cache["kn"], cache["rk"])
    dh = np.zeros_like(cache["h"])
    if c["has_ve"][layer]:
        C = c["ve_gate_ch"]
        dgate = np.sum(dv * cache["ve"], axis=-1)                # [B,T,Hk]
        dve_tok = cache["gate"][..., None] * dv                  # [B,T,Hk,hd]
        sg = cache["sg"]
        dz = dgate * 3.0 * sg * (1.0 - sg)
        g["w_ve_gate"] = _linear_wgrad(dz, cache["h"][..., :C])
        dh[..., :C] += _linear_dgrad(dz, _f64(lw["w_ve_gate"]))
        V = np.asarray(lw["ve_table"]).shape[0]
        dtab = np.zeros((V, Hk * hd))
        np.add.at(dtab, np.asarray(idx).reshape(-1), dve_tok.reshape(-1, Hk * hd))
        g["ve_table"] = dtab
    dqkv = np.concatenate([dq.reshape(B, T, H * hd), dk.reshape(B, T, Hk * hd),
                           dv.reshape(B, T, Hk * hd)], axis=-1)
    g["w_qkv"] = _linear_wgrad(dqkv, cache["h"], fp8)
    dh = dh + _linear_dgrad(dqkv, _f64(lw["w_qkv"]), fp8)
    dxm = dxm + rmsnorm_backward(dh, cache["h"], cache["r1"])
    a, b = float(lw["resid_lambda"]), float(lw["x0_lambda"])
    g["resid_lambda"] = float(np.sum(dxm * cache["x"]))
    g["x0_lambda"] = float(np.sum(dxm * cache["x0"]))
    # conditioning of the two scalar sums: sum of |terms| (used to judge a
    # rounded evaluation of a cancelling sum; not a gradient)
    g["_scale"] = {"resid_lambda": float(np.sum(np.abs(dxm * cache["x"]))),
                   "x0_lambda": float(np.sum(np.abs(dxm * cache["x0"])))}
    return a * dxm, b * dxm, g


# ---------------------------------------------------------------------------
# Smear ([AP-smear]): x[t] += smear_lambda * sigmoid(x[t, :C] . w) * x[t-1]
# for t >= 1 (reading: "x_pre_smear" is the previous token's embedding).
# ---------------------------------------------------------------------------

def smear_forward(x, w_gate, lam):
    x = _f64(x)
    C = np.asarray(w_gate).shape[0]
    sg = _sigmoid(x[..., :C] @ _f64(w_gate))                     # [B,T]
    y = x.copy()
    y[:, 1:, :] += lam * sg[:, 1:, None] * x[:, :-1, :]
    return y, sg


def smear_backward(dy, x, sg, w_gate, lam):
    """Returns (dx, d w_gate, d lambda, sum of |terms| of d lambda)."""
    x = _f64(x)
    C = np.asarray(w_gate).shape[0]
    dx = dy.copy()
    dx[:, :-1, :] += lam * sg[:, 1:, None] * dy[:, 1:, :]
    s = np.zeros(sg.shape)
    s[:, 1:] = np.sum(dy[:, 1:, :] * x[:, :-1, :], axis=-1)     # dL/dgate_t / lam
    dlam = float(np.sum(sg * s))
    dz = lam * s * sg * (1.0 - sg)
    dw = np.einsum("bt,btc->c", dz, x[..., :C])
    dx[..., :C] += dz[..., None] * _f64(w_gate)[None, None, :]
    return dx, dw, dlam, float(np.sum(np.abs(sg[:, 1:, None] * dy[:, 1:, :] * x[:, :-1, :])))


# ---------------------------------------------------------------------------
# Untied lm_head + mean next-token cross-entropy ([AP-feat] untied weights,
# [JA-tok] vocabulary 32768).  Reading: mean over all B*T positions.
# ---------------------------------------------------------------------------

def lm_head_xent(h, w_lm, targets, fp8=False):
    """Returns (loss, dh, dw_lm) for loss = mean_t(logsumexp(z_t) - z_t[y_t]).
    fp8 (True or "e5m2"): the FP8 lm_head of the module docstring."""
    h = _f64(h)
    w = _f64(w_lm)
    hf = h.reshape(-1, h.shape[-1])
    y = np.asarray(targets).reshape(-1)
    z = _mm(hf, w.T, fp8)
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    zs = e.sum(axis=1, keepdims=True)
    lse = (m + np.log(zs))[:, 0]
    n = hf.shape[0]
    loss = float(np.mean(lse - z[np.arange(n), y]))
    dz = e / zs
    dz[np.arange(n), y] -= 1.0
    dz /= n
    if not fp8:
        return loss, (dz @ w).reshape(h.shape), dz.T @ hf
    # |dz| <= 1/n fixes the per-tensor scale of the logits gradient
    fmt = "e5m2" if fp8 == "e5m2" else "e4m3"
    s_dz = bound_scale(E5M2_MAX if fmt == "e5m2" else E4M3_MAX, n)
    qdz = quantize_fixed(bf16_round(dz), s_dz, fmt)
    qw, sw = quantize_e4m3(bf16_round(w))
    qh, sh = quantize_e4m3(bf16_round(hf))
    return loss, ((qdz @ qw) / (s_dz * sw)).reshape(h.shape), (qdz.T @ qh) / (s_dz * sh)


# ---------------------------------------------------------------------------
# Whole stack: embed -> smear -> L blocks (backout saved at its layer) ->
# backout -> final norm -> lm_head + CE
# ---------------------------------------------------------------------------

def stack_forward(c, w, idx, targets, fp8=False):
    idx = np.asarray(idx)
    L = c["n_layer"]
    emb = _f64(w["wte"])[idx]                                     # [B,T,d]
    cache = dict(emb=emb)
    if c["smear_ch"] > 0:
        x, sg = smear_forward(emb, w["w_smear_gate"], float(w["smear_lambda"]))
        cache["smear_sg"] = sg
    else:
        x = emb
    x0 = x
    blocks = []
    x_bo = None
    for i in range(L):
        if i == c["backout_layer"]:
            x_bo = x
        x, bc = block_forward(c, w["layers"][i], x, x0, idx, i, fp8)
        blocks.append(bc)
    if x_bo is not None:
        xf = x - float(w["backout_lambda"]) * x_bo
    else:
        xf = x
    hf, rf = rmsnorm(xf, c["norm_eps"])
    loss, dhf, dw_lm = lm_head_xent(hf, w["w_lm"], targets, fp8 if c.get("fp8_lm_head") else False)
    cache.update(x0=x0, blocks=blocks, x_bo=x_bo, xL=x, xf=xf, hf=hf, rf=rf,
                 dhf=dhf, dw_lm=dw_lm)
    return loss, cache


def stack_backward(c, w, cache, idx, fp8=False):
    """Gradients of the mean loss w.r.t. every parameter of the stack."""
    idx = np.asarray(idx)
    L = c["n_layer"]
    grads = {"w_lm": cache["dw_lm"], "layers": [None] * L, "_scale": {}}
    dxf = rmsnorm_backward(cache["dhf"], cache["hf"], cache["rf"])
    dx = dxf
    dx_bo = None
    if cache["x_bo"] is not None:
        lam = float(w["backout_lambda"])
        grads["backout_lambda"] = float(-np.sum(dxf * cache["x_bo"]))
        grads["_scale"]["backout_lambda"] = float(np.sum(np.abs(dxf * cache["x_bo"])))
        dx_bo = -lam * dxf
    dx0 = np.zeros_like(dx)
    for i in reversed(range(L)):
        dx, dx0_i, gi = block_backward(c, w["layers"][i], cache["blocks"][i], dx, idx, i, fp8)
        dx0 = dx0 + dx0_i
        if i == c["backout_layer"] and dx_bo is not None:
            dx = dx + dx_bo
        grads["layers"][i] = gi
    dxs = dx + dx0                     # x0 is the smeared embedding itself
    if c["smear_ch"] > 0:
        demb, dws, dlam, dlam_scale = smear_backward(dxs, cache["emb"], cache["smear_sg"],
                                                     w["w_smear_gate"], float(w["smear_lambda"]))
        grads["w_smear_gate"], grads["smear_lambda"] = dws, dlam
        grads["_scale"]["smear_lambda"] = dlam_scale
    else:
        demb = dxs
    V, d = np.asarray(w["wte"]).shape
    dwte = np.zeros((V, d))
    np.add.at(dwte, idx.reshape(-1), demb.reshape(-1, d))
    grads["wte"] = dwte
    return grads

"""Planted mistakes: each test swaps one oracle function for a version with a
plausible slip (wrong sign, dropped term, wrong index, wrong scale, wrong
operand) and checks that at least one of the pins in test_oracle_pins.py /
test_oracle_fd.py fails on it.  CPU only; nothing here touches the GPU."""
import numpy as np
import pytest

from oracle import model as om
import test_oracle_pins as pins
import test_oracle_fd as fd


def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_rope_rotation_sign_is_caught(monkeypatch):
    orig = om.rope
    monkeypatch.setattr(om, "rope", lambda x, c, s: orig(x, c, -s))
    _fails(pins.test_rope_head_dim_2_is_textbook_rotation_by_t_radians)
    _fails(pins.test_block_matches_torch_library_build, 0)


def test_rope_pairing_is_caught(monkeypatch):
    def interleaved(x, cos, sin):  # pairs (2j, 2j+1) instead of (j, j + hd/2)
        y = x.copy()
        c, s = cos[None, :, None, :], sin[None, :, None, :]
        x1, x2 = x[..., 0::2], x[..., 1::2]
        y[..., 0::2] = x1 * c - x2 * s
        y[..., 1::2] = x1 * s + x2 * c
        return y
    monkeypatch.setattr(om, "rope", interleaved)
    _fails(pins.test_rope_frequencies_and_pairing)


def test_rmsnorm_backward_dropped_term_is_caught(monkeypatch):
    monkeypatch.setattr(om, "rmsnorm_backward", lambda dy, y, r: r * dy)
    _fails(pins.test_rmsnorm_backward_matches_torch_autograd)
    _fails(fd.test_block_gradients_fd, 1)


def test_gqa_head_mapping_is_caught(monkeypatch):
    orig = om.attention_forward
    # kv head h % Hkv instead of h // (H / Hkv): permute the query heads' kv source
    def bad(q, k, v, window):
        H, Hk = q.shape[2], k.shape[2]
        G = H // Hk
        perm = [(h % Hk) * G + h // Hk for h in range(H)]
        o, lse = orig(q[:, :, perm], k, v, window)
        inv = np.argsort(perm)
        return o[:, :, inv], lse[:, inv]
    monkeypatch.setattr(om, "attention_forward", bad)
    _fails(pins.test_attention_matches_torch_sdpa, 4, 2, 3)


def test_softmax_scale_is_caught(monkeypatch):
    orig = om.attention_forward
    monkeypatch.setattr(om, "attention_forward", lambda q, k, v, w: orig(q / np.sqrt(q.shape[-1]), k, v, w))
    _fails(pins.test_attention_matches_torch_sdpa, 4, 4, -1)


def test_window_off_by_one_is_caught(monkeypatch):
    orig = om.visible_mask
    monkeypatch.setattr(om, "visible_mask", lambda T, w: orig(T, w - 1 if w is not None and w > 0 else w))
    _fails(pins.test_attention_matches_torch_sdpa, 4, 2, 3)


def test_smear_uses_current_token_is_caught(monkeypatch):
    def bad(x, w_gate, lam):
        x = np.asarray(x, dtype=np.float64)
        C = np.asarray(w_gate).shape[0]
        sg = 1.0 / (1.0 + np.exp(-(x[..., :C] @ np.asarray(w_gate, dtype=np.float64))))
        y = x.copy()
        y[:, 1:, :] += lam * sg[:, 1:, None] * x[:, 1:, :]   # current token instead of the previous one
        return y, sg
    monkeypatch.setattr(om, "smear_forward", bad)
    _fails(pins.test_smear_two_token_closed_form)


def test_lm_head_transposed_weight_gradient_is_caught(monkeypatch):
    orig = om.lm_head_xent
    def bad(h, w, y):
        loss, dh, dw = orig(h, w, y)
        return loss, dh, dw[::-1]          # rows of dW_lm attached to the wrong vocabulary entries
    monkeypatch.setattr(om, "lm_head_xent", bad)
    _fails(pins.test_xent_closed_form_and_torch)


def test_ve_gate_scale_is_caught(monkeypatch):
    orig = om._sigmoid
    monkeypatch.setattr(om, "_sigmoid", lambda z: 2.0 * orig(z) / 3.0)   # gate 2*sigmoid instead of 3*sigmoid
    _fails(pins.test_block_special_cases)


def test_fp8_inverted_scale_is_caught(monkeypatch):
    from oracle import fp8 as of

    def bad(a, b):  # multiplies by the scales instead of dividing by them
        qa, sa = of.quantize_e4m3(a)
        qb, sb = of.quantize_e4m3(b)
        return (qa @ qb) * (sa * sb)
    monkeypatch.setattr(of, "fp8_matmul", bad)
    _fails(pins.test_fp8_matmul_closed_forms_at_non_unit_scales)
    _fails(pins.test_fp8_matmul_error_bound_and_torch_casts)


def test_fp8_one_scale_for_both_operands_is_caught(monkeypatch):
    from oracle import fp8 as of

    def bad(a, b):  # b quantised with a's scale
        qa, sa = of.quantize_e4m3(a)
        qb = of.e4m3_round(np.asarray(b, dtype=np.float64) * sa)
        return (qa @ qb) / (sa * sa)
    monkeypatch.setattr(of, "fp8_matmul", bad)
    _fails(pins.test_fp8_matmul_closed_forms_at_non_unit_scales)


def test_fp8_missing_bf16_rounding_is_caught(monkeypatch):
    from oracle import fp8 as of
    monkeypatch.setattr(om, "_mm", lambda a, b, fp8: of.fp8_matmul(a, b) if fp8 else a @ b)
    _fails(pins.test_fp8_block_product_quantises_bf16_tensors)


# ----------------------------------------------------------- optimizer oracle
import numpy as np  # noqa: E402
from oracle import optim as oo  # noqa: E402
import test_oracle_optim as opins  # noqa: E402


def _pe_variant(kind):
    """polar_express with one slip: the roles of b and c swapped, or the a X
    term dropped (a read as 1)."""
    def pe(G, coeffs, ns_steps=None, eps=1e-7):
        X = np.asarray(G, dtype=np.float64)
        wide = X.shape[0] < X.shape[1]
        X = X.T if wide else X
        X = X / (np.linalg.norm(X) + eps)
        for a, b, c in list(coeffs)[: (len(coeffs) if ns_steps is None else ns_steps)]:
            A = X.T @ X
            if kind == "swap_bc":
                X = a * X + X @ (c * A + b * (A @ A))
            else:
                X = X + X @ (b * A + c * (A @ A))
        return X.T if wide else X
    return pe


@pytest.mark.parametrize("kind", ["swap_bc", "drop_a"])
def test_polar_express_slips_are_caught(monkeypatch, kind):
    monkeypatch.setattr(oo, "polar_express", _pe_variant(kind))
    _fails(opins.test_one_step_maps_singular_values_by_the_odd_polynomial, (12, 7), opins.PAGE_TUPLES[0])


def test_adamw_without_bias_correction_is_caught(monkeypatch):
    def bad(p, g, m, v, t, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0):
        m = beta1 * m + (1 - beta1) * g
        v = beta2 * v + (1 - beta2) * g * g
        return p * (1 - lr * weight_decay) - lr * m / (np.sqrt(v) + eps), m, v
    monkeypatch.setattr(oo, "adamw_step", bad)
    _fails(opins.test_adamw_matches_torch_over_steps)
    _fails(opins.test_adamw_first_step_closed_form)


def test_adamw_coupled_weight_decay_is_caught(monkeypatch):
    orig = oo.adamw_step
    def bad(p, g, m, v, t, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0):
        return orig(p, np.asarray(g) + weight_decay * np.asarray(p), m, v, t, lr, beta1, beta2, eps, 0.0)
    monkeypatch.setattr(oo, "adamw_step", bad)
    _fails(opins.test_adamw_matches_torch_over_steps)


def test_normuon_reduction_axis_is_caught(monkeypatch):
    def bad(o, v, beta2, eps=1e-10):  # per-column statistics instead of per-row (neuron)
        o = np.asarray(o, dtype=np.float64)
        v_mean = np.mean(o * o, axis=0)
        v_norm = np.sqrt(np.sum(v_mean))
        v = beta2 * np.resize(np.asarray(v, dtype=np.float64), v_mean.shape) + (1.0 - beta2) * v_mean
        step = 1.0 / np.sqrt(np.maximum(v, eps))
        new = np.sqrt(np.sum(v_mean * step ** 2))
        return o * (step * v_norm / max(new, eps))[None, :], v
    monkeypatch.setattr(oo, "normuon_scale", bad)
    with pytest.raises((AssertionError, ValueError)):  # wrong shapes or wrong values
        opins.test_normuon_keeps_the_norm_and_equalises_rows()


def test_muon_without_nesterov_is_caught(monkeypatch):
    def bad(g, buf, mu):
        buf = mu * np.asarray(buf, dtype=np.float64) + np.asarray(g, dtype=np.float64)
        return buf, buf
    monkeypatch.setattr(oo, "muon_momentum", bad)
    _fails(opins.test_muon_nesterov_momentum_closed_form)


def test_polar_express_coefficient_typo_is_caught(monkeypatch):
    bad = list(oo.POLAR_EXPRESS_COEFFS)
    a, b, c = bad[3]
    bad[3] = (a + 0.05, b, c)
    monkeypatch.setattr(oo, "POLAR_EXPRESS_COEFFS", bad)
    _fails(opins.test_coefficients_follow_the_greedy_minimax_construction)



def test_fp8_lm_head_dynamic_gradient_scale_is_caught(monkeypatch):
    from oracle import fp8 as of
    orig = of.quantize_fixed

    def dynamic(t, scale, fmt="e4m3"):  # the measured amax instead of the 1/n bound
        t = np.asarray(t, dtype=np.float64)
        qmax = 448.0 if fmt == "e4m3" else 57344.0
        return orig(t, qmax / np.max(np.abs(t)), fmt) * (scale / (qmax / np.max(np.abs(t))))
    monkeypatch.setattr(om, "quantize_fixed", dynamic)
    _fails(pins.test_fp8_lm_head_matches_torch_casts_and_bound, True)


def test_fp8_e5m2_on_the_weight_operand_is_caught(monkeypatch):
    from oracle import fp8 as of
    monkeypatch.setattr(om, "fp8_matmul_grad", lambda g, w: of.fp8_matmul_grad(w.T, g.T).T)
    _fails(pins.test_fp8_e5m2_mode_quantises_only_gradient_operands)

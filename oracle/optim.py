"""fp64 oracle for the optimizer step that follows the training step — TEST
INFRASTRUCTURE ONLY (same rules as the rest of ``oracle``: imported by tests,
never by the library; shares no code with the CUDA path).

Sources (page title and section):

  [AP-muon]  apidog.com/fr "Comment Entraîner Votre Propre ChatGPT Pour 50€ ?",
             § "Comment nanochat fonctionne" › 2. "L'optimiseur Muon": the
             Polar Express orthogonalisation loop (A = X^T X, B = bA + cA^2,
             X = aX + XB over the first ns_steps coefficient tuples) and the
             first two of its five coefficient tuples.
  [JA-opt]   dev.to/aakira "ChatGPTを50ドルでトレーニングする方法",
             § 2 "Muonオプティマイザー" table: AdamW for the embeddings, the
             lm_head and the scalar parameters; Muon for the 2-D matrices.

  [AP-norm]  same page, § 2 › NorMuon lines: v_mean = mean over red_dim of
             g^2, v_norm = sqrt of the sum of v_mean, final_scale =
             step_size * v_norm / max(v_norm_new, 1e-10), g = g * final_scale.

Published sources for what the pages leave out:
  [PE-paper] N. Amsel, D. Persson, C. Musco, R. M. Gower, "The Polar Express:
             Optimal Matrix Sign Methods and Their Application to the Muon
             Algorithm" (2025): the five coefficient tuples for a lower bound
             of 1e-3 on the normalised singular values; the pages print the
             first two (to three decimals) and elide the rest.
  [Muon]     K. Jordan et al., "Muon: An optimizer for hidden layers in neural
             networks" (2024): momentum buffer B = mu B + G and the Nesterov
             update G + mu B fed to the orthogonalisation.
  [NorMuon]  Z. Li et al., "NorMuon: Making Muon more efficient and scalable"
             (2025): a per-neuron second-moment EMA v = beta2 v + (1 - beta2)
             mean(O^2 over the neuron's inputs) of the orthogonalised update
             O, which is divided by sqrt(v) per neuron and rescaled to keep
             its norm.

Readings where the pages are silent (each is also listed in the design notes):
  - the iteration starts from the update divided by its Frobenius norm, so
    every singular value lies in (0, 1], the interval its odd polynomials are
    built for;
  - A = X^T X is the Gram matrix of the smaller side: a wide update (more
    columns than rows) is transposed before the loop and back after it;
  - AdamW is the published algorithm with decoupled weight decay and bias
    correction (the pages name it and give no hyperparameters);
  - NorMuon: a neuron is a row of the weight W [out, in] (red_dim = the input
    dimension); [AP-norm]'s step_size is the per-row 1/sqrt(v) of [NorMuon]
    (v floored at 1e-10, as the printed clamp floors v_norm_new), and
    v_norm_new is v_norm measured on g * step_size, so g * final_scale has
    the Frobenius norm of g;
  - the Muon step applies W <- W (1 - lr wd) - lr * g * final_scale.
"""
import numpy as np

# [AP-muon] prints the first two tuples; [PE-paper] gives all five
POLAR_EXPRESS_COEFFS = [
    (8.156554524902461, -22.48329292557795, 15.878769915207462),
    (4.042929935166739, -2.808917465908714, 0.5000178451051316),
    (3.8916678022926607, -2.772484153217685, 0.5060648178503393),
    (3.285753657755655, -2.3681294933425376, 0.46449024233003106),
    (2.3465413258596377, -1.7097828382687081, 0.42323551169305323),
]


def polar_express(G, coeffs, ns_steps=None, eps=1e-7):
    """Orthogonalise a 2-D update by the [AP-muon] loop.

    Each step with tuple (a, b, c) replaces X by X (aI + bA + cA^2) with
    A = X^T X, i.e. maps every singular value s of X to a s + b s^3 + c s^5
    and keeps the singular vectors.
    """
    X = np.asarray(G, dtype=np.float64)
    if X.ndim != 2:
        raise ValueError("polar_express takes a 2-D matrix")
    wide = X.shape[0] < X.shape[1]
    if wide:
        X = X.T
    X = X / (np.linalg.norm(X) + eps)
    steps = list(coeffs)[: (len(coeffs) if ns_steps is None else ns_steps)]
    for a, b, c in steps:
        A = X.T @ X
        B = b * A + c * (A @ A)
        X = a * X + X @ B
    return X.T if wide else X


def adamw_step(p, g, m, v, t, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0):
    """One AdamW step (decoupled weight decay, bias-corrected moments) on
    parameter p with gradient g, moment buffers m, v and step count t >= 1.
    Returns the new (p, m, v); the inputs are not modified."""
    p = np.asarray(p, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m = beta1 * np.asarray(m, dtype=np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, dtype=np.float64) + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    p = p * (1.0 - lr * weight_decay) - lr * m_hat / (np.sqrt(v_hat) + eps)
    return p, m, v


def param_group(name):
    """[JA-opt]: which optimizer a parameter of the stack gets, by name."""
    if name in ("wte", "w_lm", "ve_table") or name.endswith("lambda"):
        return "adamw"  # embeddings, the lm_head, scalar parameters
    return "muon"       # the 2-D matrices (projections and gates)


def muon_momentum(g, buf, mu):
    """[Muon]: buf <- mu buf + g; returns (the Nesterov update g + mu buf, buf)."""
    buf = mu * np.asarray(buf, dtype=np.float64) + np.asarray(g, dtype=np.float64)
    return np.asarray(g, dtype=np.float64) + mu * buf, buf


def normuon_scale(o, v, beta2, eps=1e-10):
    """[AP-norm] with [NorMuon]'s second moment: per-row mean of o^2 (v_mean),
    its EMA v, per-row step_size = 1/sqrt(v), and the update o * final_scale
    whose Frobenius norm equals that of o.  Returns (update, new v)."""
    o = np.asarray(o, dtype=np.float64)
    v_mean = np.mean(o * o, axis=1)                        # red_dim = inputs of each neuron
    v_norm = np.sqrt(np.sum(v_mean))
    v = beta2 * np.asarray(v, dtype=np.float64) + (1.0 - beta2) * v_mean
    step_size = 1.0 / np.sqrt(np.maximum(v, eps))
    v_norm_new = np.sqrt(np.sum(v_mean * step_size ** 2))  # v_norm of o * step_size
    final_scale = step_size * (v_norm / max(v_norm_new, eps))
    return o * final_scale[:, None], v


def muon_step(W, G, buf, v, lr, mu=0.95, beta2=0.95, weight_decay=0.0, coeffs=None, ns_steps=5):
    """One Muon step on a 2-D weight W [out, in] with gradient G: momentum
    ([Muon], Nesterov), Polar Express orthogonalisation ([AP-muon] loop,
    [PE-paper] coefficients), NorMuon scaling ([AP-norm]), decoupled weight
    decay.  Returns (new W, new momentum buffer, new second moment v)."""
    u, buf = muon_momentum(G, buf, mu)
    o = polar_express(u, POLAR_EXPRESS_COEFFS if coeffs is None else coeffs, ns_steps)
    upd, v = normuon_scale(o, v, beta2)
    W = np.asarray(W, dtype=np.float64) * (1.0 - lr * weight_decay) - lr * upd
    return W, buf, v

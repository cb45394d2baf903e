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

Readings where the pages are silent (each is also listed in the design notes):
  - the iteration starts from the update divided by its Frobenius norm, so
    every singular value lies in (0, 1], the interval its odd polynomials are
    built for;
  - A = X^T X is the Gram matrix of the smaller side: a wide update (more
    columns than rows) is transposed before the loop and back after it;
  - AdamW is the published algorithm with decoupled weight decay and bias
    correction (the pages name it and give no hyperparameters).
Not covered here: the Muon momentum form and NorMuon's variance reduction
(the printed NorMuon lines use a quantity, v_norm_new, that the pages never
define), and the three elided Polar Express tuples; the coefficients are an
input of ``polar_express``.
"""
import numpy as np


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

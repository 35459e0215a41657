"""Plain fp64 CPU oracle for one Muon / DMuon optimizer step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or
executes this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it, to check
the CUDA library against a slow, obviously correct restatement of the method.
It shares no code, constants table or helper with the CUDA path.

Everything is computed in float64 with numpy; matrix products go through
``numpy.matmul`` (BLAS) and nothing is blocked, fused or reordered beyond what
each formula states.

Sources (page title, section):

* "DeepSpeed 現已支援 Muon Optimizer" (setupai.cc), section 技術深入:
  Muon orthogonalises the *momentum-based update* of each 2-D weight with
  Newton-Schulz iterations; it needs decoupled weight decay and a per-parameter
  update scale; RMS matching lets it reuse AdamW's learning rate and decay.
* DMuon release article (wjxwpt.net), section 2 "shape-adaptive execution
  stack", item 1: the NS iteration can be moved from the m x n space into the
  m x m Gram space (the sentence is cut off on the page; the recursion below
  is the plainest reading that keeps the result identical).
* DMuon release article (m.zaocj.com / wjxwpt.net): Newton-Schulz needs the
  whole weight matrix, and it is the dominant cost of the step.

The pages print no coefficient, epsilon, scale constant or momentum formula.
This oracle takes the library's documented conventions for them:

* Nesterov momentum in the SGD form  B' = mu*B + G,  U = G + mu*B'
  (``nesterov=False`` gives plain heavy-ball  U = B').
* X = U, or U^T when rows > cols, so the iteration runs on the wide side.
* X0 = X / (||X||_F + eps), eps = 1e-7 added to the norm.
* K quintic steps with fixed (a, b, c) = (3.4445, -4.7750, 2.0315):
  A = X X^T,  X <- a X + (b A + c A^2) X.
* O = X_K (transposed back), scale = 0.2 * sqrt(max(rows, cols)).
* W' = (1 - lr*wd) * W - lr * scale * O   (decay on the pre-update W).

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms (SVD of the input), special cases and hand-derived values.
"""
from __future__ import annotations

import math

import numpy as np

NS_A = 3.4445
NS_B = -4.7750
NS_C = 2.0315
NS_COEFFS = (NS_A, NS_B, NS_C)
DEFAULT_EPS = 1e-7
RMS_FACTOR = 0.2


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def nesterov_momentum(G, B, mu: float, nesterov: bool = True):
    """Momentum buffer update and the update direction it yields.

    Follows "DeepSpeed 現已支援 Muon Optimizer", 技術深入 (Muon acts on the
    momentum-based update).  The SGD-style Nesterov reading:
        B' = mu * B + G
        U  = G + mu * B'      (nesterov=True)
        U  = B'               (nesterov=False)
    Returns (B', U) in float64.
    """
    G = _f64(G)
    B = _f64(B)
    B_new = mu * B + G
    U = G + mu * B_new if nesterov else B_new
    return B_new, U


def frobenius_normalise(X, eps: float = DEFAULT_EPS):
    """X0 = X / (||X||_F + eps): puts every singular value at or below 1."""
    X = _f64(X)
    return X / (np.sqrt(np.sum(X * X)) + eps)


def newton_schulz_direct(X0, steps: int = 5, coeffs=NS_COEFFS):
    """Quintic Newton-Schulz in the m x n space (rows <= cols expected).

    For each of ``steps`` iterations:  A = X X^T,  Bp = b A + c A A,
    X <- a X + Bp X.  (The step both DMuon pages call the core of Muon.)
    """
    a, b, c = coeffs
    X = _f64(X0).copy()
    for _ in range(steps):
        A = X @ X.T
        Bp = b * A + c * (A @ A)
        X = a * X + Bp @ X
    return X


def newton_schulz_gram(X0, steps: int = 5, coeffs=NS_COEFFS):
    """Gram-space Newton-Schulz (DMuon release article, section 2, item 1).

    Writes the k-th iterate as X_k = Q_k X0 with an m x m matrix Q_k, so the
    loop only touches m x m matrices:
        G = X0 X0^T,  Q_0 = I
        A_k = Q_k G Q_k^T               (= X_k X_k^T)
        Q_{k+1} = (a I + b A_k + c A_k^2) Q_k
    and a single m x m x n product at the end:  X_K = Q_K X0.
    In exact arithmetic this equals ``newton_schulz_direct``.
    """
    a, b, c = coeffs
    X0 = _f64(X0)
    m = X0.shape[0]
    I = np.eye(m)
    G = X0 @ X0.T
    Q = I.copy()
    for _ in range(steps):
        A = Q @ G @ Q.T
        Q = (a * I + b * A + c * (A @ A)) @ Q
    return Q @ X0


def rms_scale(rows: int, cols: int) -> float:
    """Update scale 0.2 * sqrt(max(rows, cols)) that brings the update's RMS
    near AdamW's ("DeepSpeed 現已支援 Muon Optimizer", 技術深入: RMS matching)."""
    return RMS_FACTOR * math.sqrt(max(rows, cols))


def apply_update(W, O, lr: float, wd: float):
    """Decoupled weight decay and the parameter write:
        W' = (1 - lr*wd) * W - lr * 0.2 * sqrt(max(rows, cols)) * O
    ("DeepSpeed 現已支援 Muon Optimizer", 技術深入: decoupled decay and a
    per-parameter update scale)."""
    W = _f64(W)
    O = _f64(O)
    rows, cols = W.shape
    return (1.0 - lr * wd) * W - lr * rms_scale(rows, cols) * O


def muon_update(G, B, mu: float = 0.95, steps: int = 5, eps: float = DEFAULT_EPS,
                nesterov: bool = True, variant: str = "direct", coeffs=NS_COEFFS):
    """Momentum, orientation, normalisation and Newton-Schulz for one matrix.

    Returns (B', O) where O has the shape of G (transposed back when the
    iteration ran on G^T).
    """
    B_new, U = nesterov_momentum(G, B, mu, nesterov)
    transposed = U.shape[0] > U.shape[1]
    X = U.T if transposed else U
    X0 = frobenius_normalise(X, eps)
    if variant == "direct":
        XK = newton_schulz_direct(X0, steps, coeffs)
    elif variant == "gram":
        XK = newton_schulz_gram(X0, steps, coeffs)
    else:
        raise ValueError(f"unknown variant {variant!r}")
    O = XK.T if transposed else XK
    return B_new, O


def muon_step(W, G, B, lr: float = 0.02, wd: float = 0.1, mu: float = 0.95,
              steps: int = 5, eps: float = DEFAULT_EPS, nesterov: bool = True,
              variant: str = "direct", coeffs=NS_COEFFS):
    """One full Muon step for one 2-D weight.  Returns (W', B', O), float64."""
    B_new, O = muon_update(G, B, mu, steps, eps, nesterov, variant, coeffs)
    W_new = apply_update(W, O, lr, wd)
    return W_new, B_new, O

"""Plain fp64 CPU oracle for the AdamW step of the non-matrix parameters.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or
executes this module: only ``tests/`` and ``bench.py``'s CPU-baseline leg use
it.  It shares no code, constant or helper with the CUDA path.

Source (page title, section): "DeepSpeed 現已支援 Muon Optimizer"
(setupai.cc), section 技術深入: Muon is used for the matrix parameters (2-D
weights, and convolution filters once flattened); training mixes it with
AdamW for the parameters that are not matrices, such as embeddings, biases
and the final classification layer.

The pages print no AdamW formula.  This oracle restates the published AdamW
algorithm (Adam with decoupled weight decay) with bias correction, in the
convention the major frameworks use:

    m_t  = beta1 * m_{t-1} + (1 - beta1) * g
    v_t  = beta2 * v_{t-1} + (1 - beta2) * g^2
    mhat = m_t / (1 - beta1^t),   vhat = v_t / (1 - beta2^t)
    p_t  = (1 - lr*wd) * p_{t-1} - lr * mhat / (sqrt(vhat) + eps)

t counts steps from 1; the decay multiplies the pre-update parameter, and eps
is added to sqrt(vhat).  Everything is float64 and elementwise; nothing is
fused or reordered beyond the formulas.  Pinned by
``tests/test_oracle_adamw.py`` against closed forms and special cases.
"""
from __future__ import annotations

import numpy as np


def adamw_moments(g, m, v, beta1: float, beta2: float):
    """First and second moment updates (elementwise, fp64)."""
    g = np.asarray(g, np.float64)
    m_new = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v_new = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    return m_new, v_new


def adamw_direction(m, v, beta1: float, beta2: float, step: int, eps: float):
    """Bias-corrected step direction mhat / (sqrt(vhat) + eps) at step t >= 1."""
    if step < 1:
        raise ValueError("step counts from 1")
    mhat = np.asarray(m, np.float64) / (1.0 - beta1 ** step)
    vhat = np.asarray(v, np.float64) / (1.0 - beta2 ** step)
    return mhat / (np.sqrt(vhat) + eps)


def adamw_step(p, g, m, v, lr: float, beta1: float, beta2: float, eps: float, wd: float, step: int):
    """One AdamW step; returns (p', m', v') in fp64."""
    m_new, v_new = adamw_moments(g, m, v, beta1, beta2)
    d = adamw_direction(m_new, v_new, beta1, beta2, step, eps)
    p_new = (1.0 - lr * wd) * np.asarray(p, np.float64) - lr * d
    return p_new, m_new, v_new

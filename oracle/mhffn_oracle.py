"""fp64 CPU oracle for FlashFFN's multi-head feed-forward block.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library.

Source: "FlashFFN: Multi-Head Decomposition Enables I/O-Aware Feed-Forward
Networks", section "Overview".  Per head h the block computes

    O_h = sum_e R_e * ((SiLU(Q K_e^T) (.) (Q U_e^T)) V_e)

where Q is the head's RMS-normalised projection of the input and R_e are
sigmoid-normalised router weights; the model configuration table fixes
d_h = 128 and the number E of sub-networks per head, and its "intermediate
size" is the head's total sub-network width E * d_e.

Readings where the page is silent (each one is also listed in the design
notes):

* shapes: Q [T, H, d_h]; K_e, U_e, V_e [d_e, d_h] per head and sub-network,
  stacked as [H, E, d_e, d_h]; R [T, H, E]; O [T, H, d_h].  ``Q K_e^T`` is
  Q times the transpose of K_e, as in attention; ``(...) V_e`` multiplies the
  [T, d_e] activation by V_e, so V_e maps the sub-network width back to d_h.
* R_e multiplies the sub-network's whole output, so it can be applied to the
  [T, d_e] activation before V_e (the same product).
* "RMS-normalised": z / sqrt(mean(z^2) + eps) over the head's d_h entries,
  times an optional per-entry gain.
* "sigmoid-normalised router weights": sigmoid of the router logits divided
  by their sum over the head's E sub-networks.

Parity status: pinned by ``tests/test_oracle_pins.py`` (reduction to the
dense SwiGLU oracle, additivity over sub-networks and heads, an independent
float64 torch autograd for the backward, central finite differences).
"""
from __future__ import annotations

import numpy as np

from .swiglu_oracle import silu, silu_prime

__all__ = ["mhffn_forward", "mhffn_backward", "head_rmsnorm", "router_weights",
           "mhffn_prologue_forward", "mhffn_prologue_backward"]


def _f64(a):
    if hasattr(a, "detach"):
        a = a.detach().cpu().float().numpy()
    return np.asarray(a, dtype=np.float64)


def mhffn_forward(q, k, u, v, r):
    """Multi-head FFN forward ("Overview" formula).  q [T,H,dh]; k, u, v
    [H,E,de,dh]; r [T,H,E].  Returns o [T,H,dh] and the per-sub-network
    gate and up pre-activations g, up [T,H,E,de] (for the backward)."""
    q, k, u, v, r = (_f64(a) for a in (q, k, u, v, r))
    g = np.einsum("thd,hefd->thef", q, k)      # Q K_e^T
    up = np.einsum("thd,hefd->thef", q, u)     # Q U_e^T
    act = silu(g) * up                         # SiLU(Q K_e^T) (.) (Q U_e^T)
    o = np.einsum("thef,hefd->thd", act * r[..., None], v)   # sum_e R_e (.) V_e
    return {"o": o, "g": g, "up": up}


def mhffn_backward(q, k, u, v, r, do):
    """Gradients of L = sum(do * o) with respect to q, k, u, v and r, by the
    chain rule through the forward's definition."""
    q, k, u, v, r, do = (_f64(a) for a in (q, k, u, v, r, do))
    fw = mhffn_forward(q, k, u, v, r)
    g, up = fw["g"], fw["up"]
    s = silu(g)
    dact_r = np.einsum("thd,hefd->thef", do, v)          # dL/d(R_e * act)
    dr = np.einsum("thef,thef->the", dact_r, s * up)     # act summed over d_e
    dact = dact_r * r[..., None]
    dg = dact * up * silu_prime(g)
    dup = dact * s
    dq = np.einsum("thef,hefd->thd", dg, k) + np.einsum("thef,hefd->thd", dup, u)
    dk = np.einsum("thef,thd->hefd", dg, q)
    du = np.einsum("thef,thd->hefd", dup, q)
    dv = np.einsum("thef,thd->hefd", s * up * r[..., None], do)
    return {"dq": dq, "dk": dk, "du": du, "dv": dv, "dr": dr}


def head_rmsnorm(z, num_heads, eps=1e-6, weight=None):
    """Per-head RMS normalisation of a [T, H*dh] projection: each head's dh
    entries divided by sqrt(mean of their squares + eps), times an optional
    [dh] gain.  Returns [T, H, dh]."""
    z = _f64(z)
    T = z.shape[0]
    zh = z.reshape(T, num_heads, -1)
    out = zh / np.sqrt(np.mean(zh * zh, axis=-1, keepdims=True) + eps)
    if weight is not None:
        out = out * _f64(weight)
    return out


def router_weights(logits):
    """Sigmoid-normalised router weights: sigmoid(logits) / sum over the E
    sub-networks of each head.  logits [T, H, E]."""
    s = 1.0 / (1.0 + np.exp(-_f64(logits)))
    return s / np.sum(s, axis=-1, keepdims=True)


def mhffn_prologue_forward(x, w_q, w_r, num_heads, num_sub, gain=None, eps=1e-6):
    """The block's prologue: q = head_rmsnorm(x w_q^T) [T, H, dh] and router weights
    r = router_weights((x w_r^T) as [T, H, E])."""
    x, w_q, w_r = _f64(x), _f64(w_q), _f64(w_r)
    T = x.shape[0]
    q = head_rmsnorm(x @ w_q.T, num_heads, eps, gain)
    r = router_weights((x @ w_r.T).reshape(T, num_heads, num_sub))
    return {"q": q, "r": r}


def mhffn_prologue_backward(x, w_q, w_r, num_heads, num_sub, dq, dr, gain=None, eps=1e-6):
    """Gradients of L = sum(dq * q) + sum(dr * r) for the prologue above with respect to x,
    w_q, w_r and the gain (chain rule through the RMS normalisation and the normalised
    sigmoid)."""
    x, w_q, w_r, dq, dr = (_f64(a) for a in (x, w_q, w_r, dq, dr))
    T = x.shape[0]
    H, E = num_heads, num_sub
    z = (x @ w_q.T).reshape(T, H, -1)
    dh = z.shape[-1]
    inv = 1.0 / np.sqrt(np.mean(z * z, axis=-1, keepdims=True) + eps)
    n = z * inv
    g = np.ones(dh) if gain is None else _f64(gain)
    dgain = np.einsum("thd,thd->d", dq, n)
    dn = dq * g
    dz = inv * (dn - n * np.mean(dn * n, axis=-1, keepdims=True))
    l = (x @ w_r.T).reshape(T, H, E)
    sg = 1.0 / (1.0 + np.exp(-l))
    S = np.sum(sg, axis=-1, keepdims=True)
    r = sg / S
    ds = (dr - np.sum(dr * r, axis=-1, keepdims=True)) / S
    dl = ds * sg * (1.0 - sg)
    dz2, dl2 = dz.reshape(T, H * dh), dl.reshape(T, H * E)
    dx = dz2 @ w_q + dl2 @ w_r
    return {"dx": dx, "dw_q": dz2.T @ x, "dw_r": dl2.T @ x, "dgain": dgain}

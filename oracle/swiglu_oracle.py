"""fp64 CPU oracle for the SwiGLU feed-forward block and its group-sparse variant.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code, table or
helper with the CUDA library; the two meet only through the seeded inputs that
``swiglu_feed_forward_b200.synth`` draws.

Every function is the plain definition written out in float64 with numpy (a
library matmul is the only primitive; there is no blocking, fusion or
reordering).  Citations name the page and the section they follow:

* eugen_sparse README ("sparse SwiGLU FFN in Triton"), section "What it does":
  the sparse FFN formula, the group energy Sigma|SiLU(x W_gate)|, the optional
  subsample and balancing bias, the hard top-k, and the dense masked reference.
* flash-swiglu-mlp ("How pearblossom-m/flash-swiglu-mlp works"), overview:
  gate and up projections, SiLU gating, down projection; training saves
  intermediates, inference does not.
* parameter-golf PR 1105, "Fused MLP Kernels": the backward multiplies the
  down-projection gradient by an activation-gradient factor stored in the
  forward pass (here the SwiGLU analogue A = u * SiLU'(g), B = SiLU(g)).
* Megatron-Core ``sigmoid_topk`` API page: a bias that only affects selection,
  and a deterministic order among equal scores.

Readings where the pages are silent (each one is also listed in the design
notes): SiLU(z) = z * sigmoid(z); ``x W`` with nn.Linear weights means x W^T;
the balancing bias is added to the energy and used for selection only; the
subsample energy is the raw sum over the sampled rows (no rescaling); among
equal scores the lower group index wins and each row's K indices are returned
in ascending order; the subsample index is drawn per group by a partial
Fisher-Yates shuffle driven by one splitmix64 stream.

Parity status: every function here is pinned by the CPU tests in
``tests/test_oracle_pins.py`` (closed forms, finite differences, brute force,
an independent float64 torch autograd, and invariants).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "sigmoid", "silu", "silu_prime",
    "dense_forward", "dense_backward",
    "leaky_relu_sq_forward", "leaky_relu_sq_backward",
    "group_mask", "sparse_forward", "sparse_backward",
    "sparse_forward_by_groups",
    "splitmix64_stream", "make_subsample_index",
    "group_energy", "topk_groups", "topk_gap",
    "csr_buckets", "group_frequency", "update_load_balance_bias",
]


# --------------------------------------------------------------------------
# activations
# --------------------------------------------------------------------------
def sigmoid(z):
    """Logistic function 1 / (1 + e^-z), float64.  The pages never define
    SiLU; the standard reading SiLU(z) = z * sigmoid(z) is used throughout."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    """SiLU(z) = z * sigmoid(z)."""
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


def silu_prime(z):
    """d/dz SiLU(z) = sigmoid(z) * (1 + z * (1 - sigmoid(z)))."""
    z = np.asarray(z, dtype=np.float64)
    s = sigmoid(z)
    return s * (1.0 + z * (1.0 - s))


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# dense SwiGLU FFN (flash-swiglu-mlp overview; eugen_sparse "What it does")
# --------------------------------------------------------------------------
def dense_forward(x, w_gate, w_up, w_down):
    """Dense SwiGLU forward y = (SiLU(x W_g^T) * (x W_u^T)) W_d^T.

    Weights use the nn.Linear layout: w_gate, w_up are [d_ff, d_model],
    w_down is [d_model, d_ff].  Returns a dict with the pre-activations g, u,
    the product h, the output y, and the two activation-gradient factors the
    training forward saves: a = u * SiLU'(g) and b = SiLU(g) (the SwiGLU form
    of the parameter-golf "pre-computed activation gradient")."""
    x, w_gate, w_up, w_down = map(_f64, (x, w_gate, w_up, w_down))
    g = x @ w_gate.T
    u = x @ w_up.T
    b = silu(g)
    h = b * u
    a = u * silu_prime(g)
    y = h @ w_down.T
    return {"g": g, "u": u, "h": h, "y": y, "a": a, "b": b}


def dense_backward(x, w_gate, w_up, w_down, dy):
    """Gradients of L = sum(dy * y) by the chain rule:
    dH = dY W_d; dG = dH * u * SiLU'(g); dU = dH * SiLU(g);
    dx = dG W_g + dU W_u; dW_g = dG^T x; dW_u = dU^T x; dW_d = dY^T h."""
    x, w_gate, w_up, w_down, dy = map(_f64, (x, w_gate, w_up, w_down, dy))
    fw = dense_forward(x, w_gate, w_up, w_down)
    dh = dy @ w_down
    dg = dh * fw["u"] * silu_prime(fw["g"])
    du = dh * silu(fw["g"])
    return {
        "dx": dg @ w_gate + du @ w_up,
        "dw_gate": dg.T @ x,
        "dw_up": du.T @ x,
        "dw_down": dy.T @ fw["h"],
        "dh": dh, "dg": dg, "du": du,
    }


# --------------------------------------------------------------------------
# LeakyReLU(0.5)^2 MLP (parameter-golf PR 1105, "Fused MLP Kernels")
# --------------------------------------------------------------------------
def leaky_relu_sq_forward(x, w_up, w_down):
    """pre = x W_up^T; post = LeakyReLU(0.5)(pre)^2; y = post W_down^T, with the
    activation gradient the forward stores instead of the pre-activation:
    act_grad = 2 pre where pre > 0, 0.5 pre elsewhere (d post / d pre).
    w_up [hidden, d_model], w_down [d_model, hidden] (nn.Linear layout)."""
    x, w_up, w_down = map(_f64, (x, w_up, w_down))
    pre = x @ w_up.T
    leaky = np.where(pre > 0, pre, 0.5 * pre)
    post = leaky * leaky
    act_grad = np.where(pre > 0, 2.0 * pre, 0.5 * pre)
    return {"pre": pre, "post": post, "act_grad": act_grad, "y": post @ w_down.T}


def leaky_relu_sq_backward(x, w_up, w_down, dy):
    """Chain rule of L = sum(dy * y): dpre = (dy W_down) * act_grad;
    dx = dpre W_up; dW_up = dpre^T x; dW_down = dy^T post."""
    x, w_up, w_down, dy = map(_f64, (x, w_up, w_down, dy))
    fw = leaky_relu_sq_forward(x, w_up, w_down)
    dpre = (dy @ w_down) * fw["act_grad"]
    return {"dx": dpre @ w_up, "dw_up": dpre.T @ x, "dw_down": dy.T @ fw["post"], "dpre": dpre}


# --------------------------------------------------------------------------
# group-sparse variant (eugen_sparse "What it does")
# --------------------------------------------------------------------------
def group_mask(group_idx, d_ff, group_size):
    """[tokens, d_ff] 0/1 mask: column j is kept for token t when j's group
    j // group_size is among token t's selected groups."""
    group_idx = np.asarray(group_idx)
    M = group_idx.shape[0]
    ng = d_ff // group_size
    sel = np.zeros((M, ng), dtype=np.float64)
    rows = np.repeat(np.arange(M), group_idx.shape[1])
    sel[rows, group_idx.reshape(-1)] = 1.0
    return np.repeat(sel, group_size, axis=1)


def sparse_forward(x, w_gate, w_up, w_down, group_idx, group_size):
    """The dense masked reference of the eugen_sparse README: the SwiGLU
    product h is masked to each token's selected groups before the down
    projection.  Returns g, u, the masked h, and y."""
    x, w_gate, w_up, w_down = map(_f64, (x, w_gate, w_up, w_down))
    mask = group_mask(group_idx, w_gate.shape[0], group_size)
    g = x @ w_gate.T
    u = x @ w_up.T
    h = silu(g) * u * mask
    return {"g": g, "u": u, "h": h, "y": h @ w_down.T, "mask": mask}


def sparse_forward_by_groups(x, w_gate, w_up, w_down, group_idx, group_size):
    """The same output written as the README's formula: per token, the sum
    over its selected groups c of (SiLU(x W_g[c]^T) * x W_u[c]^T) W_d[:, c]^T.
    Pure per-token loop; for small cases only (it pins ``sparse_forward``)."""
    x, w_gate, w_up, w_down = map(_f64, (x, w_gate, w_up, w_down))
    G = group_size
    y = np.zeros((x.shape[0], w_down.shape[0]))
    for t in range(x.shape[0]):
        for c in np.asarray(group_idx)[t]:
            rows = slice(int(c) * G, (int(c) + 1) * G)
            hc = silu(w_gate[rows] @ x[t]) * (w_up[rows] @ x[t])
            y[t] += w_down[:, rows] @ hc
    return y


def sparse_backward(x, w_gate, w_up, w_down, group_idx, group_size, dy):
    """Gradients of L = sum(dy * y) for the masked forward: unselected
    (token, group) pairs contribute nothing, so groups chosen by no token get
    exactly zero weight gradients."""
    x, w_gate, w_up, w_down, dy = map(_f64, (x, w_gate, w_up, w_down, dy))
    fw = sparse_forward(x, w_gate, w_up, w_down, group_idx, group_size)
    mask = fw["mask"]
    dh = (dy @ w_down) * mask
    dg = dh * fw["u"] * silu_prime(fw["g"])
    du = dh * silu(fw["g"])
    return {
        "dx": dg @ w_gate + du @ w_up,
        "dw_gate": dg.T @ x,
        "dw_up": du.T @ x,
        "dw_down": dy.T @ fw["h"],
    }


# --------------------------------------------------------------------------
# subsample index (eugen_sparse "What it does" / "Parameters")
# --------------------------------------------------------------------------
_MASK64 = (1 << 64) - 1


def splitmix64_stream(seed):
    """Generator of splitmix64 outputs (Steele, Lea & Flood, "Fast splittable
    pseudorandom number generators", OOPSLA 2014; the 64-bit finaliser from
    Stafford's Mix13): state += 0x9E3779B97F4A7C15, then two xor-shift-multiply
    rounds and a final xor-shift."""
    state = int(seed) & _MASK64
    while True:
        state = (state + 0x9E3779B97F4A7C15) & _MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        yield z ^ (z >> 31)


def make_subsample_index(d_ff, group_size, samples_per_group, seed):
    """A fixed random subset of ``samples_per_group`` gate rows in every group.

    Group c owns rows [c*G, (c+1)*G).  For c = 0, 1, ... in turn, a partial
    Fisher-Yates shuffle of the offsets 0..G-1 draws its spg offsets, step i
    swapping position i with position i + (r mod (G - i)) for the next
    splitmix64 output r (one stream for all groups, seeded by ``seed``).
    Returns an int32 array [num_groups, spg] of absolute row ids, ascending
    within each group."""
    G, spg = int(group_size), int(samples_per_group)
    ng = int(d_ff) // G
    rng = splitmix64_stream(seed)
    out = np.empty((ng, spg), dtype=np.int32)
    for c in range(ng):
        perm = list(range(G))
        for i in range(spg):
            j = i + next(rng) % (G - i)
            perm[i], perm[j] = perm[j], perm[i]
        out[c] = sorted(c * G + p for p in perm[:spg])
    return out


# --------------------------------------------------------------------------
# selection (eugen_sparse "What it does"; Megatron sigmoid_topk conventions)
# --------------------------------------------------------------------------
def group_energy(x, w_gate, group_size, subsample_idx=None, bias=None):
    """Selection score per token and group:
    s[t, c] = sum over rows j of group c (or of its subsample) of
    |SiLU(x_t . W_gate[j])|, plus bias[c] when a bias is given (additive,
    selection only).  Returns [tokens, num_groups] float64."""
    x, w_gate = _f64(x), _f64(w_gate)
    G = int(group_size)
    ng = w_gate.shape[0] // G
    if subsample_idx is None:
        act = np.abs(silu(x @ w_gate.T))
        e = act.reshape(x.shape[0], ng, G).sum(axis=2)
    else:
        sub = np.asarray(subsample_idx).reshape(ng, -1)
        act = np.abs(silu(x @ w_gate[sub.reshape(-1)].T))
        e = act.reshape(x.shape[0], ng, sub.shape[1]).sum(axis=2)
    if bias is not None:
        e = e + _f64(bias)[None, :]
    return e


def topk_groups(scores, k):
    """Hard top-k per row: the k largest scores, the lower group index first
    among exactly equal scores; each row's k indices returned ascending."""
    scores = _f64(scores)
    M, ng = scores.shape
    cols = np.broadcast_to(np.arange(ng), (M, ng))
    order = np.lexsort((cols, -scores), axis=-1)  # by -score, then index
    return np.sort(order[:, :k], axis=1).astype(np.int32)


def topk_gap(scores, k):
    """Relative gap between each row's k-th and (k+1)-th largest score,
    (s_k - s_{k+1}) / |s_k|; +inf when k equals the number of groups.  Rows
    whose gap is below a tolerance are near-ties, where any top-k set is valid."""
    scores = _f64(scores)
    if k >= scores.shape[1]:
        return np.full(scores.shape[0], np.inf)
    s = -np.sort(-scores, axis=1)
    kth, nxt = s[:, k - 1], s[:, k]
    return (kth - nxt) / np.maximum(np.abs(kth), 1e-300)


def csr_buckets(group_idx, num_groups):
    """Group-major bucketing of the (token, group) pairs: offs[c] .. offs[c+1]
    index, in ``tokens``, the ids of the tokens that selected group c, in
    ascending token order (the stable order; the README states that the
    bucketing is deterministic)."""
    group_idx = np.asarray(group_idx)
    offs = np.zeros(num_groups + 1, dtype=np.int64)
    lists = []
    for c in range(num_groups):
        toks = np.nonzero((group_idx == c).any(axis=1))[0]
        lists.append(toks)
        offs[c + 1] = offs[c] + toks.size
    tokens = np.concatenate(lists) if lists else np.zeros(0, dtype=np.int64)
    return offs.astype(np.int32), tokens.astype(np.int32)


def group_frequency(group_idx, num_groups):
    """Fraction of the tokens whose selection holds each group: count[c] / tokens.  The
    frequencies of a batch sum to num_active_groups, so the balanced target of every group is
    num_active_groups / num_groups (eugen_sparse "Parameters": target_freq)."""
    group_idx = np.asarray(group_idx)
    counts = np.zeros(num_groups, dtype=np.float64)
    for row in group_idx:
        for c in set(int(v) for v in row):
            counts[c] += 1.0
    return counts / group_idx.shape[0]


def update_load_balance_bias(bias, freq_ema, current_freq, target_freq,
                             gamma, bias_max, momentum):
    """Auxiliary-loss-free balancing step (eugen_sparse "What it does" /
    "Parameters", in the DeepSeek-V3 style the README names; the formula is
    not printed, so this is the plainest reading):
    freq_ema <- momentum * freq_ema + (1 - momentum) * current_freq;
    bias <- clip(bias + gamma * sign(target_freq - freq_ema), -bias_max, bias_max).
    Returns (new_bias, new_freq_ema)."""
    freq_ema = momentum * _f64(freq_ema) + (1.0 - momentum) * _f64(current_freq)
    bias = _f64(bias) + gamma * np.sign(target_freq - freq_ema)
    return np.clip(bias, -bias_max, bias_max), freq_ema

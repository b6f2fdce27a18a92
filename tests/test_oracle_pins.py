"""Pins for the fp64 oracle: each check ties it to something other than itself
(closed forms, finite differences, brute force, an independent float64 torch
autograd, published generator outputs, invariants), so that a dropped term, a
wrong sign or a transposed operand in the oracle fails here."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def tiny(M=5, d=6, f=8, seed=0):
    return (rnd((M, d), seed), rnd((f, d), seed + 1, d ** -0.5),
            rnd((f, d), seed + 2, d ** -0.5), rnd((d, f), seed + 3, f ** -0.5),
            rnd((M, d), seed + 4, 0.1))


# ---------------------------------------------------------------- SiLU
def test_silu_closed_forms():
    assert O.silu(0.0) == 0.0
    assert O.silu_prime(0.0) == 0.5
    assert O.sigmoid(0.0) == 0.5
    z = np.linspace(-8, 8, 161)
    # SiLU(z) - SiLU(-z) = z * (s(z) + s(-z)) = z
    np.testing.assert_allclose(O.silu(z) - O.silu(-z), z, atol=1e-14)
    # asymptotes: SiLU(z) -> z for z >> 0, -> 0 for z << 0
    assert abs(O.silu(40.0) - 40.0) < 1e-12
    assert abs(O.silu(-40.0)) < 1e-12
    assert abs(O.silu_prime(40.0) - 1.0) < 1e-12 and abs(O.silu_prime(-40.0)) < 1e-12
    # SiLU(1) = 1 / (1 + 1/e)
    assert abs(O.silu(1.0) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15


def test_silu_prime_is_the_derivative():
    z = np.linspace(-10, 10, 401)
    h = 1e-5
    fd = (O.silu(z + h) - O.silu(z - h)) / (2 * h)
    np.testing.assert_allclose(O.silu_prime(z), fd, atol=1e-9)


def test_silu_matches_library():
    z = torch.linspace(-20, 20, 1001, dtype=torch.float64)
    np.testing.assert_allclose(O.silu(z.numpy()), torch.nn.functional.silu(z).numpy(),
                               rtol=1e-15, atol=1e-15)


# ---------------------------------------------------------------- dense forward
def test_dense_forward_brute_force_2x3x4():
    # every output written out with Python scalars and math.exp
    x, wg, wu, wd, _ = tiny(M=2, d=3, f=4, seed=11)
    out = O.dense_forward(x, wg, wu, wd)
    for t in range(2):
        hs = []
        for j in range(4):
            g = sum(x[t][k] * wg[j][k] for k in range(3))
            u = sum(x[t][k] * wu[j][k] for k in range(3))
            hs.append(g / (1.0 + math.exp(-g)) * u)
        for i in range(3):
            y = sum(hs[j] * wd[i][j] for j in range(4))
            assert abs(out["y"][t, i] - y) < 1e-13
        np.testing.assert_allclose(out["h"][t], hs, rtol=1e-13, atol=1e-15)


def test_dense_forward_matches_torch_float64():
    x, wg, wu, wd, _ = tiny(M=64, d=128, f=352, seed=3)
    T = lambda a: torch.from_numpy(a)
    F = torch.nn.functional
    y = F.linear(F.silu(F.linear(T(x), T(wg))) * F.linear(T(x), T(wu)), T(wd))
    np.testing.assert_allclose(O.dense_forward(x, wg, wu, wd)["y"], y.numpy(), rtol=1e-12, atol=1e-12)


def test_saved_terms_recover_gradient_factors():
    # a = u * SiLU'(g) and b = SiLU(g): b*u is h; a and b are the partials of h
    x, wg, wu, wd, _ = tiny(seed=5)
    fw = O.dense_forward(x, wg, wu, wd)
    np.testing.assert_allclose(fw["b"] * fw["u"], fw["h"], rtol=1e-14)
    eps = 1e-6
    dh_dg = (O.silu(fw["g"] + eps) * fw["u"] - O.silu(fw["g"] - eps) * fw["u"]) / (2 * eps)
    np.testing.assert_allclose(fw["a"], dh_dg, atol=1e-8)


# ---------------------------------------------------------------- dense backward
def test_dense_backward_matches_torch_autograd():
    x, wg, wu, wd, dy = tiny(M=64, d=128, f=352, seed=7)
    ts = [torch.from_numpy(a).requires_grad_(True) for a in (x, wg, wu, wd)]
    F = torch.nn.functional
    y = F.linear(F.silu(F.linear(ts[0], ts[1])) * F.linear(ts[0], ts[2]), ts[3])
    y.backward(torch.from_numpy(dy))
    bw = O.dense_backward(x, wg, wu, wd, dy)
    for name, t in zip(("dx", "dw_gate", "dw_up", "dw_down"), ts):
        np.testing.assert_allclose(bw[name], t.grad.numpy(), rtol=1e-11, atol=1e-12)


def _fd_check(loss, params, grads, eps=1e-6, tol=1e-6, sample=None, rng=None):
    for p, gref in zip(params, grads):
        idxs = list(np.ndindex(p.shape))
        if sample is not None:
            idxs = [idxs[i] for i in rng.choice(len(idxs), size=min(sample, len(idxs)), replace=False)]
        for ix in idxs:
            old = p[ix]
            p[ix] = old + eps
            lp = loss()
            p[ix] = old - eps
            lm = loss()
            p[ix] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - gref[ix]) <= tol * max(1.0, abs(gref[ix])), (ix, fd, gref[ix])


def test_dense_backward_finite_differences_every_element():
    x, wg, wu, wd, dy = tiny(M=3, d=4, f=6, seed=9)
    loss = lambda: float(np.sum(dy * O.dense_forward(x, wg, wu, wd)["y"]))
    bw = O.dense_backward(x, wg, wu, wd, dy)
    _fd_check(loss, [x, wg, wu, wd], [bw["dx"], bw["dw_gate"], bw["dw_up"], bw["dw_down"]])


def test_dense_backward_finite_differences_sampled_workload0_shape():
    x, wg, wu, wd, dy = tiny(M=64, d=128, f=352, seed=13)
    loss = lambda: float(np.sum(dy * O.dense_forward(x, wg, wu, wd)["y"]))
    bw = O.dense_backward(x, wg, wu, wd, dy)
    rng = np.random.default_rng(0)
    _fd_check(loss, [x, wg, wu, wd], [bw["dx"], bw["dw_gate"], bw["dw_up"], bw["dw_down"]],
              sample=40, rng=rng, tol=1e-6)


# ---------------------------------------------------------------- invariants
def test_dense_invariants():
    x, wg, wu, wd, dy = tiny(M=7, d=8, f=12, seed=17)
    y = O.dense_forward(x, wg, wu, wd)["y"]
    p = np.random.default_rng(1).permutation(12)
    np.testing.assert_allclose(O.dense_forward(x, wg[p], wu[p], wd[:, p])["y"], y, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(O.dense_forward(x, wg, wu, 3.0 * wd)["y"], 3.0 * y, rtol=1e-13)
    r = np.random.default_rng(2).permutation(7)
    np.testing.assert_allclose(O.dense_forward(x[r], wg, wu, wd)["y"], y[r], rtol=1e-13)
    bw = O.dense_backward(x, wg, wu, wd, dy)
    bw2 = O.dense_backward(x, wg, wu, wd, 2.0 * dy)
    for k in ("dx", "dw_gate", "dw_up", "dw_down"):
        np.testing.assert_allclose(bw2[k], 2.0 * bw[k], rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- sparse
def _sel(M, ng, K, seed):
    rng = np.random.default_rng(seed)
    return np.sort(np.stack([rng.choice(ng, size=K, replace=False) for _ in range(M)]), axis=1)


def test_sparse_all_groups_equals_dense():
    x, wg, wu, wd, dy = tiny(M=9, d=8, f=16, seed=19)
    idx = np.tile(np.arange(4), (9, 1))
    fw_s = O.sparse_forward(x, wg, wu, wd, idx, 4)
    np.testing.assert_allclose(fw_s["y"], O.dense_forward(x, wg, wu, wd)["y"], rtol=1e-13, atol=1e-15)
    bs, bd = O.sparse_backward(x, wg, wu, wd, idx, 4, dy), O.dense_backward(x, wg, wu, wd, dy)
    for k in ("dx", "dw_gate", "dw_up", "dw_down"):
        np.testing.assert_allclose(bs[k], bd[k], rtol=1e-12, atol=1e-15)


def test_sparse_masked_equals_per_group_sum_and_is_additive():
    x, wg, wu, wd, _ = tiny(M=10, d=8, f=32, seed=23)
    idx = _sel(10, 8, 3, 0)
    y = O.sparse_forward(x, wg, wu, wd, idx, 4)["y"]
    np.testing.assert_allclose(O.sparse_forward_by_groups(x, wg, wu, wd, idx, 4), y, rtol=1e-12, atol=1e-14)
    # additivity: the output is the sum of the single-group outputs
    acc = sum(O.sparse_forward(x, wg, wu, wd, idx[:, k:k + 1], 4)["y"] for k in range(3))
    np.testing.assert_allclose(acc, y, rtol=1e-12, atol=1e-14)


def test_sparse_unselected_groups_get_zero_gradients_and_fd():
    x, wg, wu, wd, dy = tiny(M=6, d=4, f=16, seed=29)
    idx = np.array([[0, 2]] * 3 + [[0, 1]] * 3)  # group 3 never chosen
    bw = O.sparse_backward(x, wg, wu, wd, idx, 4, dy)
    assert np.all(bw["dw_gate"][12:16] == 0) and np.all(bw["dw_up"][12:16] == 0)
    assert np.all(bw["dw_down"][:, 12:16] == 0)
    assert np.any(bw["dw_gate"][0:4] != 0)
    loss = lambda: float(np.sum(dy * O.sparse_forward(x, wg, wu, wd, idx, 4)["y"]))
    _fd_check(loss, [x, wg, wu, wd], [bw["dx"], bw["dw_gate"], bw["dw_up"], bw["dw_down"]])


# ---------------------------------------------------------------- energy and top-k
def test_energy_exact_and_full_subsample_agree():
    x, wg, *_ = tiny(M=11, d=8, f=32, seed=31)
    e = O.group_energy(x, wg, 8)
    assert np.all(e >= 0)
    full = np.arange(32).reshape(4, 8)
    np.testing.assert_allclose(O.group_energy(x, wg, 8, subsample_idx=full), e, rtol=1e-14)
    # independent evaluation in torch float64
    z = torch.nn.functional.silu(torch.from_numpy(x) @ torch.from_numpy(wg).T).abs()
    np.testing.assert_allclose(e, z.reshape(11, 4, 8).sum(-1).numpy(), rtol=1e-13)


def test_energy_subsample_is_raw_sum_over_sampled_rows():
    x, wg, *_ = tiny(M=5, d=8, f=16, seed=37)
    sub = np.array([[1, 3], [4, 7]])
    e = O.group_energy(x, wg, 8, subsample_idx=sub)
    a = np.abs(O.silu(x @ wg.T))
    np.testing.assert_allclose(e[:, 0], a[:, 1] + a[:, 3], rtol=1e-14)
    np.testing.assert_allclose(e[:, 1], a[:, 4] + a[:, 7], rtol=1e-14)


def test_bias_is_additive_and_forces_selection():
    x, wg, *_ = tiny(M=20, d=8, f=64, seed=41)
    bias = np.zeros(8)
    bias[[1, 4, 6]] = 10.0
    s = O.group_energy(x, wg, 8, bias=bias)
    np.testing.assert_allclose(s - O.group_energy(x, wg, 8), np.broadcast_to(bias, s.shape), atol=1e-12)
    assert np.all(O.topk_groups(s, 3) == np.array([1, 4, 6]))


def test_topk_brute_force_enumeration():
    rng = np.random.default_rng(43)
    for ng in range(1, 9):
        for K in range(1, ng + 1):
            s = rng.standard_normal((6, ng))
            got = O.topk_groups(s, K)
            for t in range(6):
                best = max(itertools.combinations(range(ng), K), key=lambda c: (s[t, list(c)].sum(), [-i for i in c]))
                assert tuple(got[t]) == tuple(sorted(best))


def test_topk_ties_lower_index_wins_and_rows_are_independent():
    s = np.array([[1.0, 2.0, 2.0, 0.5, 2.0]])
    assert tuple(O.topk_groups(s, 2)[0]) == (1, 2)
    assert tuple(O.topk_groups(s, 1)[0]) == (1,)
    rng = np.random.default_rng(47)
    S = rng.standard_normal((30, 16))
    full = O.topk_groups(S, 4)
    p = rng.permutation(30)
    np.testing.assert_array_equal(O.topk_groups(S[p], 4), full[p])
    np.testing.assert_array_equal(O.topk_groups(S[:7], 4), full[:7])
    assert np.all(np.diff(full, axis=1) > 0)


def test_topk_gap():
    s = np.array([[4.0, 3.0, 2.0, 1.0], [1.0, 1.0, 0.0, 0.0]])
    np.testing.assert_allclose(O.topk_gap(s, 2), [1.0 / 3.0, 1.0])
    assert O.topk_gap(s, 1)[1] == 0.0
    assert np.all(np.isinf(O.topk_gap(s, 4)))


# ---------------------------------------------------------------- CSR
def test_csr_buckets_brute_force():
    idx = _sel(50, 6, 3, 5)
    offs, toks = O.csr_buckets(idx, 6)
    assert offs[0] == 0 and offs[-1] == 150
    for c in range(6):
        seg = toks[offs[c]:offs[c + 1]]
        assert list(seg) == [t for t in range(50) if c in idx[t]]


# ---------------------------------------------------------------- subsample index
def _golden_splitmix():
    out = {}
    with open(os.path.join(GOLDEN, "splitmix64.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            k, v = line.split(":")
            out[int(k)] = [int(a) for a in v.split()]
    return out


def test_splitmix64_published_values():
    for seed, vals in _golden_splitmix().items():
        g = O.splitmix64_stream(seed)
        assert [next(g) for _ in vals] == vals


def test_subsample_index_properties():
    sub = O.make_subsample_index(4096, 64, 8, seed=3)
    assert sub.shape == (64, 8) and sub.dtype == np.int32
    for c in range(64):
        assert np.all(np.diff(sub[c]) > 0)
        assert sub[c].min() >= 64 * c and sub[c].max() < 64 * (c + 1)
    np.testing.assert_array_equal(sub, O.make_subsample_index(4096, 64, 8, seed=3))
    assert np.any(sub != O.make_subsample_index(4096, 64, 8, seed=4))
    full = O.make_subsample_index(256, 32, 32, seed=9)
    np.testing.assert_array_equal(full, np.arange(256).reshape(8, 32))


def test_subsample_index_is_uniform():
    # each offset within a group is drawn with probability spg/G
    counts = np.zeros(16)
    n = 0
    for seed in range(400):
        sub = O.make_subsample_index(64, 16, 4, seed)
        for c in range(4):
            np.add.at(counts, sub[c] - 16 * c, 1)
            n += 1
    expect = n * 4 / 16
    chi2 = float(((counts - expect) ** 2 / expect).sum())
    assert chi2 < 40.0, chi2  # 15 dof; p < 1e-3 at ~37.7


# ---------------------------------------------------------------- load-balance update
def test_load_balance_bias_update():
    bias = np.array([0.0, 0.0, 0.49, -0.49])
    ema = np.array([0.25, 0.25, 0.25, 0.25])
    cur = np.array([0.5, 0.0, 0.0, 0.5])
    nb, ne = O.update_load_balance_bias(bias, ema, cur, 0.25, 0.02, 0.5, 0.9)
    np.testing.assert_allclose(ne, [0.275, 0.225, 0.225, 0.275])
    # over-used groups lose bias, under-used gain it, clamped to +-bias_max
    np.testing.assert_allclose(nb, [-0.02, 0.02, 0.5, -0.5])
    nb2, _ = O.update_load_balance_bias(bias, ema, ema, 0.25, 0.02, 0.5, 0.9)
    np.testing.assert_allclose(nb2, bias)


def test_group_frequency():
    idx = np.array([[0, 2], [1, 2], [2, 3]])
    np.testing.assert_allclose(O.group_frequency(idx, 5), [1 / 3, 1 / 3, 1.0, 1 / 3, 0.0])
    rng = np.random.default_rng(3)
    big = np.sort(np.stack([rng.choice(16, size=4, replace=False) for _ in range(500)]), axis=1)
    f = O.group_frequency(big, 16)
    assert abs(f.sum() - 4.0) < 1e-12  # frequencies sum to K: the balanced target is K / groups



# ---------------------------------------------------------------- LeakyReLU(0.5)^2 MLP
def test_leaky_relu_sq_page_identity_both_signs():
    # the fused-MLP page's derivation: post = 0.5 * act_grad * pre for pre > 0 (pre^2) and
    # pre <= 0 ((0.5 pre)^2), with act_grad = 2 pre or 0.5 pre
    x, wu, wd = rnd((6, 8), 61), rnd((12, 8), 62, 8 ** -0.5), rnd((8, 12), 63, 12 ** -0.5)
    fw = O.leaky_relu_sq_forward(x, wu, wd)
    pre = fw["pre"]
    assert np.any(pre > 0) and np.any(pre < 0)
    np.testing.assert_allclose(fw["post"], 0.5 * fw["act_grad"] * pre, rtol=1e-14)
    np.testing.assert_allclose(fw["post"][pre > 0], pre[pre > 0] ** 2, rtol=1e-14)
    np.testing.assert_allclose(fw["post"][pre <= 0], (0.5 * pre[pre <= 0]) ** 2, rtol=1e-14)
    # act_grad is d post / d pre
    eps = 1e-6
    lk = lambda z: np.where(z > 0, z, 0.5 * z) ** 2
    np.testing.assert_allclose(fw["act_grad"], (lk(pre + eps) - lk(pre - eps)) / (2 * eps), atol=1e-8)


def test_leaky_relu_sq_matches_torch_autograd_and_fd():
    x, wu, wd, dy = rnd((16, 32), 71), rnd((56, 32), 72, 32 ** -0.5), rnd((32, 56), 73, 56 ** -0.5), rnd((16, 32), 74, 0.1)
    ts = [torch.from_numpy(a).requires_grad_(True) for a in (x, wu, wd)]
    F = torch.nn.functional
    y = F.linear(F.leaky_relu(F.linear(ts[0], ts[1]), 0.5) ** 2, ts[2])
    y.backward(torch.from_numpy(dy))
    fw = O.leaky_relu_sq_forward(x, wu, wd)
    np.testing.assert_allclose(fw["y"], y.detach().numpy(), rtol=1e-12, atol=1e-13)
    bw = O.leaky_relu_sq_backward(x, wu, wd, dy)
    for name, t in zip(("dx", "dw_up", "dw_down"), ts):
        np.testing.assert_allclose(bw[name], t.grad.numpy(), rtol=1e-11, atol=1e-12)
    xs, wus, wds, dys = x[:3, :4].copy(), wu[:6, :4].copy(), wd[:4, :6].copy(), dy[:3, :4].copy()
    loss = lambda: float(np.sum(dys * O.leaky_relu_sq_forward(xs, wus, wds)["y"]))
    b2 = O.leaky_relu_sq_backward(xs, wus, wds, dys)
    _fd_check(loss, [xs, wus, wds], [b2["dx"], b2["dw_up"], b2["dw_down"]])


# ---------------------------------------------------------------- FlashFFN multi-head FFN
def mh_inputs(T=5, H=2, E=3, de=4, dh=6, seed=80):
    return (rnd((T, H, dh), seed), rnd((H, E, de, dh), seed + 1, dh ** -0.5),
            rnd((H, E, de, dh), seed + 2, dh ** -0.5), rnd((H, E, de, dh), seed + 3, de ** -0.5),
            np.random.default_rng(seed + 4).uniform(0.1, 1.0, (T, H, E)), rnd((T, H, dh), seed + 5, 0.1))


def test_mhffn_one_head_one_subnetwork_is_dense_swiglu():
    # H = E = 1, R = 1: the block is a SwiGLU FFN with W_gate = K, W_up = U, W_down = V^T
    q, k, u, v, _, _ = mh_inputs(T=7, H=1, E=1, de=10, dh=6, seed=81)
    o = O.mhffn_forward(q, k, u, v, np.ones((7, 1, 1)))["o"]
    y = O.dense_forward(q[:, 0], k[0, 0], u[0, 0], v[0, 0].T)["y"]
    np.testing.assert_allclose(o[:, 0], y, rtol=1e-13, atol=1e-14)


def test_mhffn_brute_force_scalar_loops():
    q, k, u, v, r, _ = mh_inputs(T=2, H=2, E=2, de=3, dh=2, seed=82)
    sil = lambda z: z / (1.0 + math.exp(-z))
    o = np.zeros_like(q)
    for t, h, e, j, c in itertools.product(range(2), range(2), range(2), range(3), range(2)):
        g = sum(q[t, h, i] * k[h, e, j, i] for i in range(2))
        w = sum(q[t, h, i] * u[h, e, j, i] for i in range(2))
        o[t, h, c] += r[t, h, e] * sil(g) * w * v[h, e, j, c]
    np.testing.assert_allclose(O.mhffn_forward(q, k, u, v, r)["o"], o, rtol=1e-13, atol=1e-15)


def test_mhffn_additive_over_subnetworks_heads_independent_linear_in_r():
    q, k, u, v, r, _ = mh_inputs(seed=83)
    o = O.mhffn_forward(q, k, u, v, r)["o"]
    parts = sum(O.mhffn_forward(q, k[:, e:e + 1], u[:, e:e + 1], v[:, e:e + 1], r[:, :, e:e + 1])["o"]
                for e in range(k.shape[1]))
    np.testing.assert_allclose(o, parts, rtol=1e-12, atol=1e-14)
    o1 = O.mhffn_forward(q[:, 1:], k[1:], u[1:], v[1:], r[:, 1:])["o"]
    np.testing.assert_allclose(o[:, 1:], o1, rtol=1e-13)
    np.testing.assert_allclose(O.mhffn_forward(q, k, u, v, 2.5 * r)["o"], 2.5 * o, rtol=1e-12)


def test_mhffn_backward_matches_torch_autograd_and_fd():
    q, k, u, v, r, do = mh_inputs(T=6, H=2, E=3, de=5, dh=4, seed=84)
    ts = [torch.from_numpy(a.copy()).requires_grad_(True) for a in (q, k, u, v, r)]
    F = torch.nn.functional
    tq, tk, tu, tv, tr = ts
    act = F.silu(torch.einsum("thd,hefd->thef", tq, tk)) * torch.einsum("thd,hefd->thef", tq, tu)
    o = torch.einsum("thef,hefd->thd", act * tr[..., None], tv)
    o.backward(torch.from_numpy(do))
    np.testing.assert_allclose(O.mhffn_forward(q, k, u, v, r)["o"], o.detach().numpy(), rtol=1e-12, atol=1e-14)
    bw = O.mhffn_backward(q, k, u, v, r, do)
    for name, t in zip(("dq", "dk", "du", "dv", "dr"), ts):
        np.testing.assert_allclose(bw[name], t.grad.numpy(), rtol=1e-11, atol=1e-13)
    qs, ks, us, vs, rs, dos = (a.copy() for a in mh_inputs(T=2, H=1, E=2, de=2, dh=3, seed=85))
    loss = lambda: float(np.sum(dos * O.mhffn_forward(qs, ks, us, vs, rs)["o"]))
    b2 = O.mhffn_backward(qs, ks, us, vs, rs, dos)
    _fd_check(loss, [qs, ks, us, vs, rs], [b2["dq"], b2["dk"], b2["du"], b2["dv"], b2["dr"]])


def test_head_rmsnorm_and_router_weights():
    z = rnd((4, 3 * 8), 86, 3.0)
    n = O.head_rmsnorm(z, 3, eps=0.0)
    np.testing.assert_allclose(np.mean(n * n, axis=-1), 1.0, rtol=1e-12)   # unit RMS per head
    np.testing.assert_allclose(n * np.sqrt(np.mean(z.reshape(4, 3, 8) ** 2, -1, keepdims=True)),
                               z.reshape(4, 3, 8), rtol=1e-12)
    lg = rnd((4, 3, 5), 87)
    w = O.router_weights(lg)
    np.testing.assert_allclose(w.sum(-1), 1.0, rtol=1e-13)
    assert np.all(w > 0)
    np.testing.assert_allclose(O.router_weights(np.zeros((1, 1, 4))), 0.25)
    # order follows the logits; sigmoid(0) = 1/2 against sigmoid(large) ~ 1
    w2 = O.router_weights(np.array([[[0.0, 50.0]]]))
    np.testing.assert_allclose(w2[0, 0], [1 / 3, 2 / 3], rtol=1e-12)


@pytest.mark.parametrize("use_gain", [True, False])
def test_mhffn_prologue_backward_matches_autograd_and_fd(use_gain):
    T, d, H, dh, E = 5, 12, 3, 4, 3
    x, wq, wr = rnd((T, d), 90), rnd((H * dh, d), 91, d ** -0.5), rnd((H * E, d), 92, d ** -0.5)
    gain = np.random.default_rng(93).uniform(0.5, 1.5, dh) if use_gain else None
    dq, dr = rnd((T, H, dh), 94, 0.1), rnd((T, H, E), 95, 0.1)
    ts = [torch.from_numpy(a.copy()).requires_grad_(True) for a in (x, wq, wr)]
    tg = torch.from_numpy(gain.copy()).requires_grad_(True) if use_gain else None
    z = (ts[0] @ ts[1].T).reshape(T, H, dh)
    qn = z / torch.sqrt((z * z).mean(-1, keepdim=True) + 1e-6)
    if use_gain:
        qn = qn * tg
    sg = torch.sigmoid((ts[0] @ ts[2].T).reshape(T, H, E))
    rr = sg / sg.sum(-1, keepdim=True)
    fw = O.mhffn_prologue_forward(x, wq, wr, H, E, gain, 1e-6)
    np.testing.assert_allclose(fw["q"], qn.detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(fw["r"], rr.detach().numpy(), rtol=1e-12, atol=1e-14)
    ((qn * torch.from_numpy(dq)).sum() + (rr * torch.from_numpy(dr)).sum()).backward()
    bw = O.mhffn_prologue_backward(x, wq, wr, H, E, dq, dr, gain, 1e-6)
    for name, t in zip(("dx", "dw_q", "dw_r"), ts):
        np.testing.assert_allclose(bw[name], t.grad.numpy(), rtol=1e-10, atol=1e-12)
    if use_gain:
        np.testing.assert_allclose(bw["dgain"], tg.grad.numpy(), rtol=1e-10, atol=1e-12)
    xs, wqs, wrs = x[:2].copy(), wq.copy(), wr.copy()
    dqs, drs = dq[:2].copy(), dr[:2].copy()
    loss = lambda: float(np.sum(dqs * O.mhffn_prologue_forward(xs, wqs, wrs, H, E, gain, 1e-6)["q"])
                         + np.sum(drs * O.mhffn_prologue_forward(xs, wqs, wrs, H, E, gain, 1e-6)["r"]))
    b2 = O.mhffn_prologue_backward(xs, wqs, wrs, H, E, dqs, drs, gain, 1e-6)
    _fd_check(loss, [xs, wqs, wrs], [b2["dx"], b2["dw_q"], b2["dw_r"]], tol=1e-5)

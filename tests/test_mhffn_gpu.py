"""GPU parity of the FlashFFN multi-head FFN (fused forward, prologue, fused backward) against the fp64
oracle, through the C ABI: small and ragged token counts, several heads and sub-network widths,
and sampled token rows of the full 1.3B-configuration workload."""
import numpy as np
import pytest
import torch

import oracle as O
from swiglu_feed_forward_b200 import api, synth
from tests._util import assert_close, f64

pytestmark = pytest.mark.gpu


def run(inp):
    t = {k: v.cuda() for k, v in inp.items() if k != "do"}
    o = api.flash_mhffn_fwd(t["q"], t["w_k"], t["w_u"], t["w_v"], t["router"])
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return o


def reference(inp, tokens=None):
    q, k, u, v, r = (f64(inp[n]) for n in ("q", "w_k", "w_u", "w_v", "router"))
    if tokens is not None:
        q, r = q[tokens], r[tokens]
    return O.mhffn_forward(q, k, u, v, r)["o"]


@pytest.mark.parametrize("T,H,E,de", [
    (200, 2, 3, 64),     # ragged token tile, 3 sub-networks of one chunk
    (1, 1, 1, 64),       # one token, one chunk
    (260, 2, 3, 192),    # odd chunk count per sub-network
    (128, 1, 2, 256),    # exactly one tile (and an empty partner tile), two chunks per sub-network
    (300, 3, 2, 256),    # three heads, ragged
    (700, 2, 5, 384),    # the 1.3B sub-network width, several tile pairs per head
    (520, 1, 7, 384),    # the 370M configuration's E, five tile pairs
])
def test_small_and_ragged(T, H, E, de):
    inp = synth.mhffn_inputs(T, H, 128, E, de, seed=T + E, with_do=False)
    o = run(inp)
    assert o.shape == (T, H, 128)
    assert_close("o", f64(o), reference(inp), torch.bfloat16)


def test_router_weight_scales_its_subnetwork_only():
    """A sub-network whose router weight is zero for a token contributes nothing to it."""
    inp = synth.mhffn_inputs(256, 2, 128, 3, 128, seed=5, with_do=False)
    inp["router"][:, :, 1] = 0.0
    o = run(inp)
    assert_close("o", f64(o), reference(inp), torch.bfloat16)
    sub = {k: (v[:, [0, 2]].contiguous() if k in ("w_k", "w_u", "w_v") else v) for k, v in inp.items()}
    sub["router"] = inp["router"][:, :, [0, 2]].contiguous()
    o2 = run(sub)
    # exact zeros added to the fp32 accumulator change nothing: bitwise equal
    assert torch.equal(o.view(torch.int16), o2.view(torch.int16))


def test_deterministic():
    inp = synth.mhffn_inputs(384, 2, 128, 2, 128, seed=9, with_do=False)
    a, b = run(inp), run(inp)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_full_size_sampled_tokens():
    """32768 tokens x 16 heads x 15 sub-networks of 384 (the bench's launch configuration):
    sampled token rows, every head, against the oracle."""
    w = synth.WORKLOADS[6]
    inp = synth.mhffn_inputs(w["T"], w["H"], w["d_h"], w["E"], w["d_e"], w["seed"], with_do=False)
    o = run(inp)
    rng = np.random.default_rng(0)
    tokens = np.sort(np.concatenate([rng.choice(w["T"] - 128, 24, replace=False), [w["T"] - 1]]))
    assert_close("o[tokens]", f64(o)[tokens], reference(inp, tokens), torch.bfloat16)


def check_prologue(inp, H, E, use_gain, tokens=None):
    x, wq, wr = (inp[k].cuda() for k in ("x", "w_q", "w_r"))
    gain = inp["q_gain"].cuda() if use_gain else None
    q, r = api.flash_mhffn_prologue(x, wq, wr, H, E, q_gain=gain, eps=1e-6)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    xs = f64(inp["x"]) if tokens is None else f64(inp["x"])[tokens]
    q_ref = O.head_rmsnorm(xs @ f64(inp["w_q"]).T, H, eps=1e-6,
                           weight=f64(inp["q_gain"]) if use_gain else None)
    r_ref = O.router_weights((xs @ f64(inp["w_r"]).T).reshape(len(xs), H, E))
    qg, rg = f64(q), f64(r)
    if tokens is not None:
        qg, rg = qg[tokens], rg[tokens]
    assert_close("q", qg, q_ref, torch.bfloat16)
    assert_close("router", rg, r_ref, torch.float32)
    return q, r


@pytest.mark.parametrize("T,d_model,H,E,use_gain", [
    (300, 256, 3, 5, True),     # ragged tokens, E not a power of two
    (1, 64, 1, 1, False),       # one token, one head, one sub-network (router weight 1)
    (513, 768, 6, 8, True),     # the 128M configuration's heads and E
    (256, 2048, 16, 15, False), # the 1.3B configuration: 240 router columns
])
def test_prologue(T, d_model, H, E, use_gain):
    check_prologue(synth.mhffn_prologue_inputs(T, d_model, H, 128, E, seed=T + H), H, E, use_gain)


def test_block_prologue_then_fused_forward():
    """x -> (Q, R) -> O through both entry points against the oracle's whole block."""
    T, d_model, H, E, de = 700, 512, 4, 3, 128
    pro = synth.mhffn_prologue_inputs(T, d_model, H, 128, E, seed=21)
    wts = synth.mhffn_inputs(1, H, 128, E, de, seed=21, with_do=False)
    q, r = check_prologue(pro, H, E, True)
    o = api.flash_mhffn_fwd(q, wts["w_k"].cuda(), wts["w_u"].cuda(), wts["w_v"].cuda(), r)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    qr = O.head_rmsnorm(f64(pro["x"]) @ f64(pro["w_q"]).T, H, eps=1e-6, weight=f64(pro["q_gain"]))
    rr = O.router_weights((f64(pro["x"]) @ f64(pro["w_r"]).T).reshape(T, H, E))
    ref = O.mhffn_forward(qr, f64(wts["w_k"]), f64(wts["w_u"]), f64(wts["w_v"]), rr)["o"]
    assert_close("o", f64(o), ref, torch.bfloat16)


@pytest.mark.parametrize("T,H,E,de", [
    (200, 2, 3, 128),    # ragged tokens, three sub-networks
    (1, 1, 1, 128),      # one token
    (300, 1, 2, 256),    # two 128-column blocks per sub-network
    (700, 3, 2, 384),    # the 1.3B sub-network width, odd head count
    (4000, 5, 1, 128),   # two launches (four heads, then one), more units than clusters
    (333, 2, 2, 512),    # eight 64-column chunks per sub-network, ragged tokens
])
def test_backward(T, H, E, de):
    inp = synth.mhffn_inputs(T, H, 128, E, de, seed=T + 3 * E)
    t = {k: v.cuda() for k, v in inp.items()}
    grads = api.flash_mhffn_bwd(t["q"], t["w_k"], t["w_u"], t["w_v"], t["router"], t["do"])
    torch.cuda.synchronize()
    assert api.device_status() == 0
    ref = O.mhffn_backward(*(f64(inp[k]) for k in ("q", "w_k", "w_u", "w_v", "router", "do")))
    for name, got in zip(("dq", "dk", "du", "dv", "dr"), grads):
        assert_close(name, f64(got), ref[name], torch.bfloat16)


def test_backward_deterministic():
    inp = synth.mhffn_inputs(512, 2, 128, 2, 128, seed=31)
    t = {k: v.cuda() for k, v in inp.items()}
    args = (t["q"], t["w_k"], t["w_u"], t["w_v"], t["router"], t["do"])
    a, b = api.flash_mhffn_bwd(*args), api.flash_mhffn_bwd(*args)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_backward_full_size_sampled():
    """32768 tokens x 16 heads x 15 sub-networks of 384 (the bench's launch configuration):
    dq and the router gradient on sampled tokens; dK, dU, dV on sampled rows of every kind of
    sub-network (each such row sums over all 32768 tokens but needs only its own weight rows)."""
    w = synth.WORKLOADS[6]
    inp = synth.mhffn_inputs(w["T"], w["H"], w["d_h"], w["E"], w["d_e"], w["seed"])
    t = {k: v.cuda() for k, v in inp.items()}
    dq, dk, du, dv, dr = api.flash_mhffn_bwd(t["q"], t["w_k"], t["w_u"], t["w_v"], t["router"], t["do"])
    torch.cuda.synchronize()
    assert api.device_status() == 0
    q, k, u, v, r, do = (f64(inp[n]) for n in ("q", "w_k", "w_u", "w_v", "router", "do"))
    rng = np.random.default_rng(1)
    tokens = np.sort(np.concatenate([rng.choice(w["T"] - 128, 16, replace=False), [w["T"] - 1]]))
    ref = O.mhffn_backward(q[tokens], k, u, v, r[tokens], do[tokens])
    assert_close("dq[tokens]", f64(dq)[tokens], ref["dq"], torch.bfloat16)
    assert_close("dr[tokens]", f64(dr)[tokens], ref["dr"], torch.bfloat16)
    for h, e in ((0, 0), (7, 14), (15, 6)):
        rows = np.sort(rng.choice(w["d_e"], 6, replace=False))
        sub = O.mhffn_backward(q[:, [h]], k[[h]][:, [e]][:, :, rows], u[[h]][:, [e]][:, :, rows],
                               v[[h]][:, [e]][:, :, rows], r[:, [h]][:, :, [e]], do[:, [h]])
        for name, got in (("dk", dk), ("du", du), ("dv", dv)):
            assert_close(f"{name}[{h},{e},rows]", f64(got)[h, e][rows], sub[name][0, 0], torch.bfloat16)


@pytest.mark.parametrize("T,d_model,H,E,use_gain", [
    (300, 256, 3, 5, True),     # odd head count, ragged tokens
    (1, 64, 1, 1, False),       # one token, one sub-network (router gradient 0)
    (513, 512, 4, 15, True),    # the 1.3B E
])
def test_prologue_backward(T, d_model, H, E, use_gain):
    pro = synth.mhffn_prologue_inputs(T, d_model, H, 128, E, seed=T + 7)
    dq = synth.normal((T, H, 128), 0.1, T, "do")
    dr = synth.normal((T, H, E), 0.1, T, "dy", torch.float32)
    gain = pro["q_gain"] if use_gain else None
    dx, dwq, dwr, dg = api.flash_mhffn_prologue_bwd(
        pro["x"].cuda(), pro["w_q"].cuda(), pro["w_r"].cuda(), H, E, dq.cuda(), dr.cuda(),
        q_gain=None if gain is None else gain.cuda())
    torch.cuda.synchronize()
    assert api.device_status() == 0
    ref = O.mhffn_prologue_backward(f64(pro["x"]), f64(pro["w_q"]), f64(pro["w_r"]), H, E, f64(dq), f64(dr),
                                    None if gain is None else f64(gain), 1e-6)
    assert_close("dx", f64(dx), ref["dx"], torch.bfloat16)
    assert_close("dw_q", f64(dwq), ref["dw_q"], torch.bfloat16)
    if E > 1:
        assert_close("dw_r", f64(dwr), ref["dw_r"], torch.bfloat16)
    else:
        assert float(dwr.float().abs().max()) < 1e-5  # one sub-network: its weight is always 1
    if use_gain:
        assert_close("dq_gain", f64(dg), ref["dgain"], torch.float32)


def test_prologue_full_size_sampled():
    """The prologue forward and backward at the bench's block configuration (32768 tokens,
    d_model 2048, 16 heads, E = 15): q and router rows and dx on sampled tokens; the dW_q and dW_r
    rows of two heads, each a sum over all tokens that the oracle computes from that head alone."""
    T, d_model, H, E = 32768, 2048, 16, 15
    pro = synth.mhffn_prologue_inputs(T, d_model, H, 128, E, seed=6)
    dq = synth.normal((T, H, 128), 0.1, 6, "do")
    dr = synth.normal((T, H, E), 0.1, 6, "dy", torch.float32)
    g = {k: v.cuda() for k, v in pro.items()}
    q, r = api.flash_mhffn_prologue(g["x"], g["w_q"], g["w_r"], H, E, q_gain=g["q_gain"], eps=1e-6)
    dx, dwq, dwr, _ = api.flash_mhffn_prologue_bwd(g["x"], g["w_q"], g["w_r"], H, E, dq.cuda(), dr.cuda(),
                                                   q_gain=g["q_gain"])
    torch.cuda.synchronize()
    assert api.device_status() == 0
    x, wq, wr, gain = (f64(pro[k]) for k in ("x", "w_q", "w_r", "q_gain"))
    rng = np.random.default_rng(6)
    tokens = np.sort(np.concatenate([rng.choice(T, 24, replace=False), [T - 1]]))
    fw = O.mhffn_prologue_forward(x[tokens], wq, wr, H, E, gain, 1e-6)
    assert_close("q[tokens]", f64(q)[tokens], fw["q"], torch.bfloat16)
    assert_close("router[tokens]", f64(r)[tokens], fw["r"], torch.float32)
    bw = O.mhffn_prologue_backward(x[tokens], wq, wr, H, E, f64(dq)[tokens], f64(dr)[tokens], gain, 1e-6)
    assert_close("dx[tokens]", f64(dx)[tokens], bw["dx"], torch.bfloat16)
    for h in (0, 11):
        qs, rs = slice(h * 128, (h + 1) * 128), slice(h * E, (h + 1) * E)
        sub = O.mhffn_prologue_backward(x, wq[qs], wr[rs], 1, E, f64(dq)[:, [h]], f64(dr)[:, [h]], gain, 1e-6)
        assert_close(f"dw_q[head {h}]", f64(dwq)[qs], sub["dw_q"], torch.bfloat16)
        assert_close(f"dw_r[head {h}]", f64(dwr)[rs], sub["dw_r"], torch.bfloat16)


def test_block_training_step_end_to_end():
    """x -> prologue -> fused core -> O, then dO back to dx and every weight gradient, against
    the oracle's block (prologue and core chained)."""
    T, d_model, H, E, de = 260, 256, 2, 3, 128
    pro = synth.mhffn_prologue_inputs(T, d_model, H, 128, E, seed=41)
    core = synth.mhffn_inputs(T, H, 128, E, de, seed=41)
    g = {k: v.cuda() for k, v in pro.items()}
    c = {k: v.cuda() for k, v in core.items()}
    q, r = api.flash_mhffn_prologue(g["x"], g["w_q"], g["w_r"], H, E, q_gain=g["q_gain"])
    o = api.flash_mhffn_fwd(q, c["w_k"], c["w_u"], c["w_v"], r)
    dq, dk, du, dv, dr = api.flash_mhffn_bwd(q, c["w_k"], c["w_u"], c["w_v"], r, c["do"])
    dx, dwq, dwr, dg = api.flash_mhffn_prologue_bwd(g["x"], g["w_q"], g["w_r"], H, E, dq, dr,
                                                    q_gain=g["q_gain"])
    torch.cuda.synchronize()
    assert api.device_status() == 0
    x, wq, wr, gain = (f64(pro[k]) for k in ("x", "w_q", "w_r", "q_gain"))
    wk, wu, wv, do = (f64(core[k]) for k in ("w_k", "w_u", "w_v", "do"))
    pf = O.mhffn_prologue_forward(x, wq, wr, H, E, gain, 1e-6)
    ref_o = O.mhffn_forward(pf["q"], wk, wu, wv, pf["r"])["o"]
    cb = O.mhffn_backward(pf["q"], wk, wu, wv, pf["r"], do)
    pb = O.mhffn_prologue_backward(x, wq, wr, H, E, cb["dq"], cb["dr"], gain, 1e-6)
    assert_close("o", f64(o), ref_o, torch.bfloat16)
    for name, got, ref in (("dk", dk, cb["dk"]), ("du", du, cb["du"]), ("dv", dv, cb["dv"]),
                           ("dx", dx, pb["dx"]), ("dw_q", dwq, pb["dw_q"]), ("dw_r", dwr, pb["dw_r"]),
                           ("dq_gain", dg, pb["dgain"])):
        assert_close(name, f64(got), ref, torch.bfloat16)

"""GPU parity of the LeakyReLU(0.5)^2 MLP (parameter-golf PR 1105, "Fused MLP Kernels") against
the fp64 oracle through the C ABI: forward (y, post, act_grad) and backward (dx, dW_up, dW_down)."""
import numpy as np
import pytest
import torch

import oracle as O
from swiglu_feed_forward_b200 import api, synth
from tests._util import assert_close, f64

pytestmark = pytest.mark.gpu


def run_and_check(M, d, f, seed, dtype):
    inp = synth.dense_inputs(M, d, f, seed, dtype)
    t = {k: v.cuda() for k, v in inp.items()}
    y, post, ag = api.leaky_relu_sq_mlp_fwd(t["x"], t["w_up"], t["w_down"])
    dx, dwu, dwd = api.leaky_relu_sq_mlp_bwd(t["dy"], t["x"], t["w_up"], t["w_down"], post, ag)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    x, wu, wd, dy = (f64(inp[k]) for k in ("x", "w_up", "w_down", "dy"))
    fw = O.leaky_relu_sq_forward(x, wu, wd)
    bw = O.leaky_relu_sq_backward(x, wu, wd, dy)
    errs = {}
    for name, got, ref in (("y", y, fw["y"]), ("post", post, fw["post"]), ("act_grad", ag, fw["act_grad"]),
                           ("dx", dx, bw["dx"]), ("dw_up", dwu, bw["dw_up"]), ("dw_down", dwd, bw["dw_down"])):
        errs[name] = assert_close(name, f64(got), ref, dtype)
    return errs


def test_page_shape_bf16_full():
    w = synth.WORKLOADS[5]
    errs = run_and_check(16384, w["d_model"], w["d_ff"], w["seed"], torch.bfloat16)
    print({k: f"{v:.2e}" for k, v in errs.items()})


@pytest.mark.parametrize("M,d,f", [(1, 64, 128), (333, 48, 80), (1000, 512, 1792), (260, 272, 400)])
def test_bf16_small_and_ragged(M, d, f):
    run_and_check(M, d, f, 40 + M, torch.bfloat16)


@pytest.mark.parametrize("M,d,f", [(64, 128, 352), (70, 100, 130)])
def test_fp32(M, d, f):
    run_and_check(M, d, f, 50 + M, torch.float32)


def test_full_size_sampled_rows():
    """86016 tokens (the bench's launch configuration): sampled token rows of y and dx."""
    w = synth.WORKLOADS[5]
    inp = synth.workload_inputs(5)
    t = {k: v.cuda() for k, v in inp.items()}
    y, post, ag = api.leaky_relu_sq_mlp_fwd(t["x"], t["w_up"], t["w_down"])
    dx, dwu, dwd = api.leaky_relu_sq_mlp_bwd(t["dy"], t["x"], t["w_up"], t["w_down"], post, ag)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(0).choice(w["M"], 40, replace=False))
    x, wu, wd, dy = (f64(inp[k]) for k in ("x", "w_up", "w_down", "dy"))
    assert_close("y[rows]", f64(y)[rows], O.leaky_relu_sq_forward(x[rows], wu, wd)["y"], torch.bfloat16)
    assert_close("dx[rows]", f64(dx)[rows], O.leaky_relu_sq_backward(x[rows], wu, wd, dy[rows])["dx"],
                 torch.bfloat16)
    cols = np.sort(np.random.default_rng(1).choice(w["d_ff"], 16, replace=False))
    sub = O.leaky_relu_sq_backward(x, wu[cols], wd[:, cols], dy)
    assert_close("dw_up[cols]", f64(dwu)[cols], sub["dw_up"], torch.bfloat16)
    assert_close("dw_down[:,cols]", f64(dwd)[:, cols], sub["dw_down"], torch.bfloat16)

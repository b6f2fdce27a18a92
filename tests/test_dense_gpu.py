"""GPU parity of the dense SwiGLU FFN (forward, inference forward, backward) against the fp64
oracle on the same seeded inputs, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from swiglu_feed_forward_b200 import api, synth
from tests._util import TOL, assert_close, f64

pytestmark = pytest.mark.gpu


def run_dense(inp, dtype):
    dev = {k: v.cuda() for k, v in inp.items()}
    y, h, a, b = api.swiglu_ffn_fwd(dev["x"], dev["w_gate"], dev["w_up"], dev["w_down"])
    y_inf = api.swiglu_ffn_fwd_infer(dev["x"], dev["w_gate"], dev["w_up"], dev["w_down"])
    grads = api.swiglu_ffn_bwd(dev["dy"], dev["x"], dev["w_gate"], dev["w_up"], dev["w_down"], h, a, b)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return dict(y=y, h=h, a=a, b=b, y_inf=y_inf, dx=grads[0], dw_gate=grads[1], dw_up=grads[2],
                dw_down=grads[3])


def check_full(inp, out, dtype):
    x, wg, wu, wd, dy = (f64(inp[k]) for k in ("x", "w_gate", "w_up", "w_down", "dy"))
    fw = O.dense_forward(x, wg, wu, wd)
    bw = O.dense_backward(x, wg, wu, wd, dy)
    errs = {}
    for name, ref in (("y", fw["y"]), ("y_inf", fw["y"]), ("h", fw["h"]), ("a", fw["a"]), ("b", fw["b"]),
                      ("dx", bw["dx"]), ("dw_gate", bw["dw_gate"]), ("dw_up", bw["dw_up"]),
                      ("dw_down", bw["dw_down"])):
        errs[name] = assert_close(name, f64(out[name]), ref, dtype)
    return errs


def test_workload0_fp32_full():
    inp = synth.workload_inputs(0)
    out = run_dense(inp, torch.float32)
    check_full(inp, out, torch.float32)


def test_workload1_bf16_full():
    inp = synth.workload_inputs(1)
    out = run_dense(inp, torch.bfloat16)
    errs = check_full(inp, out, torch.bfloat16)
    print({k: f"{v:.2e}" for k, v in errs.items()})


@pytest.mark.parametrize("M,d,f", [
    (1, 64, 128),       # one token
    (200, 48, 352),     # ragged M, d below one k-block, f with a partial gate|up tile
    (129, 16, 16),      # smallest widths
    (333, 2048, 5504),  # full widths of the 32K-token workload, ragged M
    (512, 768, 2048),
    (260, 272, 400),    # partial 256-wide output tiles everywhere
])
def test_bf16_small_and_ragged(M, d, f):
    inp = synth.dense_inputs(M, d, f, seed=100 + M, dtype=torch.bfloat16)
    out = run_dense(inp, torch.bfloat16)
    check_full(inp, out, torch.bfloat16)


@pytest.mark.parametrize("M,d,f", [(1, 5, 7), (70, 100, 130), (64, 128, 352)])
def test_fp32_odd_shapes(M, d, f):
    inp = synth.dense_inputs(M, d, f, seed=200 + M, dtype=torch.float32)
    out = run_dense(inp, torch.float32)
    check_full(inp, out, torch.float32)


def test_workload2_full_size_sampled():
    """32768 tokens, d_model 2048, d_ff 5504 in the launch configuration the bench times;
    sampled token rows (y, dx) and sampled d_ff rows (dw_gate, dw_up, dw_down columns), each
    computed exactly by the oracle from the inputs it depends on."""
    w = synth.WORKLOADS[2]
    inp = synth.workload_inputs(2)
    out = run_dense(inp, torch.bfloat16)
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(w["M"], 48, replace=False))
    rows = np.concatenate([rows, [0, w["M"] - 1]])
    x, wg, wu, wd, dy = (f64(inp[k]) for k in ("x", "w_gate", "w_up", "w_down", "dy"))
    fw = O.dense_forward(x[rows], wg, wu, wd)
    bw = O.dense_backward(x[rows], wg, wu, wd, dy[rows])
    assert_close("y[rows]", f64(out["y"])[rows], fw["y"], torch.bfloat16)
    assert_close("y_inf[rows]", f64(out["y_inf"])[rows], fw["y"], torch.bfloat16)
    assert_close("h[rows]", f64(out["h"])[rows], fw["h"], torch.bfloat16)
    assert_close("dx[rows]", f64(out["dx"])[rows], bw["dx"], torch.bfloat16)
    cols = np.sort(rng.choice(w["d_ff"], 24, replace=False))
    cols = np.concatenate([cols, [0, w["d_ff"] - 1]])
    sub = O.dense_backward(x, wg[cols], wu[cols], wd[:, cols], dy)
    assert_close("dw_gate[cols]", f64(out["dw_gate"])[cols], sub["dw_gate"], torch.bfloat16)
    assert_close("dw_up[cols]", f64(out["dw_up"])[cols], sub["dw_up"], torch.bfloat16)
    assert_close("dw_down[:,cols]", f64(out["dw_down"])[:, cols], sub["dw_down"], torch.bfloat16)


def test_weight_gradient_last_wave_split_on_a_ragged_edge():
    """d_ff = 1200 at 16384 tokens: [dW_gate ; dW_up] is 2400 x 2048, 80 pair tiles, so its 74
    whole tiles are stored directly and the last six (the ragged 96-row block among them, all in
    dW_up) run as K splits summed per tile; every dW_up row from the split tiles and a sample of
    the others are checked against the oracle over all tokens, and the split tiles' dW_gate
    neighbours too."""
    M, d, f = 16384, 2048, 1200
    inp = synth.dense_inputs(M, d, f, seed=21, dtype=torch.bfloat16)
    dev = {k: v.cuda() for k, v in inp.items()}
    y, h, a, b = api.swiglu_ffn_fwd(dev["x"], dev["w_gate"], dev["w_up"], dev["w_down"])
    dx, dwg, dwu, dwd = api.swiglu_ffn_bwd(dev["dy"], dev["x"], dev["w_gate"], dev["w_up"], dev["w_down"], h, a, b)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    rng = np.random.default_rng(3)
    cols = np.unique(np.concatenate([np.arange(848, 1200, 11), [848, 1199], rng.choice(848, 16, replace=False), [0]]))
    x, wg, wu, wd, dy = (f64(inp[k]) for k in ("x", "w_gate", "w_up", "w_down", "dy"))
    sub = O.dense_backward(x, wg[cols], wu[cols], wd[:, cols], dy)
    assert_close("dw_gate[cols]", f64(dwg)[cols], sub["dw_gate"], torch.bfloat16)
    assert_close("dw_up[cols]", f64(dwu)[cols], sub["dw_up"], torch.bfloat16)
    assert_close("dw_down[:,cols]", f64(dwd)[:, cols], sub["dw_down"], torch.bfloat16)


def test_workload4_inference_full_size_sampled():
    """The inference forward at 262144 tokens x 2048 x 5504, the launch configuration of the
    bench's inference line: sampled token rows against the oracle."""
    w = synth.WORKLOADS[4]
    inp = synth.workload_inputs(4)
    dev = {k: v.cuda() for k, v in inp.items()}
    y = api.swiglu_ffn_fwd_infer(dev["x"], dev["w_gate"], dev["w_up"], dev["w_down"])
    torch.cuda.synchronize()
    assert api.device_status() == 0
    rng = np.random.default_rng(4)
    rows = np.sort(np.concatenate([rng.choice(w["M"], 32, replace=False), [0, w["M"] - 1]]))
    x, wg, wu, wd = (f64(inp[k]) for k in ("x", "w_gate", "w_up", "w_down"))
    assert_close("y[rows]", f64(y)[rows], O.dense_forward(x[rows], wg, wu, wd)["y"], torch.bfloat16)


def test_repeat_calls_are_bitwise_identical():
    inp = synth.dense_inputs(1000, 256, 512, seed=7, dtype=torch.bfloat16)
    o1 = run_dense(inp, torch.bfloat16)
    o2 = run_dense(inp, torch.bfloat16)
    for k in o1:
        assert torch.equal(o1[k], o2[k]), k


def test_bounded_wait_times_out_and_context_survives():
    api.device_status()  # clear
    api.selftest_wait_timeout(2000)
    assert api.device_status() == 6
    assert api.device_status() == 0
    inp = synth.dense_inputs(64, 64, 128, seed=3, dtype=torch.bfloat16)
    out = run_dense(inp, torch.bfloat16)
    check_full(inp, out, torch.bfloat16)

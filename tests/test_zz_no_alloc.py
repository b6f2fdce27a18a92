"""The inference forward that allocates nothing (swiglu_ffn_fwd_infer_noalloc).

It serves callers that cannot give the library device memory for the intermediate h: a host
program that reaches the library only through the C ABI and has no device allocator of its own,
or a plug-in inside a runtime that forbids device allocation on its execution path.  These checks
call it through the C ABI on two calls in a row (the second smaller than the first, so stale
scratch contents from the first call would show) and compare its output with the fp64 oracle
and with the workspace-taking entry point, in bf16 and in fp32, and check that an oversized
call is refused.  The file sorts last so that a run stopping at the first failure has run every
other test."""
import ctypes as C

import pytest
import torch

import oracle as O
from swiglu_feed_forward_b200 import _lib, api, synth
from tests._util import assert_close, f64

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, t, y, M, d, f, dt):
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.swiglu_ffn_fwd_infer_noalloc(
        C.c_void_p(t["x"].data_ptr()), C.c_void_p(t["w_gate"].data_ptr()),
        C.c_void_p(t["w_up"].data_ptr()), C.c_void_p(t["w_down"].data_ptr()),
        C.c_void_p(y.data_ptr()), M, d, f, dt, stream)


@pytest.mark.parametrize("dtype,calls", [
    (torch.bfloat16, [(2000, 512, 4096, 1), (700, 768, 2048, 2)]),
    # fp32 at the small dense workload's shape (64 x 128 -> 352), then a ragged larger one
    (torch.float32, [(300, 96, 1000, 5), (64, 128, 352, 0)]),
])
def test_noalloc_inference_matches_oracle_and_workspace_entry_point_on_two_calls(dtype, calls):
    lib = _lib.lib()
    dt = _lib.SWF_BF16 if dtype == torch.bfloat16 else _lib.SWF_F32
    for (M, d, f, seed) in calls:
        inp = synth.dense_inputs(M, d, f, seed, dtype, with_dy=False)
        t = {k: v.cuda() for k, v in inp.items()}
        y_ws = api.swiglu_ffn_fwd_infer(t["x"], t["w_gate"], t["w_up"], t["w_down"])
        y = torch.full_like(y_ws, float("nan"))
        assert _call_noalloc(lib, t, y, M, d, f, dt) == 0
        torch.cuda.synchronize()
        assert api.device_status() == 0
        ref = O.dense_forward(*(f64(inp[k]) for k in ("x", "w_gate", "w_up", "w_down")))["y"]
        assert_close("y_noalloc vs oracle", f64(y), ref, dtype)
        assert_close("y_noalloc vs swiglu_ffn_fwd_infer", f64(y), f64(y_ws), dtype)


def test_noalloc_refuses_sizes_beyond_its_scratch():
    lib = _lib.lib()
    d, f = 256, 4096
    M = (32 << 20) // (f * 2) + 1  # one token more than the scratch holds
    inp = synth.dense_inputs(M, d, f, 3, torch.bfloat16, with_dy=False)
    t = {k: v.cuda() for k, v in inp.items()}
    y = torch.zeros(M, d, device="cuda", dtype=torch.bfloat16)
    assert _call_noalloc(lib, t, y, M, d, f, _lib.SWF_BF16) == 4  # SWF_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0  # nothing was launched

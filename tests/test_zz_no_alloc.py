"""The inference forward that allocates nothing (swiglu_ffn_fwd_infer_noalloc).

It is for callers that cannot give the library device memory for the intermediate h -- a host
program reaching the library only through the C ABI without a device allocator, a plug-in in a
runtime that forbids allocation on its execution path, or code recording a stream capture where
cudaMalloc is an error.  These checks call it through the C ABI and compare its output with the
workspace-taking entry point on two calls in a row (the second smaller than the first, so stale
scratch contents from the first call would show), and check that an oversized call is refused.
The file sorts last so that a run stopping at the first failure has run every other test."""
import ctypes as C

import pytest
import torch

from swiglu_feed_forward_b200 import _lib, api, synth
from tests._util import assert_close, f64

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, t, y, M, d, f, dt):
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.swiglu_ffn_fwd_infer_noalloc(
        C.c_void_p(t["x"].data_ptr()), C.c_void_p(t["w_gate"].data_ptr()),
        C.c_void_p(t["w_up"].data_ptr()), C.c_void_p(t["w_down"].data_ptr()),
        C.c_void_p(y.data_ptr()), M, d, f, dt, stream)


def test_noalloc_inference_matches_workspace_entry_point_on_two_calls():
    lib = _lib.lib()
    for (M, d, f, seed) in [(2000, 512, 4096, 1), (700, 768, 2048, 2)]:
        inp = synth.dense_inputs(M, d, f, seed, torch.bfloat16, with_dy=False)
        t = {k: v.cuda() for k, v in inp.items()}
        y_ref = api.swiglu_ffn_fwd_infer(t["x"], t["w_gate"], t["w_up"], t["w_down"])
        y = torch.full_like(y_ref, float("nan"))
        assert _call_noalloc(lib, t, y, M, d, f, _lib.SWF_BF16) == 0
        torch.cuda.synchronize()
        assert api.device_status() == 0
        assert_close("y_noalloc", f64(y), f64(y_ref), torch.bfloat16)


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

"""Out-of-bounds write detection in place of compute-sanitizer (closed on this pool).

Every output, saved buffer and workspace a call receives is carved out of a larger device
buffer whose head and tail guard regions hold a sentinel byte; after the call the guards must
be byte-identical.  The outputs themselves start filled with the sentinel too, so an element a
kernel forgot to write fails the comparison with the oracle.  The cases are the ragged ones
(a row count that is not a tile multiple, widths below one k-block, a single token) of every
family: dense bf16 and fp32, inference, the no-allocation inference forward, the LeakyReLU^2
MLP, selection, bucketing, the group-sparse forward and backward (saved buffer and both
workspaces), and FlashFFN's core and prologue.  A group_idx with repeated and out-of-range
slots is covered too: in debug mode the call refuses it before launching anything; otherwise
the bucketing drops those slots and no kernel writes outside its buffers."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle as O
from swiglu_feed_forward_b200 import _lib, api, synth
from tests._util import assert_close, f64

pytestmark = pytest.mark.gpu

GUARD = 1 << 16   # bytes of sentinel before and after every buffer
SENTINEL = 0x7F   # bf16 0x7F7F and fp32 0x7F7F7F7F ~ 3.4e38: an unwritten element fails parity


class Guarded:
    """A tensor of `shape` and `dtype` inside one device buffer with sentinel guards."""

    def __init__(self, shape, dtype, fill=True):
        if isinstance(shape, int):
            shape = (shape,)
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.nbytes = n
        self.buf = torch.full((2 * GUARD + ((n + 255) // 256) * 256,), SENTINEL, dtype=torch.uint8,
                              device="cuda")
        if not fill:
            self.buf[GUARD:GUARD + n].zero_()
        self.t = self.buf[GUARD:GUARD + n].view(dtype).view(shape)

    def intact(self):
        head = self.buf[:GUARD]
        tail = self.buf[GUARD + self.nbytes:]
        return bool(torch.all(head == SENTINEL).item()) and bool(torch.all(tail == SENTINEL).item())


def guarded(**specs):
    return {k: Guarded(*v) for k, v in specs.items()}


def assert_guards(bufs, what):
    torch.cuda.synchronize()
    assert api.device_status() == 0
    bad = [k for k, g in bufs.items() if not g.intact()]
    assert not bad, f"{what}: writes outside {bad}"


def ws_guard(op, M, d, f, G=0, K=0, dtype=torch.bfloat16):
    return Guarded(max(16, api.workspace_bytes(op, M, d, f, G, K, dtype)), torch.uint8)


@pytest.mark.parametrize("M,d,f,dtype", [
    (333, 272, 560, torch.bfloat16),   # ragged M, d not a k-block multiple
    (1, 48, 96, torch.bfloat16),       # one token, d below one k-block
    (67, 100, 350, torch.float32),     # fp32 any sizes
])
def test_dense_train_and_infer_write_only_their_outputs(M, d, f, dtype):
    inp = synth.dense_inputs(M, d, f, seed=M + d, dtype=dtype)
    t = {k: v.cuda() for k, v in inp.items()}
    g = guarded(y=((M, d), dtype), h=((M, f), dtype), a=((M, f), dtype), b=((M, f), dtype),
                dx=((M, d), dtype), dwg=((f, d), dtype), dwu=((f, d), dtype), dwd=((d, f), dtype),
                yi=((M, d), dtype), yn=((M, d), dtype))
    g["ws"] = ws_guard("bwd", M, d, f, dtype=dtype)
    g["wsi"] = ws_guard("fwd_infer", M, d, f, dtype=dtype)
    api.swiglu_ffn_fwd(t["x"], t["w_gate"], t["w_up"], t["w_down"], g["y"].t, g["h"].t, g["a"].t, g["b"].t)
    api.swiglu_ffn_bwd(t["dy"], t["x"], t["w_gate"], t["w_up"], t["w_down"], g["h"].t, g["a"].t, g["b"].t,
                       g["dx"].t, g["dwg"].t, g["dwu"].t, g["dwd"].t, workspace=g["ws"].t)
    api.swiglu_ffn_fwd_infer(t["x"], t["w_gate"], t["w_up"], t["w_down"], g["yi"].t, workspace=g["wsi"].t)
    dt = _lib.SWF_BF16 if dtype == torch.bfloat16 else _lib.SWF_F32
    st = _lib.lib().swiglu_ffn_fwd_infer_noalloc(
        *(C.c_void_p(t[k].data_ptr()) for k in ("x", "w_gate", "w_up", "w_down")),
        C.c_void_p(g["yn"].t.data_ptr()), M, d, f, dt, C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    assert_guards(g, "dense")
    x, wg, wu, wd, dy = (f64(inp[k]) for k in ("x", "w_gate", "w_up", "w_down", "dy"))
    fw, bw = O.dense_forward(x, wg, wu, wd), O.dense_backward(x, wg, wu, wd, dy)
    for k in ("y", "yi", "yn"):
        assert_close(k, f64(g[k].t), fw["y"], dtype)
    for k, ref in (("dx", "dx"), ("dwg", "dw_gate"), ("dwu", "dw_up"), ("dwd", "dw_down")):
        assert_close(k, f64(g[k].t), bw[ref], dtype)


def test_mlp2_writes_only_its_outputs():
    M, d, f = 301, 80, 208
    inp = synth.dense_inputs(M, d, f, seed=4, dtype=torch.bfloat16)
    t = {k: v.cuda() for k, v in inp.items()}
    bf = torch.bfloat16
    g = guarded(y=((M, d), bf), post=((M, f), bf), ag=((M, f), bf), dx=((M, d), bf),
                dwu=((f, d), bf), dwd=((d, f), bf))
    g["ws"] = ws_guard("mlp2_bwd", M, d, f)
    api.leaky_relu_sq_mlp_fwd(t["x"], t["w_up"], t["w_down"], g["y"].t, g["post"].t, g["ag"].t)
    api.leaky_relu_sq_mlp_bwd(t["dy"], t["x"], t["w_up"], t["w_down"], g["post"].t, g["ag"].t,
                              g["dx"].t, g["dwu"].t, g["dwd"].t, workspace=g["ws"].t)
    assert_guards(g, "mlp2")
    ref = O.leaky_relu_sq_forward(*(f64(inp[k]) for k in ("x", "w_up", "w_down")))
    assert_close("y", f64(g["y"].t), ref["y"], bf)


def sparse_guarded_step(inp, idx_dev, G, K):
    M, d = inp["x"].shape
    f = inp["w_gate"].shape[0]
    t = {k: v.cuda() for k, v in inp.items()}
    bf = torch.bfloat16
    g = guarded(y=((M, d), bf), dx=((M, d), bf), dwg=((f, d), bf), dwu=((f, d), bf), dwd=((d, f), bf))
    g["saved"] = Guarded(max(16, api.sparse_saved_bytes(M, d, f, G, K)), torch.uint8)
    g["wsf"] = ws_guard("sparse_fwd", M, d, f, G, K)
    g["wsb"] = ws_guard("sparse_bwd", M, d, f, G, K)
    api.sparse_swiglu_ffn_fwd(t["x"], t["w_gate"], t["w_up"], t["w_down"], idx_dev, G, g["y"].t,
                              g["saved"].t, g["wsf"].t)
    api.sparse_swiglu_ffn_bwd(t["dy"], t["x"], t["w_gate"], t["w_up"], t["w_down"], idx_dev, G,
                              g["saved"].t, g["dx"].t, g["dwg"].t, g["dwu"].t, g["dwd"].t, g["wsb"].t)
    return g


def check_sparse_outputs(g, inp, idx, G):
    x, wg, wu, wd, dy = (f64(inp[k]) for k in ("x", "w_gate", "w_up", "w_down", "dy"))
    fw = O.sparse_forward(x, wg, wu, wd, idx, G)
    bw = O.sparse_backward(x, wg, wu, wd, idx, G, dy)
    assert_close("y", f64(g["y"].t), fw["y"], torch.bfloat16)
    for k, ref in (("dx", "dx"), ("dwg", "dw_gate"), ("dwu", "dw_up"), ("dwd", "dw_down")):
        assert_close(k, f64(g[k].t), bw[ref], torch.bfloat16)


@pytest.mark.parametrize("M,d,f,G,K,spg", [
    (513, 48, 1024, 64, 5, 8),    # ragged M, d below one k-block
    (1, 64, 256, 16, 2, None),    # one token, exact energies
    (300, 272, 768, 32, 24, 3),   # K = all groups
    (2048, 2048, 4096, 64, 8, 8),  # per-pair rows of whole 128-byte lines (dropped from L2 once summed)
])
def test_selection_and_sparse_write_only_their_buffers(M, d, f, G, K, spg):
    inp = synth.dense_inputs(M, d, f, seed=M + G, dtype=torch.bfloat16)
    x, wg = inp["x"].cuda(), inp["w_gate"].cuda()
    ng = f // G
    sub = None if spg is None else torch.from_numpy(O.make_subsample_index(f, G, spg, 3)).cuda()
    bias = synth.balance_bias(ng, 5).cuda()
    g = guarded(idx=((M, K), torch.int32), E=((M, ng), torch.float32))
    g["ws"] = ws_guard("select", M, d, f, G, K)
    api.grouped_topk_select(x, wg, G, K, subsample_idx=sub, samples_per_group=spg,
                            load_balance_bias=bias, group_idx=g["idx"].t, energies=g["E"].t,
                            workspace=g["ws"].t)
    assert_guards(g, "selection")
    idx = g["idx"].t.cpu().numpy()
    np.testing.assert_array_equal(idx, O.topk_groups(g["E"].t.cpu().numpy().astype(np.float64), K))
    # bucketing through its own entry point
    gb = guarded(offs=((ng + 1,), torch.int32), toks=((M * K,), torch.int32))
    gb["ws"] = Guarded(max(16, _lib.lib().swf_workspace_bytes(_lib.OPS["buckets"], M, 0, 0, ng, K,
                                                               _lib.SWF_BF16)), torch.uint8)
    api.swf_group_buckets(g["idx"].t, ng, gb["offs"].t, gb["toks"].t, gb["ws"].t)
    assert_guards(gb, "buckets")
    ro, rt = O.csr_buckets(idx, ng)
    np.testing.assert_array_equal(gb["offs"].t.cpu().numpy(), ro)
    np.testing.assert_array_equal(gb["toks"].t.cpu().numpy(), rt)
    gs = sparse_guarded_step(inp, g["idx"].t, G, K)
    assert_guards(gs, "sparse")
    check_sparse_outputs(gs, inp, idx, G)


def bad_group_idx(M, K, ng, seed):
    """Distinct in-range rows, then a repeated slot in some rows and an out-of-range one in
    others; also the same rows with the bad slots replaced by repeats (what the kernels use)."""
    rng = np.random.default_rng(seed)
    idx = np.sort(np.stack([rng.choice(ng, size=K, replace=False) for _ in range(M)]), axis=1).astype(np.int32)
    bad = idx.copy()
    bad[3, 1] = bad[3, 0]           # repeated
    bad[10, K - 1] = ng             # out of range (high)
    bad[11, 0] = -5                 # out of range (negative)
    bad[M - 1, 2] = bad[M - 1, 1]   # repeated in the last row
    eff = bad.copy()                # the oracle's reading: a dropped slot adds nothing
    for r in range(M):
        for k in range(K):
            if not (0 <= eff[r, k] < ng):
                eff[r, k] = eff[r, [j for j in range(K) if 0 <= bad[r, j] < ng][0]]
    return bad, eff, 4


def test_invalid_group_idx_refused_in_debug_mode_and_dropped_otherwise():
    M, d, f, G, K = 200, 64, 512, 32, 4
    ng = f // G
    bad, eff, n_bad = bad_group_idx(M, K, ng, 1)
    inp = synth.dense_inputs(M, d, f, seed=2, dtype=torch.bfloat16)
    bad_dev = torch.from_numpy(bad).cuda()
    st, count = api.validate_group_idx(bad_dev, ng)
    assert (st, count) == (1, n_bad)
    good = np.tile(np.arange(K, dtype=np.int32), (M, 1))
    assert api.validate_group_idx(torch.from_numpy(good).cuda(), ng) == (0, 0)
    prev = api.get_debug()
    try:
        api.set_debug(True)
        g = guarded(y=((M, d), torch.bfloat16))
        g["saved"] = Guarded(max(16, api.sparse_saved_bytes(M, d, f, G, K)), torch.uint8)
        g["ws"] = ws_guard("sparse_fwd", M, d, f, G, K)
        t = {k: v.cuda() for k, v in inp.items()}
        before = g["y"].buf.clone()
        with pytest.raises(api.SwfError) as e:
            api.sparse_swiglu_ffn_fwd(t["x"], t["w_gate"], t["w_up"], t["w_down"], bad_dev, G,
                                      g["y"].t, g["saved"].t, g["ws"].t)
        assert e.value.status == 1
        with pytest.raises(api.SwfError):
            api.swf_group_buckets(bad_dev, ng)
        with pytest.raises(api.SwfError):
            api.group_frequency(bad_dev, ng)
        torch.cuda.synchronize()
        assert torch.equal(g["y"].buf, before)  # nothing launched: the output is untouched
        api.set_debug(False)
        gs = sparse_guarded_step(inp, bad_dev, G, K)
        assert_guards(gs, "sparse with dropped slots")
        check_sparse_outputs(gs, inp, eff, G)
    finally:
        api.set_debug(prev)


def test_tokens_without_valid_slots_get_zero_rows_and_runs_repeat_bitwise():
    """Whole 64-token chunks and a few single tokens whose every slot is out of range: the
    bucketing drops them, so the per-token sums of the down and dx GEMMs never hear of them and
    must still write their zero rows.  The rest must match the oracle on the valid tokens alone,
    and a second run must reproduce every output bit for bit (the sums take a fixed order
    whichever CTA ends up summing a chunk)."""
    M, d, f, G, K = 300, 256, 1024, 64, 4
    ng = f // G
    rng = np.random.default_rng(7)
    idx = np.sort(np.stack([rng.choice(ng, size=K, replace=False) for _ in range(M)]), axis=1).astype(np.int32)
    dead = np.zeros(M, bool)
    dead[64:192] = True       # chunks 1 and 2
    dead[250:260] = True      # part of a chunk
    dead[M - 1] = True        # the last token
    idx[dead] = -1
    inp = synth.dense_inputs(M, d, f, seed=11, dtype=torch.bfloat16)
    idx_dev = torch.from_numpy(idx).cuda()
    g1 = sparse_guarded_step(inp, idx_dev, G, K)
    assert_guards(g1, "sparse with empty tokens")
    g2 = sparse_guarded_step(inp, idx_dev, G, K)
    assert_guards(g2, "sparse with empty tokens, second run")
    for k in ("y", "dx", "dwg", "dwu", "dwd"):
        assert torch.equal(g1[k].t, g2[k].t), f"{k} differs between two runs"
    for k in ("y", "dx"):
        assert torch.count_nonzero(g1[k].t[torch.from_numpy(dead).cuda()]).item() == 0, f"{k} rows of empty tokens"
    live = ~dead
    x, wg, wu, wd, dy = (f64(inp[k]) for k in ("x", "w_gate", "w_up", "w_down", "dy"))
    fw = O.sparse_forward(x[live], wg, wu, wd, idx[live], G)
    bw = O.sparse_backward(x[live], wg, wu, wd, idx[live], G, dy[live])
    assert_close("y", f64(g1["y"].t)[live], fw["y"], torch.bfloat16)
    assert_close("dx", f64(g1["dx"].t)[live], bw["dx"], torch.bfloat16)
    for k, ref in (("dwg", "dw_gate"), ("dwu", "dw_up"), ("dwd", "dw_down")):
        assert_close(k, f64(g1[k].t), bw[ref], torch.bfloat16)


def test_flashffn_core_and_prologue_write_only_their_buffers():
    T, H, dh, E, de = 300, 2, 128, 3, 128
    bf = torch.bfloat16
    inp = synth.mhffn_inputs(T, H, dh, E, de, 8)
    t = {k: v.cuda() for k, v in inp.items()}
    g = guarded(o=((T, H, dh), bf), dq=((T, H, dh), bf), dk=((H, E, de, dh), bf), du=((H, E, de, dh), bf),
                dv=((H, E, de, dh), bf), dr=((T, H, E), torch.float32))
    g["ws"] = Guarded(max(16, api.flash_mhffn_bwd_workspace_bytes(T, H, dh, E, de)), torch.uint8)
    api.flash_mhffn_fwd(t["q"], t["w_k"], t["w_u"], t["w_v"], t["router"], g["o"].t)
    api.flash_mhffn_bwd(t["q"], t["w_k"], t["w_u"], t["w_v"], t["router"], t["do"], g["dq"].t, g["dk"].t,
                        g["du"].t, g["dv"].t, g["dr"].t, g["ws"].t)
    assert_guards(g, "flashffn core")
    ref = O.mhffn_forward(*(f64(inp[k]) for k in ("q", "w_k", "w_u", "w_v", "router")))["o"]
    assert_close("o", f64(g["o"].t), ref, bf)
    d_model = H * dh
    pro = {k: v.cuda() for k, v in synth.mhffn_prologue_inputs(T, d_model, H, dh, E, 8).items()}
    gp = guarded(q=((T, H, dh), bf), r=((T, H, E), torch.float32), dx=((T, d_model), bf),
                 dwq=(tuple(pro["w_q"].shape), bf), dwr=(tuple(pro["w_r"].shape), bf),
                 dgain=((dh,), torch.float32))
    gp["ws"] = Guarded(max(16, api.flash_mhffn_prologue_bwd_workspace_bytes(T, d_model, H, dh, E)), torch.uint8)
    api.flash_mhffn_prologue(pro["x"], pro["w_q"], pro["w_r"], H, E, q_gain=pro["q_gain"], q=gp["q"].t,
                             router=gp["r"].t)
    api.flash_mhffn_prologue_bwd(pro["x"], pro["w_q"], pro["w_r"], H, E, g["dq"].t, g["dr"].t,
                                 q_gain=pro["q_gain"], dx=gp["dx"].t, dw_q=gp["dwq"].t, dw_r=gp["dwr"].t,
                                 dq_gain=gp["dgain"].t, workspace=gp["ws"].t)
    assert_guards(gp, "flashffn prologue")
    assert torch.isfinite(gp["dx"].t.float()).all()

"""Run one operation of the library on seeded synthetic inputs and print per-kernel timings.

python -m swiglu_feed_forward_b200.run_case --op fwd --M 32768 --d 2048 --f 5504 [--reps 5]
python -m swiglu_feed_forward_b200.run_case --op sparse_step --M 16384 --d 1024 --f 4096 \
    --G 64 --K 8 --spg 8

Ops: fwd, fwd_infer, bwd (fwd once, then timed bwd), step (fwd + bwd), select, sparse_step
(select + sparse fwd + sparse bwd), mhffn_fwd, mhffn_bwd (FlashFFN block core, --T --H --E --de).  Each rep is timed with CUDA events; the per-kernel split
comes from the library's profiling hooks.  Also a convenient target for ncu (-k regex:...)."""
from __future__ import annotations

import argparse
import json

import torch

from . import api, synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", default="step",
                    choices=["fwd", "fwd_infer", "bwd", "step", "select", "sparse_step", "mlp2_step",
                             "mhffn_fwd", "mhffn_bwd"])
    ap.add_argument("--M", type=int, default=32768)
    ap.add_argument("--d", type=int, default=2048)
    ap.add_argument("--f", type=int, default=5504)
    ap.add_argument("--G", type=int, default=64)
    ap.add_argument("--K", type=int, default=8)
    ap.add_argument("--spg", type=int, default=8)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--T", type=int, default=32768)   # mhffn_fwd: tokens, heads, sub-networks, width
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--E", type=int, default=15)
    ap.add_argument("--de", type=int, default=384)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--reps", type=int, default=5)
    a = ap.parse_args()
    dev = torch.device("cuda")
    if a.op in ("mhffn_fwd", "mhffn_bwd"):
        return run_mhffn(a, dev)
    M, d, f, G, K = a.M, a.d, a.f, a.G, a.K
    inp = synth.dense_inputs(M, d, f, a.seed, torch.bfloat16)
    t = {k: v.to(dev) for k, v in inp.items()}
    e = lambda *s: torch.empty(*s, device=dev, dtype=torch.bfloat16)
    y, h, ga, gb, dx = e(M, d), e(M, f), e(M, f), e(M, f), e(M, d)
    dwg, dwu, dwd = e(f, d), e(f, d), e(d, f)
    ws = torch.empty(max(16, api.workspace_bytes("bwd", M, d, f), api.workspace_bytes("fwd_infer", M, d, f)),
                     device=dev, dtype=torch.uint8)
    ops = {}
    ops["fwd"] = lambda: api.swiglu_ffn_fwd(t["x"], t["w_gate"], t["w_up"], t["w_down"], y, h, ga, gb)
    ops["fwd_infer"] = lambda: api.swiglu_ffn_fwd_infer(t["x"], t["w_gate"], t["w_up"], t["w_down"], y, ws)
    ops["bwd"] = lambda: api.swiglu_ffn_bwd(t["dy"], t["x"], t["w_gate"], t["w_up"], t["w_down"], h, ga, gb,
                                            dx, dwg, dwu, dwd, ws)
    ops["step"] = lambda: (ops["fwd"](), ops["bwd"]())
    ws2 = torch.empty(max(16, api.workspace_bytes("mlp2_bwd", M, d, f)), device=dev, dtype=torch.uint8)
    ops["mlp2_step"] = lambda: (
        api.leaky_relu_sq_mlp_fwd(t["x"], t["w_up"], t["w_down"], y, h, ga),
        api.leaky_relu_sq_mlp_bwd(t["dy"], t["x"], t["w_up"], t["w_down"], h, ga, dx, dwu, dwd, ws2))
    if a.op in ("select", "sparse_step"):
        ng = f // G
        sub, _ = api.make_subsample_index(f, G, a.spg, a.seed)
        sub = sub.to(dev)
        bias = synth.balance_bias(ng, a.seed).to(dev)
        idx = torch.empty(M, K, device=dev, dtype=torch.int32)
        wsel = torch.empty(max(16, api.workspace_bytes("select", M, d, f, G, K)), device=dev, dtype=torch.uint8)
        wsf = torch.empty(max(16, api.workspace_bytes("sparse_fwd", M, d, f, G, K)), device=dev, dtype=torch.uint8)
        wsb = torch.empty(max(16, api.workspace_bytes("sparse_bwd", M, d, f, G, K)), device=dev, dtype=torch.uint8)
        saved = torch.empty(max(16, api.sparse_saved_bytes(M, d, f, G, K)), device=dev, dtype=torch.uint8)
        ops["select"] = lambda: api.grouped_topk_select(t["x"], t["w_gate"], G, K, subsample_idx=sub,
                                                        samples_per_group=a.spg, load_balance_bias=bias,
                                                        group_idx=idx, workspace=wsel)

        def sparse_step():
            ops["select"]()
            api.sparse_swiglu_ffn_fwd(t["x"], t["w_gate"], t["w_up"], t["w_down"], idx, G, y, saved, wsf)
            api.sparse_swiglu_ffn_bwd(t["dy"], t["x"], t["w_gate"], t["w_up"], t["w_down"], idx, G, saved,
                                      dx, dwg, dwu, dwd, wsb)
        ops["sparse_step"] = sparse_step
    if a.op == "bwd":
        ops["fwd"]()
    fn = ops[a.op]
    for _ in range(a.warmup):
        fn()
    torch.cuda.synchronize()
    api.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    kern = api.profile_read()
    api.profile_enable(False)
    status = api.device_status()
    ms = e0.elapsed_time(e1) / a.reps
    out = {"op": a.op, "M": M, "d": d, "f": f, "ms_per_rep": round(ms, 4), "status": status,
           "kernels": {k: {"launches": n, "avg_ms": round(v / n, 4), "share": round(v / max(1e-9, sum(x for _, x in kern.values())), 4)}
                       for k, (n, v) in sorted(kern.items(), key=lambda kv: -kv[1][1])}}
    print(json.dumps(out))
    return 0 if status == 0 else 1


def timed_reps(fn, a):
    for _ in range(a.warmup):
        fn()
    torch.cuda.synchronize()
    api.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    kern = api.profile_read()
    api.profile_enable(False)
    return e0.elapsed_time(e1) / a.reps, kern


def run_mhffn(a, dev):
    bwd = a.op == "mhffn_bwd"
    inp = synth.mhffn_inputs(a.T, a.H, 128, a.E, a.de, a.seed, with_do=bwd)
    t = {k: v.to(dev) for k, v in inp.items()}
    if bwd:
        ws = torch.empty(max(16, api.flash_mhffn_bwd_workspace_bytes(a.T, a.H, 128, a.E, a.de)),
                         device=dev, dtype=torch.uint8)
        outs = [torch.empty_like(t[k]) for k in ("q", "w_k", "w_u", "w_v", "router")]
        fn = lambda: api.flash_mhffn_bwd(t["q"], t["w_k"], t["w_u"], t["w_v"], t["router"], t["do"],
                                         *outs, workspace=ws)
        flops = 16.0 * a.T * a.H * 128 * a.E * a.de
    else:
        o = torch.empty_like(t["q"])
        fn = lambda: api.flash_mhffn_fwd(t["q"], t["w_k"], t["w_u"], t["w_v"], t["router"], o)
        flops = 6.0 * a.T * a.H * 128 * a.E * a.de
    ms, kern = timed_reps(fn, a)
    status = api.device_status()
    print(json.dumps({"op": a.op, "T": a.T, "H": a.H, "E": a.E, "de": a.de,
                      "ms_per_rep": round(ms, 4), "tflops": round(flops / (ms / 1e3) / 1e12, 1),
                      "status": status,
                      "kernels": {k: {"launches": n, "avg_ms": round(v / n, 4)} for k, (n, v) in kern.items()}}))
    return 0 if status == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())

"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This module holds no arithmetic of the method: it only draws random tensors
with the shapes and value distributions of the workloads (x ~ N(0, 1),
dY ~ N(0, 1e-2) read as a variance, weights ~ N(0, 1/fan_in) as in the
eugen_sparse README's quick start, balancing bias ~ U(-0.1, 0.1)) and rounds
them to the compute dtype.  Each tensor has its own torch CPU generator seeded
from (workload seed, tensor id), so a tensor does not depend on the sizes of
the others.  It imports nothing else from the package.
"""
from __future__ import annotations

import torch

# Workloads: shapes of the pages' SwiGLU configurations (FlashFFN model table:
# d_model 768/2048 with d_ff 2048/5504, batch 8 at 2K-32K tokens per sequence)
# and of the eugen_sparse training setting (d_ff 4096, 64 groups, 8 active).
WORKLOADS = {
    0: dict(name="dense_f32_m64_d128_f352", kind="dense", dtype="f32",
            M=64, d_model=128, d_ff=352, seed=0),
    1: dict(name="dense_bf16_m16384_d768_f2048", kind="dense", dtype="bf16",
            M=16384, d_model=768, d_ff=2048, seed=1),
    2: dict(name="dense_bf16_m32768_d2048_f5504", kind="dense", dtype="bf16",
            M=32768, d_model=2048, d_ff=5504, seed=2),
    3: dict(name="sparse_bf16_m16384_d1024_f4096_g64_k8_spg8", kind="sparse",
            dtype="bf16", M=16384, d_model=1024, d_ff=4096, group_size=64,
            num_active_groups=8, samples_per_group=8, seed=3),
    4: dict(name="infer_bf16_m262144_d2048_f5504", kind="infer", dtype="bf16",
            M=262144, d_model=2048, d_ff=5504, seed=4),
    # parameter-golf PR 1105's MLP: d_model 512, hidden 1792 (3.5x), LeakyReLU(0.5)^2; its
    # "302 MB intermediate" of [tokens, 1792] bf16 is about 86K tokens
    5: dict(name="leaky_relu_sq_mlp_bf16_m86016_d512_f1792", kind="mlp2", dtype="bf16",
            M=86016, d_model=512, d_ff=1792, seed=5),
    # FlashFFN's 1.3B configuration (d_model 2048 = 16 heads x d_h 128, E = 15 sub-networks,
    # intermediate size 5760 = 15 x 384 per head) at batch 8 x 4096 tokens
    6: dict(name="flashffn_bf16_t32768_h16_dh128_e15_de384", kind="mhffn", dtype="bf16",
            T=32768, H=16, d_h=128, E=15, d_e=384, seed=6),
}

_TENSOR_IDS = {"x": 1, "w_gate": 2, "w_up": 3, "w_down": 4, "dy": 5, "bias": 6,
               "q": 7, "w_k": 8, "w_u": 9, "w_v": 10, "router": 11, "do": 12,
               "w_q": 13, "w_r": 14, "q_gain": 15}

DY_STD = 0.1  # N(0, 1e-2) as a variance


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _gen(seed: int, tensor: str) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1_000_003 + _TENSOR_IDS[tensor])
    return g


def normal(shape, std, seed, tensor, dtype=torch.bfloat16):
    """std * N(0, 1) drawn in fp32 and rounded (nearest-even) to ``dtype``."""
    t = torch.randn(*shape, generator=_gen(seed, tensor), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def dense_inputs(M, d_model, d_ff, seed, dtype=torch.bfloat16, with_dy=True):
    """x [M, d_model], w_gate / w_up [d_ff, d_model], w_down [d_model, d_ff]
    (nn.Linear layout), dy [M, d_model]; CPU tensors."""
    out = {
        "x": normal((M, d_model), 1.0, seed, "x", dtype),
        "w_gate": normal((d_ff, d_model), d_model ** -0.5, seed, "w_gate", dtype),
        "w_up": normal((d_ff, d_model), d_model ** -0.5, seed, "w_up", dtype),
        "w_down": normal((d_model, d_ff), d_ff ** -0.5, seed, "w_down", dtype),
    }
    if with_dy:
        out["dy"] = normal((M, d_model), DY_STD, seed, "dy", dtype)
    return out


def balance_bias(num_groups, seed, lo=-0.1, hi=0.1):
    """Per-group load-balance bias ~ U(lo, hi), fp32."""
    u = torch.rand(num_groups, generator=_gen(seed, "bias"), dtype=torch.float32)
    return u * (hi - lo) + lo


def mhffn_inputs(T, H, d_h, E, d_e, seed, dtype=torch.bfloat16, with_do=True):
    """Multi-head FFN inputs: q [T, H, d_h] ~ N(0, 1) (unit RMS, as after the per-head norm);
    w_k, w_u [H, E, d_e, d_h] ~ N(0, 1/d_h); w_v [H, E, d_e, d_h] ~ N(0, 1/d_e); router
    [T, H, E] fp32, positive and summing to one over E (U(0.05, 1) draws divided by their sum);
    do [T, H, d_h] ~ N(0, 1e-2).  CPU tensors."""
    u = torch.rand(T, H, E, generator=_gen(seed, "router"), dtype=torch.float32) * 0.95 + 0.05
    out = {
        "q": normal((T, H, d_h), 1.0, seed, "q", dtype),
        "w_k": normal((H, E, d_e, d_h), d_h ** -0.5, seed, "w_k", dtype),
        "w_u": normal((H, E, d_e, d_h), d_h ** -0.5, seed, "w_u", dtype),
        "w_v": normal((H, E, d_e, d_h), d_e ** -0.5, seed, "w_v", dtype),
        "router": u / u.sum(-1, keepdim=True),
    }
    if with_do:
        out["do"] = normal((T, H, d_h), DY_STD, seed, "do", dtype)
    return out


def mhffn_prologue_inputs(T, d_model, H, d_h, E, seed, dtype=torch.bfloat16):
    """Inputs of the multi-head block's prologue: x [T, d_model] ~ N(0, 1); w_q [H*d_h, d_model]
    and w_r [H*E, d_model] ~ N(0, 1/d_model); q_gain [d_h] fp32 ~ U(0.5, 1.5).  CPU tensors."""
    return {
        "x": normal((T, d_model), 1.0, seed, "x", dtype),
        "w_q": normal((H * d_h, d_model), d_model ** -0.5, seed, "w_q", dtype),
        "w_r": normal((H * E, d_model), d_model ** -0.5, seed, "w_r", dtype),
        "q_gain": torch.rand(d_h, generator=_gen(seed, "q_gain"), dtype=torch.float32) + 0.5,
    }


def skewed_balance_bias(num_groups, seed):
    """The load-imbalance variant of the group-sparse workload: the U(-0.1, 0.1) bias with groups
    0 and 1 raised to +0.5 and groups 2 and 3 lowered to -0.5."""
    b = balance_bias(num_groups, seed)
    b[:2] = 0.5
    b[2:4] = -0.5
    return b


def workload_inputs(cfg_id: int, with_dy=True):
    w = WORKLOADS[cfg_id]
    return dense_inputs(w["M"], w["d_model"], w["d_ff"], w["seed"],
                        torch_dtype(w["dtype"]), with_dy=with_dy and w["kind"] != "infer")

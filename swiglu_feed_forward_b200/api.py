"""Python binding of the C ABI: same names as include/swiglu_ffn.h, argument marshalling only.

Tensors are torch CUDA tensors (PyTorch supplies device memory and the stream); every step of
the computation runs in the library's CUDA kernels.  Output tensors may be passed in; those
left as None are allocated with torch.empty.  A non-OK status raises SwfError."""
from __future__ import annotations

import ctypes as C

import torch

from . import _lib
from ._lib import OPS, SWF_BF16, SWF_F32, swf_plan_info


class SwfError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = _lib.lib().swf_status_string(status)
        super().__init__(f"{fn}: {msg.decode() if msg else status}")
        self.status = status


def _check(fn: str, status: int) -> None:
    if status != _lib.SWF_OK:
        raise SwfError(fn, status)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SWF_BF16
    if t.dtype == torch.float32:
        return SWF_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _p(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _empty(shape, like, dtype=None):
    return torch.empty(shape, device=like.device, dtype=dtype or like.dtype)


def _workspace(op, M, d, f, G, K, dt, like, workspace):
    n = _lib.lib().swf_workspace_bytes(OPS[op], M, d, f, G, K, dt)
    if workspace is None:
        workspace = torch.empty(max(n, 16), device=like.device, dtype=torch.uint8)
    return workspace, workspace.numel() * workspace.element_size()


# ------------------------------------------------------------------ dense
def swiglu_ffn_fwd(x, w_gate, w_up, w_down, y=None, saved_h=None, saved_a=None, saved_b=None,
                   stream=None):
    """Training forward: returns (y, saved_h, saved_a, saved_b)."""
    M, d = x.shape
    f = w_gate.shape[0]
    y = _empty((M, d), x) if y is None else y
    saved_h = _empty((M, f), x) if saved_h is None else saved_h
    saved_a = _empty((M, f), x) if saved_a is None else saved_a
    saved_b = _empty((M, f), x) if saved_b is None else saved_b
    _check("swiglu_ffn_fwd", _lib.lib().swiglu_ffn_fwd(
        _p(x), _p(w_gate), _p(w_up), _p(w_down), _p(y), _p(saved_h), _p(saved_a), _p(saved_b),
        M, d, f, _dt(x), _stream(stream)))
    return y, saved_h, saved_a, saved_b


def swiglu_ffn_fwd_infer(x, w_gate, w_up, w_down, y=None, workspace=None, stream=None):
    M, d = x.shape
    f = w_gate.shape[0]
    y = _empty((M, d), x) if y is None else y
    ws, nb = _workspace("fwd_infer", M, d, f, 0, 0, _dt(x), x, workspace)
    _check("swiglu_ffn_fwd_infer", _lib.lib().swiglu_ffn_fwd_infer(
        _p(x), _p(w_gate), _p(w_up), _p(w_down), _p(y), _p(ws), nb, M, d, f, _dt(x),
        _stream(stream)))
    return y


def swiglu_ffn_bwd(dy, x, w_gate, w_up, w_down, saved_h, saved_a, saved_b, dx=None, dw_gate=None,
                   dw_up=None, dw_down=None, workspace=None, stream=None):
    """Backward: returns (dx, dw_gate, dw_up, dw_down)."""
    M, d = x.shape
    f = w_gate.shape[0]
    dx = _empty((M, d), x) if dx is None else dx
    dw_gate = _empty((f, d), x) if dw_gate is None else dw_gate
    dw_up = _empty((f, d), x) if dw_up is None else dw_up
    dw_down = _empty((d, f), x) if dw_down is None else dw_down
    ws, nb = _workspace("bwd", M, d, f, 0, 0, _dt(x), x, workspace)
    _check("swiglu_ffn_bwd", _lib.lib().swiglu_ffn_bwd(
        _p(dy), _p(x), _p(w_gate), _p(w_up), _p(w_down), _p(saved_h), _p(saved_a), _p(saved_b),
        _p(dx), _p(dw_gate), _p(dw_up), _p(dw_down), _p(ws), nb, M, d, f, _dt(x),
        _stream(stream)))
    return dx, dw_gate, dw_up, dw_down


# ------------------------------------------------------------------ LeakyReLU(0.5)^2 MLP
def leaky_relu_sq_mlp_fwd(x, w_up, w_down, y=None, saved_post=None, saved_act_grad=None, stream=None):
    """Returns (y, saved_post, saved_act_grad)."""
    M, d = x.shape
    f = w_up.shape[0]
    y = _empty((M, d), x) if y is None else y
    saved_post = _empty((M, f), x) if saved_post is None else saved_post
    saved_act_grad = _empty((M, f), x) if saved_act_grad is None else saved_act_grad
    _check("leaky_relu_sq_mlp_fwd", _lib.lib().leaky_relu_sq_mlp_fwd(
        _p(x), _p(w_up), _p(w_down), _p(y), _p(saved_post), _p(saved_act_grad), M, d, f, _dt(x),
        _stream(stream)))
    return y, saved_post, saved_act_grad


def leaky_relu_sq_mlp_bwd(dy, x, w_up, w_down, saved_post, saved_act_grad, dx=None, dw_up=None,
                          dw_down=None, workspace=None, stream=None):
    """Returns (dx, dw_up, dw_down)."""
    M, d = x.shape
    f = w_up.shape[0]
    dx = _empty((M, d), x) if dx is None else dx
    dw_up = _empty((f, d), x) if dw_up is None else dw_up
    dw_down = _empty((d, f), x) if dw_down is None else dw_down
    ws, nb = _workspace("mlp2_bwd", M, d, f, 0, 0, _dt(x), x, workspace)
    _check("leaky_relu_sq_mlp_bwd", _lib.lib().leaky_relu_sq_mlp_bwd(
        _p(dy), _p(x), _p(w_up), _p(w_down), _p(saved_post), _p(saved_act_grad), _p(dx), _p(dw_up),
        _p(dw_down), _p(ws), nb, M, d, f, _dt(x), _stream(stream)))
    return dx, dw_up, dw_down


# ------------------------------------------------------------------ FlashFFN multi-head FFN
def flash_mhffn_fwd(q, w_k, w_u, w_v, router, o=None, stream=None):
    """q [T, H, d_h]; w_k, w_u, w_v [H, E, d_e, d_h]; router [T, H, E] fp32.
    Returns o [T, H, d_h]."""
    T, H, dh = q.shape
    E, de = w_k.shape[1], w_k.shape[2]
    for t in (q, w_k, w_u, w_v, router):
        if not t.is_contiguous():
            raise ValueError("flash_mhffn_fwd: tensors must be contiguous")
    if router.dtype != torch.float32 or tuple(router.shape) != (T, H, E):
        raise ValueError("flash_mhffn_fwd: router must be fp32 [T, H, E]")
    o = _empty((T, H, dh), q) if o is None else o
    _check("flash_mhffn_fwd", _lib.lib().flash_mhffn_fwd(
        _p(q), _p(w_k), _p(w_u), _p(w_v), _p(router), _p(o), T, H, dh, E, de, _dt(q),
        _stream(stream)))
    return o


def flash_mhffn_bwd_workspace_bytes(T, num_heads, head_dim, num_sub, sub_dim, dtype=torch.bfloat16):
    return _lib.lib().flash_mhffn_bwd_workspace_bytes(T, num_heads, head_dim, num_sub, sub_dim,
                                                      SWF_BF16 if dtype == torch.bfloat16 else SWF_F32)


def flash_mhffn_bwd(q, w_k, w_u, w_v, router, d_o, dq=None, dw_k=None, dw_u=None, dw_v=None,
                    drouter=None, workspace=None, stream=None):
    """Gradients of sum(d_o * flash_mhffn_fwd(q, w_k, w_u, w_v, router)).
    Returns (dq, dw_k, dw_u, dw_v, drouter)."""
    T, H, dh = q.shape
    E, de = w_k.shape[1], w_k.shape[2]
    dq = torch.empty_like(q) if dq is None else dq
    dw_k = torch.empty_like(w_k) if dw_k is None else dw_k
    dw_u = torch.empty_like(w_u) if dw_u is None else dw_u
    dw_v = torch.empty_like(w_v) if dw_v is None else dw_v
    drouter = torch.empty_like(router) if drouter is None else drouter
    nb = flash_mhffn_bwd_workspace_bytes(T, H, dh, E, de, q.dtype)
    if workspace is None:
        workspace = torch.empty(max(16, nb), device=q.device, dtype=torch.uint8)
    _check("flash_mhffn_bwd", _lib.lib().flash_mhffn_bwd(
        _p(q), _p(w_k), _p(w_u), _p(w_v), _p(router), _p(d_o), _p(dq), _p(dw_k), _p(dw_u), _p(dw_v),
        _p(drouter), _p(workspace), workspace.numel() * workspace.element_size(), T, H, dh, E, de,
        _dt(q), _stream(stream)))
    return dq, dw_k, dw_u, dw_v, drouter


def flash_mhffn_prologue(x, w_q, w_r, num_heads, num_sub, q_gain=None, eps=1e-6, q=None, router=None,
                         stream=None):
    """x [T, d_model]; w_q [H * 128, d_model]; w_r [H * E, d_model]; q_gain [128] fp32 or None.
    Returns (q [T, H, 128], router [T, H, E] fp32): the inputs of flash_mhffn_fwd."""
    T, d = x.shape
    dh = w_q.shape[0] // num_heads
    q = _empty((T, num_heads, dh), x) if q is None else q
    router = _empty((T, num_heads, num_sub), x, torch.float32) if router is None else router
    _check("flash_mhffn_prologue", _lib.lib().flash_mhffn_prologue(
        _p(x), _p(w_q), _p(q_gain), _p(w_r), _p(q), _p(router), T, d, num_heads, dh, num_sub,
        float(eps), _dt(x), _stream(stream)))
    return q, router


def flash_mhffn_prologue_bwd_workspace_bytes(T, d_model, num_heads, head_dim, num_sub, dtype=torch.bfloat16):
    return _lib.lib().flash_mhffn_prologue_bwd_workspace_bytes(T, d_model, num_heads, head_dim, num_sub,
                                                               SWF_BF16 if dtype == torch.bfloat16 else SWF_F32)


def flash_mhffn_prologue_bwd(x, w_q, w_r, num_heads, num_sub, dq, drouter, q_gain=None, eps=1e-6,
                             dx=None, dw_q=None, dw_r=None, dq_gain=None, workspace=None, stream=None):
    """Backward of flash_mhffn_prologue: returns (dx, dw_q, dw_r, dq_gain or None)."""
    T, d = x.shape
    dh = w_q.shape[0] // num_heads
    dx = torch.empty_like(x) if dx is None else dx
    dw_q = torch.empty_like(w_q) if dw_q is None else dw_q
    dw_r = torch.empty_like(w_r) if dw_r is None else dw_r
    if q_gain is not None and dq_gain is None:
        dq_gain = torch.empty_like(q_gain)
    nb = flash_mhffn_prologue_bwd_workspace_bytes(T, d, num_heads, dh, num_sub, x.dtype)
    if workspace is None:
        workspace = torch.empty(max(16, nb), device=x.device, dtype=torch.uint8)
    _check("flash_mhffn_prologue_bwd", _lib.lib().flash_mhffn_prologue_bwd(
        _p(x), _p(w_q), _p(q_gain), _p(w_r), _p(dq), _p(drouter), _p(dx), _p(dw_q), _p(dq_gain), _p(dw_r),
        _p(workspace), workspace.numel() * workspace.element_size(), T, d, num_heads, dh, num_sub,
        float(eps), _dt(x), _stream(stream)))
    return dx, dw_q, dw_r, dq_gain


# ------------------------------------------------------------------ group-sparse
def make_subsample_index(d_ff, group_size, samples_per_group, seed):
    """Host call: returns (int32 CPU tensor [d_ff // group_size, spg], spg)."""
    ng = d_ff // group_size
    out = torch.empty((ng, samples_per_group), dtype=torch.int32)
    _check("swf_make_subsample_index", _lib.lib().swf_make_subsample_index(
        d_ff, group_size, samples_per_group, int(seed) & (2 ** 64 - 1), C.c_void_p(out.data_ptr())))
    return out, samples_per_group


def grouped_topk_select(x, w_gate, group_size, num_active_groups, subsample_idx=None,
                        samples_per_group=None, load_balance_bias=None, group_idx=None,
                        energies=None, want_energies=False, workspace=None, stream=None):
    """Returns group_idx [M, K] int32 (and energies [M, ng] fp32 when requested)."""
    M, d = x.shape
    f = w_gate.shape[0]
    ng = f // group_size
    spg = samples_per_group if samples_per_group is not None else (
        subsample_idx.shape[1] if subsample_idx is not None else group_size)
    if group_idx is None:
        group_idx = torch.empty((M, num_active_groups), device=x.device, dtype=torch.int32)
    if energies is None and want_energies:
        energies = torch.empty((M, ng), device=x.device, dtype=torch.float32)
    ws, nb = _workspace("select", M, d, f, group_size, num_active_groups, _dt(x), x, workspace)
    _check("grouped_topk_select", _lib.lib().grouped_topk_select(
        _p(x), _p(w_gate), _p(subsample_idx), spg, _p(load_balance_bias), group_size,
        num_active_groups, _p(group_idx), _p(energies), _p(ws), nb, M, d, f, _dt(x),
        _stream(stream)))
    return (group_idx, energies) if want_energies or energies is not None else group_idx


def swf_group_buckets(group_idx, num_groups, offsets=None, tokens=None, workspace=None,
                      stream=None):
    """Returns (offsets [ng + 1] int32, tokens [M * K] int32)."""
    M, K = group_idx.shape
    dev = group_idx.device
    offsets = torch.empty(num_groups + 1, device=dev, dtype=torch.int32) if offsets is None else offsets
    tokens = torch.empty(M * K, device=dev, dtype=torch.int32) if tokens is None else tokens
    n = _lib.lib().swf_workspace_bytes(OPS["buckets"], M, 0, 0, num_groups, K, SWF_BF16)
    ws = torch.empty(max(n, 16), device=dev, dtype=torch.uint8) if workspace is None else workspace
    _check("swf_group_buckets", _lib.lib().swf_group_buckets(
        _p(group_idx), M, K, num_groups, _p(offsets), _p(tokens), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    return offsets, tokens


def group_frequency(group_idx, num_groups, freq=None, stream=None):
    """Fraction of tokens that selected each group (fp32 [num_groups])."""
    M, K = group_idx.shape
    freq = torch.empty(num_groups, device=group_idx.device, dtype=torch.float32) if freq is None else freq
    _check("swf_group_frequency", _lib.lib().swf_group_frequency(
        _p(group_idx), M, K, num_groups, _p(freq), _stream(stream)))
    return freq


def validate_group_idx(group_idx, num_groups, stream=None):
    """Counts the slots of group_idx [M, K] that are out of [0, num_groups) or repeat an earlier
    slot of their row; synchronises the stream.  Returns (status, count): status 0 when every
    slot is valid, 1 (SWF_ERR_INVALID_ARG) otherwise."""
    M, K = group_idx.shape
    bad = C.c_int64(-1)
    st = _lib.lib().swf_validate_group_idx(_p(group_idx), M, K, num_groups, C.byref(bad), _stream(stream))
    if st not in (_lib.SWF_OK, 1):
        raise SwfError("swf_validate_group_idx", st)
    return st, int(bad.value)


def set_debug(enable: bool) -> None:
    """Debug mode: entry points that read group_idx validate it first (and synchronise)."""
    _check("swf_set_debug", _lib.lib().swf_set_debug(1 if enable else 0))


def get_debug() -> bool:
    return bool(_lib.lib().swf_get_debug())


def update_load_balance_bias(bias, freq_ema, current_freq, target_freq, gamma=1e-3, bias_max=0.5,
                             momentum=0.99, stream=None):
    """In-place balancing step on the device buffers bias and freq_ema (fp32 [num_groups])."""
    _check("update_load_balance_bias", _lib.lib().update_load_balance_bias(
        _p(bias), _p(freq_ema), _p(current_freq), float(target_freq), float(gamma),
        float(bias_max), float(momentum), bias.numel(), _stream(stream)))
    return bias, freq_ema


def sparse_saved_bytes(M, d, f, group_size, num_active_groups, dtype=torch.bfloat16):
    return _lib.lib().swf_sparse_saved_bytes(M, d, f, group_size, num_active_groups,
                                             SWF_BF16 if dtype == torch.bfloat16 else SWF_F32)


def sparse_swiglu_ffn_fwd(x, w_gate, w_up, w_down, group_idx, group_size, y=None, saved=None,
                          workspace=None, stream=None):
    """Returns (y, saved)."""
    M, d = x.shape
    f = w_gate.shape[0]
    K = group_idx.shape[1]
    y = _empty((M, d), x) if y is None else y
    sb = sparse_saved_bytes(M, d, f, group_size, K, x.dtype)
    saved = torch.empty(max(sb, 16), device=x.device, dtype=torch.uint8) if saved is None else saved
    ws, nb = _workspace("sparse_fwd", M, d, f, group_size, K, _dt(x), x, workspace)
    _check("sparse_swiglu_ffn_fwd", _lib.lib().sparse_swiglu_ffn_fwd(
        _p(x), _p(w_gate), _p(w_up), _p(w_down), _p(group_idx), group_size, K, _p(y), _p(saved),
        saved.numel(), _p(ws), nb, M, d, f, _dt(x), _stream(stream)))
    return y, saved


def sparse_swiglu_ffn_bwd(dy, x, w_gate, w_up, w_down, group_idx, group_size, saved, dx=None,
                          dw_gate=None, dw_up=None, dw_down=None, workspace=None, stream=None):
    """Returns (dx, dw_gate, dw_up, dw_down)."""
    M, d = x.shape
    f = w_gate.shape[0]
    K = group_idx.shape[1]
    dx = _empty((M, d), x) if dx is None else dx
    dw_gate = _empty((f, d), x) if dw_gate is None else dw_gate
    dw_up = _empty((f, d), x) if dw_up is None else dw_up
    dw_down = _empty((d, f), x) if dw_down is None else dw_down
    ws, nb = _workspace("sparse_bwd", M, d, f, group_size, K, _dt(x), x, workspace)
    _check("sparse_swiglu_ffn_bwd", _lib.lib().sparse_swiglu_ffn_bwd(
        _p(dy), _p(x), _p(w_gate), _p(w_up), _p(w_down), _p(group_idx), _p(saved), saved.numel(),
        _p(dx), _p(dw_gate), _p(dw_up), _p(dw_down), _p(ws), nb, M, d, f, group_size, K,
        _dt(x), _stream(stream)))
    return dx, dw_gate, dw_up, dw_down


# ------------------------------------------------------------------ queries
def workspace_bytes(op, M, d, f, group_size=0, num_active_groups=0, dtype=torch.bfloat16):
    return _lib.lib().swf_workspace_bytes(OPS[op], M, d, f, group_size, num_active_groups,
                                          SWF_BF16 if dtype == torch.bfloat16 else SWF_F32)


def supported(op, M, d, f, group_size=0, num_active_groups=0, samples_per_group=0,
              dtype=torch.bfloat16) -> int:
    """Status code (0 = supported) without touching the GPU."""
    return _lib.lib().swf_supported(OPS[op], M, d, f, group_size, num_active_groups,
                                    samples_per_group,
                                    SWF_BF16 if dtype == torch.bfloat16 else SWF_F32)


def plan(op, M, d, f, group_size=0, num_active_groups=0, samples_per_group=0,
         dtype=torch.bfloat16) -> dict:
    info = swf_plan_info()
    _check("swf_plan", _lib.lib().swf_plan(
        OPS[op], M, d, f, group_size, num_active_groups, samples_per_group,
        SWF_BF16 if dtype == torch.bfloat16 else SWF_F32, C.byref(info)))
    return {name: getattr(info, name) for name, _ in info._fields_}


def device_status(stream=None) -> int:
    """Synchronises the stream; returns and clears the device status word (0 or 6 = timeout)."""
    return _lib.lib().swf_device_status(_stream(stream))


def selftest_wait_timeout(limit_us: int, stream=None) -> None:
    _check("swf_selftest_wait_timeout", _lib.lib().swf_selftest_wait_timeout(limit_us, _stream(stream)))


# ------------------------------------------------------------------ profiling aid
def profile_enable(enable: bool = True) -> None:
    _check("swf_profile_enable", _lib.lib().swf_profile_enable(1 if enable else 0))


def profile_read() -> dict:
    """{kernel name: (launches, total ms)} for the launches bracketed since the last read."""
    import numpy as np
    n = 64
    launches = np.zeros(n, dtype=np.int64)
    total = np.zeros(n, dtype=np.float64)
    k = _lib.lib().swf_profile_read(n, C.c_void_p(launches.ctypes.data), C.c_void_p(total.ctypes.data))
    if k < 0:
        raise SwfError("swf_profile_read", _lib.SWF_ERR_LAUNCH if hasattr(_lib, "SWF_ERR_LAUNCH") else 5)
    return {_lib.lib().swf_kernel_name(i).decode(): (int(launches[i]), float(total[i]))
            for i in range(k) if launches[i] > 0}

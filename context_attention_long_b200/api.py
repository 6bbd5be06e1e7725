"""Thin PyTorch binding of the C ABI (include/cpattn.h), same function names.

Argument marshalling only: shapes and pointers are read from torch tensors,
outputs are allocated with torch when not given, and every step of the hot path
runs in libcpattn.so's CUDA kernels on the current (or given) CUDA stream.
There is no CPU path: calling without a CUDA device or without the built
library raises.

Layouts: Q/K/V/out are bf16 (B, S, H, D) contiguous; LSE is float32 (B, H, S),
natural log.  See include/cpattn.h for the exact semantics of each call.
"""
from __future__ import annotations

import ctypes

import torch

from . import _native

__all__ = [
    "CpattnError", "cpattn_ring_attention", "cpattn_causal_ring_attention", "cpattn_ring_step",
    "cpattn_causal_ring_step", "cpattn_lse_merge", "cpattn_kv_gather_attention", "cpattn_ulysses_permute",
    "cpattn_ulysses_permute_qkv", "cpattn_ulysses_unpermute", "cpattn_ulysses_qkv_projection",
    "cpattn_ulysses_output_projection", "cpattn_head_sharded_attention",
    "cpattn_causal_head_sharded_attention", "cpattn_ulysses_workspace_bytes",
    "cpattn_unified_workspace_bytes", "cpattn_ulysses_attention", "cpattn_causal_ulysses_attention",
    "cpattn_unified_attention", "cpattn_causal_unified_attention",
    "cpattn_attention_backward_workspace_bytes", "cpattn_attention_backward_ds_bytes", "cpattn_attention_backward",
    "backward_workspace_bytes", "BACKWARD_DS_BUDGET",
    "cpattn_ulysses_attention_backward_workspace_bytes", "cpattn_ulysses_attention_backward",
    "cpattn_ulysses_attention_noalloc", "cpattn_ring_chunk_attention", "cpattn_gathered_kv_attention",
    "cpattn_rank_buffer_attention", "cpattn_front_loaded_splits", "cpattn_exchange_bytes",
    "cpattn_plan_exchange", "cpattn_device_status", "cpattn_debug_wait_timeout", "NOALLOC_SCRATCH_BYTES",
    "status_string",
]


CPATTN_ERR_CUDA = 6


class CpattnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)} ({status})"
        if status == CPATTN_ERR_CUDA:
            msg += " -- " + _native.load().cpattn_last_cuda_error_string().decode()
        super().__init__(msg)


def status_string(status: int) -> str:
    return _native.load().cpattn_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != 0:
        raise CpattnError(status, where)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    """Device address of a tensor the library may read or write.  The kernels
    launch on the current CUDA device and index the memory densely, so a host
    tensor, a tensor on another device or a non-contiguous view is refused
    here, before the library sees the pointer."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("tensor arguments must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensor on {t.device}, but the current device is cuda:{torch.cuda.current_device()}")
    return ctypes.c_void_p(t.data_ptr())


def _need(t, numel, dtype, name):
    """A tensor argument must hold at least `numel` elements of `dtype`: the
    library indexes the memory behind the pointer by the sizes it is given."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements, {numel} needed")


def _bshd(q: torch.Tensor, name="q"):
    if q.dim() != 4:
        raise ValueError(f"{name} must be (B, S, H, D)")
    if not q.is_cuda or q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    B, S, H, D = q.shape
    return B, S, H, D


def _ring(entry, q, k, v, ring_degree, chunk_lens, out, lse, want_lse, stream):
    B, S, H, D = _bshd(q)
    out = torch.empty_like(q) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    for t, name in ((k, "k"), (v, "v"), (out, "out")):
        _need(t, q.numel(), torch.bfloat16, name)
    _need(lse, B * H * S, torch.float32, "lse")
    _check(getattr(_native.load(), entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S, D,
                                          int(ring_degree), _native.int_array(chunk_lens), _stream(stream)), entry)
    return out, lse


def cpattn_ring_attention(q, k, v, ring_degree, chunk_lens=None, out=None, lse=None, want_lse=True, stream=None):
    """Fused ring attention; returns (out bf16 (B,S,H,D), lse float32 (B,H,S) or None)."""
    return _ring("cpattn_ring_attention", q, k, v, ring_degree, chunk_lens, out, lse, want_lse, stream)


def cpattn_causal_ring_attention(q, k, v, ring_degree, chunk_lens=None, out=None, lse=None, want_lse=True,
                                 stream=None):
    """Fused causal ring attention (key j visible to query i iff j <= i); returns (out, lse)."""
    return _ring("cpattn_causal_ring_attention", q, k, v, ring_degree, chunk_lens, out, lse, want_lse, stream)


def _ring_step(entry, q, k, v, ring_degree, step, chunk_lens, part_out, part_lse, stream):
    B, S, H, D = _bshd(q)
    if part_out is None:
        part_out = torch.empty((B, S, H, D), dtype=torch.float32, device=q.device)
    if part_lse is None:
        part_lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    _need(k, q.numel(), torch.bfloat16, "k")
    _need(v, q.numel(), torch.bfloat16, "v")
    _need(part_out, q.numel(), torch.float32, "part_out")
    _need(part_lse, B * H * S, torch.float32, "part_lse")
    _check(getattr(_native.load(), entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(part_out), _ptr(part_lse), B, H, S, D,
                                          int(ring_degree), _native.int_array(chunk_lens), int(step),
                                          _stream(stream)), entry)
    return part_out, part_lse


def cpattn_ring_step(q, k, v, ring_degree, step, chunk_lens=None, part_out=None, part_lse=None, stream=None):
    """One ring step for every rank; returns float32 (partial out (B,S,H,D), partial lse (B,H,S))."""
    return _ring_step("cpattn_ring_step", q, k, v, ring_degree, step, chunk_lens, part_out, part_lse, stream)


def cpattn_causal_ring_step(q, k, v, ring_degree, step, chunk_lens=None, part_out=None, part_lse=None,
                            stream=None):
    """One causal ring step for every rank (a chunk after the rank's shard gives out 0, lse -inf)."""
    return _ring_step("cpattn_causal_ring_step", q, k, v, ring_degree, step, chunk_lens, part_out, part_lse, stream)


def cpattn_lse_merge(part_out, part_lse, out_f32=None, out_bf16=None, lse_out=None, want_f32=False,
                     want_bf16=True, stream=None):
    """Merge P float32 partials: part_out (P,B,S,H,D), part_lse (P,B,H,S).
    Returns (out_f32 or None, out_bf16 or None, lse_out)."""
    P, B, S, H, D = part_out.shape
    dev = part_out.device
    if out_f32 is None and want_f32:
        out_f32 = torch.empty((B, S, H, D), dtype=torch.float32, device=dev)
    if out_bf16 is None and want_bf16:
        out_bf16 = torch.empty((B, S, H, D), dtype=torch.bfloat16, device=dev)
    if lse_out is None:
        lse_out = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    n = B * S * H * D
    _need(part_out, P * n, torch.float32, "part_out")
    _need(part_lse, P * B * H * S, torch.float32, "part_lse")
    _need(out_f32, n, torch.float32, "out_f32")
    _need(out_bf16, n, torch.bfloat16, "out_bf16")
    _need(lse_out, B * H * S, torch.float32, "lse_out")
    _check(_native.load().cpattn_lse_merge(_ptr(part_out), _ptr(part_lse), P, B, H, S, D, _ptr(out_f32),
                                           _ptr(out_bf16), _ptr(lse_out), _stream(stream)), "cpattn_lse_merge")
    return out_f32, out_bf16, lse_out


def cpattn_kv_gather_attention(q, k, v, degree, q_lens=None, out=None, lse=None, want_lse=True, stream=None):
    """kv_gather attention; returns (out, lse)."""
    B, S, H, D = _bshd(q)
    out = torch.empty_like(q) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    for t, name in ((k, "k"), (v, "v"), (out, "out")):
        _need(t, q.numel(), torch.bfloat16, name)
    _need(lse, B * H * S, torch.float32, "lse")
    _check(_native.load().cpattn_kv_gather_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S, D,
                                                     int(degree), _native.int_array(q_lens), _stream(stream)),
           "cpattn_kv_gather_attention")
    return out, lse


def _flat_numel(B, S, H, D):
    return B * S * H * D


def cpattn_ulysses_permute(x, B, S, H, D, degree, seq_splits=None, head_splits=None, y=None, stream=None):
    """Sequence-sharded rank buffers (flat, any 1/2/4/8-byte dtype) -> head-sharded rank buffers."""
    if y is None:
        y = torch.empty_like(x)
    _need(x, _flat_numel(B, S, H, D), None, "x")
    _need(y, _flat_numel(B, S, H, D), x.dtype, "y")
    _check(_native.load().cpattn_ulysses_permute(_ptr(x), _ptr(y), B, S, H, D, x.element_size(), int(degree),
                                                 _native.int_array(seq_splits), _native.int_array(head_splits),
                                                 _stream(stream)), "cpattn_ulysses_permute")
    return y


def cpattn_ulysses_permute_qkv(q, k, v, B, S, H, D, degree, seq_splits=None, head_splits=None, yq=None, yk=None,
                               yv=None, stream=None):
    """The Q, K and V permutes of the first all-to-all in one launch; returns (yq, yk, yv)."""
    yq = torch.empty_like(q) if yq is None else yq
    yk = torch.empty_like(k) if yk is None else yk
    yv = torch.empty_like(v) if yv is None else yv
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (yq, "yq"), (yk, "yk"), (yv, "yv")):
        _need(t, _flat_numel(B, S, H, D), q.dtype, name)
    _check(_native.load().cpattn_ulysses_permute_qkv(_ptr(q), _ptr(k), _ptr(v), _ptr(yq), _ptr(yk), _ptr(yv), B, S,
                                                     H, D, q.element_size(), int(degree),
                                                     _native.int_array(seq_splits), _native.int_array(head_splits),
                                                     _stream(stream)), "cpattn_ulysses_permute_qkv")
    return yq, yk, yv


def cpattn_ulysses_unpermute(y, B, S, H, D, degree, seq_splits=None, head_splits=None, x=None, stream=None):
    """Head-sharded rank buffers -> sequence-sharded rank buffers (inverse permute)."""
    if x is None:
        x = torch.empty_like(y)
    _need(y, _flat_numel(B, S, H, D), None, "y")
    _need(x, _flat_numel(B, S, H, D), y.dtype, "x")
    _check(_native.load().cpattn_ulysses_unpermute(_ptr(y), _ptr(x), B, S, H, D, y.element_size(), int(degree),
                                                   _native.int_array(seq_splits), _native.int_array(head_splits),
                                                   _stream(stream)), "cpattn_ulysses_unpermute")
    return x


def cpattn_ulysses_qkv_projection(x, w_qkv, B, S, H, D, Dm, degree, seq_splits=None, head_splits=None, yq=None,
                                  yk=None, yv=None, stream=None):
    """Q, K, V projections of the sequence-side activations x (rank buffers
    (B, S_r, Dm) concatenated, bf16) by w_qkv (3*H*D, Dm), stored straight into
    the head-sharded layout; returns flat (yq, yk, yv) of B*S*H*D bf16 each."""
    n = _flat_numel(B, S, H, D)
    yq, yk, yv = (torch.empty(n, dtype=torch.bfloat16, device=x.device) if t is None else t for t in (yq, yk, yv))
    _need(x, B * S * Dm, torch.bfloat16, "x")
    _need(w_qkv, 3 * H * D * Dm, torch.bfloat16, "w_qkv")
    for t, name in ((yq, "yq"), (yk, "yk"), (yv, "yv")):
        _need(t, n, torch.bfloat16, name)
    _check(_native.load().cpattn_ulysses_qkv_projection(_ptr(x), _ptr(w_qkv), _ptr(yq), _ptr(yk), _ptr(yv), B, S, H,
                                                        D, Dm, int(degree), _native.int_array(seq_splits),
                                                        _native.int_array(head_splits), _stream(stream)),
           "cpattn_ulysses_qkv_projection")
    return yq, yk, yv


def cpattn_ulysses_output_projection(yo, w_o, B, S, H, D, Dm, degree, seq_splits=None, head_splits=None, out=None,
                                     stream=None):
    """Output projection by w_o (Dm, H*D) of the head-sharded attention output yo,
    read in place; returns the sequence-side result (rank buffers (B, S_r, Dm)
    concatenated), flat bf16 of B*S*Dm."""
    out = torch.empty(B * S * Dm, dtype=torch.bfloat16, device=yo.device) if out is None else out
    _need(yo, _flat_numel(B, S, H, D), torch.bfloat16, "yo")
    _need(w_o, Dm * H * D, torch.bfloat16, "w_o")
    _need(out, B * S * Dm, torch.bfloat16, "out")
    _check(_native.load().cpattn_ulysses_output_projection(_ptr(yo), _ptr(w_o), _ptr(out), B, S, H, D, Dm,
                                                           int(degree), _native.int_array(seq_splits),
                                                           _native.int_array(head_splits), _stream(stream)),
           "cpattn_ulysses_output_projection")
    return out


def _head_sharded(entry, yq, yk, yv, B, S, H, D, degree, head_splits, yo, lse, want_lse, stream):
    yo = torch.empty_like(yq) if yo is None else yo
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=yq.device)
    for t, name in ((yq, "yq"), (yk, "yk"), (yv, "yv"), (yo, "yo")):
        _need(t, _flat_numel(B, S, H, D), torch.bfloat16, name)
    _need(lse, B * H * S, torch.float32, "lse")
    _check(getattr(_native.load(), entry)(_ptr(yq), _ptr(yk), _ptr(yv), _ptr(yo), _ptr(lse), B, H, S, D,
                                          int(degree), _native.int_array(head_splits), _stream(stream)), entry)
    return yo, lse


def cpattn_head_sharded_attention(yq, yk, yv, B, S, H, D, degree, head_splits=None, yo=None, lse=None,
                                  want_lse=True, stream=None):
    """Local attention on head-sharded rank buffers; returns (yo, lse (B,H,S))."""
    return _head_sharded("cpattn_head_sharded_attention", yq, yk, yv, B, S, H, D, degree, head_splits, yo, lse,
                         want_lse, stream)


def cpattn_causal_head_sharded_attention(yq, yk, yv, B, S, H, D, degree, head_splits=None, yo=None, lse=None,
                                         want_lse=True, stream=None):
    """Causal local attention on head-sharded rank buffers; returns (yo, lse (B,H,S))."""
    return _head_sharded("cpattn_causal_head_sharded_attention", yq, yk, yv, B, S, H, D, degree, head_splits, yo,
                         lse, want_lse, stream)


def cpattn_ulysses_workspace_bytes(B, H, S, D) -> int:
    return int(_native.load().cpattn_ulysses_workspace_bytes(B, H, S, D))


def cpattn_unified_workspace_bytes(B, H, S, D) -> int:
    return int(_native.load().cpattn_unified_workspace_bytes(B, H, S, D))


def _workspace(nbytes, device, workspace):
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace


def _ulysses(entry, q, k, v, B, S, H, D, degree, seq_splits, head_splits, out, lse, want_lse, workspace, stream):
    out = torch.empty_like(q) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    nbytes = cpattn_ulysses_workspace_bytes(B, H, S, D)
    workspace = _workspace(nbytes, q.device, workspace)
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _need(t, _flat_numel(B, S, H, D), torch.bfloat16, name)
    _need(lse, B * H * S, torch.float32, "lse")
    _check(getattr(_native.load(), entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S, D,
                                          int(degree), _native.int_array(seq_splits),
                                          _native.int_array(head_splits), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream)), entry)
    return out, lse


def cpattn_ulysses_attention(q, k, v, B, S, H, D, degree, seq_splits=None, head_splits=None, out=None, lse=None,
                             want_lse=True, workspace=None, stream=None):
    """Ulysses attention on sequence-sharded rank buffers (flat bf16); returns (out, lse)."""
    return _ulysses("cpattn_ulysses_attention", q, k, v, B, S, H, D, degree, seq_splits, head_splits, out, lse,
                    want_lse, workspace, stream)


def cpattn_causal_ulysses_attention(q, k, v, B, S, H, D, degree, seq_splits=None, head_splits=None, out=None,
                                    lse=None, want_lse=True, workspace=None, stream=None):
    """Causal Ulysses attention on sequence-sharded rank buffers (flat bf16); returns (out, lse)."""
    return _ulysses("cpattn_causal_ulysses_attention", q, k, v, B, S, H, D, degree, seq_splits, head_splits, out,
                    lse, want_lse, workspace, stream)


def _unified(entry, q, k, v, ring_degree, ulysses_degree, ring_lens, head_splits, out, lse, want_lse, workspace,
             stream):
    B, S, H, D = _bshd(q)
    out = torch.empty_like(q) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    nbytes = cpattn_unified_workspace_bytes(B, H, S, D)
    workspace = _workspace(nbytes, q.device, workspace)
    for t, name in ((k, "k"), (v, "v"), (out, "out")):
        _need(t, q.numel(), torch.bfloat16, name)
    _need(lse, B * H * S, torch.float32, "lse")
    _check(getattr(_native.load(), entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S, D,
                                          int(ring_degree), int(ulysses_degree), _native.int_array(ring_lens),
                                          _native.int_array(head_splits), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream)), entry)
    return out, lse


def cpattn_unified_attention(q, k, v, ring_degree, ulysses_degree, ring_lens=None, head_splits=None, out=None,
                             lse=None, want_lse=True, workspace=None, stream=None):
    """Unified ring x Ulysses attention on full (B,S,H,D) tensors; returns (out, lse)."""
    return _unified("cpattn_unified_attention", q, k, v, ring_degree, ulysses_degree, ring_lens, head_splits, out,
                    lse, want_lse, workspace, stream)


def cpattn_causal_unified_attention(q, k, v, ring_degree, ulysses_degree, ring_lens=None, head_splits=None,
                                    out=None, lse=None, want_lse=True, workspace=None, stream=None):
    """Causal unified ring x Ulysses attention on full (B,S,H,D) tensors; returns (out, lse)."""
    return _unified("cpattn_causal_unified_attention", q, k, v, ring_degree, ulysses_degree, ring_lens,
                    head_splits, out, lse, want_lse, workspace, stream)


def cpattn_attention_backward_workspace_bytes(B, H, S) -> int:
    return int(_native.load().cpattn_attention_backward_workspace_bytes(B, H, S))


def cpattn_attention_backward_ds_bytes(B, S, causal) -> int:
    return int(_native.load().cpattn_attention_backward_ds_bytes(B, S, 1 if causal else 0))


# Default cap on the dS scratch the backward bindings add to a workspace they
# allocate: the library groups the heads so that their dS tiles fit it, and
# when one head's tiles exceed it the dQ kernel runs instead.
BACKWARD_DS_BUDGET = 8 << 30


def _ds_scratch_bytes(B, H, S, causal, ds_budget):
    """Whole heads of dS scratch within the budget, plus the 256 bytes the
    library may skip to align it (0: no scratch)."""
    per = cpattn_attention_backward_ds_bytes(B, S, causal)
    budget = BACKWARD_DS_BUDGET if ds_budget is None else int(ds_budget)
    heads = min(H, budget // per) if per > 0 else 0
    return 256 + heads * per if heads > 0 else 0


def backward_workspace_bytes(B, H, S, causal=False, ds_budget=None, ulysses_D=None) -> int:
    """Bytes of the workspace the backward bindings allocate: the minimum of
    cpattn_attention_backward (or, given ulysses_D, of the Ulysses backward
    flow) plus whole heads of dS scratch within ds_budget.  A workspace sized
    for causal=False also serves the causal backward."""
    base = (cpattn_attention_backward_workspace_bytes(B, H, S) if ulysses_D is None else
            cpattn_ulysses_attention_backward_workspace_bytes(B, H, S, ulysses_D))
    return base + _ds_scratch_bytes(B, H, S, causal, ds_budget)


def _allocation_budget(device, ds_budget):
    """The dS budget for a workspace the binding allocates itself: the given
    one, or by default BACKWARD_DS_BUDGET capped at half the device's free
    memory (a smaller scratch only means more head groups)."""
    if ds_budget is not None:
        return int(ds_budget)
    free, _ = torch.cuda.mem_get_info(device)
    return min(BACKWARD_DS_BUDGET, free // 2)


def cpattn_attention_backward(q, k, v, out, lse, dout, causal=False, dq=None, dk=None, dv=None, workspace=None,
                              stream=None, ds_budget=None):
    """Gradient of attention over full (B,S,H,D) bf16 tensors given the
    forward's output and LSE; returns (dq, dk, dv) in bf16.  An allocated
    workspace holds up to ds_budget bytes of dS scratch (default
    BACKWARD_DS_BUDGET, capped at half the device's free memory); 0 selects
    the dQ kernel that recomputes S and dP."""
    B, S, H, D = _bshd(q)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = _workspace(backward_workspace_bytes(B, H, S, causal, _allocation_budget(q.device, ds_budget)),
                               q.device, None)
    for t, name in ((k, "k"), (v, "v"), (out, "out"), (dout, "dout"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, q.numel(), torch.bfloat16, name)
    _need(lse, B * H * S, torch.float32, "lse")
    if lse is None:
        raise ValueError("lse is required")
    _check(_native.load().cpattn_attention_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout),
                                                    _ptr(dq), _ptr(dk), _ptr(dv), B, H, S, D, 1 if causal else 0,
                                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                                    _stream(stream)), "cpattn_attention_backward")
    return dq, dk, dv


def cpattn_ulysses_attention_backward_workspace_bytes(B, H, S, D) -> int:
    return int(_native.load().cpattn_ulysses_attention_backward_workspace_bytes(B, H, S, D))


def cpattn_ulysses_attention_backward(q, k, v, out, lse, dout, B, S, H, D, degree, seq_splits=None,
                                      head_splits=None, causal=False, dq=None, dk=None, dv=None, workspace=None,
                                      stream=None, ds_budget=None):
    """Backward of the Ulysses flow on sequence-sharded rank buffers (flat
    bf16); returns (dq, dk, dv) in the same layout.  ds_budget as
    cpattn_attention_backward."""
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = _workspace(backward_workspace_bytes(B, H, S, causal, _allocation_budget(q.device, ds_budget),
                                                        ulysses_D=D), q.device, None)
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, _flat_numel(B, S, H, D), torch.bfloat16, name)
    _need(lse, B * H * S, torch.float32, "lse")
    if lse is None:
        raise ValueError("lse is required")
    _check(_native.load().cpattn_ulysses_attention_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), B, H, S, D,
        int(degree), _native.int_array(seq_splits), _native.int_array(head_splits), 1 if causal else 0,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
        "cpattn_ulysses_attention_backward")
    return dq, dk, dv


# Size of the library-held scratch of cpattn_ulysses_attention_noalloc
# (CPATTN_NOALLOC_SCRATCH_BYTES in cpattn.h).
NOALLOC_SCRATCH_BYTES = 64 << 20


def cpattn_ulysses_attention_noalloc(q, k, v, B, S, H, D, degree, seq_splits=None, head_splits=None, out=None,
                                     lse=None, want_lse=True, stream=None):
    """Ulysses attention for callers that cannot allocate device memory when
    they call: the scratch lives in a fixed 64 MiB array inside the library
    (see cpattn.h).  `out` and `lse` should be passed in by such callers; when
    omitted they are allocated here with torch for convenience.  Concurrent
    calls on different streams race on the shared scratch."""
    out = torch.empty_like(q) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _need(t, _flat_numel(B, S, H, D), torch.bfloat16, name)
    _need(lse, B * H * S, torch.float32, "lse")
    _check(_native.load().cpattn_ulysses_attention_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S,
                                                           D, int(degree), _native.int_array(seq_splits),
                                                           _native.int_array(head_splits), _stream(stream)),
           "cpattn_ulysses_attention_noalloc")
    return out, lse


def cpattn_ring_chunk_attention(q, k, v, Skv, out, lse, prev_out=None, q_pos0=0, kv_pos0=0, causal=False,
                                kv_batch_rows=None, stream=None):
    """One ring step of one rank over separate buffers, merged into its running
    result.  q (B, Sq, H, D) bf16; k, v (B, kv_batch_rows, H, D) bf16 whose
    first Skv rows per batch element are the chunk; out float32 (an
    intermediate state) or bf16 (the final output), (B, Sq, H, D); lse
    (B, H, Sq) float32, holding prev_out's LSE on entry when prev_out (float32,
    may be `out` itself) is given.  Returns (out, lse)."""
    B, Sq, H, D = _bshd(q)
    rows = k.shape[1] if kv_batch_rows is None else int(kv_batch_rows)
    for t, name in ((k, "k"), (v, "v")):
        _need(t, B * rows * H * D, torch.bfloat16, name)
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("out must be float32 or bf16")
    _need(out, B * Sq * H * D, out.dtype, "out")
    _need(lse, B * H * Sq, torch.float32, "lse")
    _need(prev_out, B * Sq * H * D, torch.float32, "prev_out")
    _check(_native.load().cpattn_ring_chunk_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                                      _ptr(prev_out), B, H, Sq, int(Skv), rows, D, int(q_pos0),
                                                      int(kv_pos0), int(bool(causal)),
                                                      int(out.dtype == torch.float32), _stream(stream)),
           "cpattn_ring_chunk_attention")
    return out, lse


def cpattn_gathered_kv_attention(q, k, v, degree, rank, kv_lens=None, out=None, lse=None, want_lse=True,
                                 causal=False, stream=None):
    """Attention of one rank's query shard q (B, kv_lens[rank], H, D) against
    `degree` gathered K/V chunks, k and v (degree, B, kv_batch_rows, H, D)
    bf16, chunk c holding kv_lens[c] valid rows.  Returns (out, lse)."""
    B, Sq, H, D = _bshd(q)
    if k.dim() != 5 or k.shape[0] != degree or k.shape[1] != B:
        raise ValueError("k and v must be (degree, B, kv_batch_rows, H, D)")
    rows = k.shape[2]
    for t, name in ((k, "k"), (v, "v")):
        _need(t, degree * B * rows * H * D, torch.bfloat16, name)
    out = torch.empty_like(q) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    _need(out, B * Sq * H * D, torch.bfloat16, "out")
    _need(lse, B * H * Sq, torch.float32, "lse")
    _check(_native.load().cpattn_gathered_kv_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, D,
                                                       int(degree), _native.int_array(kv_lens), rows, int(rank),
                                                       int(bool(causal)), _stream(stream)),
           "cpattn_gathered_kv_attention")
    return out, lse


def cpattn_rank_buffer_attention(q, k, v, B, S, H, D, degree, seq_splits=None, out=None, lse=None, want_lse=True,
                                 causal=False, stream=None):
    """Attention over a sequence held as rank buffers (B, S_u, H, D)
    concatenated (flat bf16), the layout an all-to-all delivers; every query
    attends all S keys.  Returns (out in the same layout, lse (B, H, S))."""
    out = torch.empty_like(q) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _need(t, _flat_numel(B, S, H, D), torch.bfloat16, name)
    _need(lse, B * H * S, torch.float32, "lse")
    _check(_native.load().cpattn_rank_buffer_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S, D,
                                                       int(degree), _native.int_array(seq_splits),
                                                       int(bool(causal)), _stream(stream)),
           "cpattn_rank_buffer_attention")
    return out, lse


def cpattn_front_loaded_splits(total, parts):
    arr = (ctypes.c_int * max(1, int(parts)))()
    _check(_native.load().cpattn_front_loaded_splits(int(total), int(parts), arr), "cpattn_front_loaded_splits")
    return [int(arr[i]) for i in range(int(parts))]


EXCHANGE_MODES = {"ring": 0, "ulysses": 1, "kv_gather": 2}


def cpattn_exchange_bytes(mode, B, H, S, D, degree, seq_splits=None, head_splits=None, elem_bytes=2):
    """Per-rank (send, recv) bytes of one attention call under an exchange
    ('ring', 'ulysses' or 'kv_gather'); host arithmetic only."""
    send = (ctypes.c_ulonglong * int(degree))()
    recv = (ctypes.c_ulonglong * int(degree))()
    _check(_native.load().cpattn_exchange_bytes(EXCHANGE_MODES[mode], B, H, S, D, elem_bytes, int(degree),
                                                _native.int_array(seq_splits), _native.int_array(head_splits),
                                                send, recv), "cpattn_exchange_bytes")
    return [int(x) for x in send], [int(x) for x in recv]


class _ExchangeEnv(ctypes.Structure):
    _fields_ = [("link_gbs", ctypes.c_double), ("attn_tflops", ctypes.c_double), ("hbm_gbs", ctypes.c_double),
                ("causal", ctypes.c_int)]


class _ExchangePlan(ctypes.Structure):
    _fields_ = [("seconds", ctypes.c_double * 3), ("recv_bytes", ctypes.c_ulonglong * 3),
                ("resident_bytes", ctypes.c_ulonglong * 3), ("flops", ctypes.c_double * 3), ("best", ctypes.c_int)]


def cpattn_plan_exchange(B, H, S, D, degree, link_gbs, attn_tflops, hbm_gbs, causal=False, seq_splits=None,
                         head_splits=None, elem_bytes=2):
    """Exchange-selection model for one attention call over `degree` ranks.
    Returns {"best": mode name, mode name: {"seconds" (None if infeasible),
    "recv_bytes", "resident_bytes", "flops"}}; host arithmetic only."""
    env = _ExchangeEnv(float(link_gbs), float(attn_tflops), float(hbm_gbs), 1 if causal else 0)
    plan = _ExchangePlan()
    _check(_native.load().cpattn_plan_exchange(B, H, S, D, elem_bytes, int(degree), _native.int_array(seq_splits),
                                               _native.int_array(head_splits), ctypes.byref(env),
                                               ctypes.byref(plan)), "cpattn_plan_exchange")
    names = {v: k for k, v in EXCHANGE_MODES.items()}
    out = {"best": names[plan.best]}
    for m, name in names.items():
        out[name] = {"seconds": None if plan.seconds[m] < 0 else float(plan.seconds[m]),
                     "recv_bytes": int(plan.recv_bytes[m]), "resident_bytes": int(plan.resident_bytes[m]),
                     "flops": float(plan.flops[m])}
    return out


def cpattn_device_status(stream=None):
    """Synchronise the stream and read-and-clear the device status word.
    Returns (status, code)."""
    code = ctypes.c_uint(0)
    st = _native.load().cpattn_device_status(_stream(stream), ctypes.byref(code))
    return int(st), int(code.value)


def cpattn_debug_wait_timeout(timeout_us, stream=None):
    _check(_native.load().cpattn_debug_wait_timeout(int(timeout_us), _stream(stream)), "cpattn_debug_wait_timeout")

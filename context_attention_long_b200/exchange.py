"""Context-parallel attention across GPUs: the exchanges as real collectives.

One process per GPU; torch.distributed (NCCL over NVLink / NVSwitch) moves the
data, and every arithmetic step runs in libcpattn.so's CUDA kernels through the
C ABI.  Each rank holds its sequence shard of Q, K and V as a contiguous bf16
(B, S_r, H, D) tensor; the shards of all ranks, concatenated in rank order,
are the full sequence.

  ring_attention       diffusers "Context parallelism", "Ring Attention": each
                       rank attends its queries to one K/V chunk at a time and
                       passes the chunk on; after a full ring every query has
                       seen every key.  rotate_method "p2p" pipelines the
                       point-to-point rotation against the attention of the
                       chunk already held (SGLang "Sequence Parallelism",
                       "Cross-Node Sequence Parallelism"); "allgather" gathers
                       the chunks first (diffusers "parallel", rotate_method)
                       and then runs the very same per-chunk steps, so the two
                       give byte-identical results.  Uneven chunk lengths are
                       Ring Anything: chunks are padded to the longest for the
                       all-gather and sliced back before attention.
  ulysses_attention    diffusers "Ulysses Attention"; "Ulysses Sequence
                       Parallelism" article, section 4: an all-to-all from the
                       sequence-sharded to the head-sharded layout, local
                       attention over all tokens of the rank's heads, and the
                       inverse all-to-all.  Uneven splits are Ulysses Anything.
  kv_gather_attention  SGLang "Sequence Parallelism", "Choosing The Attention
                       Exchange": K and V are all-gathered, Q and the output
                       stay sequence-sharded; non-causal.
  unified_attention    diffusers "Unified Attention": Ulysses inside each
                       Ulysses group, ring across the groups, on a
                       ring_degree x ulysses_degree grid of ranks.

Every rank of a group must call the same function with the same split
arguments.  Collectives move raw bytes (uint8 views), so any backend that
moves bytes carries them.  The local compute is the `kernels` object:
CudaKernels (the default) calls the library and refuses host tensors, so there
is no CPU path; tests substitute a stand-in with the same contract to check
the data movement on CPU ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import api

__all__ = ["CudaKernels", "ring_attention", "ulysses_attention", "kv_gather_attention", "unified_attention",
           "unified_groups", "equal_splits", "front_loaded_splits"]


def equal_splits(total: int, parts: int) -> list[int]:
    if total % parts:
        raise ValueError(f"{total} is not divisible by {parts}: pass explicit splits (the 'anything' modes)")
    return [total // parts] * parts


def front_loaded_splits(total: int, parts: int) -> list[int]:
    """The first total % parts entries get ceil(total / parts), the rest the floor."""
    base, extra = divmod(total, parts)
    return [base + (1 if i < extra else 0) for i in range(parts)]


def _prefix(lens):
    off = [0]
    for n in lens:
        off.append(off[-1] + n)
    return off


class CudaKernels:
    """The library's CUDA entry points (the only compute this module runs)."""

    def ring_chunk(self, q, k, v, Skv, out, lse, prev, q_pos0, kv_pos0, causal, kv_batch_rows):
        api.cpattn_ring_chunk_attention(q, k, v, Skv, out, lse, prev_out=prev, q_pos0=q_pos0, kv_pos0=kv_pos0,
                                        causal=causal, kv_batch_rows=kv_batch_rows)

    def gathered(self, q, k, v, degree, rank, kv_lens, causal):
        return api.cpattn_gathered_kv_attention(q, k, v, degree, rank, kv_lens, causal=causal)

    def rank_buffer(self, q, k, v, B, S, H, D, degree, seq_splits, causal):
        return api.cpattn_rank_buffer_attention(q, k, v, B, S, H, D, degree, seq_splits, causal=causal)

    def permute_qkv(self, q, k, v, B, S, H, D, degree, seq_splits, head_splits):
        return api.cpattn_ulysses_permute_qkv(q, k, v, B, S, H, D, degree, seq_splits, head_splits)

    def permute(self, x, B, S, H, D, degree, seq_splits, head_splits):
        return api.cpattn_ulysses_permute(x, B, S, H, D, degree, seq_splits, head_splits)

    def unpermute(self, y, B, S, H, D, degree, seq_splits, head_splits):
        return api.cpattn_ulysses_unpermute(y, B, S, H, D, degree, seq_splits, head_splits)

    def backward(self, q, k, v, out, lse, dout, causal):
        return api.cpattn_attention_backward(q, k, v, out, lse, dout, causal)


def _bytes(t: torch.Tensor) -> torch.Tensor:
    return t.reshape(-1).view(torch.uint8)


def _shape4(q):
    if q.dim() != 4 or q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise ValueError("q, k and v must be contiguous bf16 (B, S_r, H, D) tensors")
    return tuple(q.shape)


def _group_rank(group):
    return dist.get_world_size(group), dist.get_rank(group)


def _global_rank(group, r):
    return r if group is None else dist.get_global_rank(group, r)


# ------------------------------------------------------------------- ring

def _ring(q, k, v, group, lens, causal, rotate_method, kernels, pos_base=0):
    """Ring attention of this rank's queries over the chunks `lens` of `group`
    (chunk c at positions pos_base + off_c).  Returns (out bf16, lse float32
    (B, H, S_r))."""
    P, r = _group_rank(group)
    B, Sr, H, D = _shape4(q)
    if len(lens) != P or lens[r] != Sr or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("chunk lengths must have one entry per rank, and entry `rank` must be this rank's length")
    off = _prefix(lens)
    Smax = max(lens)
    order = [(r - t) % P for t in range(P)]          # chunk held after t hand-offs
    visible = [(not causal) or order[t] <= r for t in range(P)]
    steps = [t for t in range(P) if visible[t] and lens[order[t]] > 0]
    out = torch.empty_like(q)
    lse = torch.empty((B, H, Sr), dtype=torch.float32, device=q.device)
    state = torch.empty((B, Sr, H, D), dtype=torch.float32, device=q.device) if len(steps) > 1 else None

    def compute(t, kc, vc, rows):
        if Sr == 0 or t not in steps:
            return
        c = order[t]
        first, last = t == steps[0], t == steps[-1]
        kernels.ring_chunk(q, kc, vc, lens[c], out if last else state, lse, None if first else state,
                           pos_base + off[r], pos_base + off[c], causal, rows)

    if rotate_method == "p2p":
        nxt_rank, prv_rank = _global_rank(group, (r + 1) % P), _global_rank(group, (r - 1) % P)
        n = B * Smax * H * D
        bufs = [(torch.empty(n, dtype=q.dtype, device=q.device), torch.empty(n, dtype=q.dtype, device=q.device))
                for _ in range(2 if P > 2 else 1)]
        cur_k, cur_v, cur_rows = k, v, Sr
        for t in range(P):
            works = []
            if t < P - 1:
                # pass the chunk held now to the next rank, take the next one
                # from the previous rank; both sides agree on every size.
                send_n = B * lens[order[t]] * H * D
                recv_n = B * lens[order[t + 1]] * H * D
                nk, nv = bufs[t % len(bufs)]
                ops = []
                if send_n:
                    ops += [dist.P2POp(dist.isend, _bytes(cur_k)[:2 * send_n], nxt_rank, group),
                            dist.P2POp(dist.isend, _bytes(cur_v)[:2 * send_n], nxt_rank, group)]
                if recv_n:
                    ops += [dist.P2POp(dist.irecv, _bytes(nk)[:2 * recv_n], prv_rank, group),
                            dist.P2POp(dist.irecv, _bytes(nv)[:2 * recv_n], prv_rank, group)]
                if ops:
                    works = dist.batch_isend_irecv(ops)
            compute(t, cur_k, cur_v, cur_rows)
            for w in works:
                w.wait()
            if t < P - 1:
                c1 = order[t + 1]
                cur_k = nk[:B * lens[c1] * H * D].view(B, lens[c1], H, D)
                cur_v = nv[:B * lens[c1] * H * D].view(B, lens[c1], H, D)
                cur_rows = lens[c1]
    elif rotate_method == "allgather":
        gk, gv = _gather_padded(k, v, group, lens)
        for t in range(P):
            c = order[t]
            compute(t, gk[c], gv[c], Smax)
    else:
        raise ValueError("rotate_method must be 'p2p' or 'allgather'")
    return out, lse


def _gather_padded(k, v, group, lens):
    """All-gather of every rank's K and V chunk padded to the longest chunk:
    two (P, B, Smax, H, D) tensors (rows past a chunk's length are padding)."""
    P, r = _group_rank(group)
    B, Sr, H, D = k.shape
    Smax = max(lens)
    if Sr == Smax:
        kp, vp = k, v
    else:
        kp = torch.empty((B, Smax, H, D), dtype=k.dtype, device=k.device)
        vp = torch.empty_like(kp)
        if Sr:
            kp[:, :Sr].copy_(k)
            vp[:, :Sr].copy_(v)
    gk = torch.empty((P, B, Smax, H, D), dtype=k.dtype, device=k.device)
    gv = torch.empty_like(gk)
    dist.all_gather_into_tensor(_bytes(gk), _bytes(kp), group=group)
    dist.all_gather_into_tensor(_bytes(gv), _bytes(vp), group=group)
    return gk, gv


def ring_attention(q, k, v, group=None, chunk_lens=None, causal=False, rotate_method="p2p", kernels=None):
    """Ring attention over the ranks of `group`.  q, k, v: this rank's shard,
    contiguous bf16 (B, S_r, H, D).  chunk_lens: every rank's S_r (None: all
    equal).  causal: key j visible to query i iff j <= i (positions in the full
    sequence).  Returns (out (B, S_r, H, D) bf16, lse (B, H, S_r) float32)."""
    P, r = _group_rank(group)
    lens = list(chunk_lens) if chunk_lens is not None else [q.shape[1]] * P
    return _ring(q, k, v, group, lens, causal, rotate_method, kernels or CudaKernels())


# ---------------------------------------------------------------- Ulysses

def _all_to_all(recv, send, recv_splits, send_splits, group):
    """all_to_all_single on the bytes of two bf16 buffers; splits in elements."""
    dist.all_to_all_single(_bytes(recv), _bytes(send), [2 * n for n in recv_splits], [2 * n for n in send_splits],
                           group=group)


def _ulysses_to_heads(tensors, group, seq, heads, kernels):
    """First all-to-all: this rank's (B, S_r, H, D) tokens -> every token of
    its heads, as rank buffers (B, S_u, H_r, D) concatenated (flat)."""
    P, r = _group_rank(group)
    B, Sr, H, D = tensors[0].shape
    S, Hr = sum(seq), heads[r]
    pack_seq = [Sr] + [0] * (P - 1)          # all local tokens as "rank 0"
    if not Sr:
        packed = [torch.empty(0, dtype=tensors[0].dtype, device=tensors[0].device)] * len(tensors)
    elif len(tensors) == 3:
        packed = kernels.permute_qkv(*tensors, B, Sr, H, D, P, pack_seq, heads)
    else:
        packed = [kernels.permute(x, B, Sr, H, D, P, pack_seq, heads) for x in tensors]
    send_splits = [B * Sr * heads[u] * D for u in range(P)]
    recv_splits = [B * seq[u] * Hr * D for u in range(P)]
    out = []
    for y in packed:
        recv = torch.empty(B * S * Hr * D, dtype=y.dtype, device=y.device)
        _all_to_all(recv, y, recv_splits, send_splits, group)
        out.append(recv)
    return out


def _ulysses_to_tokens(yo, group, seq, heads, B, H, D, kernels):
    """Second all-to-all: this rank's heads for every token (rank buffers) ->
    all heads of its own tokens, (B, S_r, H, D)."""
    P, r = _group_rank(group)
    Sr, Hr = seq[r], heads[r]
    send_splits = [B * seq[u] * Hr * D for u in range(P)]
    recv_splits = [B * Sr * heads[u] * D for u in range(P)]
    recv = torch.empty(B * Sr * H * D, dtype=yo.dtype, device=yo.device)
    _all_to_all(recv, yo, recv_splits, send_splits, group)
    if Sr == 0:
        return recv.view(B, 0, H, D)
    x = kernels.unpermute(recv, B, Sr, H, D, P, [Sr] + [0] * (P - 1), heads)
    return x.view(B, Sr, H, D)


def ulysses_attention(q, k, v, group=None, seq_splits=None, head_splits=None, causal=False, kernels=None):
    """Ulysses attention over the ranks of `group`.  q, k, v: this rank's
    tokens (B, S_r, H, D) bf16.  seq_splits: every rank's S_r (None: equal);
    head_splits: the heads of every rank (None: equal; uneven = Ulysses
    Anything).  Returns (out (B, S_r, H, D) bf16, lse (B, H_r, S) float32 for
    this rank's heads hoff_r .. hoff_r + H_r - 1 and every token)."""
    kernels = kernels or CudaKernels()
    P, r = _group_rank(group)
    B, Sr, H, D = _shape4(q)
    seq = list(seq_splits) if seq_splits is not None else [Sr] * P
    heads = list(head_splits) if head_splits is not None else equal_splits(H, P)
    if len(seq) != P or seq[r] != Sr or len(heads) != P or sum(heads) != H:
        raise ValueError("splits must have one entry per rank; seq_splits[rank] must be this rank's length")
    S, Hr = sum(seq), heads[r]
    yq, yk, yv = _ulysses_to_heads((q, k, v), group, seq, heads, kernels)
    if Hr:
        yo, lse = kernels.rank_buffer(yq, yk, yv, B, S, Hr, D, P, seq, causal)
    else:
        yo, lse = yq, torch.empty((B, 0, S), dtype=torch.float32, device=q.device)
    return _ulysses_to_tokens(yo, group, seq, heads, B, H, D, kernels), lse


# ---------------------------------------------------- Ulysses, training

def _heads_dense(y, B, S, Hr, D, P, seq, kernels):
    """Head-side rank buffers (B, S_u, H_r, D), concatenated -> (B, S, H_r, D).
    For B = 1 the two layouts are the same bytes."""
    if B == 1 or not Hr or not S:
        return y.view(B, S, Hr, D)
    return kernels.permute(y, B, S, Hr, D, P, seq, [Hr] + [0] * (P - 1)).view(B, S, Hr, D)


def _heads_rank_buffers(x, B, S, Hr, D, P, seq, kernels):
    """The inverse of _heads_dense."""
    if B == 1 or not Hr or not S:
        return x.reshape(-1)
    return kernels.unpermute(x.reshape(-1), B, S, Hr, D, P, seq, [Hr] + [0] * (P - 1))


class UlyssesAttentionFunction(torch.autograd.Function):
    """Ulysses attention over the ranks of a group, differentiable ("Ulysses
    Sequence Parallelism" article, sections 1, 4 and 7: training over long
    contexts).  The forward is ulysses_attention's and keeps the head-side Q,
    K, V and output.  The backward sends dO through the same all-to-all, runs
    the attention backward on this rank's heads over every token, and sends
    dQ, dK and dV back through the inverse all-to-all."""

    @staticmethod
    def forward(ctx, q, k, v, group, seq, heads, causal, kernels):
        P, r = _group_rank(group)
        B, Sr, H, D = _shape4(q)
        S, Hr = sum(seq), heads[r]
        yq, yk, yv = _ulysses_to_heads((q, k, v), group, seq, heads, kernels)
        if Hr:
            yo, lse = kernels.rank_buffer(yq, yk, yv, B, S, Hr, D, P, seq, causal)
        else:
            yo, lse = yq, torch.empty((B, 0, S), dtype=torch.float32, device=q.device)
        ctx.save_for_backward(yq, yk, yv, yo, lse)
        ctx.meta = (group, list(seq), list(heads), bool(causal), kernels, (B, Sr, H, D))
        return _ulysses_to_tokens(yo, group, seq, heads, B, H, D, kernels)

    @staticmethod
    def backward(ctx, dout):
        yq, yk, yv, yo, lse = ctx.saved_tensors
        group, seq, heads, causal, kernels, (B, Sr, H, D) = ctx.meta
        dq, dk, dv = _ulysses_backward(yq, yk, yv, yo, lse, dout, group, seq, heads, causal, kernels, B, H, D)
        return dq, dk, dv, None, None, None, None, None


def _ulysses_backward(yq, yk, yv, yo, lse, dout, group, seq, heads, causal, kernels, B, H, D):
    """dQ, dK, dV of this rank's token shard from the head-side Q, K, V,
    output and LSE of its heads: dO through the first all-to-all, the
    attention backward on the heads over every token, the gradients through
    the inverse all-to-all."""
    P, r = _group_rank(group)
    S, Hr = sum(seq), heads[r]
    (ydo,) = _ulysses_to_heads((dout.contiguous(),), group, seq, heads, kernels)
    if Hr and S:
        dense = [_heads_dense(y, B, S, Hr, D, P, seq, kernels) for y in (yq, yk, yv, yo, ydo)]
        dqh, dkh, dvh = kernels.backward(dense[0], dense[1], dense[2], dense[3], lse, dense[4], causal)
        grads = [_heads_rank_buffers(g, B, S, Hr, D, P, seq, kernels) for g in (dqh, dkh, dvh)]
    else:
        grads = [torch.empty(0, dtype=yq.dtype, device=yq.device)] * 3
    return tuple(_ulysses_to_tokens(g, group, seq, heads, B, H, D, kernels) for g in grads)


class HeadSideBackwardFunction(torch.autograd.Function):
    """An exchange's forward (ring or unified) with its gradient taken on the
    head side: the gradient of attention depends only on the attention of the
    full sequence, not on how the forward moved the data.  The backward sends
    Q, K, V and dO through a Ulysses all-to-all over `group` (whose rank order
    is the sequence order), recomputes this rank's heads' output and LSE there
    (one extra forward), runs the attention backward, and sends the gradients
    back.  Heads are split front-loaded (the Ulysses Anything rule), so any H
    works, and a rank without heads only moves data."""

    @staticmethod
    def forward(ctx, q, k, v, forward_fn, group, seq, causal, kernels):
        ctx.save_for_backward(q, k, v)
        ctx.meta = (group, list(seq), bool(causal), kernels)
        with torch.no_grad():
            return forward_fn(q, k, v)

    @staticmethod
    def backward(ctx, dout):
        q, k, v = ctx.saved_tensors
        group, seq, causal, kernels = ctx.meta
        P, r = _group_rank(group)
        B, Sr, H, D = q.shape
        S, heads = sum(seq), front_loaded_splits(H, P)
        yq, yk, yv = _ulysses_to_heads((q, k, v), group, seq, heads, kernels)
        if heads[r] and S:
            yo, lse = kernels.rank_buffer(yq, yk, yv, B, S, heads[r], D, P, seq, causal)
        else:
            yo, lse = yq, torch.empty((B, 0, S), dtype=torch.float32, device=q.device)
        dq, dk, dv = _ulysses_backward(yq, yk, yv, yo, lse, dout, group, seq, heads, causal, kernels, B, H, D)
        return dq, dk, dv, None, None, None, None, None


def ring_attention_trainable(q, k, v, group=None, chunk_lens=None, causal=False, rotate_method="p2p", kernels=None):
    """ring_attention's output with a gradient (HeadSideBackwardFunction): the
    forward is the ring exchange; the backward goes through a Ulysses
    all-to-all over the same group.  Every rank of the group must run the
    backward."""
    kernels = kernels or CudaKernels()
    P, r = _group_rank(group)
    B, Sr, H, D = _shape4(q)
    lens = list(chunk_lens) if chunk_lens is not None else [Sr] * P
    if len(lens) != P or lens[r] != Sr:
        raise ValueError("chunk_lens must have one entry per rank; entry `rank` must be this rank's length")
    fwd = lambda a, b, c: ring_attention(a, b, c, group, lens, causal, rotate_method, kernels)[0]
    return HeadSideBackwardFunction.apply(q, k, v, fwd, group, lens, causal, kernels)


def ulysses_attention_trainable(q, k, v, group=None, seq_splits=None, head_splits=None, causal=False, kernels=None):
    """ulysses_attention as an autograd function: returns out (B, S_r, H, D)
    bf16 whose gradient flows back to this rank's q, k and v.  Arguments as
    ulysses_attention's; every rank of the group must run the backward."""
    kernels = kernels or CudaKernels()
    P, r = _group_rank(group)
    B, Sr, H, D = _shape4(q)
    seq = list(seq_splits) if seq_splits is not None else [Sr] * P
    heads = list(head_splits) if head_splits is not None else equal_splits(H, P)
    if len(seq) != P or seq[r] != Sr or len(heads) != P or sum(heads) != H:
        raise ValueError("splits must have one entry per rank; seq_splits[rank] must be this rank's length")
    return UlyssesAttentionFunction.apply(q, k, v, group, seq, heads, causal, kernels)


# -------------------------------------------------------------- kv_gather

def kv_gather_attention(q, k, v, group=None, q_lens=None, kernels=None):
    """kv_gather over the ranks of `group`: all-gather K and V (padded to the
    longest shard), then attention of this rank's queries against every key.
    Returns (out (B, S_r, H, D) bf16, lse (B, H, S_r) float32)."""
    kernels = kernels or CudaKernels()
    P, r = _group_rank(group)
    B, Sr, H, D = _shape4(q)
    lens = list(q_lens) if q_lens is not None else [Sr] * P
    if len(lens) != P or lens[r] != Sr:
        raise ValueError("q_lens must have one entry per rank; entry `rank` must be this rank's length")
    gk, gv = _gather_padded(k, v, group, lens)
    if Sr == 0:
        return torch.empty_like(q), torch.empty((B, H, 0), dtype=torch.float32, device=q.device)
    return kernels.gathered(q, gk, gv, P, r, lens, False)


# ---------------------------------------------------------------- unified

def unified_groups(ring_degree, ulysses_degree, backend=None):
    """Process groups of a ring_degree x ulysses_degree grid of the default
    group's ranks, rank = i * ulysses_degree + j (a Ulysses group holds
    consecutive ranks, i.e. the GPUs of one NVLink domain).  Every rank must
    call this (each group is created on all ranks).  Returns (ring_group,
    ulysses_group) of the calling rank."""
    world, rank = dist.get_world_size(), dist.get_rank()
    R, U = ring_degree, ulysses_degree
    if R * U != world:
        raise ValueError(f"ring_degree x ulysses_degree = {R * U}, but the world has {world} ranks")
    mine_ring = mine_uly = None
    for i in range(R):
        g = dist.new_group([i * U + j for j in range(U)], backend=backend)
        if rank // U == i:
            mine_uly = g
    for j in range(U):
        g = dist.new_group([i * U + j for i in range(R)], backend=backend)
        if rank % U == j:
            mine_ring = g
    return mine_ring, mine_uly


def unified_attention(q, k, v, ring_group, ulysses_group, ring_lens=None, sub_splits=None, head_splits=None,
                      causal=False, rotate_method="p2p", kernels=None):
    """Unified (ring x Ulysses) attention.  The rank at (i, j) of the grid
    holds sub-shard j of ring chunk i: q, k, v (B, S_ij, H, D) bf16.
    ring_lens: the R chunk lengths (None: equal, derived from the local length
    and the sub-splits); sub_splits: for every chunk i the U sub-shard lengths
    (None: front-loaded splits of each chunk); head_splits: the U head groups
    (None: equal).  Returns (out (B, S_ij, H, D) bf16, lse (B, H_j, S_i)
    float32 for head group j over chunk i)."""
    kernels = kernels or CudaKernels()
    R, i = _group_rank(ring_group)
    U, j = _group_rank(ulysses_group)
    B, Sij, H, D = _shape4(q)
    if ring_lens is None:
        if sub_splits is not None:
            ring_lens = [sum(s) for s in sub_splits]
        else:
            ring_lens = [Sij * U] * R
    ring_lens = list(ring_lens)
    subs = [list(s) for s in sub_splits] if sub_splits is not None else [front_loaded_splits(n, U) for n in ring_lens]
    heads = list(head_splits) if head_splits is not None else equal_splits(H, U)
    if len(ring_lens) != R or len(subs) != R or any(len(s) != U for s in subs) or subs[i][j] != Sij:
        raise ValueError("ring_lens / sub_splits do not match the grid or this rank's length")
    Si, Hj = ring_lens[i], heads[j]
    off = _prefix(ring_lens)
    # 1. Ulysses all-to-all inside the group: chunk i, head group j
    yq, yk, yv = _ulysses_to_heads((q, k, v), ulysses_group, subs[i], heads, kernels)
    if Hj and Si:
        if B > 1:   # rank buffers (B, S_iu, H_j, D) -> (B, S_i, H_j, D)
            lead = [Hj] + [0] * (U - 1)
            yq, yk, yv = (kernels.permute(y, B, Si, Hj, D, U, subs[i], lead) for y in (yq, yk, yv))
        qc, kc, vc = (y.view(B, Si, Hj, D) for y in (yq, yk, yv))
    else:
        qc = kc = vc = torch.empty((B, Si, Hj, D), dtype=q.dtype, device=q.device)
    # 2. ring over the chunks, inside the ring group of head group j (every
    #    rank of that ring group holds head group j, so all of them skip it
    #    together when the group has no heads)
    if Hj:
        oc, lse = _ring(qc, kc, vc, ring_group, ring_lens, causal, rotate_method, kernels)
    else:
        oc, lse = qc, torch.empty((B, 0, Si), dtype=torch.float32, device=q.device)
    # 3. back to rank buffers and through the inverse all-to-all
    yo = oc.reshape(-1)
    if B > 1 and Hj and Si:
        yo = kernels.unpermute(yo, B, Si, Hj, D, U, subs[i], [Hj] + [0] * (U - 1))
    return _ulysses_to_tokens(yo, ulysses_group, subs[i], heads, B, H, D, kernels), lse


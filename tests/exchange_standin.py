"""A stand-in for the library's kernels on CPU ranks, used by the tests of the
multi-GPU exchanges (context_attention_long_b200.exchange) with gloo process
groups: the contract of exchange.CudaKernels, computed by the oracle in
float64 on host tensors and stored in the kernels' output types (bf16 outputs,
float32 partial states and LSEs).  Test infrastructure only: the product path
always runs the CUDA kernels."""
import numpy as np
import torch

import oracle


def _f64(t):
    return t.detach().double().numpy()


def _full_from_rank_buffers(x, B, H, D, seq):
    off = np.concatenate([[0], np.cumsum(seq)]).astype(int)
    parts, pos = [], 0
    for n in seq:
        parts.append(x[pos:pos + B * n * H * D].reshape(B, n, H, D))
        pos += B * n * H * D
    return np.concatenate(parts, axis=1), off


def _rank_buffers_from_full(x, seq):
    off = np.concatenate([[0], np.cumsum(seq)]).astype(int)
    return np.concatenate([np.ascontiguousarray(x[:, off[u]:off[u + 1]]).reshape(-1) for u in range(len(seq))])


class OracleKernels:
    def ring_chunk(self, q, k, v, Skv, out, lse, prev, q_pos0, kv_pos0, causal, kv_batch_rows):
        B, Sq, H, D = q.shape
        kk = k.reshape(B, kv_batch_rows, H, D)[:, :Skv]
        vv = v.reshape(B, kv_batch_rows, H, D)[:, :Skv]
        qpos = q_pos0 + np.arange(Sq)
        kpos = kv_pos0 + np.arange(Skv)
        o, l = oracle.attention(_f64(q), _f64(kk), _f64(vv), qpos if causal else None, kpos if causal else None)
        if prev is not None:
            o, l = oracle.lse_merge([_f64(prev), o], [_f64(lse), l])
        out.copy_(torch.from_numpy(o).to(out.dtype))
        lse.copy_(torch.from_numpy(l).float())

    def gathered(self, q, k, v, degree, rank, kv_lens, causal):
        B, Sq, H, D = q.shape
        kf = np.concatenate([_f64(k[c][:, :kv_lens[c]]) for c in range(degree)], axis=1)
        vf = np.concatenate([_f64(v[c][:, :kv_lens[c]]) for c in range(degree)], axis=1)
        off = int(sum(kv_lens[:rank]))
        qpos, kpos = off + np.arange(Sq), np.arange(kf.shape[1])
        o, l = oracle.attention(_f64(q), kf, vf, qpos if causal else None, kpos if causal else None)
        return torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(l).float()

    def rank_buffer(self, q, k, v, B, S, H, D, degree, seq_splits, causal):
        (qf, _), (kf, _), (vf, _) = (_full_from_rank_buffers(_f64(t), B, H, D, seq_splits) for t in (q, k, v))
        pos = np.arange(S)
        o, l = oracle.attention(qf, kf, vf, pos if causal else None, pos if causal else None)
        return torch.from_numpy(_rank_buffers_from_full(o, seq_splits)).to(torch.bfloat16), torch.from_numpy(l).float()

    @staticmethod
    def _bits(t):
        return t.detach().reshape(-1).view(torch.int16).numpy()

    @staticmethod
    def _from_bits(a):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16)

    def permute_qkv(self, q, k, v, B, S, H, D, degree, seq_splits, head_splits):
        return tuple(self.permute(t, B, S, H, D, degree, seq_splits, head_splits) for t in (q, k, v))

    def permute(self, x, B, S, H, D, degree, seq_splits, head_splits):
        return self._from_bits(oracle.ulysses_permute(self._bits(x), B, S, H, D, degree, seq_splits, head_splits))

    def unpermute(self, y, B, S, H, D, degree, seq_splits, head_splits):
        return self._from_bits(oracle.ulysses_unpermute(self._bits(y), B, S, H, D, degree, seq_splits, head_splits))

    def backward(self, q, k, v, out, lse, dout, causal):
        grads = oracle.attention_backward(_f64(q), _f64(k), _f64(v), _f64(dout), causal=causal)
        return tuple(torch.from_numpy(g).to(torch.bfloat16) for g in grads)

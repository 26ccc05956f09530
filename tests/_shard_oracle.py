"""An exact host backend for the sharded-step phases (test only): the oracle's float64
arithmetic behind the same phase interface as the CUDA backend, so that the exchange logic of
learned_sparse_kv_decode_b200.sharded can run with real gloo collectives on the CPU."""
import math

import numpy as np
import torch

import oracle
from learned_sparse_kv_decode_b200.sharded import Candidates, Partial

NEG = -np.finfo(np.float32).max


class OracleShardBackend:
    def __init__(self, plan, local_emb, local_K, local_V):
        self.plan = plan
        self.emb, self.K, self.V = local_emb, local_K, local_V  # per sequence float64 arrays

    def candidates(self, q_emb, _unused=None) -> Candidates:
        p = self.plan
        s = np.full((p.B, p.k_pad), NEG)
        ids = np.full((p.B, p.k_pad), -1, dtype=np.int64)
        for b in range(p.B):
            sc = oracle.chunk_scores(q_emb[b], self.emb[b])
            loc = oracle.topk(sc, p.k_local[b])
            s[b, :len(loc)] = sc[loc]
            ids[b, :len(loc)] = loc + p.global_offset[b]
        return Candidates(torch.from_numpy(s), torch.from_numpy(ids))

    def select(self, all_scores, all_ids) -> None:
        p = self.plan
        s = all_scores.numpy()
        ids = all_ids.numpy()
        self.global_ids, self.local_ids = [], []
        for b in range(p.B):
            seq_s = s[:, b, :].reshape(-1)       # rank-major: ascending global ids, padding after
            seq_i = ids[:, b, :].reshape(-1)
            pos = oracle.topk(seq_s, p.k[b])
            gid = seq_i[pos]
            self.global_ids.append(gid)
            lo, hi = p.global_offset[b], p.global_offset[b] + p.local_n[b]
            self.local_ids.append(gid[(gid >= lo) & (gid < hi)] - lo)

    def attend(self, q, K=None, V=None) -> Partial:
        p = self.plan
        out = np.zeros((p.B, p.H, 128))
        lse = np.full((p.B, p.H), -np.inf)
        for b in range(p.B):
            if len(self.local_ids[b]) == 0:
                continue
            tok = oracle.kept_tokens(self.local_ids[b], p.C)
            out[b], lse[b] = oracle.attention(q[b], self.K[b][tok], self.V[b][tok], 1.0 / math.sqrt(128))
        return Partial(torch.from_numpy(out), torch.from_numpy(lse))

    def merge(self, all_out, all_lse):
        o, l = all_out.numpy(), all_lse.numpy()
        M = l.max(axis=0)
        wgt = np.where(np.isfinite(l), np.exp(l - M[None]), 0.0)
        L = wgt.sum(axis=0)
        return (wgt[..., None] * o).sum(axis=0) / L[..., None], M + np.log(L)

"""Chunk-sharded LSA decode step: one sequence's chunks split across G ranks.

The step (include/lsa.h, "Chunk-sharded step across G ranks") runs in phases; the two
exchanges between them are all-gathers of fixed-size tensors:

    cand = step.candidates(q_emb, chunk_emb)          # local score + top-k -> (score, gid)
    step.select(all_gather(cand.scores), all_gather(cand.ids))
    part = step.attend(q, K, V)                       # local attention over own kept chunks
    out, lse = step.merge(all_gather(part.out), all_gather(part.lse))

`run_distributed` drives the phases with torch.distributed (NCCL over NVLink on GPUs, one
process per GPU; the only collectives are those two all-gathers, each carried out as one
all_gather_into_tensor per tensor; under a host backend such as gloo the device tensors are
gathered through host memory). `run_emulated` drives G shard objects in one process
(the all-gathers become stacks), which exercises every kernel of the sharded path on one
GPU. All arithmetic happens in the library's CUDA kernels (`CudaShardBackend`); the backend
object exists so that the exchange logic can also be checked on the host with an exact
reference backend.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import abi


@dataclass
class ShardPlan:
    """Which chunks of each sequence this rank owns, and the step's shape."""
    B: int
    Q: int
    E: int
    H: int
    C: int
    G: int
    rank: int
    k: list             # global kept chunks per sequence
    local_n: list       # this rank's chunks per sequence
    global_offset: list  # global id of this rank's first chunk per sequence
    emb_dtype: str = "bf16"
    kv_dtype: str = "bf16"

    @property
    def k_local(self) -> list:
        return [min(kb, nb) for kb, nb in zip(self.k, self.local_n)]

    @property
    def k_pad(self) -> int:
        return max(self.k)


def split_chunks(n_chunks: list, G: int) -> list:
    """Contiguous near-equal runs: rank g owns chunks [off, off + n) of each sequence.
    Returns [(local_n list, global_offset list)] per rank."""
    out = []
    for g in range(G):
        ln, go = [], []
        for n in n_chunks:
            lo, hi = (n * g) // G, (n * (g + 1)) // G
            if hi <= lo:
                raise ValueError("every rank needs at least one chunk of every sequence")
            ln.append(hi - lo)
            go.append(lo)
        out.append((ln, go))
    return out


@dataclass
class Candidates:
    scores: torch.Tensor  # [B][k_pad] float32
    ids: torch.Tensor     # [B][k_pad] int32 global chunk ids (-1 = padding)


@dataclass
class Partial:
    out: torch.Tensor  # [B][H][Dh] float32
    lse: torch.Tensor  # [B][H] float32


class CudaShardBackend:
    """The sharded phases through the C ABI (device tensors; torch only allocates)."""

    def __init__(self, plan: ShardPlan, device="cuda"):
        self.plan = plan
        p = plan
        off = np.concatenate([[0], np.cumsum(p.local_n)]).astype(np.int64).tolist()
        self.local_dims = abi.Dims(p.B, p.Q, p.E, p.H, p.C, chunk_offsets=off, k_per_seq=p.k_local,
                                   emb_dtype=p.emb_dtype, kv_dtype=p.kv_dtype)
        self.global_dims = abi.Dims(p.B, 1, p.E, p.H, p.C, N=p.G * p.k_pad, k_per_seq=p.k,
                                    emb_dtype=p.emb_dtype, kv_dtype=p.kv_dtype)
        self.ws_local = abi.alloc_workspace(self.local_dims, device)
        self.ws_global = abi.alloc_workspace(self.global_dims, device)
        n_local, kl, kg = int(sum(p.local_n)), int(sum(p.k_local)), int(sum(p.k))
        f32, i32 = torch.float32, torch.int32
        self.scores = torch.empty(n_local, dtype=f32, device=device)
        self.local_cand = torch.empty(kl, dtype=i32, device=device)
        self.cand_s = torch.empty((p.B, p.k_pad), dtype=f32, device=device)
        self.cand_i = torch.empty((p.B, p.k_pad), dtype=i32, device=device)
        self.seq_s = torch.empty((p.B, p.G * p.k_pad), dtype=f32, device=device)
        self.seq_i = torch.empty((p.B, p.G * p.k_pad), dtype=i32, device=device)
        self.global_ids = torch.empty(kg, dtype=i32, device=device)
        self.local_ids = torch.empty(kl, dtype=i32, device=device)
        self.local_count = torch.empty(p.B, dtype=i32, device=device)
        self.out_g = torch.empty((p.B, p.H, abi.LSA_HEAD_DIM), dtype=f32, device=device)
        self.lse_g = torch.empty((p.B, p.H), dtype=f32, device=device)
        self.out = torch.empty_like(self.out_g)
        self.lse = torch.empty_like(self.lse_g)

    def candidates(self, q_emb, chunk_emb) -> Candidates:
        abi.lsa_score_chunks(self.local_dims, q_emb, chunk_emb, self.scores, self.ws_local)
        abi.lsa_topk_select(self.local_dims, self.scores, self.local_cand, self.ws_local)
        abi.lsa_shard_candidates(self.local_dims, self.scores, self.local_cand, self.plan.global_offset,
                                 self.plan.k_pad, self.cand_s, self.cand_i)
        return Candidates(self.cand_s, self.cand_i)

    def select(self, all_scores, all_ids) -> None:
        p = self.plan
        abi.lsa_shard_global_select(self.global_dims, p.G, p.global_offset, p.local_n, all_scores, all_ids,
                                    self.seq_s, self.seq_i, self.global_ids, self.local_ids, self.local_count,
                                    self.ws_global)

    def attend(self, q, K, V) -> Partial:
        abi.lsa_sparse_decode_attn_counts(self.local_dims, q, K, V, self.local_ids, self.local_count,
                                          self.out_g, self.lse_g, self.ws_local)
        return Partial(self.out_g, self.lse_g)

    def merge(self, all_out, all_lse):
        abi.lsa_merge_partials(self.plan.G, self.plan.B, self.plan.H, all_out, all_lse, self.out, self.lse)
        return self.out, self.lse


def run_emulated(backends: list, q_emb, chunk_embs: list, q, Ks: list, Vs: list):
    """All G shards in one process: the all-gathers become stacks (rank-major, as all_gather)."""
    cands = [bk.candidates(q_emb, ce) for bk, ce in zip(backends, chunk_embs)]
    all_s = torch.stack([c.scores for c in cands]).contiguous()
    all_i = torch.stack([c.ids for c in cands]).contiguous()
    for bk in backends:
        bk.select(all_s, all_i)
    parts = [bk.attend(q, K, V) for bk, K, V in zip(backends, Ks, Vs)]
    all_o = torch.stack([pt.out for pt in parts]).contiguous()
    all_l = torch.stack([pt.lse for pt in parts]).contiguous()
    return [bk.merge(all_o, all_l) for bk in backends], backends[0].global_ids


def _all_gather(t: torch.Tensor, world: int) -> torch.Tensor:
    """[world, *t.shape] in rank order (gathered as a concatenation along dim 0, the form
    every backend accepts)."""
    import torch.distributed as dist
    if t.is_cuda and dist.get_backend() != "nccl":  # a host collective backend (gloo): via host memory
        return _all_gather(t.cpu(), world).to(t.device)
    t = t.contiguous()
    out = torch.empty((world * t.shape[0], *t.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(out, t)
    return out.view(world, *t.shape)


def run_distributed(backend, q_emb, chunk_emb, q, K, V):
    """This rank's phases with torch.distributed all-gathers (every rank calls it)."""
    world = backend.plan.G
    cand = backend.candidates(q_emb, chunk_emb)
    backend.select(_all_gather(cand.scores, world), _all_gather(cand.ids, world))
    part = backend.attend(q, K, V)
    return backend.merge(_all_gather(part.out, world), _all_gather(part.lse, world))

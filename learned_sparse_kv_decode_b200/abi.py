"""ctypes binding of include/lsa.h (liblsa_b200.so): argument marshalling only.

Every Python function here has the name of the C entry point it calls and does
nothing but check tensor types, take raw device pointers and the stream handle,
and call the library; all work runs in the CUDA kernels. Tensors are torch CUDA
tensors (torch is used for device memory and streams only). A missing library
raises at import time: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblsa_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "lsa.h")

LSA_OK, LSA_ERR_INVALID_ARG, LSA_ERR_WORKSPACE, LSA_ERR_CUDA = 0, 1, 2, 3
LSA_ERR_NONFINITE, LSA_ERR_TIMEOUT, LSA_ERR_UNSUPPORTED, LSA_ERR_BAD_ID = 4, 5, 6, 7
LSA_F32, LSA_BF16 = 0, 1
LSA_ENSEMBLE_MAX, LSA_ENSEMBLE_MEAN = 0, 1
LSA_INDEX_DIM = 128
LSA_MAX_BATCH = 256
LSA_HEAD_DIM = 128


class LsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {string(status)}")


class _Dims(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Q", ctypes.c_int32), ("E", ctypes.c_int32),
        ("H", ctypes.c_int32), ("Dh", ctypes.c_int32), ("chunk_len", ctypes.c_int32),
        ("N", ctypes.c_int32), ("k", ctypes.c_int32),
        ("chunk_offsets", ctypes.POINTER(ctypes.c_int64)),
        ("k_per_seq", ctypes.POINTER(ctypes.c_int32)),
        ("emb_dtype", ctypes.c_int), ("kv_dtype", ctypes.c_int),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with learned_sparse_kv_decode_b200.build.build()")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, dp = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(_Dims)
    sig = {
        "lsa_abi_version": ([], ctypes.c_int),
        "lsa_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "lsa_workspace_size": ([dp, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
        "lsa_workspace_init": ([vp, sz, vp], ctypes.c_int),
        "lsa_score_chunks": ([dp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_topk_select": ([dp, vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_gather_kv": ([dp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_sparse_decode_attn": ([dp, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_decode_step": ([dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_sparse_decode_attn_lookahead": ([dp, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_decode_step_lookahead": ([dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_get_device_status": ([vp, vp], ctypes.c_int),
        "lsa_lookahead_partition": ([dp, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)],
                                    ctypes.c_int),
        "lsa_sparse_decode_attn_noalloc": ([dp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsa_refresh_resident": ([dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_threshold_select": ([dp, vp, ctypes.c_float, ctypes.c_int32, vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_decode_step_threshold": ([dp, vp, vp, vp, vp, vp, ctypes.c_float, ctypes.c_int32, vp, vp, vp, vp,
                                       vp, sz, vp], ctypes.c_int),
        "lsa_indexer_score_fp8": ([dp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int, vp, vp, vp, vp, vp, vp, sz, vp],
                                  ctypes.c_int),
        "lsa_decode_step_fp8": ([dp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp,
                                 vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_sparse_decode_attn_counts": ([dp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_shard_candidates": ([dp, vp, vp, ctypes.POINTER(ctypes.c_int32), ctypes.c_int32, vp, vp, vp],
                                 ctypes.c_int),
        "lsa_shard_global_select": ([dp, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32),
                                     vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "lsa_merge_partials": ([ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, vp, vp, vp, vp, vp], ctypes.c_int),
        "lsa_read_stream": ([vp, sz, vp], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def header_symbols() -> list:
    """Names of the entry points declared in include/lsa.h."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"LSA_API\s+[\w\s\*]*?\b(lsa_\w+)\s*\(", text)


def string(status: int) -> str:
    return lib.lsa_status_string(int(status)).decode()


def lsa_abi_version() -> int:
    return lib.lsa_abi_version()


class Dims:
    """lsa_dims plus the host arrays it points to (kept alive with it)."""

    def __init__(self, B, Q, E, H, chunk_len, N=None, k=None, chunk_offsets=None, k_per_seq=None,
                 emb_dtype="bf16", kv_dtype="bf16", Dh=LSA_HEAD_DIM):
        def dt(x):
            return LSA_BF16 if x in ("bf16", torch.bfloat16, LSA_BF16) else LSA_F32
        self._off = None if chunk_offsets is None else (ctypes.c_int64 * len(chunk_offsets))(*map(int, chunk_offsets))
        self._k = None if k_per_seq is None else (ctypes.c_int32 * len(k_per_seq))(*map(int, k_per_seq))
        self.c = _Dims(int(B), int(Q), int(E), int(H), int(Dh), int(chunk_len),
                       int(N or 0), int(k or 0),
                       ctypes.cast(self._off, ctypes.POINTER(ctypes.c_int64)) if self._off is not None else None,
                       ctypes.cast(self._k, ctypes.POINTER(ctypes.c_int32)) if self._k is not None else None,
                       dt(emb_dtype), dt(kv_dtype))

    @property
    def ptr(self):
        return ctypes.byref(self.c)


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, where: str):
    if rc != LSA_OK:
        raise LsaError(rc, where)


def _nbytes(t):
    return t.numel() * t.element_size()


def lsa_workspace_size(dims: Dims) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.lsa_workspace_size(dims.ptr, ctypes.byref(n)), "lsa_workspace_size")
    return n.value


def lsa_workspace_init(ws, stream=None) -> None:
    _check(lib.lsa_workspace_init(_p(ws), _nbytes(ws), _stream(stream)), "lsa_workspace_init")


def lsa_score_chunks(dims, q_emb, chunk_emb, scores, ws, stream=None) -> None:
    _check(lib.lsa_score_chunks(dims.ptr, _p(q_emb), _p(chunk_emb), _p(scores), _p(ws), _nbytes(ws),
                                _stream(stream)), "lsa_score_chunks")


def lsa_topk_select(dims, scores, chunk_ids, ws, stream=None) -> None:
    _check(lib.lsa_topk_select(dims.ptr, _p(scores), _p(chunk_ids), _p(ws), _nbytes(ws), _stream(stream)),
           "lsa_topk_select")


def lsa_gather_kv(dims, K, V, chunk_ids, K_res, V_res, ws, stream=None) -> None:
    _check(lib.lsa_gather_kv(dims.ptr, _p(K), _p(V), _p(chunk_ids), _p(K_res), _p(V_res), _p(ws),
                             _nbytes(ws), _stream(stream)), "lsa_gather_kv")


def lsa_sparse_decode_attn(dims, q, K, V, chunk_ids, out, lse, ws, stream=None) -> None:
    _check(lib.lsa_sparse_decode_attn(dims.ptr, _p(q), _p(K), _p(V), _p(chunk_ids), _p(out), _p(lse),
                                      _p(ws), _nbytes(ws), _stream(stream)), "lsa_sparse_decode_attn")


def lsa_decode_step(dims, q_emb, chunk_emb, q, K, V, chunk_ids_out, out, lse, ws, stream=None) -> None:
    _check(lib.lsa_decode_step(dims.ptr, _p(q_emb), _p(chunk_emb), _p(q), _p(K), _p(V), _p(chunk_ids_out),
                               _p(out), _p(lse), _p(ws), _nbytes(ws), _stream(stream)), "lsa_decode_step")


def lsa_sparse_decode_attn_lookahead(dims, q, K, V, chunk_ids, out, lse, ws, stream=None) -> None:
    _check(lib.lsa_sparse_decode_attn_lookahead(dims.ptr, _p(q), _p(K), _p(V), _p(chunk_ids), _p(out), _p(lse),
                                                _p(ws), _nbytes(ws), _stream(stream)),
           "lsa_sparse_decode_attn_lookahead")


def lsa_decode_step_lookahead(dims, q_emb, chunk_emb, q, K, V, chunk_ids_out, out, lse, ws, stream=None) -> None:
    _check(lib.lsa_decode_step_lookahead(dims.ptr, _p(q_emb), _p(chunk_emb), _p(q), _p(K), _p(V),
                                         _p(chunk_ids_out), _p(out), _p(lse), _p(ws), _nbytes(ws),
                                         _stream(stream)), "lsa_decode_step_lookahead")


def lsa_lookahead_partition(dims, max_ctas: int) -> list:
    """First tile of each CTA of the lookahead attention's split, then the tile count (host only)."""
    n = min(int(max_ctas), 256) + 1 if max_ctas >= 1 else 1
    starts = (ctypes.c_int32 * n)()
    g = ctypes.c_int32(0)
    _check(lib.lsa_lookahead_partition(dims.ptr, int(max_ctas), starts, ctypes.byref(g)), "lsa_lookahead_partition")
    return list(starts[:g.value + 1])


def lsa_indexer_score_fp8(dims, n_layers, n_heads, ensemble, compressed_k, q_fp8, q_scale, head_w, scores, ws,
                          stream=None) -> None:
    _check(lib.lsa_indexer_score_fp8(dims.ptr, int(n_layers), int(n_heads), int(ensemble), _p(compressed_k),
                                     _p(q_fp8), _p(q_scale), _p(head_w), _p(scores), _p(ws), _nbytes(ws),
                                     _stream(stream)), "lsa_indexer_score_fp8")


def lsa_decode_step_fp8(dims, n_layers, n_heads, ensemble, compressed_k, q_fp8, q_scale, head_w, q, K, V,
                        chunk_ids_out, out, lse, ws, stream=None) -> None:
    _check(lib.lsa_decode_step_fp8(dims.ptr, int(n_layers), int(n_heads), int(ensemble), _p(compressed_k),
                                   _p(q_fp8), _p(q_scale), _p(head_w), _p(q), _p(K), _p(V), _p(chunk_ids_out),
                                   _p(out), _p(lse), _p(ws), _nbytes(ws), _stream(stream)), "lsa_decode_step_fp8")


def lsa_threshold_select(dims, scores, tau, k_min, chunk_ids, kept_count, ws, stream=None) -> None:
    _check(lib.lsa_threshold_select(dims.ptr, _p(scores), float(tau), int(k_min), _p(chunk_ids), _p(kept_count),
                                    _p(ws), _nbytes(ws), _stream(stream)), "lsa_threshold_select")


def lsa_decode_step_threshold(dims, q_emb, chunk_emb, q, K, V, tau, k_min, chunk_ids_out, kept_count_out, out,
                              lse, ws, stream=None) -> None:
    _check(lib.lsa_decode_step_threshold(dims.ptr, _p(q_emb), _p(chunk_emb), _p(q), _p(K), _p(V), float(tau),
                                         int(k_min), _p(chunk_ids_out), _p(kept_count_out), _p(out), _p(lse),
                                         _p(ws), _nbytes(ws), _stream(stream)), "lsa_decode_step_threshold")


def _i32(values):
    return (ctypes.c_int32 * len(values))(*map(int, values))


def lsa_sparse_decode_attn_counts(dims, q, K, V, chunk_ids, kept_count, out, lse, ws, stream=None) -> None:
    _check(lib.lsa_sparse_decode_attn_counts(dims.ptr, _p(q), _p(K), _p(V), _p(chunk_ids), _p(kept_count), _p(out),
                                             _p(lse), _p(ws), _nbytes(ws), _stream(stream)),
           "lsa_sparse_decode_attn_counts")


def lsa_shard_candidates(local_dims, scores, local_ids, global_offset, k_pad, cand_scores, cand_ids,
                         stream=None) -> None:
    _check(lib.lsa_shard_candidates(local_dims.ptr, _p(scores), _p(local_ids), _i32(global_offset), int(k_pad),
                                    _p(cand_scores), _p(cand_ids), _stream(stream)), "lsa_shard_candidates")


def lsa_shard_global_select(global_dims, G, global_offset, local_n, all_scores, all_ids, seq_scores, seq_ids,
                            global_ids, local_ids, local_count, ws, stream=None) -> None:
    _check(lib.lsa_shard_global_select(global_dims.ptr, int(G), _i32(global_offset), _i32(local_n), _p(all_scores),
                                       _p(all_ids), _p(seq_scores), _p(seq_ids), _p(global_ids), _p(local_ids),
                                       _p(local_count), _p(ws), _nbytes(ws), _stream(stream)),
           "lsa_shard_global_select")


def lsa_merge_partials(G, B, H, outs, lses, out, lse, stream=None) -> None:
    _check(lib.lsa_merge_partials(int(G), int(B), int(H), _p(outs), _p(lses), _p(out), _p(lse), _stream(stream)),
           "lsa_merge_partials")


def lsa_refresh_resident(dims, q_emb, chunk_emb, K, V, slot_ids, K_res, V_res, moved, ws, stream=None) -> None:
    _check(lib.lsa_refresh_resident(dims.ptr, _p(q_emb), _p(chunk_emb), _p(K), _p(V), _p(slot_ids), _p(K_res),
                                    _p(V_res), _p(moved), _p(ws), _nbytes(ws), _stream(stream)),
           "lsa_refresh_resident")


def lsa_sparse_decode_attn_noalloc(dims, q, K, V, chunk_ids, out, lse, stream=None) -> None:
    """lsa_sparse_decode_attn without a workspace, for callers that cannot allocate device
    memory: the partials live in a fixed scratch array inside the library (see include/lsa.h)."""
    _check(lib.lsa_sparse_decode_attn_noalloc(dims.ptr, _p(q), _p(K), _p(V), _p(chunk_ids), _p(out), _p(lse),
                                              _stream(stream)), "lsa_sparse_decode_attn_noalloc")


def lsa_get_device_status(ws, stream=None) -> int:
    """Synchronise, read and clear the sticky device error word; returns the status code."""
    return lib.lsa_get_device_status(_p(ws), _stream(stream))


def lsa_read_stream(buf, stream=None) -> None:
    """Read every byte of the device tensor ``buf`` and discard it (a read-bandwidth probe)."""
    _check(lib.lsa_read_stream(_p(buf), _nbytes(buf), _stream(stream)), "lsa_read_stream")


def alloc_workspace(dims: Dims, device=None, stream=None):
    """Allocate (with torch) and initialise a workspace for ``dims``."""
    ws = torch.empty(lsa_workspace_size(dims), dtype=torch.uint8, device=device or "cuda")
    lsa_workspace_init(ws, stream)
    return ws

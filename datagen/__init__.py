"""Seeded synthetic inputs for the LSA decode step (host side).

This module only MAKES inputs. It holds none of the arithmetic of the method
(no score, no selection, no attention): both the float64 oracle and the CUDA
path consume what it produces, and nothing else is shared between them.

Generator
---------
Every random value is drawn from a counter-based form of SplitMix64
(Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014; the finaliser constants are Vigna's ``splitmix64.c``):

* ``mix64`` is the SplitMix64 output function;
* the stream for ``(seed, tensor_id)`` starts at state
  ``key = mix64((seed << 32) | tensor_id)``; its n-th output (n >= 1) is
  ``mix64(key + n * GAMMA)`` with ``GAMMA = 0x9E3779B97F4A7C15`` (mod 2**64);
* element ``i`` of a tensor uses outputs ``3i+1, 3i+2, 3i+3``; each 64-bit
  output is split into four 16-bit uniforms, and the Irwin-Hall sum of the
  twelve uniforms, minus its mean ``12 * 65535 / 2 = 393210``, times ``2**-16``
  is ``x_i`` ~ N(0, 1) (variance ``1 - 2**-32``, tails cut at +-6).
  ``x_i`` is an integer times ``2**-16`` with ``|integer| < 2**19``, so it is
  exact in float32 on every machine; bf16 tensors round it to nearest-even.

The same definition is implemented for the GPU in ``datagen/csrc/fill.cu``
(used to fill the multi-GB K/V caches in place); ``tests`` check that both
agree bit for bit.

Workloads
---------
The five decode workloads follow the configurations of the FlashMemory-
DeepSeek-V4 LSA decode step (128K / 500K / 1M-token contexts, plus a tiny fp32
case and a mixed-length serving batch). The pages name LongBench-v2,
LongMemEval, RULER and MRCR contexts of 46K-512K tokens; these seeded
synthetic inputs stand in for them (no item of those suites is used).
"""
from __future__ import annotations

import math
import subprocess
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "GAMMA", "mix64", "stream_key", "normal_f32", "uniform_f64", "bf16_bits",
    "bf16_to_f32", "Workload", "workload", "WORKLOADS", "make_inputs",
    "kv_rows", "TENSOR_IDS", "make_lookahead_queries",
]

_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)
GAMMA = np.uint64(0x9E3779B97F4A7C15)
_C1 = np.uint64(0xBF58476D1CE4E5B9)
_C2 = np.uint64(0x94D049BB133111EB)
_IH_MEAN = 393210  # 12 * 65535 / 2

# Tensor ids of the generator streams (one stream per logical tensor).
TENSOR_IDS = {
    "chunk_emb": 1,   # chunk-side embeddings, N(0,1) noise
    "q_emb": 2,       # query-side embeddings
    "q": 3,           # decode query [B, H, Dh]
    "K": 4,           # key cache [sum L, H, Dh]
    "V": 5,           # value cache [sum L, H, Dh]
    "plant_noise": 6, # noise added to planted chunks
    "plant_pos": 7,   # planted positions (permutation keys)
    "zipf_rank": 8,   # Zipf rank permutation keys
    "lengths": 9,     # mixed-batch sequence lengths
    "plant_query": 10,  # which lookahead query a planted chunk copies
}


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wraps mod 2**64)."""
    z = np.asarray(z, dtype=np.uint64)
    z = (z ^ (z >> np.uint64(30))) * _C1
    z = (z ^ (z >> np.uint64(27))) * _C2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_id: int) -> np.uint64:
    """Initial SplitMix64 state of the stream for ``(seed, tensor_id)``."""
    if not (0 <= seed < 2**32 and 0 <= tensor_id < 2**32):
        raise ValueError("seed and tensor_id must fit in 32 bits")
    return mix64(np.array([(seed << 32) | tensor_id], dtype=np.uint64))[0]


def _words(seed: int, tensor_id: int, n: np.ndarray) -> np.ndarray:
    """Outputs number ``n`` (uint64 array, n >= 1) of the stream."""
    key = np.array([stream_key(seed, tensor_id)], dtype=np.uint64)
    return mix64(key + np.asarray(n, dtype=np.uint64) * GAMMA)


def normal_f32(seed: int, tensor_id: int, idx) -> np.ndarray:
    """x_i ~ N(0,1) for element indices ``idx`` (any int array), float32, exact."""
    idx = np.asarray(idx, dtype=np.uint64)
    acc = np.zeros(idx.shape, dtype=np.int64)
    three = np.uint64(3)
    for j in range(3):
        w = _words(seed, tensor_id, three * idx + np.uint64(j + 1))
        for m in range(4):
            acc += ((w >> np.uint64(16 * m)) & np.uint64(0xFFFF)).astype(np.int64)
    return (acc - _IH_MEAN).astype(np.float32) * np.float32(2.0 ** -16)


def uniform_f64(seed: int, tensor_id: int, idx) -> np.ndarray:
    """u_i ~ U[0,1) from the top 53 bits of output ``idx + 1`` of the stream."""
    idx = np.asarray(idx, dtype=np.uint64)
    w = _words(seed, tensor_id, idx + np.uint64(1))
    return (w >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def _perm(seed: int, tensor_id: int, n: int) -> np.ndarray:
    """A seeded permutation of 0..n-1 (argsort of stream outputs; ties impossible in practice, stable anyway)."""
    w = _words(seed, tensor_id, np.arange(1, n + 1, dtype=np.uint64))
    return np.argsort(w, kind="stable").astype(np.int64)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16, nearest-even; returns the uint16 bit patterns (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return (u >> np.uint64(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 values -> storage array (float32 or bf16 bit patterns)."""
    return x.astype(np.float32) if dtype == "f32" else bf16_bits(x)


def _value(a: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array -> exact float32 values."""
    return a if dtype == "f32" else bf16_to_f32(a)


@dataclass
class Workload:
    """One decode-step workload: shapes, dtypes, seed and planted structure."""
    name: str
    B: int
    N: list            # chunks per sequence (length B)
    E: int             # embedding dim
    Q: int             # query embeddings per sequence (1, or 64 for the lookahead window)
    k: list            # kept chunks per sequence (length B)
    H: int             # attention heads (query heads = KV heads)
    Dh: int = 128      # head dim
    C: int = 64        # tokens per chunk
    emb_dtype: str = "bf16"
    kv_dtype: str = "bf16"
    seed: int = 0
    plant: str = "copy"          # "copy" (q_emb + 0.1 noise), "zipf", "copy_query"
    plant_count: list = field(default_factory=list)  # planted chunks per sequence
    zipf_s: float = 1.0
    zipf_c: float = 4.0
    uniform: bool = True         # all sequences have the same N and k

    @property
    def L(self) -> list:
        return [n * self.C for n in self.N]

    @property
    def chunk_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.N)]).astype(np.int64)

    @property
    def k_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.k)]).astype(np.int64)

    @property
    def total_chunks(self) -> int:
        return int(sum(self.N))

    @property
    def total_kept(self) -> int:
        return int(sum(self.k))

    def esize(self, which: str) -> int:
        return 4 if getattr(self, which) == "f32" else 2

    def kv_elems(self) -> int:
        return int(sum(self.L)) * self.H * self.Dh

    def algorithmic_bytes(self) -> int:
        """Bytes one fused step must touch: every chunk embedding, the query
        embeddings, the decode queries and the kept chunks' K and V (read once),
        plus the outputs (ids and attention output)."""
        e = self.esize("emb_dtype")
        kv = self.esize("kv_dtype")
        emb = self.total_chunks * self.E * e + self.B * self.Q * self.E * e
        q = self.B * self.H * self.Dh * kv
        kept = self.total_kept * self.C * self.H * self.Dh * kv * 2
        out = self.B * self.H * self.Dh * 4 + self.total_kept * 4
        return emb + q + kept + out


def round_half_up(x: float) -> int:
    return int(math.floor(x + 0.5))


def _mixed_lengths(seed: int, B: int) -> list:
    u = uniform_f64(seed, TENSOR_IDS["lengths"], np.arange(B))
    lo, hi = math.log(32768.0), math.log(524288.0)
    L = np.exp(lo + (hi - lo) * u)
    return [int(l) // 64 * 64 for l in L]


def workload(name: str) -> Workload:
    """The decode workloads by name: tiny, 128k, 500k, 1m, mixed (plus 'small-*' test variants)."""
    if name == "tiny":
        return Workload("tiny", 1, [64], 128, 1, [8], 8, emb_dtype="f32", kv_dtype="f32",
                        seed=0, plant="copy", plant_count=[4])
    if name == "128k":
        return Workload("128k", 8, [2048] * 8, 128, 1, [256] * 8, 16, seed=1, plant="copy",
                        plant_count=[32] * 8)
    if name == "128k-b2":  # the 128K shape with batch 2: a profiling case (2.1 GB of K/V, kept set > L2)
        return Workload("128k-b2", 2, [2048] * 2, 128, 1, [256] * 2, 16, seed=1, plant="copy",
                        plant_count=[32] * 2)
    if name == "500k":
        return Workload("500k", 4, [8192] * 4, 256, 1, [819] * 4, 16, seed=2, plant="zipf")
    if name == "1m":
        return Workload("1m", 1, [16384], 256, 64, [2212], 16, seed=3, plant="copy_query",
                        plant_count=[164])
    if name == "1m-h2":  # the 1M lookahead shape with 2 heads: a profiling case (1.1 GB of K/V)
        return Workload("1m-h2", 1, [16384], 256, 64, [2212], 2, seed=3, plant="copy_query",
                        plant_count=[164])
    if name == "mixed":
        L = _mixed_lengths(4, 32)
        N = [l // 64 for l in L]
        k = [max(1, round_half_up(0.135 * n)) for n in N]
        pc = [max(1, n // 100) for n in N]
        return Workload("mixed", 32, N, 128, 1, k, 8, seed=4, plant="copy", plant_count=pc,
                        uniform=False)
    raise KeyError(name)


WORKLOADS = ("tiny", "128k", "500k", "1m", "mixed")


def small_workload(B=2, N=(40, 72), E=64, Q=1, k=(5, 9), H=4, Dh=128, C=64,
                   emb_dtype="f32", kv_dtype="f32", seed=11, plant="copy", plant_count=None,
                   name="small") -> Workload:
    """A small, possibly ragged workload for tests (several tiles and a ragged tail)."""
    N = list(N)
    k = list(k)
    if plant_count is None:
        plant_count = [max(1, n // 16) for n in N]
    return Workload(name, B, N, E, Q, k, H, Dh, C, emb_dtype, kv_dtype, seed, plant,
                    list(plant_count), uniform=(len(set(N)) == 1 and len(set(k)) == 1))


def make_inputs(w: Workload) -> dict:
    """Query embeddings, chunk embeddings and decode queries of a workload.

    Returns storage arrays (float32, or bf16 bit patterns as uint16):
      q_emb [B, Q, E], chunk_emb [sum N, E], q [B, H, Dh].
    The planted structure is built in float32 with separate multiply and add
    (no fused multiply-add), then rounded to the storage type.
    """
    E, Q = w.E, w.Q
    q_emb = normal_f32(w.seed, TENSOR_IDS["q_emb"], np.arange(w.B * Q * E)).reshape(w.B, Q, E)
    q_emb = _value(_store(q_emb, w.emb_dtype), w.emb_dtype)  # planted copies use the stored q_emb
    emb = normal_f32(w.seed, TENSOR_IDS["chunk_emb"],
                     np.arange(w.total_chunks * E)).reshape(w.total_chunks, E)
    off = w.chunk_offsets
    tenth = np.float32(0.1)
    for b in range(w.B):
        n = w.N[b]
        rows = slice(int(off[b]), int(off[b + 1]))
        if w.plant in ("copy", "copy_query"):
            # positions: the first plant_count entries of a seeded permutation of this sequence
            perm = _perm(w.seed, TENSOR_IDS["plant_pos"] + (b << 8), n)
            pos = np.sort(perm[: w.plant_count[b]])
            noise = normal_f32(w.seed, TENSOR_IDS["plant_noise"],
                               (off[b] + pos)[:, None] * E + np.arange(E)[None, :])
            if w.plant == "copy":
                src = np.broadcast_to(q_emb[b, 0], (len(pos), E))
            else:
                j = (uniform_f64(w.seed, TENSOR_IDS["plant_query"], off[b] + pos) * Q).astype(np.int64)
                src = q_emb[b, j]
            seg = emb[rows]
            seg[pos] = src.astype(np.float32) + (tenth * noise).astype(np.float32)
            emb[rows] = seg
        elif w.plant == "zipf":
            rank = _perm(w.seed, TENSOR_IDS["zipf_rank"] + (b << 8), n) + 1  # rank_i in 1..n
            wgt = (w.zipf_c / np.power(rank.astype(np.float64), w.zipf_s)).astype(np.float32)
            seg = emb[rows]
            seg = seg + (wgt[:, None] * q_emb[b, 0][None, :]).astype(np.float32)
            emb[rows] = seg.astype(np.float32)
        else:
            raise ValueError(w.plant)
    q = normal_f32(w.seed, TENSOR_IDS["q"], np.arange(w.B * w.H * w.Dh)).reshape(w.B, w.H, w.Dh)
    return {
        "q_emb": _store(q_emb, w.emb_dtype),
        "chunk_emb": _store(emb, w.emb_dtype),
        "q": _store(q, w.kv_dtype),
    }


def planted_positions(w: Workload, b: int) -> np.ndarray:
    """Chunk indices (within sequence b) that carry planted relevance ('copy' plants)."""
    perm = _perm(w.seed, TENSOR_IDS["plant_pos"] + (b << 8), w.N[b])
    return np.sort(perm[: w.plant_count[b]])


_NATIVE_MIN = 1 << 16  # elements from which kv_rows uses the C generator
_host = None


def _host_lib():
    """The C side of the generator (datagen/csrc/normal_host.c), built on first use; None
    when it cannot be built (kv_rows then stays in numpy)."""
    global _host
    if _host is None:
        import ctypes
        try:
            from . import build as _build
            lib = ctypes.CDLL(_build.build_host())
        except (OSError, subprocess.CalledProcessError):
            _host = False
            return None
        i64, u32, vp = ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p
        lib.dg_cache_rows.argtypes = [u32, u32, i64, i64, vp, i64, vp, i64, ctypes.c_int, vp]
        lib.dg_cache_rows.restype = None
        lib.dg_normal_f32.argtypes = [u32, u32, vp, i64, vp]
        lib.dg_normal_f32.restype = None
        _host = lib
    return _host or None


def kv_rows(w: Workload, which: str, tokens, heads=None) -> np.ndarray:
    """Exact float32 values of K or V at global token indices ``tokens`` (and heads).

    The cache layout is [sum L, H, Dh] row-major; element (t, h, d) is element
    ``(t * H + h) * Dh + d`` of the stream. Returns [len(tokens), len(heads), Dh].
    """
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    heads = np.ascontiguousarray(np.arange(w.H) if heads is None else heads, dtype=np.int64)
    if tokens.size * heads.size * w.Dh >= _NATIVE_MIN:
        lib = _host_lib()
        if lib is not None:  # the same definition in C (bit-identical, tested), for large slices
            out = np.empty((tokens.size, heads.size, w.Dh), dtype=np.float32)
            lib.dg_cache_rows(w.seed, TENSOR_IDS[which], w.H, w.Dh, tokens.ctypes.data, tokens.size,
                              heads.ctypes.data, heads.size, 1 if w.kv_dtype == "bf16" else 0, out.ctypes.data)
            return out
    idx = ((tokens[:, None, None] * w.H + heads[None, :, None]) * w.Dh
           + np.arange(w.Dh)[None, None, :])
    x = normal_f32(w.seed, TENSOR_IDS[which], idx.reshape(-1)).reshape(idx.shape)
    return _value(_store(x, w.kv_dtype), w.kv_dtype)


def as_f32(a: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array -> exact float32 values (public helper)."""
    return _value(a, dtype)


def make_query_variant(w: Workload, r: int) -> dict:
    """Query embeddings and decode queries of rotation r (r = 0 is make_inputs' own).

    Variant r > 0 draws q_emb and q from seed ``w.seed + 1000 * r``; the chunk
    embeddings and caches stay those of the workload, so each variant keeps a
    different set of chunks with the same byte count."""
    if r == 0:
        x = make_inputs(w)
        return {"q_emb": x["q_emb"], "q": x["q"]}
    seed = w.seed + 1000 * r
    q_emb = normal_f32(seed, TENSOR_IDS["q_emb"], np.arange(w.B * w.Q * w.E)).reshape(w.B, w.Q, w.E)
    q = normal_f32(seed, TENSOR_IDS["q"], np.arange(w.B * w.H * w.Dh)).reshape(w.B, w.H, w.Dh)
    return {"q_emb": _store(q_emb, w.emb_dtype), "q": _store(q, w.kv_dtype)}


TENSOR_IDS["q_la"] = 17  # attention queries of the lookahead window [B, Q, H, Dh]


def make_lookahead_queries(w: Workload, seed: int | None = None) -> np.ndarray:
    """Attention queries of the Q-token lookahead window, [B, Q, H, Dh], in the K/V storage
    type: element (b, j, h, d) is element ((b*Q + j)*H + h)*Dh + d of stream 'q_la'."""
    s = w.seed if seed is None else seed
    q = normal_f32(s, TENSOR_IDS["q_la"], np.arange(w.B * w.Q * w.H * w.Dh)).reshape(w.B, w.Q, w.H, w.Dh)
    return _store(q, w.kv_dtype)


TENSOR_IDS.update({"idx_q": 11, "idx_k": 12, "idx_qs": 13, "idx_ks": 14, "idx_w": 15, "idx_plant": 16})


def e4m3_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> float8_e4m3 bit patterns (round to nearest even, saturated to +-448)."""
    import torch
    t = torch.from_numpy(np.clip(np.asarray(x, dtype=np.float32), -448.0, 448.0))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()


def make_indexer_inputs(w: Workload, layers: int = 3, heads: int = 128, dim: int = 128) -> dict:
    """Inputs of the FP8 compressed-K indexer score for a workload.

    compressed_k [layers][sum N][132] uint8 (128 e4m3 key values + float32 scale), q_fp8
    [B][layers][heads][dim] e4m3, q_scale [B][layers][heads] and head_w [layers][heads]
    float32. Keys and queries are N(0, 8^2) before quantisation, both dequant scales are
    about 1/27 (so a dequantised head logit is about N(0, 1)) and the head weights are
    N(0, 1) / (4 sqrt(heads)). In every layer, the chunks of `planted_positions` copy (plus
    0.5 noise) the query of that layer's head with the largest weight, so they score high."""
    n = w.total_chunks
    q = normal_f32(w.seed, TENSOR_IDS["idx_q"], np.arange(w.B * layers * heads * dim))
    q = (q * np.float32(8.0)).reshape(w.B, layers, heads, dim)
    q8 = e4m3_bits(q)
    qv = e4m3_bits_to_f32(q8)
    k = normal_f32(w.seed, TENSOR_IDS["idx_k"], np.arange(layers * n * dim))
    k = (k * np.float32(8.0)).reshape(layers, n, dim)
    hw = (normal_f32(w.seed, TENSOR_IDS["idx_w"], np.arange(layers * heads)).reshape(layers, heads)
          / np.float32(4.0 * math.sqrt(heads))).astype(np.float32)
    off = w.chunk_offsets
    for b in range(w.B):
        pos = planted_positions(w, b) if w.plant_count else np.zeros(0, np.int64)
        for l in range(layers):
            hstar = int(np.argmax(hw[l]))
            noise = normal_f32(w.seed, TENSOR_IDS["idx_plant"] + (l << 8),
                               (off[b] + pos)[:, None] * dim + np.arange(dim)[None, :])
            k[l, off[b] + pos] = qv[b, l, hstar][None, :] + np.float32(0.5) * noise
    k8 = e4m3_bits(k)
    base = np.float32(1.0 / 27.0)
    ks = base * (np.float32(1.0) + np.float32(0.1) * uniform_f64(w.seed, TENSOR_IDS["idx_ks"],
                                                                  np.arange(layers * n)).astype(np.float32))
    qs = base * (np.float32(1.0) + np.float32(0.1) * uniform_f64(w.seed, TENSOR_IDS["idx_qs"],
                                                                  np.arange(w.B * layers * heads)).astype(np.float32))
    ck = np.empty((layers, n, dim + 4), dtype=np.uint8)
    ck[..., :dim] = k8
    ck[..., dim:] = ks.astype("<f4").reshape(layers, n, 1).view(np.uint8).reshape(layers, n, 4)
    return {"compressed_k": ck, "q_fp8": q8, "q_scale": qs.reshape(w.B, layers, heads).astype(np.float32),
            "head_w": hw, "layers": layers, "heads": heads}


def e4m3_bits_to_f32(codes: np.ndarray) -> np.ndarray:
    """float8_e4m3 bit patterns -> float32 (input construction only)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).float().numpy()

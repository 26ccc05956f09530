"""lsa_sparse_decode_attn_noalloc: the attention call for callers that cannot allocate.

Some callers cannot call cudaMalloc (an engine that has reserved nearly all device
memory for its own pool, a plugin that must not allocate behind its host framework's
allocator, a latency-critical path that cannot afford cudaMalloc's implicit device
synchronisation). This entry point keeps its scratch in a fixed array inside the
library. These tests call it through the C ABI and check it against the workspace
entry point, lsa_sparse_decode_attn, and against the float64 oracle, on two calls
in a row (the second call must not be fooled by what the first left in the shared
array). The file is named so that pytest collects it last.
"""
import math

import numpy as np
import pytest
import torch

import datagen
import oracle
from tests import _gpu as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lsa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from learned_sparse_kv_decode_b200 import build
    build.build()
    import learned_sparse_kv_decode_b200 as m
    return m


def _ids(w, seed):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(np.concatenate(
        [np.sort(rng.permutation(n)[:k]) for n, k in zip(w.N, w.k)]).astype(np.int32)).cuda()


@pytest.mark.parametrize("kv_dtype,H", [("bf16", 16), ("f32", 8)])
def test_noalloc_matches_workspace_entry_point_twice(lsa, kv_dtype, H):
    w = datagen.small_workload(B=3, N=(40, 9, 70), k=(11, 9, 25), E=64, H=H, kv_dtype=kv_dtype, seed=71)
    dw = G.DeviceWorkload(w, lsa)
    for call, seed in enumerate((1, 2)):  # two calls in a row, different kept sets and queries
        ids = _ids(w, seed)
        q = dw.q if call == 0 else (dw.q * -0.5).contiguous()
        ref_out = torch.empty_like(dw.out)
        ref_lse = torch.empty_like(dw.lse)
        lsa.lsa_sparse_decode_attn(dw.dims, q, dw.K, dw.V, ids, ref_out, ref_lse, dw.ws)
        # the workspace call's own error word (the no-alloc call's is internal to the library)
        assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
        out = torch.full_like(dw.out, float("nan"))
        lse = torch.full_like(dw.lse, float("nan"))
        lsa.lsa_sparse_decode_attn_noalloc(dw.dims, q, dw.K, dw.V, ids, out, lse)
        torch.cuda.synchronize()
        got_o, got_l = out.cpu().numpy(), lse.cpu().numpy()
        np.testing.assert_allclose(got_o, ref_out.cpu().numpy(), rtol=0, atol=1e-4)
        np.testing.assert_allclose(got_l, ref_lse.cpu().numpy(), rtol=0, atol=1e-4)
        # and against the float64 oracle directly, at the problem statement's tolerance for
        # the K/V dtype and at 1e-4 (fp32 arithmetic on exact inputs)
        ids_h = ids.cpu().numpy()
        qf = datagen.as_f32(dw.host["q"], kv_dtype) * (1.0 if call == 0 else -0.5)
        for b in range(w.B):
            tok = oracle.kept_tokens(ids_h[w.k_offsets[b]:w.k_offsets[b + 1]], w.C)
            ref_o, ref_l = oracle.attention(qf[b], dw.kv_f("K", b, tok), dw.kv_f("V", b, tok),
                                            1.0 / math.sqrt(w.Dh))
            np.testing.assert_allclose(got_o[b], ref_o, rtol=0, atol=G.ATTN_ATOL[kv_dtype])
            np.testing.assert_allclose(got_o[b], ref_o, rtol=0, atol=1e-4)
            np.testing.assert_allclose(got_l[b], ref_l, rtol=0, atol=1e-4)


def test_noalloc_resident_buffer_mode(lsa):
    w = datagen.small_workload(B=2, N=(20, 33), k=(7, 12), E=64, H=16, kv_dtype="bf16", seed=72)
    dw = G.DeviceWorkload(w, lsa)
    ids = _ids(w, 3)
    Kr = torch.empty((w.total_kept * w.C, w.H, w.Dh), dtype=torch.bfloat16, device="cuda")
    Vr = torch.empty_like(Kr)
    lsa.lsa_gather_kv(dw.dims, dw.K, dw.V, ids, Kr, Vr, dw.ws)
    ref = torch.empty_like(dw.out)
    lsa.lsa_sparse_decode_attn(dw.dims, dw.q, Kr, Vr, None, ref, None, dw.ws)
    for _ in range(2):
        out = torch.full_like(dw.out, float("nan"))
        lsa.lsa_sparse_decode_attn_noalloc(dw.dims, dw.q, Kr, Vr, None, out, None)
        np.testing.assert_allclose(out.cpu().numpy(), ref.cpu().numpy(), rtol=0, atol=1e-4)


def test_noalloc_rejects_shapes_beyond_its_scratch(lsa):
    # 256 sequences x 128 heads need far more than the fixed 4 MiB of partials
    dims = lsa.Dims(256, 1, 64, 128, 64, N=4, k=2, emb_dtype="bf16", kv_dtype="bf16")
    t = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(16, dtype=torch.int32, device="cuda")
    out = torch.empty(16, dtype=torch.float32, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_sparse_decode_attn_noalloc(dims, t, t, t, ids, out, None)
    assert e.value.status == lsa.LSA_ERR_WORKSPACE

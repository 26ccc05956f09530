"""CPU checks of the C ABI: the library builds for sm_100a, loads, exports every
entry point of include/lsa.h, and rejects bad arguments on the host before any
CUDA call (so these run without a GPU)."""
import ctypes

import pytest

from learned_sparse_kv_decode_b200 import build as lsa_build

lsa_build.build()
import learned_sparse_kv_decode_b200 as lsa  # noqa: E402
from learned_sparse_kv_decode_b200 import abi  # noqa: E402


def test_exports_every_header_symbol():
    names = lsa.header_symbols()
    assert len(names) == 24
    for n in names:
        assert hasattr(abi.lib, n), n


def test_version_and_status_strings():
    assert lsa.lsa_abi_version() == 1
    for s in range(8):
        assert lsa.string(s).startswith("LSA_")
    assert "unknown" in lsa.string(99)


def _ws_size_status(**kw):
    base = dict(B=2, Q=1, E=128, H=16, chunk_len=64, N=100, k=10)
    base.update(kw)
    d = lsa.Dims(**base)
    n = ctypes.c_size_t(0)
    return abi.lib.lsa_workspace_size(d.ptr, ctypes.byref(n))


@pytest.mark.parametrize("kw,expect", [
    (dict(B=0), lsa.LSA_ERR_INVALID_ARG),
    (dict(B=257), lsa.LSA_ERR_INVALID_ARG),
    (dict(Q=0), lsa.LSA_ERR_INVALID_ARG),
    (dict(Q=257), lsa.LSA_ERR_INVALID_ARG),
    (dict(k=0), lsa.LSA_ERR_INVALID_ARG),
    (dict(k=101), lsa.LSA_ERR_INVALID_ARG),
    (dict(N=0), lsa.LSA_ERR_INVALID_ARG),
    (dict(Dh=64), lsa.LSA_ERR_UNSUPPORTED),
    (dict(H=12), lsa.LSA_ERR_UNSUPPORTED),
    (dict(H=256), lsa.LSA_ERR_UNSUPPORTED),
    (dict(chunk_len=48), lsa.LSA_ERR_UNSUPPORTED),
    (dict(chunk_len=4), lsa.LSA_ERR_UNSUPPORTED),
    (dict(E=100), lsa.LSA_ERR_UNSUPPORTED),       # 200 bytes: not a multiple of 16
    (dict(E=96), lsa.LSA_ERR_UNSUPPORTED),        # 12 pieces of 16 bytes
    (dict(chunk_offsets=[1, 5, 9], N=None), lsa.LSA_ERR_INVALID_ARG),     # must start at 0
    (dict(chunk_offsets=[0, 5, 5], N=None), lsa.LSA_ERR_INVALID_ARG),     # empty sequence
    (dict(chunk_offsets=[0, 5, 9], N=None, k_per_seq=[5, 5], k=None), lsa.LSA_ERR_INVALID_ARG),  # k_1 > N_1
])
def test_host_validation_rejects(kw, expect):
    assert _ws_size_status(**kw) == expect


@pytest.mark.parametrize("ptr,nbytes", [(None, 16), (16, 0), (0x1008, 16), (0x1000, 24)])
def test_read_stream_rejects_bad_buffers(ptr, nbytes):
    # null, empty, not 16-byte aligned, not a multiple of 16 bytes: rejected before any CUDA call
    assert abi.lib.lsa_read_stream(ptr, nbytes, None) == lsa.LSA_ERR_INVALID_ARG


def test_null_arguments_rejected():
    d = lsa.Dims(B=1, Q=1, E=128, H=8, chunk_len=64, N=4, k=2)
    assert abi.lib.lsa_workspace_size(None, None) == lsa.LSA_ERR_INVALID_ARG
    assert abi.lib.lsa_workspace_size(d.ptr, None) == lsa.LSA_ERR_INVALID_ARG
    assert abi.lib.lsa_workspace_init(None, 4096, None) == lsa.LSA_ERR_INVALID_ARG
    assert abi.lib.lsa_workspace_init(ctypes.c_void_p(0x1001), 4096, None) == lsa.LSA_ERR_INVALID_ARG
    assert abi.lib.lsa_decode_step(None, *([None] * 9), 0, None) == lsa.LSA_ERR_INVALID_ARG
    assert abi.lib.lsa_get_device_status(None, None) == lsa.LSA_ERR_INVALID_ARG


def test_valid_dims_need_a_device_here():
    # valid shapes pass host validation and then need the CUDA runtime: with no GPU
    # in this container the call reports a CUDA error instead of guessing
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _ws_size_status() == lsa.LSA_ERR_CUDA


def test_missing_library_fails_loudly(tmp_path):
    # no fallback: without the CUDA library the binding refuses to load
    old = abi.LIB_PATH
    abi.LIB_PATH = str(tmp_path / "liblsa_b200.so")
    try:
        with pytest.raises(ImportError):
            abi._load()
    finally:
        abi.LIB_PATH = old

"""A bounded device wait that runs out: the kernel records LSA_ERR_TIMEOUT in the workspace's
sticky error word and returns, and the CUDA context stays usable for the next call.

The wait is the library's own helper (mbar_wait in csrc/lsa_device.cuh), compiled into a
test-only kernel that waits on an mbarrier nothing arrives on. No fault, trap or hang."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import datagen
from tests import _gpu as G

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def waitlib(tmp_path_factory):
    out = tmp_path_factory.mktemp("wt") / "libwait_timeout.so"
    subprocess.check_call([os.environ.get("NVCC", "nvcc"), "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-O2", "-std=c++17", "-Xcompiler", "-fPIC", "-I", os.path.join(os.path.dirname(HERE), "include"),
                           os.path.join(HERE, "csrc", "wait_timeout.cu"), "-o", str(out)])
    lib = ctypes.CDLL(str(out))
    lib.wt_run.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.wt_run.restype = ctypes.c_int
    return lib


def test_bounded_wait_times_out_and_context_survives(waitlib):
    assert torch.cuda.is_available()
    import learned_sparse_kv_decode_b200 as lsa
    w = datagen.small_workload(B=2, N=(40, 72), k=(5, 9), E=64, H=4)
    dw = G.DeviceWorkload(w, lsa)
    elapsed = torch.zeros(2, dtype=torch.int64, device="cuda")
    rc = waitlib.wt_run(ctypes.c_void_p(dw.ws.data_ptr()), ctypes.c_void_p(elapsed.data_ptr()))
    assert rc == 0, f"CUDA error {rc}"
    ns, ok = elapsed.cpu().numpy().tolist()
    assert ok == 0 and 1.0e9 < ns < 30e9, (ok, ns)  # gave up after its ~2 s limit
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_ERR_TIMEOUT
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK  # read-and-clear
    # the context is intact: a full decode step still runs and matches its own rerun
    lsa.lsa_decode_step(dw.dims, dw.q_emb, dw.chunk_emb, dw.q, dw.K, dw.V, dw.ids, dw.out, dw.lse, dw.ws)
    assert lsa.lsa_get_device_status(dw.ws) == lsa.LSA_OK
    first = dw.out.clone()
    lsa.lsa_decode_step(dw.dims, dw.q_emb, dw.chunk_emb, dw.q, dw.K, dw.V, dw.ids, dw.out, dw.lse, dw.ws)
    assert torch.equal(first, dw.out) and np.isfinite(first.cpu().numpy()).all()

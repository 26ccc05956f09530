"""Host-side checks of the seeded input generator (datagen)."""
import numpy as np
import torch

import datagen


def test_splitmix64_known_answers():
    # SplitMix64 seeded with 0: the first three outputs of the published generator
    key = np.array([0], dtype=np.uint64)
    n = np.arange(1, 4, dtype=np.uint64)
    got = datagen.mix64(key + n * datagen.GAMMA)
    assert [int(v) for v in got] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_normal_statistics_and_exactness():
    x = datagen.normal_f32(123, 4, np.arange(400_000))
    assert abs(float(x.mean())) < 0.01
    assert abs(float(x.var()) - 1.0) < 0.01
    assert float(np.abs(x).max()) < 6.0
    # every value is an integer multiple of 2**-16 (exact in float32)
    r = x.astype(np.float64) * 65536.0
    np.testing.assert_array_equal(r, np.round(r))


def test_normal_is_counter_based():
    a = datagen.normal_f32(5, 4, np.arange(1000))
    b = datagen.normal_f32(5, 4, np.arange(500, 1000))
    np.testing.assert_array_equal(a[500:], b)
    c = datagen.normal_f32(6, 4, np.arange(1000))
    assert not np.array_equal(a, c)


def test_bf16_rounding_matches_torch():
    x = np.concatenate([datagen.normal_f32(1, 1, np.arange(100_000)) * np.float32(37.0),
                        np.array([1.00390625, 1.01171875, -1.00390625, 0.0, -0.0], np.float32)])
    ours = datagen.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    np.testing.assert_array_equal(datagen.bf16_to_f32(ours),
                                  torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_workload_shapes():
    for name in datagen.WORKLOADS:
        w = datagen.workload(name)
        assert len(w.N) == w.B and len(w.k) == w.B
        assert all(1 <= k <= n for k, n in zip(w.k, w.N))
    w = datagen.workload("mixed")
    assert w.B == 32 and not w.uniform
    assert all(32768 <= l <= 524288 and l % 64 == 0 for l in w.L)
    assert all(k == int(np.floor(0.135 * n + 0.5)) for k, n in zip(w.k, w.N))
    assert datagen.workload("500k").k[0] == 819 and datagen.workload("1m").k[0] == 2212


def test_kv_rows_layout():
    w = datagen.small_workload()
    r = datagen.kv_rows(w, "K", [3, 0], [1])
    idx = (np.array([3, 0])[:, None] * w.H + 1) * w.Dh + np.arange(w.Dh)[None, :]
    np.testing.assert_array_equal(r[:, 0, :], datagen.normal_f32(w.seed, 4, idx))


def test_make_inputs_tiny_planting():
    w = datagen.workload("tiny")
    x = datagen.make_inputs(w)
    assert x["q_emb"].shape == (1, 1, 128) and x["chunk_emb"].shape == (64, 128)
    pos = datagen.planted_positions(w, 0)
    d = x["chunk_emb"][pos] - x["q_emb"][0, 0][None, :]
    assert float(np.abs(d).max()) < 0.1 * 6.0 + 1e-6


def test_lookahead_queries_layout_and_storage():
    w = datagen.small_workload(Q=5, H=3, kv_dtype="bf16")
    x = datagen.make_lookahead_queries(w)
    assert x.shape == (w.B, 5, 3, w.Dh) and x.dtype == np.uint16
    b, j, h, d = 1, 4, 2, 77
    idx = ((b * w.Q + j) * w.H + h) * w.Dh + d
    v = datagen.normal_f32(w.seed, datagen.TENSOR_IDS["q_la"], np.array([idx]))[0]
    assert x[b, j, h, d] == datagen.bf16_bits(np.array([v], np.float32))[0]
    assert datagen.TENSOR_IDS["q_la"] not in [t for k, t in datagen.TENSOR_IDS.items() if k != "q_la"]


def test_kv_rows_native_matches_numpy_definition():
    # the C regenerator of large cache slices against the numpy definition, bit for bit,
    # for both storage types, unordered tokens and a head subset
    lib = datagen._host_lib()
    assert lib is not None, "the host generator must build (gcc)"
    for kv in ("f32", "bf16"):
        w = datagen.small_workload(H=16, kv_dtype=kv, seed=9)
        tokens = np.array([4095, 0, 17, 3000, 63, 64, 2047, 5], dtype=np.int64)
        heads = np.array([15, 0, 7], dtype=np.int64)
        saved = datagen._NATIVE_MIN
        try:
            datagen._NATIVE_MIN = 0
            native = datagen.kv_rows(w, "V", tokens, heads)
            datagen._NATIVE_MIN = 1 << 62
            ref = datagen.kv_rows(w, "V", tokens, heads)
        finally:
            datagen._NATIVE_MIN = saved
        np.testing.assert_array_equal(native.view(np.uint32), ref.view(np.uint32))
    idx = np.array([0, 1, 2**40 + 3, 123456789], dtype=np.uint64)
    out = np.empty(idx.size, dtype=np.float32)
    lib.dg_normal_f32(3, 4, idx.ctypes.data, idx.size, out.ctypes.data)
    np.testing.assert_array_equal(out, datagen.normal_f32(3, 4, idx))

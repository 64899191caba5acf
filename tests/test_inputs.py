"""The seeded input generator: shapes, determinism, distinct top-k, hot expert."""
import numpy as np

from moe_expert_load_ue_b200 import inputs


def test_shapes_distinct_and_deterministic():
    w = inputs.CLASS_671B.with_(tokens_per_rank=64)
    a = inputs.topk_ids(w, 2)
    b = inputs.topk_ids(w, 2)
    assert a.shape == (w.T, w.K) and a.dtype == np.int32
    assert np.array_equal(a, b)
    assert not np.array_equal(a, inputs.topk_ids(w, 3))
    srt = np.sort(a, axis=1)
    assert (np.diff(srt, axis=1) > 0).all()            # K distinct experts per token
    assert a.min() >= 0 and a.max() < w.E


def test_zipf_skew_orders_popularity():
    w = inputs.CLASS_106B.with_(tokens_per_rank=256)
    ids = inputs.topk_ids(w, 0)
    cnt = np.bincount(ids.ravel(), minlength=w.E)
    p = inputs.popularity(w, 0)
    # the most popular expert by construction is among the most frequent
    assert cnt[np.argmax(p)] >= np.sort(cnt)[-3]


def test_nonstationary_permutation():
    w = inputs.CLASS_671B.with_(tokens_per_rank=64)
    c0 = np.bincount(inputs.topk_ids(w, 0).ravel(), minlength=w.E)
    c1 = np.bincount(inputs.topk_ids(w, 1).ravel(), minlength=w.E)
    assert np.argmax(c0) != np.argmax(c1) or not np.array_equal(c0, c1)


def test_extreme_hot_expert_exact_count():
    w = inputs.EXTREME.with_(tokens_per_rank=128)
    ids = inputs.topk_ids(w, 0)
    hot = inputs.hot_expert(w, 0)
    n_hot = int(np.floor(w.hot_fraction * w.T))
    assert np.count_nonzero(ids == hot) == n_hot
    assert np.count_nonzero(ids[:, 0] == hot) == n_hot
    assert (np.diff(np.sort(ids, axis=1), axis=1) > 0).all()


def test_full_size_extreme_hot_count():
    w = inputs.EXTREME
    assert int(np.floor(0.3 * w.T)) == 78643
    assert w.T == 262144 and w.L // w.N == 8192


def test_gates_are_softmax():
    w = inputs.TINY
    ids = inputs.topk_ids(w, 0)
    g = inputs.gates(ids, w, 0)
    assert g.shape == ids.shape and g.dtype == np.float32
    assert np.allclose(g.sum(1), 1.0, atol=1e-6)
    assert (np.diff(g, axis=1) <= 0).all()


def test_bf16_bits_round_to_nearest():
    x = inputs.random_bf16_bits((1000,), 0.02, 3)
    f = (x.astype(np.uint32) << 16).view(np.float32)
    assert abs(float(f.std()) - 0.02) < 0.003


def test_device_generator_shapes_and_distinct():
    w = inputs.CLASS_671B.with_(tokens_per_rank=64)
    a = inputs.topk_ids_device(w, 1, "cpu").numpy()
    assert a.shape == (w.T, w.K) and a.dtype == np.int32
    assert (np.diff(np.sort(a, axis=1), axis=1) > 0).all()
    assert a.min() >= 0 and a.max() < w.E
    b = inputs.topk_ids_device(w, 1, "cpu").numpy()
    assert np.array_equal(a, b)

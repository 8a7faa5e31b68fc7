"""The seeded input generators (workloads/) follow their stated recipe.

Both the oracle and the CUDA path draw their inputs here, so the recipe is
checked on its own:
  * bf16 rounding is round-to-nearest-even (against torch's conversion and
    hand-picked ties);
  * generation is deterministic and per head (a head subset, or another
    thread count, gives the same bits);
  * clusters are 64 tokens laid out per segment, each segment's last one
    possibly short;
  * clustered heads: X = c_g + sigma_g * eps per 64-token cluster, sigma_g in
    [0.05, 1] shared by Q, K and V, context centroids at half scale, Q
    multiplied by one temperature tau in [0.5, 2] per head;
  * the iid kind is standard normal.
"""
import numpy as np
import torch

from workloads import (CLUSTER, CTX_CENTROID_SCALE, Workload, _cluster_ids, bf16_to_f32, f32_to_bf16_bits,
                       generate_bits, generate_dout_bits, head_f32)


def torch_bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_bf16_rounding_is_nearest_even():
    ties = np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, -2.5, 0.0, -0.0], np.float32)
    assert f32_to_bf16_bits(ties).tolist() == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xC020, 0x0000, 0x8000]
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 10.0
    assert np.array_equal(f32_to_bf16_bits(x), torch_bf16_bits(x))
    b = f32_to_bf16_bits(x)
    assert np.array_equal(f32_to_bf16_bits(bf16_to_f32(b)), b)      # bf16 values are fixed points


def test_generation_is_deterministic_and_per_head():
    w = Workload("det", 2, 3, 64, 150, 90, seed=42)
    full = generate_bits(w)
    again = generate_bits(w, threads=1)
    for a, b in zip(full, again):
        assert np.array_equal(a, b)
    sub = generate_bits(w, heads=[4, 1])
    for a, s in zip(full, sub):
        flat = a.reshape(w.BH, w.L, w.D)
        assert np.array_equal(s[0], flat[4]) and np.array_equal(s[1], flat[1])
    assert not np.array_equal(full[0], generate_bits(w.replace(seed=43))[0])
    d = generate_dout_bits(w)
    assert np.array_equal(d, generate_dout_bits(w, threads=1))
    assert np.array_equal(generate_dout_bits(w, heads=[5])[0], d.reshape(w.BH, w.L, w.D)[5])


def test_clusters_are_laid_out_per_segment():
    cid, is_ctx, n = _cluster_ids(100, 70)
    assert CLUSTER == 64 and n == 4
    assert cid.tolist() == [0] * 64 + [1] * 36 + [2] * 64 + [3] * 6
    assert is_ctx.tolist() == [False] * 100 + [True] * 70


def cluster_stats(x: np.ndarray, cid: np.ndarray, n: int):
    means = np.stack([x[cid == g].mean(axis=0) for g in range(n)])
    spread = np.array([(x[cid == g] - means[g]).std() for g in range(n)])
    return means, spread


def test_clustered_recipe():
    w = Workload("recipe", 1, 1, 128, 32 * CLUSTER, 32 * CLUSTER, seed=7)
    q, k, v = (x.astype(np.float64) for x in head_f32(w, 0))
    cid, is_ctx, n = _cluster_ids(w.L_src, w.L_ctx)
    mq, sq = cluster_stats(q, cid, n)
    mk, sk = cluster_stats(k, cid, n)
    mv, sv = cluster_stats(v, cid, n)
    # sigma_g in [0.05, 1] (64 x 128 samples per cluster: ~1 % estimates)
    assert sk.min() > 0.05 * 0.95 and sk.max() < 1.0 * 1.05
    assert sk.max() / sk.min() > 3.0                       # sigma varies over clusters
    # one sigma_g per cluster for all three tensors; Q carries one tau per head
    assert np.all(np.abs(sv / sk - 1.0) < 0.05)
    tau = sq / sk
    assert 0.5 * 0.95 < tau.mean() < 2.0 * 1.05 and tau.std() / tau.mean() < 0.05
    # context centroids at CTX_CENTROID_SCALE of the source ones (squared norms
    # of the cluster means: D * scale^2 plus the small sigma^2 D / 64 term)
    src = (mk[:32] ** 2).sum(axis=1) - sk[:32] ** 2 * w.D / CLUSTER
    ctx = (mk[32:] ** 2).sum(axis=1) - sk[32:] ** 2 * w.D / CLUSTER
    ratio = ctx.mean() / src.mean()
    assert abs(ratio - CTX_CENTROID_SCALE ** 2) < 0.08, ratio
    # the three tensors have their own centroids
    assert abs(np.corrcoef(mk.ravel(), mv.ravel())[0, 1]) < 0.1


def test_iid_kind_is_standard_normal():
    w = Workload("iid", 1, 1, 64, 2048, 2048, kind="iid", seed=3)
    for x in head_f32(w, 0):
        assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01

"""The synthetic input recipe (prototype-Voronoi tokens), host and device
generators.  No GPU: the device generator runs on the CPU here."""
import numpy as np
import torch

from block_sparse_attention_20_b200 import synth


def _voronoi_labels(w, grid_seeds):
    return synth.nearest_seed(synth.token_coords(w.grid, w.N), grid_seeds)


def test_host_generator_follows_the_recipe():
    # regenerate head 0 by hand from the same draw order and compare
    w = synth.TINY
    Q, K, V = synth.generate(w, heads=1)
    rng = np.random.Generator(np.random.PCG64(w.seed))
    seeds = rng.random((w.prototypes, 3))
    proto = rng.standard_normal((w.prototypes, w.d)).astype(np.float32)
    lab = _voronoi_labels(w, seeds)
    q = proto[lab] + np.float32(w.noise) * rng.standard_normal((w.N, w.d), dtype=np.float32)
    assert np.array_equal(Q[0, 0].float().numpy(), torch.from_numpy(q).to(torch.bfloat16).float().numpy())
    # every token's query sits within the noise of its prototype
    resid = Q[0, 0].float().numpy() - proto[lab]
    assert abs(resid.std() - w.noise) < 0.01


def test_device_generator_is_seeded_and_has_the_recipes_spread():
    w = synth.sweep(8192, 10, 16).with_(H=2)
    a = synth.generate_on_device(w, torch.device("cpu"))
    b = synth.generate_on_device(w, torch.device("cpu"))
    c = synth.generate_on_device(w.with_(seed=1), torch.device("cpu"))
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert not torch.equal(a[0], c[0])
    Q, K, V = (x.float() for x in a)
    assert Q.shape == (1, 2, 8192, 128)
    # q = proto + 0.5 n: variance 1 + 0.25; v ~ N(0, 1)
    assert abs(Q.std().item() - np.sqrt(1.25)) < 0.03
    assert abs(V.std().item() - 1.0) < 0.01
    # tokens of one Voronoi cell share a prototype: their keys agree far more
    # than keys of random token pairs
    k0 = K[0, 0]
    near = torch.nn.functional.cosine_similarity(k0[:-1], k0[1:]).mean().item()
    perm = torch.randperm(8192, generator=torch.Generator().manual_seed(0))
    rand = torch.nn.functional.cosine_similarity(k0, k0[perm]).mean().item()
    assert near > 0.5 and rand < 0.2


def test_sweep_points():
    w = synth.sweep(65536, 25, 64)
    assert (w.B, w.H, w.d, w.N, w.Bk, w.budget_bp) == (1, 24, 128, 65536, 64, 2500)
    assert w.grid == (19, 45, 80) and w.nK == 1024

"""The seeded generator: determinism, shapes and the distributions the recipe states."""
import torch

from synth import CONFIGS, IVF, LARGE, TINY, gaussian_mixture, init_indices, make_config


def test_deterministic_and_seed_sensitive():
    a = gaussian_mixture(1000, 16, 8, seed=3)
    b = gaussian_mixture(1000, 16, 8, seed=3)
    c = gaussian_mixture(1000, 16, 8, seed=4)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert not torch.equal(a[0], c[0])


def test_bf16_storage_is_rounded_fp32_mixture():
    X, comp, cen = gaussian_mixture(500, 8, 4, dtype="bf16", seed=1)
    assert X.dtype == torch.bfloat16 and X.shape == (500, 8)
    X32, comp32, _ = gaussian_mixture(500, 8, 4, dtype="f32", seed=1)
    assert torch.equal(comp, comp32)
    assert torch.equal(X, X32.to(torch.bfloat16))


def test_zipf_top_component_share():
    # w_j ~ j^-1.2 over 65536 components: the top share is 1/H with H ~ 5.05.
    _, comp, _ = gaussian_mixture(200_000, 2, 65536, weights="zipf", zipf_s=1.2)
    share = (comp == 0).float().mean().item()
    w = torch.arange(1, 65537, dtype=torch.float64) ** -1.2
    expect = (1 / w.sum()).item()
    assert abs(share - expect) < 0.01
    assert comp.max() < 65536 and comp.min() >= 0


def test_noise_scale_matches_sigma():
    X, comp, cen = gaussian_mixture(20000, 32, 4, sigma=0.3, centers="normal")
    resid = X - cen[comp.long()]
    assert abs(resid.std().item() - 0.3) < 0.01


def test_init_indices_distinct():
    idx = init_indices(1000, 256, seed=0)
    assert len(set(idx.tolist())) == 256 and idx.max() < 1000


def test_make_config_shapes():
    spec, X, C0, comp, cen = make_config(TINY, n=4096, k=32)
    assert X.shape == (4096, 128) and C0.shape == (32, 128) and C0.dtype == torch.float32
    assert CONFIGS[LARGE].dtype == "bf16" and CONFIGS[IVF].metric == "cosine"


def test_shards_share_the_mixture_and_draw_their_own_points():
    """A data-parallel rank's points (shard r) come from the same centers with their own
    component and noise draws; shard 0 is the plain draw."""
    X0, c0, cen0 = gaussian_mixture(4000, 16, 10, sigma=0.05, seed=3)
    Xa, ca, cena = gaussian_mixture(4000, 16, 10, sigma=0.05, seed=3, shard=0)
    X1, c1, cen1 = gaussian_mixture(4000, 16, 10, sigma=0.05, seed=3, shard=1)
    assert torch.equal(X0, Xa) and torch.equal(c0, ca)
    assert torch.equal(cen0, cen1)
    assert not torch.equal(X0, X1) and not torch.equal(c0, c1)
    # every shard's points sit around the shared centers
    err = (X1 - cen1[c1.long()]).std()
    assert abs(float(err) - 0.05) < 0.005

"""The seeded input generators (bit_w4a4_quantised_b200.workloads), the one
module both the oracle side and the device side draw from.  It holds none of
the method's arithmetic; these checks pin the input recipe itself: values
exact in bf16 where the device takes bf16, V with orthonormal columns, the
alpha = 0.5 smoothing rule, the outlier channels, determinism per seed, and
the denoising step's layer list."""
import numpy as np
import pytest

from bit_w4a4_quantised_b200 import workloads


def small(seed=0, layer=0, **kw):
    args = dict(seed=seed, config_id=99, layer=layer, n_outliers=5, outlier_scale=20.0)
    args.update(kw)
    return workloads.draw_layer("t", 48, 384, 80, 16, 64, **args)


def test_bf16_round_is_nearest_even_and_idempotent():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1) wins; 1 + 3 * 2^-8
    # ties between 1 + 2^-7 and 1 + 2^-6: the even one is 1 + 2^-6
    v = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 1 + 2.0 ** -9], dtype=np.float32)
    got = workloads.bf16_round(v)
    assert got.tolist() == [1.0, 1 + 2.0 ** -6, -1.0, 1.0]
    x = np.random.default_rng(0).standard_normal(1000).astype(np.float32)
    once = workloads.bf16_round(x)
    assert np.array_equal(workloads.bf16_round(once), once)
    assert np.all(workloads.bf16_bits(once).astype(np.uint32) << 16 == once.view(np.uint32))


def test_layer_arrays_are_exact_in_bf16_and_shaped():
    c = small()
    assert c.x.shape == (48, 384) and c.W.shape == (80, 384) and c.bias.shape == (80,)
    assert c.s.shape == (384,) and c.V.shape == (384, 16)
    for a in (c.x, c.W, c.bias):
        assert a.dtype == np.float32
        assert np.array_equal(workloads.bf16_round(a), a)


def test_v_has_orthonormal_columns():
    V = small().V.astype(np.float64)
    assert np.abs(V.T @ V - np.eye(16)).max() < 1e-6


def test_smoothing_vector_is_the_alpha_half_rule():
    c = small()
    ax = np.abs(c.x).max(axis=0).astype(np.float64)
    aw = np.abs(c.W).max(axis=0).astype(np.float64)
    want = np.sqrt(ax) / np.sqrt(aw)
    assert np.allclose(c.s, want, rtol=1e-6)
    assert np.all(c.s > 0)


def test_outlier_channels():
    c = small(n_outliers=5, outlier_scale=20.0)
    col = np.abs(c.x).max(axis=0)
    top = np.sort(col)[::-1]
    # five channels scaled x20 stand far above the Gaussian rest
    assert top[4] > 3 * top[5]
    assert workloads.outlier_count(3072, 0.005) == 15
    assert workloads.outlier_count(14336, 0.005) == 72


def test_draws_are_seeded():
    a, b = small(seed=3, layer=1), small(seed=3, layer=1)
    for f in ("x", "W", "bias", "V", "s"):
        assert np.array_equal(getattr(a, f), getattr(b, f))
    c = small(seed=3, layer=2)
    assert not np.array_equal(a.x, c.x)
    d = small(seed=4, layer=1)
    assert not np.array_equal(a.W, d.W)


def test_rank_variants_share_x_w_and_bias():
    lo = workloads.draw_layer("t", 40, 256, 32, 0, 128, seed=1, config_id=99, v_rank=32)
    hi = workloads.draw_layer("t", 40, 256, 32, 32, 128, seed=1, config_id=99, v_rank=32)
    for f in ("x", "W", "bias", "s"):
        assert np.array_equal(getattr(lo, f), getattr(hi, f))
    assert lo.V.shape == (256, 0) and hi.V.shape == (256, 32)


@pytest.mark.parametrize("ctx", [True, False])
def test_denoising_step_layer_list(ctx):
    specs = workloads.c5_layer_specs(cross_kv_context=ctx)
    assert len(specs) == 600
    video = [s for s in specs if s.name.startswith("video.")]
    action = [s for s in specs if s.name.startswith("action.")]
    assert len(video) == 300 and len(action) == 300
    assert all(s.M == 4096 and s.r == 0 for s in video)
    assert sum(1 for s in video if (s.K, s.N) == (3072, 3072)) == 240
    assert sum(1 for s in video if (s.K, s.N) == (3072, 14336)) == 30
    assert sum(1 for s in video if (s.K, s.N) == (14336, 3072)) == 30
    assert all(s.r == 32 for s in action)
    kv = [s for s in action if s.name.split(".")[-1] in ("cross_k", "cross_v")]
    assert len(kv) == 60 and all(s.M == (4096 if ctx else 32) for s in kv)
    assert all(s.M == 32 for s in action if s not in kv)
    # the named single layers of the step are the ones the FFN workloads draw
    assert (specs[8].name, specs[8].N) == ("video.0.ffn0", 14336)
    assert (specs[9].name, specs[9].K) == ("video.0.ffn2", 14336)

"""Host-side checks of the runtime path selector (gqla_select_path): no GPU.

The selector predicts both decode calls' device times from a model of the
library's kernels and picks the faster one ("GQLA" chatpaper.ai Abstract: the
runtime takes the path that suits the hardware; "GQLA" scholarbro.com
Abstract: the preference follows the compute-to-bandwidth balance)."""
import pytest
import torch

from latent_kv_cache_flash_b200 import synth

B200 = (148, 6559.0, 1656.2)   # SMs, copy GB/s, dense bf16 TFLOP/s (measured on a B200)

# Faster path per (G, s_q) on the crossover grid (n_h 128, r 512, rope 64,
# d = v = 128, B32, L 32K), measured on one B200 with `bench.py --sweep
# crossover` (absorb ms, GQA ms).  A performance record, not an oracle value.
MEASURED_B200 = {
    (1, 1): (0.489, 0.133), (1, 2): (0.924, 0.227), (1, 4): (1.710, 0.413),
    (2, 1): (0.488, 0.237), (2, 2): (0.922, 0.246), (2, 4): (1.710, 0.417),
    (4, 1): (0.487, 0.485), (4, 2): (0.923, 0.460), (4, 4): (1.710, 0.476),
    (8, 1): (0.487, 0.759), (8, 2): (0.923, 0.855), (8, 4): (1.712, 0.912),
    (16, 1): (0.498, 1.509), (16, 2): (0.928, 1.512), (16, 4): (1.711, 1.615),
    (32, 1): (0.502, 2.986), (32, 2): (0.930, 2.998), (32, 4): (1.723, 3.031),
    (128, 1): (0.497, 12.161), (128, 2): (0.926, 12.171), (128, 4): (1.710, 12.175),
}

# The DeepSeek-V3-shaped layer (n_h 128, G 16, B64) over context lengths,
# `bench.py --sweep context` on the same B200: (L, s_q) -> (absorb ms, GQA ms).
MEASURED_CONTEXT_B200 = {
    (8192, 1): (0.279, 0.779), (8192, 2): (0.531, 0.803),
    (16384, 1): (0.501, 1.507), (16384, 2): (0.958, 1.532),
    (32768, 1): (0.934, 2.978), (32768, 2): (1.744, 3.001),
    (65536, 1): (1.728, 5.970), (65536, 2): (3.281, 6.001),
}


@pytest.fixture(scope="module")
def G():
    from latent_kv_cache_flash_b200 import build, gqla
    build.build()
    return gqla


def _est(gq, n_h, groups, s_q, B, L, hw=B200, shared=False, total=None):
    d = synth.Dims(n_h=n_h, G=groups, d_nope=128, d_rope=64, d_v=128, r=512, s_q=s_q, k_shared_rope=shared)
    lens = torch.full((B,), L, dtype=torch.int32)
    lay = gq.make_layout(lens, L, 0, L)
    return gq.gqla_select_path(gq.make_dims(d), lay, B * L if total is None else total, gq.GqlaHw(*hw))


def test_reproduces_the_measured_crossover(G):
    for (groups, s_q), (ms_a, ms_g) in MEASURED_B200.items():
        path, a_us, g_us = _est(G, 128, groups, s_q, 32, 32768)
        want = G.GQLA_PATH_GQA if ms_g < ms_a else G.GQLA_PATH_ABSORB
        assert path == want, (groups, s_q, a_us, g_us)
        # and the predicted times are within 15% of the measured ones
        assert abs(a_us / (ms_a * 1e3) - 1) < 0.15, (groups, s_q, a_us, ms_a)
        assert abs(g_us / (ms_g * 1e3) - 1) < 0.15, (groups, s_q, g_us, ms_g)


def test_reproduces_the_measured_context_sweep(G):
    for (L, s_q), (ms_a, ms_g) in MEASURED_CONTEXT_B200.items():
        path, a_us, g_us = _est(G, 128, 16, s_q, 64, L)
        assert path == (G.GQLA_PATH_GQA if ms_g < ms_a else G.GQLA_PATH_ABSORB), (L, s_q)
        assert abs(a_us / (ms_a * 1e3) - 1) < 0.10, (L, s_q, a_us, ms_a)
        assert abs(g_us / (ms_g * 1e3) - 1) < 0.10, (L, s_q, g_us, ms_g)


def test_structure_of_the_estimates(G):
    # absorb reads the joint latent whatever G is; the GQA stream grows with G
    a = [_est(G, 128, g, 1, 32, 32768)[1] for g in (8, 16, 32, 128)]
    q = [_est(G, 128, g, 1, 32, 32768)[2] for g in (8, 16, 32, 128)]
    assert max(a) - min(a) < 1e-6 * max(a)
    for (g0, t0), (g1, t1) in zip(zip((8, 16, 32), q), zip((16, 32, 128), q[1:])):
        assert abs(t1 / t0 - g1 / g0) < 0.02 * g1 / g0
    # the shared-RoPE K pool streams fewer bytes
    assert _est(G, 128, 16, 1, 64, 16384, shared=True)[2] < _est(G, 128, 16, 1, 64, 16384)[2]
    # doubling the context nearly doubles both (long-context regime); the
    # absorbed call's side GEMMs and merge do not grow with L (measured: 0.501
    # -> 0.934 ms, a factor 1.87)
    p1, a1, g1 = _est(G, 128, 16, 1, 64, 16384)
    p2, a2, g2 = _est(G, 128, 16, 1, 64, 32768)
    assert 1.7 < a2 / a1 < 2.1 and 1.9 < g2 / g1 < 2.1


def test_preference_follows_the_compute_to_bandwidth_ratio(G):
    # The same DeepSeek-V3-shaped layer on machines of other balance, with the
    # kernels' B200 efficiencies: a compute-rich part (H100-like: 132 SMs,
    # 3350 GB/s, 989 TFLOP/s) keeps absorb, as the pages report for H100; a
    # bandwidth-rich, compute-poor part (H20-like: 78 SMs, 4000 GB/s, 148
    # TFLOP/s) prefers GQA on the 8-way head-sharded layer the pages ran there
    # (16 heads, 2 groups per rank).
    assert _est(G, 128, 16, 1, 64, 32768, hw=(132, 3350.0, 989.0))[0] == G.GQLA_PATH_ABSORB
    assert _est(G, 16, 2, 1, 64, 32768, hw=(78, 4000.0, 148.0))[0] == G.GQLA_PATH_GQA
    # lowering only the tensor rate moves the crossover towards GQA
    slow_tc = (148, 6559.0, 400.0)
    assert _est(G, 128, 16, 2, 32, 32768)[0] == G.GQLA_PATH_ABSORB
    assert _est(G, 128, 16, 2, 32, 32768, hw=slow_tc)[0] == G.GQLA_PATH_GQA


def test_ragged_total_and_validation(G):
    # fewer cached tokens than the uniform bound: both estimates shrink
    full = _est(G, 128, 16, 1, 128, 65536)
    ragged = _est(G, 128, 16, 1, 128, 65536, total=128 * 33280)
    assert ragged[1] < full[1] and ragged[2] < full[2]
    with pytest.raises(G.GqlaError):
        _est(G, 128, 16, 1, 4, 1024, total=4 * 1024 + 1)       # above batch * max_seq_len
    with pytest.raises(G.GqlaError):
        _est(G, 128, 16, 2, 4, 1024, total=7)                  # below batch * s_q
    with pytest.raises(G.GqlaError):
        _est(G, 128, 16, 1, 4, 1024, hw=(0, 6559.0, 1656.2))

"""The path selector against live timings on this GPU: on shapes where one
path is clearly faster (margin above 20%), gqla_select_path must name it, and
its predicted times must be within a factor of 2 of the measured ones."""
import pytest
import torch

from latent_kv_cache_flash_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from latent_kv_cache_flash_b200 import build
    build.build()


def _time_us(fn, reps=20):
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps * 1e3


@pytest.mark.parametrize("n_h,G,s_q,B,L", [(128, 2, 2, 16, 8192), (128, 32, 1, 16, 8192), (32, 8, 1, 32, 8192),
                                           (128, 4, 4, 8, 16384)])
def test_selector_names_the_faster_path(n_h, G, s_q, B, L):
    from latent_kv_cache_flash_b200 import gqla
    d = synth.Dims(n_h=n_h, G=G, d_nope=128, d_rope=64, d_v=128, r=512, s_q=s_q)
    wl = synth.Workload("select", d, batch=B, seq_len=L, seed=70)
    inp = synth.make_inputs(wl, DEV)
    dims = gqla.make_dims(d)
    lay = gqla.make_layout(inp.seq_lens, L, 0, inp.capacity)
    ks, vs = synth.expanded_pool_shapes(inp)
    g = torch.Generator(device=DEV)
    g.manual_seed(1)
    kp = synth._randn_chunked(ks, g, DEV, d.torch_dtype)   # decode time does not depend on the values
    vp = synth._randn_chunked(vs, g, DEV, d.torch_dtype)
    out = torch.empty((B, s_q, n_h, d.d_v), dtype=d.torch_dtype, device=DEV)
    lse = torch.empty((B, s_q, n_h), device=DEV)
    ws_a = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_ABSORB, DEV)
    ws_g = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_GQA, DEV)
    t_a = _time_us(lambda: gqla.gqla_decode_absorb(dims, lay, inp.q, inp.latent, inp.W_uk, inp.W_uv, out, lse, 0,
                                                   ws_a))
    t_g = _time_us(lambda: gqla.gqla_decode_gqa(dims, lay, inp.q, kp, vp, out, lse, 0, ws_g))
    path, e_a, e_g = gqla.gqla_select_path(dims, lay, B * L)
    assert max(t_a, t_g) > 1.2 * min(t_a, t_g), "shape without a clear winner: %.1f vs %.1f us" % (t_a, t_g)
    assert path == (gqla.GQLA_PATH_GQA if t_g < t_a else gqla.GQLA_PATH_ABSORB), (t_a, t_g, e_a, e_g)
    assert 0.5 < e_a / t_a < 2.0 and 0.5 < e_g / t_g < 2.0, (t_a, t_g, e_a, e_g)

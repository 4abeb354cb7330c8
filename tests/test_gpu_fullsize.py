"""GPU parity at full size: the DeepSeek-V3-shaped batch the bench times (B64,
L65536) and the corners of the path-crossover grid (B32, L32768), each decoded
by both paths in the launch configuration the bench uses (the library's own
split plan), compared with the fp64 oracle on sampled (sequence, group) units.

Tolerances as everywhere: bf16 max|err| <= 1e-2 max|ref| + 1e-3, applied to
the output and to the log-sum-exp of the sampled units."""
import pytest
import torch

from latent_kv_cache_flash_b200 import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from latent_kv_cache_flash_b200 import build
    build.build()
    yield
    torch.cuda.empty_cache()


def _both_paths(inp, n_units, seed, what):
    for path in ("absorb", "gqa"):
        out, lse = H.run_decode(inp, path)
        torch.cuda.synchronize()
        H.check_units(inp, out, lse, H.sample_units(inp, n_units, seed=seed), "%s %s" % (what, path))
        del out, lse
        torch.cuda.empty_cache()


@pytest.mark.parametrize("s_q", [1, 2])
def test_dsv3_b64_l64k_full_batch(s_q):
    """The bench's headline workload: every sequence of the B64 batch at 64K
    context decoded in one call per path; sampled units against the oracle."""
    torch.cuda.empty_cache()
    inp = synth.make_inputs(synth.dsv3(seq_len=65536, s_q=s_q, batch=64), DEV)
    _both_paths(inp, 3, 10 + s_q, "dsv3 B64 L64K s_q=%d" % s_q)
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("G,s_q", [(1, 4), (2, 2), (128, 1), (16, 2)])
def test_crossover_corners_b32_l32k(G, s_q):
    """Corners of the crossover grid (n_h 128, B32, L32K) at full size: the
    tensor-bound GQA shapes (G 1 with s_q 4, G 2 with s_q 2), the 86 GB
    expanded cache of G 128, and the DeepSeek group count with s_q 2."""
    torch.cuda.empty_cache()
    inp = synth.make_inputs(synth.crossover(G, s_q), DEV)
    _both_paths(inp, 3, 20 + G + s_q, "crossover G=%d s_q=%d B32 L32K" % (G, s_q))
    del inp
    torch.cuda.empty_cache()

"""Group tensor parallelism on one GPU: the ranks' shares of a batch
(multi.tp_shard: a rank's groups, their heads and up-projections; the whole
latent cache) are decoded one after another, and their outputs, put side by
side along the heads, must equal the unsharded decode.  A group's heads read
only that group's K/V, so with the same split plan the shares give the very
same numbers, bit for bit; both match the fp64 oracle on sampled units."""
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


@pytest.mark.parametrize("world", [2, 4, 8])
@pytest.mark.parametrize("path", ["gqa", "absorb"])
def test_group_shards_reassemble_the_batch(world, path):
    from latent_kv_cache_flash_b200 import multi
    d = synth.Dims(n_h=32, G=8, d_nope=128, d_rope=64, d_v=128, r=512, s_q=2)
    wl = synth.Workload("tp", d, batch=3, seq_len=1500, page_size=64, seed=80)
    inp = synth.make_inputs(wl, DEV, seq_lens=[1500, 130, 777])
    full_o, full_l = H.run_decode(inp, path, num_splits=3)
    outs, lses = [], []
    for rank in range(world):
        sh = multi.tp_shard(inp, world, rank)
        o, l = H.run_decode(sh, path, num_splits=3)
        outs.append(o)
        lses.append(l)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(outs, dim=2), full_o) and torch.equal(torch.cat(lses, dim=2), full_l)
    H.check_units(inp, full_o, full_l, H.sample_units(inp, 4, seed=world), "tp %s x%d" % (path, world))

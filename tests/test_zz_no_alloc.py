"""The allocation-free GQA decode entry point (gqla_decode_gqa_noalloc).

Some callers cannot allocate device memory: a plug-in running inside a host
framework that owns all device memory and hands it no allocator, or a decode
loop that must not call cudaMalloc/cudaFree (which synchronise the device) on
its hot path.  For them the library keeps its split-KV scratch in a fixed
device array of its own.  This file checks, through the C ABI, that two calls
in a row give the same results as the workspace-taking gqla_decode_gqa on the
same inputs (within the tolerance the other GPU tests use), and that a problem
whose scratch would not fit is refused before anything is launched.

It sits in a file of its own, named so that pytest collects it last.
"""
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


def _inputs(seed, lens, s_q=2, page=64):
    d = synth.Dims(n_h=32, G=8, d_nope=128, d_rope=64, d_v=128, r=512, s_q=s_q)
    wl = synth.Workload("noalloc", d, batch=len(lens), seq_len=max(lens), page_size=page, seed=seed)
    return synth.make_inputs(wl, DEV, seq_lens=lens)


def _run_noalloc(inp, pools, num_splits):
    from latent_kv_cache_flash_b200 import gqla
    d = inp.dims
    out = torch.empty((inp.wl.batch, d.s_q, d.n_h, d.d_v), dtype=d.torch_dtype, device=DEV)
    lse = torch.empty((inp.wl.batch, d.s_q, d.n_h), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    gqla.gqla_decode_gqa_noalloc(gqla.make_dims(d), H.layout_of(inp), inp.q, pools[0], pools[1], out, lse,
                                 num_splits, dev_status=st)
    return out, lse, st


def test_noalloc_matches_workspace_entry_point_twice():
    # two different problems back to back: the second call must not see
    # anything the first one left in the shared scratch
    cases = [(_inputs(31, [1500, 777, 4096]), 0), (_inputs(32, [2048, 3000]), 5)]
    for inp, splits in cases:
        pools = H.run_expand(inp)
        ref_o, ref_l = H.run_decode(inp, "gqa", num_splits=splits, pools=pools)
        got_o, got_l, st = _run_noalloc(inp, pools, splits)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        H.assert_close(got_o.float().cpu().numpy(), ref_o.float().cpu().numpy(), "bf16", "noalloc out")
        H.assert_close(got_l.cpu().numpy(), ref_l.cpu().numpy(), "bf16", "noalloc lse")
        # and against the oracle on a few (sequence, group) units
        H.check_units(inp, got_o, got_l, H.sample_units(inp, 3), "noalloc vs oracle")


def test_noalloc_refuses_scratch_beyond_limit():
    from latent_kv_cache_flash_b200 import gqla
    # 64 sequences x 2 new tokens x 128 heads x (128 + 1) floats x 128 splits is
    # far above the 32 MiB scratch: refused before any launch
    d = synth.Dims(n_h=128, G=16, d_nope=128, d_rope=64, d_v=128, r=512, s_q=2)
    lens = torch.full((64,), 65536, dtype=torch.int32, device=DEV)
    lay = gqla.make_layout(lens, 65536, 0, 65536)
    dummy = torch.empty(16, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(gqla.GqlaError) as ei:
        gqla.gqla_decode_gqa_noalloc(gqla.make_dims(d), lay, dummy, dummy, dummy, dummy, None, 128)
    assert ei.value.status == gqla.GQLA_ERR_WORKSPACE

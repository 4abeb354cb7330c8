"""GPU checks of the shared-RoPE layout of the expanded K pool.

The decoupled RoPE key is one vector per token shared by all heads ("GQLA"
scholarbro.com Abstract), so the per-group K rows [k_nope_g ; k_rope] may keep
k_rope once per token row instead of once per group.  The scores are the same
numbers either way, so with the same inputs the two layouts must give
bit-identical expansions (rearranged) and bit-identical decode outputs, and
both must match the fp64 oracle."""
import dataclasses

import pytest
import torch

from latent_kv_cache_flash_b200 import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu

DEV = "cuda"
LLAMA = dict(n_h=32, G=8, d_nope=128, d_rope=64, d_v=128, r=512)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from latent_kv_cache_flash_b200 import build
    build.build()


def _pair(dims, lens, page, seed):
    """The same seeded inputs under both K layouts."""
    wl = synth.Workload("klayout", dims, batch=len(lens), seq_len=max(lens), page_size=page, seed=seed)
    a = synth.make_inputs(wl, DEV, seq_lens=lens)
    wl2 = dataclasses.replace(wl, dims=dataclasses.replace(dims, k_shared_rope=True))
    b = synth.make_inputs(wl2, DEV, seq_lens=lens)
    assert torch.equal(a.latent, b.latent) and torch.equal(a.q, b.q)
    return a, b


def _check_rearranged(dims, kp, vp, kp_s, vp_s, slots):
    G, dn = dims.G, dims.d_nope
    K = kp[slots]
    Ks = kp_s[slots]
    for g in range(G):
        assert torch.equal(Ks[:, g * dn:(g + 1) * dn], K[:, g, :dn]), g
        assert torch.equal(Ks[:, G * dn:], K[:, g, dn:]), g
    assert torch.equal(vp_s[slots], vp[slots])


def _valid_slots(inp):
    """Boolean mask over the pool's leading two dims: slots holding a token."""
    lead = inp.latent.shape[:2]
    mask = torch.zeros(lead, dtype=torch.bool)
    ps = inp.wl.page_size
    for b, L in enumerate(inp.seq_lens_host):
        if ps == 0:
            mask[b, :L] = True
        else:
            nb = (L + ps - 1) // ps
            for j in range(nb):
                page = int(inp.block_table[b, j])
                mask[page, : min(ps, L - j * ps)] = True
    return mask.to(DEV)


@pytest.mark.parametrize("page", [0, 64])
def test_shared_rope_expansion_is_a_rearrangement(page):
    d = synth.Dims(**LLAMA, s_q=1)
    a, b = _pair(d, [300, 64, 1000], page, seed=60)
    kp, vp = H.run_expand(a)
    kp_s, vp_s = H.run_expand(b)
    assert kp_s.shape[-1] == d.G * d.d_nope + d.d_rope
    _check_rearranged(d, kp, vp, kp_s, vp_s, _valid_slots(a))


@pytest.mark.parametrize("G,s_q,splits", [(8, 1, 0), (8, 2, 3), (16, 1, 0), (2, 2, 0), (1, 4, 2), (2, 4, 0), (1, 2, 3)])
def test_shared_rope_decode_matches_per_group(G, s_q, splits):
    # narrow (mma.sync, m*s_q < 64) and wide (tcgen05, m*s_q >= 64) kernels
    n_h = 32 if G <= 8 else 128
    d = synth.Dims(n_h=n_h, G=G, d_nope=128, d_rope=64, d_v=128, r=512, s_q=s_q)
    a, b = _pair(d, [700, 64 + s_q, 2049], 64, seed=61 + G + s_q)
    out_a, lse_a = H.run_decode(a, "gqa", num_splits=splits)
    out_b, lse_b = H.run_decode(b, "gqa", num_splits=splits)
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b)
    H.check_units(b, out_b, lse_b, H.sample_units(b, 6, seed=G), "shared rope G=%d s_q=%d" % (G, s_q))


def test_shared_rope_f32():
    d = synth.Dims(n_h=8, G=2, d_nope=32, d_rope=16, d_v=32, r=64, s_q=2, dtype="f32")
    a, b = _pair(d, [5, 129, 70], 0, seed=62)
    out_a, lse_a = H.run_decode(a, "gqa", num_splits=2)
    out_b, lse_b = H.run_decode(b, "gqa", num_splits=2)
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b)
    H.check_units(b, out_b, lse_b, H.all_units(b), "shared rope f32")


def test_shared_rope_append():
    from latent_kv_cache_flash_b200 import gqla
    d = synth.Dims(**LLAMA, s_q=2, k_shared_rope=True)
    wl = synth.Workload("klayout", d, batch=3, seq_len=500, page_size=64, seed=63)
    inp = synth.make_inputs(wl, DEV, seq_lens=[500, 65, 128])
    kp_ref, vp_ref = H.run_expand(inp)
    kp, vp = torch.zeros_like(kp_ref), torch.zeros_like(vp_ref)
    H.run_expand(inp, pools=(kp, vp))
    sentinel = -5.0
    for b_, L in enumerate(inp.seq_lens_host):   # poison the new tokens' slots
        for t in range(L - 2, L):
            page = int(inp.block_table[b_, t // 64])
            kp[page, t % 64] = sentinel
            vp[page, t % 64] = sentinel
    new_rows = torch.stack([inp.logical_latent(b_)[L - 2:L] for b_, L in enumerate(inp.seq_lens_host)]).contiguous()
    gqla.gqla_append_tokens(gqla.make_dims(d), H.layout_of(inp), new_rows, inp.latent, inp.W_uk, inp.W_uv, kp, vp)
    torch.cuda.synchronize()
    assert torch.equal(kp, kp_ref) and torch.equal(vp, vp_ref)

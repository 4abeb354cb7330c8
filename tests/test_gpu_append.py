"""GPU checks of the decode-time cache append (gqla_append_tokens).

The append writes the step's new rows [c_KV ; k_rope] at positions
L - s_q .. L - 1 of every sequence and, for the GQA path, expands exactly
those tokens into the per-group K/V pools ("GQLA" chatpaper.ai Abstract: the
latent cache of the absorb path, the expanded per-group cache of the GQA
path).  The latent write is a copy, so it is checked bit for bit; the
expanded rows against the fp64 oracle's expansion (bf16 tolerance) and bit for
bit against a full expansion of the same pool; and a decode after the append
against the oracle on the whole sequences."""
import numpy as np
import pytest
import torch

from latent_kv_cache_flash_b200 import synth
from oracle import gqla_oracle as O
from tests import helpers as H

pytestmark = pytest.mark.gpu

DEV = "cuda"
LLAMA = dict(n_h=32, G=8, d_nope=128, d_rope=64, d_v=128, r=512)
SENTINEL = -3.0


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from latent_kv_cache_flash_b200 import build
    build.build()


def _inputs(dims, lens, page, seed):
    wl = synth.Workload("append", dims, batch=len(lens), seq_len=max(lens), page_size=page, seed=seed)
    return synth.make_inputs(wl, DEV, seq_lens=lens)


def _slots(inp, b, t0, t1):
    """Pool indices (first two dims) of tokens t0..t1-1 of sequence b."""
    ps = inp.wl.page_size
    ts = torch.arange(t0, t1)
    if ps == 0:
        return torch.full_like(ts, b), ts
    return inp.block_table[b].cpu()[ts // ps].long(), ts % ps


def _new_rows(inp):
    s_q = inp.dims.s_q
    return torch.stack([inp.logical_latent(b)[L - s_q:L] for b, L in enumerate(inp.seq_lens_host)]).contiguous()


def _poison_new_slots(t, inp):
    s_q = inp.dims.s_q
    for b, L in enumerate(inp.seq_lens_host):
        i0, i1 = _slots(inp, b, L - s_q, L)
        t[i0.to(t.device), i1.to(t.device)] = SENTINEL


def _append(inp, new_rows, latent, pools=None, st=None):
    from latent_kv_cache_flash_b200 import gqla
    kp, vp = pools if pools is not None else (None, None)
    gqla.gqla_append_tokens(gqla.make_dims(inp.dims), H.layout_of(inp), new_rows, latent, inp.W_uk, inp.W_uv, kp,
                            vp, dev_status=st)


@pytest.mark.parametrize("page", [0, 64])
@pytest.mark.parametrize("s_q", [1, 2, 4])
def test_append_writes_latent_and_expanded_rows(page, s_q):
    d = synth.Dims(**LLAMA, s_q=s_q)
    inp = _inputs(d, [700, 64 + s_q, 129, 2048], page, seed=40 + s_q)
    ref_latent = inp.latent.clone()
    kp_ref, vp_ref = H.run_expand(inp)                 # full expansion of the intact pool
    new_rows = _new_rows(inp)
    _poison_new_slots(inp.latent, inp)
    kp, vp = kp_ref.clone(), vp_ref.clone()
    _poison_new_slots(kp, inp)
    _poison_new_slots(vp, inp)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    _append(inp, new_rows, inp.latent, (kp, vp), st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(inp.latent, ref_latent)         # a copy: bit for bit, nothing else touched
    assert torch.equal(kp, kp_ref) and torch.equal(vp, vp_ref)
    # the appended tokens' expansion against the oracle's
    W_uk = inp.W_uk.double().cpu().numpy()
    W_uv = inp.W_uv.double().cpu().numpy()
    for b, L in enumerate(inp.seq_lens_host):
        i0, i1 = _slots(inp, b, L - s_q, L)
        rows = new_rows[b].double().cpu().numpy()
        K = kp[i0.to(DEV), i1.to(DEV)].double().cpu().numpy()
        V = vp[i0.to(DEV), i1.to(DEV)].double().cpu().numpy()
        for g in range(d.G):
            Kr, Vr = O.expand_group(rows[:, : d.r], rows[:, d.r:], W_uk[g], W_uv[g])
            H.assert_close(K[:, g], Kr, "bf16", "K b=%d g=%d" % (b, g))
            H.assert_close(V[:, g], Vr, "bf16", "V b=%d g=%d" % (b, g))
    # and a decode step over the appended caches, both paths, against the oracle
    for path in ("absorb", "gqa"):
        out, lse = H.run_decode(inp, path, pools=(kp, vp))
        H.check_units(inp, out, lse, H.all_units(inp), "after append " + path)


def test_append_latent_only_leaves_pools_alone():
    d = synth.Dims(**LLAMA, s_q=2)
    inp = _inputs(d, [333, 80], 64, seed=50)
    ref_latent = inp.latent.clone()
    new_rows = _new_rows(inp)
    _poison_new_slots(inp.latent, inp)
    _append(inp, new_rows, inp.latent)
    torch.cuda.synchronize()
    assert torch.equal(inp.latent, ref_latent)


def test_append_expansion_only_without_latent_pool():
    """latent = NULL: the GQA-only cache gets the new tokens' K/V from the
    dense rows alone, bit for bit as the full expansion gives them."""
    d = synth.Dims(**LLAMA, s_q=3)
    inp = _inputs(d, [500, 3, 64, 1000], 64, seed=53)
    kp_ref, vp_ref = H.run_expand(inp)
    new_rows = _new_rows(inp)
    before = inp.latent.clone()
    kp, vp = kp_ref.clone(), vp_ref.clone()
    _poison_new_slots(kp, inp)
    _poison_new_slots(vp, inp)
    from latent_kv_cache_flash_b200 import gqla
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    gqla.gqla_append_tokens(gqla.make_dims(inp.dims), H.layout_of(inp), new_rows, None, inp.W_uk, inp.W_uv, kp, vp,
                            dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(kp, kp_ref) and torch.equal(vp, vp_ref)
    assert torch.equal(inp.latent, before)


def test_append_f32_contiguous():
    d = synth.Dims(n_h=8, G=2, d_nope=32, d_rope=16, d_v=32, r=64, s_q=3, dtype="f32")
    inp = _inputs(d, [5, 3, 70], 0, seed=51)
    ref_latent = inp.latent.clone()
    kp_ref, vp_ref = H.run_expand(inp)
    new_rows = _new_rows(inp)
    _poison_new_slots(inp.latent, inp)
    kp, vp = kp_ref.clone(), vp_ref.clone()
    _poison_new_slots(kp, inp)
    _append(inp, new_rows, inp.latent, (kp, vp))
    torch.cuda.synchronize()
    assert torch.equal(inp.latent, ref_latent)
    assert torch.equal(kp, kp_ref) and torch.equal(vp, vp_ref)
    out, lse = H.run_decode(inp, "gqa", pools=(kp, vp))
    H.check_units(inp, out, lse, H.all_units(inp), "f32 after append")


def test_append_flags_bad_sequences_and_skips_them():
    from latent_kv_cache_flash_b200 import gqla
    d = synth.Dims(**LLAMA, s_q=2)
    inp = _inputs(d, [100, 200, 300], 64, seed=52)
    new_rows = _new_rows(inp)
    before = inp.latent.clone()
    inp.seq_lens[0] = 1                           # shorter than s_q
    inp.block_table[2, 4] = inp.num_pages + 9     # the page of tokens 256..299, outside the pool
    poison = torch.full_like(new_rows, SENTINEL)
    poison[1] = new_rows[1]
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    _append(inp, poison, inp.latent, st=st)
    torch.cuda.synchronize()
    flags = int(st.item())
    assert flags & gqla.DEV_SHORT_SEQ and flags & gqla.DEV_BAD_PAGE
    # sequence 1 rewrote its own (identical) rows, 0 and 2 wrote nothing
    assert torch.equal(inp.latent, before)


@pytest.mark.parametrize("shape", ["llama", "wide"])
@pytest.mark.parametrize("page", [0, 64])
def test_chained_calls_without_host_sync(shape, page):
    # the append, then both decode paths, queued back to back on one stream
    # with no host synchronisation: every call must see all that the one
    # before it wrote (its kernels may launch early, but the first waits for
    # the kernel ahead before any access).  New slots are poisoned first, so a
    # decode that read too early would differ from the synchronised run.
    dims_kw = LLAMA if shape == "llama" else dict(n_h=128, G=2, d_nope=128, d_rope=64, d_v=128, r=512)
    d = synth.Dims(**dims_kw, s_q=2)
    inp = _inputs(d, [700, 66, 1029, 2048], page, seed=77)
    kp0, vp0 = H.run_expand(inp)
    new_rows = _new_rows(inp)
    lat0 = inp.latent.clone()

    def run(sync):
        inp.latent.copy_(lat0)
        kp, vp = kp0.clone(), vp0.clone()
        for t in (inp.latent, kp, vp):
            _poison_new_slots(t, inp)
        if sync:
            torch.cuda.synchronize()
        _append(inp, new_rows, inp.latent, (kp, vp))
        if sync:
            torch.cuda.synchronize()
        res = [H.run_decode(inp, "absorb")]
        if sync:
            torch.cuda.synchronize()
        res.append(H.run_decode(inp, "gqa", pools=(kp, vp)))
        torch.cuda.synchronize()
        return res

    ref = run(True)
    for _ in range(3):
        for (o1, l1), (o2, l2) in zip(ref, run(False)):
            assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)

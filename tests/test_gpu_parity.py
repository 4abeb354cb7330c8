"""GPU parity: the CUDA path (through the C-ABI binding) against the fp64
oracle on the same seeded inputs, plus structural invariances and edge cases.

Tolerances: fp32 max|err| <= 1e-5 max|ref|; bf16 max|err| <= 1e-2 max|ref| +
1e-3 (fp32 accumulation), applied to the output and to the log-sum-exp."""
import numpy as np
import pytest
import torch

from latent_kv_cache_flash_b200 import synth
from oracle import gqla_oracle as O
from tests import helpers as H

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from latent_kv_cache_flash_b200 import build
    build.build()


def _wl(dims, B, lens, page=0, seed=0):
    wl = synth.Workload("t", dims, batch=B, seq_len=max(lens), page_size=page, seed=seed)
    return synth.make_inputs(wl, DEV, seq_lens=lens)


LLAMA = dict(n_h=32, G=8, d_nope=128, d_rope=64, d_v=128, r=512)
DSV3 = dict(n_h=128, G=16, d_nope=128, d_rope=64, d_v=128, r=512)


# ---- the tiny fp32 workload, whole output, both paths ----------------------
@pytest.mark.parametrize("path", ["absorb", "gqa"])
def test_tiny_f32_full(path):
    inp = synth.make_inputs(synth.tiny_f32(), DEV)
    out, lse = H.run_decode(inp, path)
    H.check_units(inp, out, lse, H.all_units(inp), "tiny_f32 " + path)


@pytest.mark.parametrize("path", ["absorb", "gqa"])
@pytest.mark.parametrize("splits", [1, 2, 5])
def test_f32_ragged_splits(path, splits):
    d = synth.Dims(n_h=8, G=2, d_nope=32, d_rope=16, d_v=32, r=64, s_q=2, dtype="f32")
    inp = _wl(d, 3, [2, 301, 700])
    out, lse = H.run_decode(inp, path, num_splits=splits)
    H.check_units(inp, out, lse, H.all_units(inp), "f32 ragged %s S=%d" % (path, splits))


# ---- bf16, LLaMA-3-8B and DeepSeek-V3 head shapes at short contexts --------
@pytest.mark.parametrize("s_q", [1, 2, 3, 4])
@pytest.mark.parametrize("path", ["absorb", "gqa"])
@pytest.mark.parametrize("page", [0, 64])
def test_bf16_llama_shapes(s_q, path, page):
    d = synth.Dims(**LLAMA, s_q=s_q)
    inp = _wl(d, 3, [s_q, 517, 1100], page=page, seed=s_q)
    out, lse = H.run_decode(inp, path)
    H.check_units(inp, out, lse, H.all_units(inp), "llama bf16 %s s_q=%d page=%d" % (path, s_q, page))


@pytest.mark.parametrize("s_q", [1, 2])
@pytest.mark.parametrize("path", ["absorb", "gqa"])
def test_bf16_dsv3_shapes(s_q, path):
    d = synth.Dims(**DSV3, s_q=s_q)
    inp = _wl(d, 2, [640, 1313], page=64, seed=7)
    out, lse = H.run_decode(inp, path)
    H.check_units(inp, out, lse, H.sample_units(inp, 8), "dsv3 bf16 %s s_q=%d" % (path, s_q))


@pytest.mark.parametrize("B", [5, 33, 61])
def test_bf16_absorb_merge_row_tiles(B):
    """The absorbed call's split merge and up-projection take 16, 32 or 64
    rows of a group per CTA, the largest that still fills the SMs: at G 16
    (8 rows a group per token) B 5 takes 16-row tiles, B 33 32-row tiles with
    a ragged last tile, B 61 64-row tiles with a ragged last tile.  Three
    splits, so every row merges several partials."""
    d = synth.Dims(**DSV3, s_q=1)
    g = torch.Generator()
    g.manual_seed(B)
    lens = torch.randint(200, 700, (B,), generator=g).tolist()
    inp = _wl(d, B, lens, seed=B)
    out, lse = H.run_decode(inp, "absorb", num_splits=3)
    H.check_units(inp, out, lse, H.sample_units(inp, 6, seed=B), "absorb merge tiles B=%d" % B)


@pytest.mark.parametrize("page", [128, 256])
@pytest.mark.parametrize("path", ["absorb", "gqa"])
def test_bf16_large_pages(page, path):
    """Pages of 128 and 256 tokens (any multiple of the 64-token tile):
    lengths that end inside a page, on a page boundary and past several
    pages, through a permuted block table."""
    d = synth.Dims(**DSV3, s_q=2)
    inp = _wl(d, 3, [130, 2 * page, 1500], page=page, seed=page)
    out, lse = H.run_decode(inp, path)
    H.check_units(inp, out, lse, H.sample_units(inp, 6, seed=page), "dsv3 bf16 %s page=%d" % (path, page))


@pytest.mark.parametrize("G", [1, 2])
@pytest.mark.parametrize("splits", [0, 3])
def test_gqa_wide_three_new_tokens(G, splits):
    """The tcgen05 GQA kernel at s_q 3: 384 rows a group at G 1 (three full
    128-row blocks), 192 at G 2 (the second block half empty), paged."""
    d = synth.Dims(n_h=128, G=G, d_nope=128, d_rope=64, d_v=128, r=512, s_q=3)
    inp = _wl(d, 2, [300, 777], page=128, seed=50 + G)
    out, lse = H.run_decode(inp, "gqa", num_splits=splits)
    H.check_units(inp, out, lse, H.sample_units(inp, 4, seed=G), "gqa_wide G=%d s_q=3 splits=%d" % (G, splits))


@pytest.mark.parametrize("G", [1, 2, 4, 32, 128])
@pytest.mark.parametrize("s_q", [1, 4])
def test_bf16_group_counts(G, s_q):
    d = synth.Dims(n_h=128, G=G, d_nope=128, d_rope=64, d_v=128, r=512, s_q=s_q)
    inp = _wl(d, 1, [777], seed=G)
    for path in ("absorb", "gqa"):
        out, lse = H.run_decode(inp, path)
        H.check_units(inp, out, lse, H.sample_units(inp, 4, seed=G), "G=%d s_q=%d %s" % (G, s_q, path))


# ---- expansion --------------------------------------------------------------
def test_expand_matches_oracle():
    d = synth.Dims(**LLAMA)
    inp = _wl(d, 2, [130, 257], page=64, seed=3)
    kp, vp = H.run_expand(inp)
    W_uk = inp.W_uk.double().cpu().numpy()
    W_uv = inp.W_uv.double().cpu().numpy()
    for b in range(2):
        rows = inp.logical_latent(b).double().cpu().numpy()
        L = inp.seq_lens_host[b]
        nb = (L + 63) // 64
        pages = inp.block_table[b, :nb].long()
        K = kp[pages].reshape(nb * 64, d.G, d.d_qk)[:L].double().cpu().numpy()
        V = vp[pages].reshape(nb * 64, d.G, d.d_v)[:L].double().cpu().numpy()
        for g in range(d.G):
            Kr, Vr = O.expand_group(rows[:, : d.r], rows[:, d.r:], W_uk[g], W_uv[g])
            H.assert_close(K[:, g], Kr, "bf16", "K b=%d g=%d" % (b, g))
            H.assert_close(V[:, g], Vr, "bf16", "V b=%d g=%d" % (b, g))
            assert torch.equal(torch.tensor(K[:, g, d.d_nope:]), torch.tensor(rows[:, d.r:]))


@pytest.mark.parametrize("lens,page,G", [([100], 0, 8), ([1], 0, 8), ([64, 1, 300], 0, 8), ([64, 1, 300], 64, 8),
                                         ([129, 257, 1], 64, 16), ([700], 64, 1)])
def test_expand_odd_tile_counts(lens, page, G):
    """The whole-cache expansion runs two 128-token tiles per MMA (one per CTA
    of a pair): an odd tile count, a pair whose second tile lies past its
    sequence, one-token sequences, G = 1 and G = 16.  Every token's rows
    against the oracle; the slots past each sequence's end keep the sentinel
    the pools were filled with."""
    d = synth.Dims(**dict(LLAMA, G=G))
    inp = _wl(d, len(lens), lens, page=page, seed=21)
    ks, vs = synth.expanded_pool_shapes(inp)
    sentinel = 5.0
    kp = torch.full(ks, sentinel, dtype=d.torch_dtype, device=DEV)
    vp = torch.full(vs, sentinel, dtype=d.torch_dtype, device=DEV)
    H.run_expand(inp, pools=(kp, vp))
    torch.cuda.synchronize()
    W_uk = inp.W_uk.double().cpu().numpy()
    W_uv = inp.W_uv.double().cpu().numpy()
    for b, L in enumerate(lens):
        rows = inp.logical_latent(b).double().cpu().numpy()
        if page:
            nb = (L + page - 1) // page
            pages = inp.block_table[b, :nb].long()
            K = kp[pages].reshape(nb * page, d.G, d.d_qk)
            V = vp[pages].reshape(nb * page, d.G, d.d_v)
        else:
            K, V = kp[b], vp[b]
        assert bool((K[L:] == sentinel).all()) and bool((V[L:] == sentinel).all()), "written past the end, b=%d" % b
        K = K[:L].double().cpu().numpy()
        V = V[:L].double().cpu().numpy()
        for g in range(d.G):
            Kr, Vr = O.expand_group(rows[:, : d.r], rows[:, d.r:], W_uk[g], W_uv[g])
            H.assert_close(K[:, g], Kr, "bf16", "K b=%d g=%d" % (b, g))
            H.assert_close(V[:, g], Vr, "bf16", "V b=%d g=%d" % (b, g))
            assert torch.equal(torch.tensor(K[:, g, d.d_nope:]), torch.tensor(rows[:, d.r:]))


@pytest.mark.parametrize("page", [0, 64])
def test_expand_flags_bad_sequences_and_skips_them(page):
    """Whole-cache expansion with an empty sequence and one longer than the
    host bound: both flagged, their slots keep the sentinel, and the healthy
    sequence's rows equal an expansion without the bad ones, bit for bit."""
    from latent_kv_cache_flash_b200 import gqla
    d = synth.Dims(**LLAMA)
    inp = _wl(d, 3, [200, 300, 150], page=page, seed=14)
    kp_ref, vp_ref = H.run_expand(inp)
    ks, vs = synth.expanded_pool_shapes(inp)
    kp = torch.full(ks, 5.0, dtype=d.torch_dtype, device=DEV)
    vp = torch.full(vs, 5.0, dtype=d.torch_dtype, device=DEV)
    inp.seq_lens[0] = 0                       # empty
    inp.seq_lens[2] = 400                     # above the host bound max_seq_len = 300
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    H.run_expand(inp, dev_status=st, pools=(kp, vp))
    torch.cuda.synchronize()
    flags = int(st.item())
    assert flags & gqla.DEV_SHORT_SEQ and flags & gqla.DEV_OVERFLOW
    if page:
        rows = lambda b: inp.block_table[b, : (inp.seq_lens_host[b] + 63) // 64].long()
        for b in (0, 2):
            assert bool((kp[rows(b)] == 5.0).all()) and bool((vp[rows(b)] == 5.0).all())
        flat = lambda t: t[rows(1)].reshape((-1,) + tuple(t.shape[2:]))[:300]
        assert torch.equal(flat(kp), flat(kp_ref)) and torch.equal(flat(vp), flat(vp_ref))
    else:
        for b in (0, 2):
            assert bool((kp[b] == 5.0).all()) and bool((vp[b] == 5.0).all())
        assert torch.equal(kp[1, :300], kp_ref[1, :300]) and torch.equal(vp[1, :300], vp_ref[1, :300])


def test_expand_tail_only_touches_new_tokens():
    d = synth.Dims(**LLAMA, s_q=2)
    inp = _wl(d, 2, [300, 41], seed=5)
    kp, vp = H.run_expand(inp)
    sentinel = 7.0
    kp2 = torch.full_like(kp, sentinel)
    vp2 = torch.full_like(vp, sentinel)
    H.run_expand(inp, tail=2, pools=(kp2, vp2))
    for b, L in enumerate(inp.seq_lens_host):
        assert torch.equal(kp2[b, L - 2:L], kp[b, L - 2:L])
        assert torch.equal(vp2[b, L - 2:L], vp[b, L - 2:L])
        assert bool((kp2[b, :L - 2] == sentinel).all()) and bool((vp2[b, L:] == sentinel).all())


def test_expand_flags_bad_page_and_writes_nothing_for_it():
    """A block-table entry outside the pool: flagged, and no row is written in
    its place; every other page is expanded as without it."""
    from latent_kv_cache_flash_b200 import gqla
    d = synth.Dims(**LLAMA)
    inp = _wl(d, 2, [300, 200], page=64, seed=12)
    kp_ref, vp_ref = H.run_expand(inp)
    replaced = int(inp.block_table[1, 1])
    inp.block_table[1, 1] = inp.num_pages + 3
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    kp, vp = H.run_expand(inp, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & gqla.DEV_BAD_PAGE
    others = [pg for pg in range(inp.num_pages) if pg != replaced]
    assert torch.equal(kp[others], kp_ref[others]) and torch.equal(vp[others], vp_ref[others])
    assert not bool(kp[replaced].any()) and not bool(vp[replaced].any())


# ---- combine ------------------------------------------------------------
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_combine_matches_oracle(dtype):
    from latent_kv_cache_flash_b200 import gqla
    g = torch.Generator(device=DEV)
    g.manual_seed(0)
    S, R, D = 5, 77, 512
    o = torch.randn((S, R, D), generator=g, device=DEV)
    l = torch.randn((S, R), generator=g, device=DEV) * 3
    l[1, :10] = -float("inf")
    l[:, 20] = -float("inf")       # a row with no keys at all
    out = torch.empty((R, D), dtype=dtype, device=DEV)
    lse = torch.empty((R,), device=DEV)
    gqla.gqla_splitkv_combine(o, l, out, lse)
    ro, rl = O.splitkv_combine(o.double().cpu().numpy(), l.double().cpu().numpy())
    H.assert_close(out.float().cpu().numpy(), ro, "f32" if dtype == torch.float32 else "bf16", "combine out")
    H.assert_close(lse.cpu().numpy(), rl, "f32", "combine lse")
    assert torch.all(out[20] == 0)


# ---- invariances ------------------------------------------------------------
@pytest.mark.parametrize("path", ["absorb", "gqa"])
def test_paged_equals_contiguous_and_padding_poison(path):
    d = synth.Dims(**LLAMA, s_q=2)
    lens = [390, 1000]
    a = _wl(d, 2, lens, page=0, seed=9)
    # the same logical tokens in a permuted paged pool
    b = _wl(d, 2, lens, page=64, seed=9)
    for bb in range(2):
        L = lens[bb]
        nb = (L + 63) // 64
        pages = b.block_table[bb, :nb].long()
        pool = b.latent[pages].reshape(nb * 64, -1)
        pool[:L] = a.latent[bb, :L]
        pool[L:] = 1e4                       # finite poison past the end
        b.latent[pages] = pool.reshape(nb, 64, -1)
    b.q.copy_(a.q)
    b.W_uk.copy_(a.W_uk)
    b.W_uv.copy_(a.W_uv)
    a.latent[0, lens[0]:] = -1e4
    oa, la = H.run_decode(a, path, num_splits=3)
    ob, lb = H.run_decode(b, path, num_splits=3)
    assert torch.equal(oa, ob) and torch.equal(la, lb)


@pytest.mark.parametrize("path", ["absorb", "gqa"])
def test_split_count_invariance(path):
    d = synth.Dims(**LLAMA)
    inp = _wl(d, 2, [2000, 3000], seed=4)
    ref_o, ref_l = H.run_decode(inp, path, num_splits=1)
    for S in (2, 7, 24):
        o, l = H.run_decode(inp, path, num_splits=S)
        H.assert_close(o.float().cpu().numpy(), ref_o.float().cpu().numpy(), "bf16", "splits %d" % S)
        np.testing.assert_allclose(l.cpu().numpy(), ref_l.cpu().numpy(), rtol=0, atol=2e-3)


def test_paths_agree_full_tensor():
    """absorb and GQA outputs of the same weights agree on the whole tensor."""
    d = synth.Dims(**DSV3, s_q=2)
    inp = _wl(d, 3, [700, 2048, 4000], page=64, seed=12)
    oa, la = H.run_decode(inp, "absorb")
    og, lg = H.run_decode(inp, "gqa")
    H.assert_close(oa.float().cpu().numpy(), og.float().cpu().numpy(), "bf16", "absorb vs gqa")
    np.testing.assert_allclose(la.cpu().numpy(), lg.cpu().numpy(), rtol=0, atol=2e-2)


# ---- edge cases and device status -------------------------------------------
@pytest.mark.parametrize("path", ["absorb", "gqa"])
def test_edge_lengths(path):
    d = synth.Dims(**LLAMA, s_q=3)
    inp = _wl(d, 4, [3, 4, 129, 128], page=64, seed=2)   # L == s_q, page-boundary lengths
    out, lse = H.run_decode(inp, path)
    H.check_units(inp, out, lse, H.all_units(inp), "edge " + path)
    d1 = synth.Dims(**LLAMA, s_q=1)
    inp = _wl(d1, 1, [1], seed=2)
    out, lse = H.run_decode(inp, path)
    H.check_units(inp, out, lse, H.all_units(inp), "L=1 " + path)


@pytest.mark.parametrize("path", ["absorb", "gqa"])
@pytest.mark.parametrize("splits", [0, 3])
def test_device_status_flags(path, splits):
    from latent_kv_cache_flash_b200 import gqla
    d = synth.Dims(**LLAMA, s_q=2)
    inp = _wl(d, 3, [100, 200, 300], page=64, seed=1)
    pools = H.run_expand(inp) if path == "gqa" else None
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    inp.seq_lens[0] = 1                       # shorter than s_q
    inp.block_table[2, 1] = inp.num_pages + 5  # page id outside the pool
    out, lse = H.run_decode(inp, path, pools=pools, dev_status=st, num_splits=splits)
    torch.cuda.synchronize()
    flags = int(st.item())
    assert flags & gqla.DEV_SHORT_SEQ and flags & gqla.DEV_BAD_PAGE
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))
    assert torch.all(out[2] == 0) and torch.all(torch.isneginf(lse[2]))
    inp.seq_lens_host[0] = 1
    inp.block_table[2, 1] = 0
    H.check_units(inp, out, lse, [(1, g) for g in range(d.G)], "healthy row " + path)
    st.zero_()
    inp.seq_lens[1] = 400                     # above the host bound max_seq_len=300
    H.run_decode(inp, path, pools=pools, dev_status=st, max_seq_len=300, num_splits=splits)
    torch.cuda.synchronize()
    assert int(st.item()) & gqla.DEV_OVERFLOW


# ---- full-size workloads: whole GPU launch, sampled oracle units ------------
@pytest.mark.parametrize("s_q", [1, 2])
def test_llama3_8b_full_size(s_q):
    inp = synth.make_inputs(synth.llama3_8b(s_q=s_q), DEV)
    for path in ("absorb", "gqa"):
        out, lse = H.run_decode(inp, path)
        H.check_units(inp, out, lse, H.sample_units(inp, 4, seed=s_q), "llama full %s s_q=%d" % (path, s_q))


def test_dsv3_64k_sampled():
    inp = synth.make_inputs(synth.dsv3(seq_len=65536, s_q=2, batch=8), DEV)
    for path in ("absorb", "gqa"):
        out, lse = H.run_decode(inp, path)
        H.check_units(inp, out, lse, H.sample_units(inp, 3, seed=5), "dsv3 64K %s" % path)


def test_ragged_paged_full_size():
    inp = synth.make_inputs(synth.ragged_paged(), DEV)
    for path in ("absorb", "gqa"):
        out, lse = H.run_decode(inp, path)
        H.check_units(inp, out, lse, H.sample_units(inp, 4, seed=8), "ragged paged %s" % path)


# ---- rescaling paths: scores that grow along the sequence ---------------------
@pytest.mark.parametrize("path", ["absorb", "gqa"])
@pytest.mark.parametrize("peak", [1.0, 3.0])
def test_growing_and_peaked_scores(path, peak):
    """Every query's RoPE part is a shared direction u and the RoPE key of token
    t is 0.1 noise + (4 t / L) u, so scores rise by ~18 (natural units) along
    the sequence: the running maximum keeps growing past the first tile's,
    which forces the online-softmax rescale of the accumulator (lazy in the
    absorb kernel).  Values keep unit scale.  peak scales u (a sharper
    softmax)."""
    d = synth.Dims(**LLAMA, s_q=2)
    lens = [1500, 700]
    inp = _wl(d, 2, lens, page=64, seed=21)
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    u = torch.randn(d.d_rope, generator=g, device=DEV) * peak
    q = inp.q.float()
    q[..., d.d_nope:] = u + 0.05 * torch.randn(q[..., d.d_nope:].shape, generator=g, device=DEV)
    inp.q.copy_(q.to(inp.q.dtype))
    for b, L in enumerate(lens):
        nb = (L + 63) // 64
        pages = inp.block_table[b, :nb].long()
        rows = inp.latent[pages].reshape(nb * 64, -1).float()
        t = torch.arange(nb * 64, device=DEV, dtype=torch.float32)[:, None]
        rows[:, d.r:] = 0.1 * rows[:, d.r:] + (4.0 * t / L) * u[None, :] / peak
        inp.latent[pages] = rows.to(inp.latent.dtype).reshape(nb, 64, -1)
    out, lse = H.run_decode(inp, path, num_splits=1)
    H.check_units(inp, out, lse, H.all_units(inp), "growing scores %s peak=%g" % (path, peak))
    out2, lse2 = H.run_decode(inp, path)
    H.check_units(inp, out2, lse2, H.all_units(inp), "growing scores %s peak=%g auto splits" % (path, peak))


@pytest.mark.parametrize("G,s_q", [(2, 2), (1, 2), (4, 4)])
@pytest.mark.parametrize("splits", [0, 3])
def test_gqa_many_rows_per_group_paged(G, s_q, splits):
    """m * s_q >= 64 rows per group (the tensor-core GQA kernel), paged and
    ragged, with and without split-KV."""
    d = synth.Dims(n_h=128, G=G, d_nope=128, d_rope=64, d_v=128, r=512, s_q=s_q)
    inp = _wl(d, 3, [777, 1500, 64], page=64, seed=40 + G)
    out, lse = H.run_decode(inp, "gqa", num_splits=splits)
    H.check_units(inp, out, lse, H.sample_units(inp, 5, seed=G), "gqa wide G=%d s_q=%d S=%d" % (G, s_q, splits))


# ---- absorb at 128 heads: several 64-row blocks per sequence -------------------
@pytest.mark.parametrize("s_q,splits", [(1, 0), (1, 4), (2, 3), (4, 0)])
def test_absorb_128_heads_paged_ragged_edges(s_q, splits):
    """n_h = 128 (2 to 8 row blocks a sequence): paged, ragged, with
    page-boundary and tiny lengths (L = s_q, one page, one token past a page),
    every unit against the oracle."""
    d = synth.Dims(**DSV3, s_q=s_q)
    lens = [s_q, 64, 65, 1313, 2048]
    inp = _wl(d, len(lens), lens, page=64, seed=90 + s_q)
    out, lse = H.run_decode(inp, "absorb", num_splits=splits)
    H.check_units(inp, out, lse, H.all_units(inp), "absorb 128 heads s_q=%d S=%d" % (s_q, splits))


@pytest.mark.parametrize("peak", [1.0, 3.0])
def test_absorb_128_heads_growing_scores(peak):
    """Scores that rise along the sequence force the lazy rescale in every row
    block; contiguous cache, n_h = 128, s_q = 2."""
    d = synth.Dims(**DSV3, s_q=2)
    lens = [1500, 700]
    inp = _wl(d, 2, lens, seed=23)
    g = torch.Generator(device=DEV)
    g.manual_seed(6)
    u = torch.randn(d.d_rope, generator=g, device=DEV) * peak
    q = inp.q.float()
    q[..., d.d_nope:] = u + 0.05 * torch.randn(q[..., d.d_nope:].shape, generator=g, device=DEV)
    inp.q.copy_(q.to(inp.q.dtype))
    for b, L in enumerate(lens):
        rows = inp.latent[b].float()
        t = torch.arange(rows.shape[0], device=DEV, dtype=torch.float32)[:, None]
        rows[:, d.r:] = 0.1 * rows[:, d.r:] + (4.0 * t / L) * u[None, :] / peak
        inp.latent[b] = rows.to(inp.latent.dtype)
    for splits in (1, 0):
        out, lse = H.run_decode(inp, "absorb", num_splits=splits)
        H.check_units(inp, out, lse, H.all_units(inp), "absorb 128 heads growing peak=%g S=%d" % (peak, splits))


def test_absorb_128_heads_matches_gqa_full_tensor():
    """Absorb and GQA on the same weights at n_h = 128, whole tensors."""
    d = synth.Dims(**DSV3, s_q=1)
    inp = _wl(d, 4, [3000, 1, 777, 4096], page=64, seed=95)
    a_o, a_l = H.run_decode(inp, "absorb")
    g_o, g_l = H.run_decode(inp, "gqa")
    H.assert_close(a_o.float().cpu().numpy(), g_o.float().cpu().numpy(), "bf16", "absorb vs gqa out")
    H.assert_close(a_l.cpu().numpy(), g_l.cpu().numpy(), "bf16", "absorb vs gqa lse")


@pytest.mark.parametrize("G,s_q,splits", [(1, 2, 1), (2, 4, 0), (2, 2, 3)])
def test_gqa_wide_growing_scores(G, s_q, splits):
    """The tcgen05 GQA kernel (m * s_q >= 64 rows a group) with scores that
    rise along the sequence: both softmax warpgroups rescale their own
    accumulator, and their states merge at the end."""
    d = synth.Dims(n_h=128, G=G, d_nope=128, d_rope=64, d_v=128, r=512, s_q=s_q)
    lens = [1500, 193]
    inp = _wl(d, 2, lens, seed=31 + G)
    g = torch.Generator(device=DEV)
    g.manual_seed(7)
    u = torch.randn(d.d_rope, generator=g, device=DEV) * 2.0
    q = inp.q.float()
    q[..., d.d_nope:] = u + 0.05 * torch.randn(q[..., d.d_nope:].shape, generator=g, device=DEV)
    inp.q.copy_(q.to(inp.q.dtype))
    for b, L in enumerate(lens):
        rows = inp.latent[b].float()
        t = torch.arange(rows.shape[0], device=DEV, dtype=torch.float32)[:, None]
        rows[:, d.r:] = 0.1 * rows[:, d.r:] + (4.0 * t / L) * u[None, :] / 2.0
        inp.latent[b] = rows.to(inp.latent.dtype)
    out, lse = H.run_decode(inp, "gqa", num_splits=splits)
    H.check_units(inp, out, lse, H.all_units(inp), "gqa wide growing G=%d s_q=%d S=%d" % (G, s_q, splits))


@pytest.mark.parametrize("G,s_q", [(1, 2), (8, 1)])
def test_negative_and_tiny_scales(G, s_q):
    """The softmax scale is any finite number: a negative one flips which
    score is largest (the tcgen05 GQA kernel scales the extreme raw score),
    and a tiny one gives near-uniform weights."""
    for scale in (-0.09, 1e-4):
        d = synth.Dims(n_h=128, G=G, d_nope=128, d_rope=64, d_v=128, r=512, s_q=s_q, scale=scale)
        inp = _wl(d, 2, [700, 131], page=64, seed=77)
        for path in ("absorb", "gqa"):
            out, lse = H.run_decode(inp, path)
            H.check_units(inp, out, lse, H.sample_units(inp, 4, seed=G), "scale %g %s G=%d" % (scale, path, G))

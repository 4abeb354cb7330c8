"""Pins for the fp64 oracle: checks against what the pages and the mathematics
fix, independent of the oracle's own code (brute force in 40-digit decimal
arithmetic, torch's float64 scaled_dot_product_attention, closed forms, and
the figures the pages print).  A final group plants plausible mistakes in the
oracle and checks that a pin catches each of them."""
import json
import math
import os
from decimal import Decimal, localcontext

import numpy as np
import pytest
import torch

from oracle import gqla_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


def _rand_problem(seed, B=1, s_q=1, n_h=4, G=2, d_n=3, d_r=2, d_v=3, r=5, L=6):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, s_q, n_h, d_n + d_r))
    c = rng.standard_normal((B, L, r))
    kr = rng.standard_normal((B, L, d_r))
    W_uk = rng.standard_normal((G, r, d_n)) / math.sqrt(r)
    W_uv = rng.standard_normal((G, r, d_v)) / math.sqrt(r)
    return q, c, kr, W_uk, W_uv


def _brute_force(q_b, c, kr, W_uk, W_uv, L, scale):
    """Definition written out in 40-digit decimals: no max-subtraction, no
    matrix routines, keys and values built element by element."""
    s_q, n_h, D = q_b.shape
    G, r, d_n = W_uk.shape
    d_v = W_uv.shape[2]
    m = n_h // G
    out = np.zeros((s_q, n_h, d_v))
    lse = np.zeros((s_q, n_h))
    with localcontext() as ctx:
        ctx.prec = 40
        dsc = Decimal(float(scale))
        for i in range(s_q):
            for h in range(n_h):
                g = h // m
                last = L - s_q + i          # newest token query i may see
                ws, vs = [], []
                for t in range(last + 1):
                    key = []
                    for a in range(d_n):
                        key.append(sum(Decimal(float(c[t, j])) * Decimal(float(W_uk[g, j, a]))
                                       for j in range(r)))
                    for a in range(kr.shape[1]):
                        key.append(Decimal(float(kr[t, a])))
                    val = [sum(Decimal(float(c[t, j])) * Decimal(float(W_uv[g, j, a])) for j in range(r))
                           for a in range(d_v)]
                    sc = dsc * sum(Decimal(float(q_b[i, h, a])) * key[a] for a in range(D))
                    ws.append(sc.exp())
                    vs.append(val)
                Z = sum(ws)
                for a in range(d_v):
                    out[i, h, a] = float(sum(w * v[a] for w, v in zip(ws, vs)) / Z)
                lse[i, h] = float(Z.ln())
    return out, lse


@pytest.mark.parametrize("s_q,L", [(1, 1), (1, 6), (2, 2), (2, 5), (3, 7)])
@pytest.mark.parametrize("form", ["gqa", "absorb"])
def test_brute_force_tiny(s_q, L, form):
    q, c, kr, W_uk, W_uv = _rand_problem(11 * s_q + L, s_q=s_q, L=L)
    scale = 0.37
    fn = O.decode_sequence_gqa if form == "gqa" else O.decode_sequence_absorb
    o, l = fn(q[0], c[0], kr[0], W_uk, W_uv, L, scale)
    bo, bl = _brute_force(q[0], c[0], kr[0], W_uk, W_uv, L, scale)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, bl, rtol=1e-12, atol=1e-13)


def _sdpa_gqa(q_b, c, kr, W_uk, W_uv, L, scale):
    """torch float64 SDPA with enable_gqa and an explicit bottom-right causal
    mask; the per-group keys are built with torch matmuls."""
    s_q, n_h, D = q_b.shape
    G = W_uk.shape[0]
    C = torch.tensor(c[:L])
    K = torch.stack([torch.cat([C @ torch.tensor(W_uk[g]), torch.tensor(kr[:L])], dim=1) for g in range(G)])
    V = torch.stack([C @ torch.tensor(W_uv[g]) for g in range(G)])
    Q = torch.tensor(q_b).permute(1, 0, 2).unsqueeze(0)          # [1, n_h, s_q, D]
    mask = torch.zeros((s_q, L), dtype=torch.bool)
    for i in range(s_q):
        mask[i, : L - s_q + i + 1] = True
    out = torch.nn.functional.scaled_dot_product_attention(
        Q, K.unsqueeze(0), V.unsqueeze(0), attn_mask=mask, scale=scale, enable_gqa=True)
    return out[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("n_h,G,s_q,L", [(8, 2, 1, 40), (8, 8, 2, 33), (8, 1, 3, 17), (12, 3, 4, 64)])
def test_library_sdpa_crosscheck(n_h, G, s_q, L):
    q, c, kr, W_uk, W_uv = _rand_problem(5 + L, s_q=s_q, n_h=n_h, G=G, d_n=16, d_r=8, d_v=12, r=24, L=L)
    scale = 1 / math.sqrt(24)
    o, _ = O.decode_sequence_gqa(q[0], c[0], kr[0], W_uk, W_uv, L, scale)
    ref = _sdpa_gqa(q[0], c[0], kr[0], W_uk, W_uv, L, scale)
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("n_h,G,s_q,L", [(8, 2, 1, 50), (16, 4, 2, 70), (8, 1, 4, 33), (8, 8, 1, 9)])
def test_absorb_equals_expanded(n_h, G, s_q, L):
    """The two paths are algebraically equivalent over the same weights
    (GQLA, chatpaper.ai and scholarbro.com abstracts)."""
    q, c, kr, W_uk, W_uv = _rand_problem(100 + L, s_q=s_q, n_h=n_h, G=G, d_n=16, d_r=8, d_v=16, r=32, L=L)
    a = O.decode_sequence_absorb(q[0], c[0], kr[0], W_uk, W_uv, L, 0.2)
    e = O.decode_sequence_gqa(q[0], c[0], kr[0], W_uk, W_uv, L, 0.2)
    np.testing.assert_allclose(a[0], e[0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(a[1], e[1], rtol=1e-12, atol=1e-14)


def test_grouping_limits_mha_mqa():
    """G = n_h is MHA (each head its own projections) and G = 1 is MQA (one
    shared K/V) -- Grouped Query Attention glossary, 'Fonctionnement de la GQA'."""
    n_h, L, s_q = 6, 20, 2
    q, c, kr, W_uk, W_uv = _rand_problem(7, s_q=s_q, n_h=n_h, G=n_h, d_n=8, d_r=4, d_v=8, r=10, L=L)
    Kh = np.stack([np.concatenate([c[0] @ W_uk[h], kr[0]], 1) for h in range(n_h)])
    Vh = np.stack([c[0] @ W_uv[h] for h in range(n_h)])
    ref = O.mha_decode(q[0], Kh, Vh, L, 0.3)
    got = O.decode_sequence_gqa(q[0], c[0], kr[0], W_uk, W_uv, L, 0.3)
    np.testing.assert_allclose(got[0], ref[0], rtol=1e-13, atol=1e-14)
    # MQA: one group, every head uses the same K/V
    W1k, W1v = W_uk[:1], W_uv[:1]
    K1 = np.concatenate([c[0] @ W1k[0], kr[0]], 1)
    V1 = c[0] @ W1v[0]
    ref = O.mha_decode(q[0], np.stack([K1] * n_h), np.stack([V1] * n_h), L, 0.3)
    got = O.decode_sequence_gqa(q[0], c[0], kr[0], W1k, W1v, L, 0.3)
    np.testing.assert_allclose(got[0], ref[0], rtol=1e-13, atol=1e-14)


def test_gqa_equals_repeated_heads_example():
    """The glossary's enable_gqa example: 8 query heads, 2 KV heads, 16 tokens,
    head dim 64; output shape (1, 8, 16, 64) and equal (atol 1e-6) to MHA with
    each KV head copied to its 4 query heads; 256 vs 1024 cached values."""
    gold = json.load(open(GOLDEN))["sdpa_gqa_example"]
    rng = np.random.default_rng(0)
    n_h, G, T, D = gold["n_q_heads"], gold["n_kv_heads"], gold["tokens"], gold["head_dim"]
    q = rng.standard_normal((T, n_h, D))
    k = rng.standard_normal((G, T, D))
    v = rng.standard_normal((G, T, D))
    # all T tokens are new (s_q = L = T), which reproduces the example's causal
    # mask; the grouped form maps head h to KV head h // m
    m = n_h // G
    grouped = O.mha_decode(q, np.stack([k[h // m] for h in range(n_h)]),
                           np.stack([v[h // m] for h in range(n_h)]), T, 1 / math.sqrt(D))[0]
    k_full = np.repeat(k, m, axis=0)
    v_full = np.repeat(v, m, axis=0)
    rep = O.mha_decode(q, k_full, v_full, T, 1 / math.sqrt(D))[0]
    out = grouped.transpose(1, 0, 2)[None]
    assert list(out.shape) == gold["output_shape"]
    assert np.allclose(grouped, rep, atol=gold["atol"]) == gold["same_as_copied_heads"]
    assert O.cache_elems_per_token("gqa_baseline", n_kv_heads=G, head_dim=D) == gold["cached_values_per_token_gqa"]
    assert O.cache_elems_per_token("gqa_baseline", n_kv_heads=n_h, head_dim=D) == gold["cached_values_per_token_mha"]
    # and against torch's own enable_gqa on the same tensors (library cross-check)
    t = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q).permute(1, 0, 2)[None], torch.tensor(k)[None], torch.tensor(v)[None],
        is_causal=True, enable_gqa=True)
    np.testing.assert_allclose(out, t.numpy(), rtol=1e-12, atol=1e-12)


def test_cache_size_figures():
    gold = json.load(open(GOLDEN))
    a = gold["absorb_cache_fraction_llama3_8b"]
    frac = O.cache_elems_per_token("absorb", r=a["r"], d_r=a["d_rope"]) / \
        O.cache_elems_per_token("gqa_baseline", n_kv_heads=a["n_kv_heads"], head_dim=a["head_dim"])
    assert frac == a["value"]
    l = gold["llama31_8b_cache"]
    e_gqa = O.cache_elems_per_token("gqa_baseline", n_kv_heads=l["n_kv_heads"], head_dim=l["head_dim"])
    per_tok = O.cache_bytes_per_token(e_gqa, l["n_layers"], l["bytes_per_elem"])
    assert per_tok == l["kib_per_token_gqa"] * 1024
    assert per_tok * l["window_tokens"] == l["gib_at_full_window_gqa"] * 2 ** 30
    e_mha = O.cache_elems_per_token("gqa_baseline", n_kv_heads=l["n_q_heads"], head_dim=l["head_dim"])
    per_tok_mha = O.cache_bytes_per_token(e_mha, l["n_layers"], l["bytes_per_elem"])
    assert per_tok_mha == l["kib_per_token_mha"] * 1024
    assert per_tok_mha * l["window_tokens"] == l["gib_at_full_window_mha"] * 2 ** 30


def test_softmax_closed_forms():
    q, c, kr, W_uk, W_uv = _rand_problem(3, s_q=1, L=9)
    # L = 1: the only key gets weight 1, lse is its score
    o, l = O.decode_sequence_gqa(q[0], c[0], kr[0], W_uk, W_uv, 1, 0.5)
    for h in range(q.shape[2]):
        g = h // (q.shape[2] // W_uk.shape[0])
        K, V = c[0][:1] @ W_uk[g], c[0][:1] @ W_uv[g]
        s0 = 0.5 * (q[0, 0, h, :3] @ K[0] + q[0, 0, h, 3:] @ kr[0][0])
        np.testing.assert_allclose(o[0, h], V[0], rtol=1e-14)
        np.testing.assert_allclose(l[0, h], s0, rtol=1e-13)
    # identical keys: uniform weights, o = mean of the values, lse = s + ln n
    c_same = np.repeat(c[0][:1], 9, axis=0)
    kr_same = np.repeat(kr[0][:1], 9, axis=0)
    o, l = O.decode_sequence_gqa(q[0], c_same, kr_same, W_uk, W_uv, 9, 0.5)
    o1, l1 = O.decode_sequence_gqa(q[0], c_same, kr_same, W_uk, W_uv, 1, 0.5)
    np.testing.assert_allclose(o, o1, rtol=1e-13)
    np.testing.assert_allclose(l, l1 + math.log(9), rtol=1e-13)
    # weights sum to one: with all values equal to a constant vector, o equals it
    W_uv_c = np.zeros_like(W_uv)
    o, _ = O.decode_sequence_gqa(q[0], c[0], kr[0], W_uk, W_uv_c, 9, 0.5)
    np.testing.assert_allclose(o, 0.0, atol=1e-15)


def test_causality_multi_token():
    """Query i sees tokens 0..L-s_q+i: changing the newest token moves only the
    last query's output."""
    q, c, kr, W_uk, W_uv = _rand_problem(9, s_q=2, L=12)
    o, _ = O.decode_sequence_gqa(q[0], c[0], kr[0], W_uk, W_uv, 12, 0.4)
    c2 = c[0].copy()
    c2[11] += 1.0
    o2, _ = O.decode_sequence_gqa(q[0], c2, kr[0], W_uk, W_uv, 12, 0.4)
    np.testing.assert_array_equal(o[0], o2[0])
    assert np.abs(o[1] - o2[1]).max() > 1e-6


def test_splitkv_combine_identity():
    """Attention over a union of disjoint key ranges equals the LSE merge of the
    per-range results; ranges with no key carry lse = -inf and weight 0."""
    rng = np.random.default_rng(4)
    L, D, R = 37, 6, 5
    K = rng.standard_normal((R, L, 4))
    V = rng.standard_normal((R, L, D))
    qv = rng.standard_normal((R, 4))
    cuts = [0, 0, 10, 11, 30, 37, 37]     # includes empty ranges
    S = len(cuts) - 1
    o_part = np.zeros((S, R, D))
    lse_part = np.full((S, R), -np.inf)
    for s in range(S):
        a, b = cuts[s], cuts[s + 1]
        for row in range(R):
            if b > a:
                o_part[s, row], lse_part[s, row] = O.attend(qv[row], K[row, a:b], V[row, a:b], b - a, 0.7)
    o, lse = O.splitkv_combine(o_part, lse_part)
    for row in range(R):
        ro, rl = O.attend(qv[row], K[row], V[row], L, 0.7)
        np.testing.assert_allclose(o[row], ro, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse[row], rl, rtol=1e-13)
    o, lse = O.splitkv_combine(np.zeros((2, 1, 3)), np.full((2, 1), -np.inf))
    assert np.all(o == 0) and np.isneginf(lse[0])


def test_divisibility_error():
    q, c, kr, W_uk, W_uv = _rand_problem(1, n_h=6, G=4)
    with pytest.raises(ValueError):
        O.decode_sequence_gqa(q[0], c[0], kr[0], W_uk, W_uv, 6, 0.3)
    with pytest.raises(ValueError):
        O.visible_keys(1, 2, 0)


# --- planted mistakes: each must be caught by one of the pins above --------

def _mutant_results(monkeypatch, name, fn):
    monkeypatch.setattr(O, name, fn)
    q, c, kr, W_uk, W_uv = _rand_problem(21, s_q=2, L=5)
    o, l = O.decode_sequence_gqa(q[0], c[0], kr[0], W_uk, W_uv, 5, 0.37)
    bo, bl = _brute_force(q[0], c[0], kr[0], W_uk, W_uv, 5, 0.37)
    return np.allclose(o, bo, rtol=1e-12, atol=1e-13) and np.allclose(l, bl, rtol=1e-12, atol=1e-13)


def test_planted_mistakes_are_caught(monkeypatch):
    orig_expand, orig_vis, orig_attend = O.expand_group, O.visible_keys, O.attend

    def no_rope(c, k_rope, W_uk_g, W_uv_g):
        K, V = orig_expand(c, k_rope, W_uk_g, W_uv_g)
        K[:, W_uk_g.shape[1]:] = 0.0
        return K, V
    assert not _mutant_results(monkeypatch, "expand_group", no_rope)
    monkeypatch.setattr(O, "expand_group", orig_expand)

    assert not _mutant_results(monkeypatch, "visible_keys", lambda L, s_q, i: orig_vis(L, s_q, i) - 1 or 1)
    monkeypatch.setattr(O, "visible_keys", orig_vis)

    def lse_no_scale(q_vec, K, V, n, scale):
        o, l = orig_attend(q_vec, K, V, n, scale)
        return o, l / scale
    assert not _mutant_results(monkeypatch, "attend", lse_no_scale)
    monkeypatch.setattr(O, "attend", orig_attend)

    def swapped_uv(c, k_rope, W_uk_g, W_uv_g):
        return orig_expand(c, k_rope, W_uk_g, W_uv_g * -1.0)
    assert not _mutant_results(monkeypatch, "expand_group", swapped_uv)
    monkeypatch.setattr(O, "expand_group", orig_expand)
    assert _mutant_results(monkeypatch, "attend", orig_attend)   # the unmutated oracle passes


def test_planted_group_map_mistake_caught_by_sdpa():
    """A head-to-group map of h % G instead of h // m is caught by the library
    cross-check (enable_gqa copies KV head g to heads g*m .. g*m+m-1)."""
    n_h, G, L = 8, 2, 10
    q, c, kr, W_uk, W_uv = _rand_problem(2, n_h=n_h, G=G, d_n=4, d_r=2, d_v=4, r=6, L=L)
    m = n_h // G
    Kh = np.stack([np.concatenate([c[0] @ W_uk[h % G], kr[0]], 1) for h in range(n_h)])
    Vh = np.stack([c[0] @ W_uv[h % G] for h in range(n_h)])
    wrong = O.mha_decode(q[0], Kh, Vh, L, 0.3)[0]
    ref = _sdpa_gqa(q[0], c[0], kr[0], W_uk, W_uv, L, 0.3)
    assert not np.allclose(wrong, ref, atol=1e-6)
    right = O.decode_sequence_gqa(q[0], c[0], kr[0], W_uk, W_uv, L, 0.3)[0]
    np.testing.assert_allclose(right, ref, rtol=1e-11, atol=1e-12)
    assert m == 4


# --- the batch driver -------------------------------------------------------

def _ragged_batch(seed, lens, s_q=2):
    """Three sequences of different lengths, each with its own rows; the
    logical rows past a sequence's length are never read."""
    rng = np.random.default_rng(seed)
    n_h, G, d_n, d_r, d_v, r = 4, 2, 3, 2, 3, 5
    q = rng.standard_normal((len(lens), s_q, n_h, d_n + d_r))
    c_list = [rng.standard_normal((L + 3, r)) for L in lens]
    kr_list = [rng.standard_normal((L + 3, d_r)) for L in lens]
    W_uk = rng.standard_normal((G, r, d_n)) / math.sqrt(r)
    W_uv = rng.standard_normal((G, r, d_v)) / math.sqrt(r)
    return q, c_list, kr_list, W_uk, W_uv


@pytest.mark.parametrize("form", ["gqa", "absorb"])
def test_decode_batch_ragged_brute_force(form):
    """decode_batch over a ragged batch (lengths 2, 7, 4; s_q 2) equals the
    definition written out for every sequence with its own length and rows."""
    lens = [2, 7, 4]
    q, c_list, kr_list, W_uk, W_uv = _ragged_batch(31, lens)
    o, l = O.decode_batch(q, c_list, kr_list, W_uk, W_uv, np.array(lens), 0.41, form=form)
    assert o.shape == (3, 2, 4, 3) and l.shape == (3, 2, 4)
    for b, L in enumerate(lens):
        bo, bl = _brute_force(q[b], c_list[b], kr_list[b], W_uk, W_uv, L, 0.41)
        np.testing.assert_allclose(o[b], bo, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(l[b], bl, rtol=1e-12, atol=1e-13)


def test_decode_batch_planted_mistakes_caught(monkeypatch):
    """A batch driver that decodes every sequence with the first one's length,
    or reads the next sequence's rows, fails the brute-force pin above."""
    lens = [2, 7, 4]
    q, c_list, kr_list, W_uk, W_uv = _ragged_batch(31, lens)

    def pinned(res):
        o, l = res
        for b, L in enumerate(lens):
            bo, bl = _brute_force(q[b], c_list[b], kr_list[b], W_uk, W_uv, L, 0.41)
            if not (np.allclose(o[b], bo, rtol=1e-12, atol=1e-13) and np.allclose(l[b], bl, rtol=1e-12, atol=1e-13)):
                return False
        return True

    assert pinned(O.decode_batch(q, c_list, kr_list, W_uk, W_uv, np.array(lens), 0.41))
    first_len = np.array([lens[0]] * 3)
    assert not pinned(O.decode_batch(q, c_list, kr_list, W_uk, W_uv, first_len, 0.41))
    shifted = c_list[1:] + c_list[:1]
    shifted_kr = kr_list[1:] + kr_list[:1]
    # rows of sequence b + 1 with the right lengths (trimmed to fit the shorter buffers)
    rows = [np.resize(shifted[b], c_list[b].shape) for b in range(3)]
    rows_kr = [np.resize(shifted_kr[b], kr_list[b].shape) for b in range(3)]
    assert not pinned(O.decode_batch(q, rows, rows_kr, W_uk, W_uv, np.array(lens), 0.41))

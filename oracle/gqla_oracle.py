"""fp64 CPU oracle for GQLA decode attention.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import or run this module.
The product path (the CUDA library and its Python binding) never calls it and
shares no code with it.

What it computes, and where the pages define it
-----------------------------------------------
Sources (web pages on Group-Query Latent Attention):

* [GQLA-chatpaper] "GQLA: Group-Query Latent Attention ..." (chatpaper.ai),
  Abstract (English): the trained weights expose two algebraically equivalent
  decoding paths over the same parameters -- an MQA-absorb path identical to
  MLA's, and a GQA path with a per-group expanded cache; per-token cache of the
  absorb path is (512+64)/(2*8*128) = 28.125 % of the GQA baseline at
  LLaMA-3-8B shapes.
* [GQLA-scholarbro] "GQLA: Group-Query Latent Attention for Hardware-Adaptive
  Decoding" (scholarbro.com), Abstract: the up-projections are group-shared and
  preserve a joint latent; the same weights run as MQA-absorb or as GQA.
* [GQA-glossary] "Grouped Query Attention (GQA)" (ultralytics.com glossary),
  sections "Fonctionnement de la GQA" (grouped heads = MHA with each KV head
  copied to its group; one group = MQA, one group per head = MHA) and
  "Pourquoi la GQA reduit le cache KV" (cache sizes).
* [gqla_attn] "gqla_attn" module page (frankenstein-transformer docs),
  GQLAAttention docstring: knob names (decode_path, num_groups), the
  divisibility rule, causal masking in decoder mode.

Readings taken where the pages are silent:
head h belongs to group g = h // m with m = n_h / G; the key of token t for
group g is [c_t W_uk^g ; k_rope_t] (the decoupled RoPE key is shared by all
heads and already rotated); the value is c_t W_uv^g; the cache of length L
already holds the s_q new tokens and query i sees tokens 0 .. L - s_q + i;
scores are scale * <q, k>; lse is the natural log of the softmax normaliser
with the scale included.

Every function works on fp64 copies of the (already rounded) inputs. Matrix
products use numpy's matmul as the library primitive; there is no blocking,
no online softmax and no split of the key range.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "expand_group",
    "visible_keys",
    "attend",
    "decode_sequence_gqa",
    "decode_sequence_absorb",
    "decode_batch",
    "absorb_query",
    "mha_decode",
    "splitkv_combine",
    "cache_elems_per_token",
    "cache_bytes_per_token",
]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def expand_group(c, k_rope, W_uk_g, W_uv_g):
    """Per-group expanded cache of one sequence.

    [GQLA-chatpaper] Abstract ("GQA path with a per-group expanded cache") and
    [GQLA-scholarbro] Abstract ("group-shared up-projections preserve a joint
    latent"): the keys of group g are the latent lifted by the group's W_uk^g,
    with the shared decoupled RoPE key appended; the values are the latent
    lifted by W_uv^g.

    c: [L, r]; k_rope: [L, d_r]; W_uk_g: [r, d_nope]; W_uv_g: [r, d_v].
    Returns K_g [L, d_nope + d_r] and V_g [L, d_v].
    """
    c = _f64(c)
    K_nope = c @ _f64(W_uk_g)
    K = np.concatenate([K_nope, _f64(k_rope)], axis=1)
    V = c @ _f64(W_uv_g)
    return K, V


def visible_keys(L, s_q, i):
    """Number of cache tokens query i (0-based among the s_q new tokens) sees.

    The cache of length L already contains the s_q new tokens; query i is the
    token at position L - s_q + i and attends causally (decoder-mode causal
    mask of [gqla_attn] GQLAAttention.forward, bottom-right aligned).
    """
    n = L - s_q + i + 1
    if n < 1:
        raise ValueError("sequence length %d is shorter than s_q=%d" % (L, s_q))
    return n


def attend(q_vec, K, V, n_keys, scale):
    """Scaled dot-product attention of one query vector over the first n_keys.

    Plain definition: s_t = scale * <q, k_t>; p = softmax(s); o = sum_t p_t v_t;
    lse = max(s) + ln sum_t exp(s_t - max(s)).
    """
    s = scale * (_f64(K)[:n_keys] @ _f64(q_vec))
    mx = s.max()
    w = np.exp(s - mx)
    Z = w.sum()
    o = (w / Z) @ _f64(V)[:n_keys]
    return o, mx + np.log(Z)


def decode_sequence_gqa(q_b, c, k_rope, W_uk, W_uv, L, scale, groups=None):
    """Fully expanded per-head decode of one sequence (the GQA form).

    q_b: [s_q, n_h, d_nope + d_r] (nope part first); c: [>=L, r];
    k_rope: [>=L, d_r]; W_uk: [G, r, d_nope]; W_uv: [G, r, d_v].
    groups: optional iterable of group ids to compute (others are left NaN),
    used to check sampled (sequence, group) units at full context.
    Returns out [s_q, n_h, d_v] and lse [s_q, n_h].
    """
    q_b = _f64(q_b)
    s_q, n_h, _ = q_b.shape
    G = W_uk.shape[0]
    if n_h % G != 0:
        raise ValueError("number of groups must divide the number of heads")
    m = n_h // G
    d_v = W_uv.shape[2]
    out = np.full((s_q, n_h, d_v), np.nan)
    lse = np.full((s_q, n_h), np.nan)
    for g in (range(G) if groups is None else groups):
        K, V = expand_group(c[:L], k_rope[:L], W_uk[g], W_uv[g])
        for i in range(s_q):
            n = visible_keys(L, s_q, i)
            for h in range(g * m, (g + 1) * m):
                out[i, h], lse[i, h] = attend(q_b[i, h], K, V, n, scale)
    return out, lse


def absorb_query(q_nope_h, W_uk_g):
    """q~ = W_uk^g q_nope, the query carried into the latent space.

    [GQLA-chatpaper] Abstract ("absorbed MQA form"): <q_nope, c W_uk^g> equals
    <W_uk^g q_nope, c>, so the up-projection moves onto the query.
    """
    return _f64(W_uk_g) @ _f64(q_nope_h)


def decode_sequence_absorb(q_b, c, k_rope, W_uk, W_uv, L, scale, groups=None):
    """MQA-absorb form of the same decode (used to pin the equivalence).

    Every head attends over the shared cache rows [c_t ; k_rope_t] with the
    absorbed query [q~ ; q_rope]; its latent output sum_t p_t c_t is lifted by
    the group's W_uv^g.  [GQLA-chatpaper] and [GQLA-scholarbro] Abstracts.
    """
    q_b = _f64(q_b)
    s_q, n_h, D = q_b.shape
    G, r, d_n = W_uk.shape
    m = n_h // G
    C = _f64(c)[:L]
    KR = _f64(k_rope)[:L]
    keys = np.concatenate([C, KR], axis=1)          # [L, r + d_r]
    d_v = W_uv.shape[2]
    out = np.full((s_q, n_h, d_v), np.nan)
    lse = np.full((s_q, n_h), np.nan)
    for g in (range(G) if groups is None else groups):
        for i in range(s_q):
            n = visible_keys(L, s_q, i)
            for h in range(g * m, (g + 1) * m):
                qt = absorb_query(q_b[i, h, :d_n], W_uk[g])
                qa = np.concatenate([qt, q_b[i, h, d_n:]])
                o_lat, lse[i, h] = attend(qa, keys, C, n, scale)
                out[i, h] = o_lat @ _f64(W_uv[g])
    return out, lse


def decode_batch(q, c_list, k_rope_list, W_uk, W_uv, seq_lens, scale, form="gqa"):
    """Decode a whole batch: out [B, s_q, n_h, d_v], lse [B, s_q, n_h].

    c_list[b] / k_rope_list[b] hold sequence b's logical token rows.
    """
    fn = decode_sequence_gqa if form == "gqa" else decode_sequence_absorb
    outs, lses = [], []
    for b in range(q.shape[0]):
        o, l = fn(q[b], c_list[b], k_rope_list[b], W_uk, W_uv, int(seq_lens[b]), scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def mha_decode(q_b, K_heads, V_heads, L, scale):
    """Multi-head decode where every query head h has its own K_heads[h], V_heads[h].

    Independent of the grouping code above: used for the [GQA-glossary]
    statement that grouped-query attention equals MHA with each KV head copied
    to the query heads of its group (and that G = n_h is MHA, G = 1 is MQA).
    """
    q_b = _f64(q_b)
    s_q, n_h, _ = q_b.shape
    d_v = V_heads.shape[2]
    out = np.empty((s_q, n_h, d_v))
    lse = np.empty((s_q, n_h))
    for i in range(s_q):
        n = visible_keys(L, s_q, i)
        for h in range(n_h):
            out[i, h], lse[i, h] = attend(q_b[i, h], K_heads[h], V_heads[h], n, scale)
    return out, lse


def splitkv_combine(o_part, lse_part):
    """Merge attention results computed over disjoint key ranges.

    o_part: [S, rows, D] (each normalised over its own range), lse_part:
    [S, rows]. Ranges with no key carry lse = -inf and weight 0.
    lse = ln sum_j exp(lse_j); o = sum_j exp(lse_j - lse) o_j.
    This is the identity softmax over a union of key sets obeys; the pages
    name FlashAttention-style kernels ([GQA-glossary], "GQA et techniques
    connexes") but print no combine rule.
    """
    o_part = _f64(o_part)
    lse_part = _f64(lse_part)
    mx = lse_part.max(axis=0)
    finite = np.isfinite(mx)
    safe = np.where(finite, mx, 0.0)
    w = np.exp(lse_part - safe[None, :])          # exp(-inf) = 0
    Z = w.sum(axis=0)
    lse = np.where(finite, safe + np.log(np.where(finite, Z, 1.0)), -np.inf)
    wn = np.where(finite[None, :], w / np.where(finite, Z, 1.0)[None, :], 0.0)
    o = np.einsum("sr,srd->rd", wn, o_part)
    return o, lse


def cache_elems_per_token(path, n_kv_heads=None, head_dim=None, r=None, d_r=None,
                          G=None, d_nope=None, d_v=None):
    """Cached elements per token per layer.

    path "gqa_baseline": K and V of n_kv_heads heads of head_dim each
    ([GQA-glossary] "Pourquoi la GQA reduit le cache KV").
    path "absorb": the joint latent plus the shared RoPE key, r + d_r
    ([GQLA-chatpaper] Abstract, 28.125 %).
    path "gqla_expanded": G groups of K (d_nope + d_r) and V (d_v).
    """
    if path == "gqa_baseline":
        return 2 * n_kv_heads * head_dim
    if path == "absorb":
        return r + d_r
    if path == "gqla_expanded":
        return G * (d_nope + d_r + d_v)
    raise ValueError(path)


def cache_bytes_per_token(elems_per_layer, n_layers, bytes_per_elem):
    """Bytes per token over all layers (16-bit values: 2 bytes each)."""
    return elems_per_layer * n_layers * bytes_per_elem

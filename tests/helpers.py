"""Test plumbing: run the CUDA path through the C-ABI binding and the fp64
oracle on the same seeded inputs, and compare with the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

from latent_kv_cache_flash_b200 import synth
from oracle import gqla_oracle as O

# Tolerances (stated for the kernels): fp32 max|err| <= 1e-5 * max|ref|;
# bf16 inputs with fp32 accumulation max|err| <= 1e-2 * max|ref| + 1e-3.
# The same rule is applied to the log-sum-exp output as a tensor of its own.


def tol(dtype: str, ref: np.ndarray) -> float:
    mx = float(np.max(np.abs(ref))) if ref.size else 0.0
    return 1e-5 * mx if dtype == "f32" else 1e-2 * mx + 1e-3


# Diagnostics of every decode comparison (what, max|err|, tol, rel-RMS error,
# max|ref|), printed at the end of the run beside the gates: at long contexts
# the softmax is nearly flat, |out| is small and the +1e-3 term of the bf16
# rule is a large share of it, so the relative RMS error and the absolute
# log-sum-exp error (lse grows like ln L) are the sharper readings.
DIAG = []

# Sharper gates at long context (bf16, every sampled sequence >= 8192 tokens).
# The lse is compared in absolute terms: it grows like ln L while its error
# shrinks as the per-score rounding errors (q~ or the expanded K rounded to
# bf16, about 2^-9 relative per product, independent across tokens) average
# out over the softmax weights; measured at most 3.2e-4 at 8K-64K on B200, so
# 2e-3 keeps a margin of six and is 55 times tighter than the output rule
# gives it at L = 64K (1e-2 * 11.7 + 1e-3).  The output's relative RMS error
# is bounded by the few bf16 roundings on the way (P, the merged latent
# output, the expanded cache: each about 2^-9 / sqrt(3) = 1.1e-3 relative RMS),
# measured at most 3.0e-3; the gate is 1e-2.
LONG_CONTEXT = 8192
LSE_ABS_TOL_LONG = 2e-3
OUT_REL_RMS_TOL_LONG = 1e-2


def rel_rms(got, ref):
    den = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    return float(np.sqrt(np.mean((got - ref) ** 2))) / den if den > 0 else 0.0


def assert_close(got, ref, dtype, what="", record=False):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), "%s: non-finite pattern differs" % what
    err = float(np.max(np.abs(got[fin] - ref[fin]))) if fin.any() else 0.0
    t = tol(dtype, ref[fin])
    if record:
        DIAG.append((what, err, t, rel_rms(got[fin], ref[fin]), float(np.max(np.abs(ref[fin]))) if fin.any() else 0.0))
    assert err <= t, "%s: max|err| %.3e > tol %.3e (max|ref| %.3e)" % (what, err, t, np.max(np.abs(ref[fin])))
    return err


def layout_of(inp: synth.Inputs, max_seq_len=None):
    from latent_kv_cache_flash_b200 import gqla
    return gqla.make_layout(inp.seq_lens, max_seq_len or inp.max_seq_len, inp.wl.page_size,
                            inp.capacity if inp.wl.page_size == 0 else 0, inp.block_table, inp.num_pages)


def run_expand(inp: synth.Inputs, tail=0, dev_status=None, pools=None):
    from latent_kv_cache_flash_b200 import gqla
    d = inp.dims
    ks, vs = synth.expanded_pool_shapes(inp)
    if pools is None:
        kp = torch.zeros(ks, dtype=d.torch_dtype, device=inp.latent.device)
        vp = torch.zeros(vs, dtype=d.torch_dtype, device=inp.latent.device)
    else:
        kp, vp = pools
    gqla.gqla_expand_cache(gqla.make_dims(d), layout_of(inp), inp.latent, inp.W_uk, inp.W_uv, kp, vp,
                           tail_tokens=tail, dev_status=dev_status)
    return kp, vp


def run_decode(inp: synth.Inputs, path: str, num_splits=0, pools=None, dev_status=None, max_seq_len=None):
    """Returns (out, lse) torch tensors on the inputs' device."""
    from latent_kv_cache_flash_b200 import gqla
    d = inp.dims
    B = inp.wl.batch
    out = torch.empty((B, d.s_q, d.n_h, d.d_v), dtype=d.torch_dtype, device=inp.q.device)
    lse = torch.empty((B, d.s_q, d.n_h), dtype=torch.float32, device=inp.q.device)
    dims = gqla.make_dims(d)
    lay = layout_of(inp, max_seq_len)
    if path == "absorb":
        gqla.gqla_decode_absorb(dims, lay, inp.q, inp.latent, inp.W_uk, inp.W_uv, out, lse, num_splits,
                                dev_status=dev_status)
    else:
        kp, vp = pools if pools is not None else run_expand(inp)
        gqla.gqla_decode_gqa(dims, lay, inp.q, kp, vp, out, lse, num_splits, dev_status=dev_status)
    return out, lse


def oracle_units(inp: synth.Inputs, units, form="gqa"):
    """Oracle outputs for (sequence, group) units: dict b -> (out, lse) with only
    the requested groups filled (others NaN)."""
    d = inp.dims
    by_b = {}
    for b, g in units:
        by_b.setdefault(b, []).append(g)
    res = {}
    W_uk = inp.W_uk.double().cpu().numpy()
    W_uv = inp.W_uv.double().cpu().numpy()
    for b, gs in by_b.items():
        rows = inp.logical_latent(b).double().cpu().numpy()
        c, kr = rows[:, : d.r], rows[:, d.r:]
        qb = inp.q[b].double().cpu().numpy()
        fn = O.decode_sequence_gqa if form == "gqa" else O.decode_sequence_absorb
        res[b] = fn(qb, c, kr, W_uk, W_uv, inp.seq_lens_host[b], d.softmax_scale, groups=gs)
    return res


def check_units(inp: synth.Inputs, out, lse, units, what=""):
    """Compares the GPU output of the sampled units with the oracle."""
    d = inp.dims
    ref = oracle_units(inp, units)
    got_o, got_l, ref_o, ref_l = [], [], [], []
    o_np = out.float().cpu().numpy()
    l_np = lse.float().cpu().numpy()
    for b, g in units:
        hs = slice(g * d.m, (g + 1) * d.m)
        got_o.append(o_np[b, :, hs])
        got_l.append(l_np[b, :, hs])
        ref_o.append(ref[b][0][:, hs])
        ref_l.append(ref[b][1][:, hs])
    go, ro, gl, rl = np.stack(got_o), np.stack(ref_o), np.stack(got_l), np.stack(ref_l)
    e1 = assert_close(go, ro, d.dtype, what + " out", record=True)
    e2 = assert_close(gl, rl, d.dtype, what + " lse", record=True)
    if d.dtype == "bf16" and min(inp.seq_lens_host[b] for b, _ in units) >= LONG_CONTEXT:
        fin = np.isfinite(rl)
        dl = float(np.max(np.abs(gl[fin].astype(np.float64) - rl[fin]))) if fin.any() else 0.0
        assert dl <= LSE_ABS_TOL_LONG, "%s: max|d lse| %.3e > %.1e at L >= %d" % (what, dl, LSE_ABS_TOL_LONG,
                                                                                 LONG_CONTEXT)
        rr = rel_rms(go.astype(np.float64)[np.isfinite(ro)], ro[np.isfinite(ro)])
        assert rr <= OUT_REL_RMS_TOL_LONG, "%s: out rel-RMS %.2e > %.1e at L >= %d" % (
            what, rr, OUT_REL_RMS_TOL_LONG, LONG_CONTEXT)
    return e1, e2


def all_units(inp: synth.Inputs):
    return [(b, g) for b in range(inp.wl.batch) for g in range(inp.dims.G)]


def sample_units(inp: synth.Inputs, n: int, seed: int = 1):
    rng = np.random.default_rng(seed)
    allu = all_units(inp)
    idx = rng.choice(len(allu), size=min(n, len(allu)), replace=False)
    return [allu[i] for i in sorted(idx)]

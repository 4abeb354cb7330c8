"""ctypes binding of libgqla.so (declared in include/gqla.h).

Argument marshalling only: every step of the decode path runs in the
library's CUDA kernels.  torch tensors supply device pointers, the current
CUDA stream and, when the caller passes none, the workspace buffer.  The
functions keep the C names; a non-OK status raises :class:`GqlaError`.
There is no fallback: if the library is missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgqla.so")

GQLA_OK, GQLA_ERR_INVALID_ARG, GQLA_ERR_UNSUPPORTED, GQLA_ERR_ALIGNMENT, GQLA_ERR_WORKSPACE, GQLA_ERR_CUDA = range(6)
GQLA_F32, GQLA_BF16 = 0, 1
GQLA_PATH_ABSORB, GQLA_PATH_GQA = 0, 1
GQLA_K_PER_GROUP, GQLA_K_SHARED_ROPE = 0, 1
DEV_SHORT_SEQ, DEV_OVERFLOW, DEV_BAD_PAGE, DEV_TIMEOUT = 1, 2, 4, 8


class GqlaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


class GqlaDims(ctypes.Structure):
    _fields_ = [("n_h", ctypes.c_int32), ("G", ctypes.c_int32), ("d_nope", ctypes.c_int32),
                ("d_rope", ctypes.c_int32), ("d_v", ctypes.c_int32), ("r", ctypes.c_int32),
                ("s_q", ctypes.c_int32), ("scale", ctypes.c_float), ("dtype", ctypes.c_int),
                ("k_layout", ctypes.c_int32)]


class GqlaKvLayout(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("seq_lens", ctypes.c_void_p), ("max_seq_len", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("capacity", ctypes.c_int32), ("block_table", ctypes.c_void_p),
                ("max_blocks_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32)]


class GqlaHw(ctypes.Structure):
    _fields_ = [("sms", ctypes.c_int32), ("hbm_gbs", ctypes.c_double), ("tc_tflops", ctypes.c_double)]


class GqlaPathEstimate(ctypes.Structure):
    _fields_ = [("absorb_us", ctypes.c_double), ("gqa_us", ctypes.c_double), ("path", ctypes.c_int)]


_lib = None


def lib():
    """Loads libgqla.so once; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError("libgqla.so not built: run python -m latent_kv_cache_flash_b200.build")
        L = ctypes.CDLL(_LIB_PATH)
        P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        pd, pl = ctypes.POINTER(GqlaDims), ctypes.POINTER(GqlaKvLayout)
        L.gqla_expand_cache.argtypes = [pd, pl, P, P, P, P, P, I32, P, P]
        L.gqla_decode_absorb.argtypes = [pd, pl, P, P, P, P, P, P, I32, P, SZ, P, P]
        L.gqla_decode_gqa.argtypes = [pd, pl, P, P, P, P, P, I32, P, SZ, P, P]
        L.gqla_decode_gqa_noalloc.argtypes = [pd, pl, P, P, P, P, P, I32, P, P]
        L.gqla_splitkv_combine.argtypes = [I32, I32, I32, P, P, P, ctypes.c_int, P, P]
        L.gqla_append_tokens.argtypes = [pd, pl, P, P, P, P, P, P, P, P]
        L.gqla_select_path.argtypes = [pd, pl, ctypes.c_int64, ctypes.POINTER(GqlaHw),
                                       ctypes.POINTER(GqlaPathEstimate)]
        L.gqla_workspace_bytes.argtypes = [pd, pl, I32, ctypes.c_int]
        L.gqla_workspace_bytes.restype = SZ
        L.gqla_num_splits.argtypes = [pd, pl, I32, ctypes.c_int]
        L.gqla_num_splits.restype = I32
        L.gqla_cache_bytes_per_token.argtypes = [pd, ctypes.c_int]
        L.gqla_cache_bytes_per_token.restype = SZ
        L.gqla_status_string.argtypes = [ctypes.c_int]
        L.gqla_status_string.restype = ctypes.c_char_p
        L.gqla_version.restype = ctypes.c_char_p
        L.gqla_launch_counter.restype = ctypes.c_uint64
        for name in ("gqla_expand_cache", "gqla_decode_absorb", "gqla_decode_gqa", "gqla_decode_gqa_noalloc",
                     "gqla_splitkv_combine", "gqla_append_tokens", "gqla_select_path"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is not None:
        return ctypes.c_void_p(stream)
    if device is not None and device.type == "cuda":
        return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    return None


def _check(status: int, what: str):
    if status != GQLA_OK:
        raise GqlaError(status, "%s: %s" % (what, gqla_status_string(status)))


def make_dims(d) -> GqlaDims:
    """Builds the C struct from any object with n_h, G, d_nope, d_rope, d_v, r,
    s_q, softmax_scale (or scale), dtype ("f32"/"bf16") and optionally
    k_shared_rope (the expanded K pool stores the RoPE key once per token)."""
    scale = getattr(d, "softmax_scale", None)
    if scale is None:
        scale = d.scale
    dt = GQLA_F32 if d.dtype in ("f32", torch.float32) else GQLA_BF16
    kl = GQLA_K_SHARED_ROPE if getattr(d, "k_shared_rope", False) else GQLA_K_PER_GROUP
    return GqlaDims(d.n_h, d.G, d.d_nope, d.d_rope, d.d_v, d.r, d.s_q, float(scale), dt, kl)


def make_layout(seq_lens: torch.Tensor, max_seq_len: int, page_size: int = 0, capacity: int = 0,
                block_table: Optional[torch.Tensor] = None, num_pages: int = 0) -> GqlaKvLayout:
    """seq_lens and block_table are int32 device tensors (kept alive by the caller)."""
    mbps = 0 if block_table is None else int(block_table.shape[1])
    return GqlaKvLayout(int(seq_lens.shape[0]), _ptr(seq_lens), int(max_seq_len), int(page_size),
                        int(capacity), _ptr(block_table), mbps, int(num_pages))


def gqla_status_string(status: int) -> str:
    return lib().gqla_status_string(status).decode()


def gqla_version() -> str:
    return lib().gqla_version().decode()


def gqla_launch_counter() -> int:
    return int(lib().gqla_launch_counter())


def gqla_cache_bytes_per_token(dims: GqlaDims, path: int) -> int:
    return int(lib().gqla_cache_bytes_per_token(ctypes.byref(dims), path))


def gqla_workspace_bytes(dims: GqlaDims, layout: GqlaKvLayout, num_splits: int, path: int) -> int:
    return int(lib().gqla_workspace_bytes(ctypes.byref(dims), ctypes.byref(layout), num_splits, path))


def gqla_num_splits(dims: GqlaDims, layout: GqlaKvLayout, num_splits: int, path: int) -> int:
    return int(lib().gqla_num_splits(ctypes.byref(dims), ctypes.byref(layout), num_splits, path))


def gqla_select_path(dims: GqlaDims, layout: GqlaKvLayout, total_tokens: int, hw: Optional[GqlaHw] = None):
    """(path, absorb_us, gqa_us): the library's prediction of both decode calls."""
    est = GqlaPathEstimate()
    s = lib().gqla_select_path(ctypes.byref(dims), ctypes.byref(layout), int(total_tokens),
                               ctypes.byref(hw) if hw is not None else None, ctypes.byref(est))
    _check(s, "gqla_select_path")
    return int(est.path), float(est.absorb_us), float(est.gqa_us)


def workspace_for(dims: GqlaDims, layout: GqlaKvLayout, num_splits: int, path: int, device) -> torch.Tensor:
    n = gqla_workspace_bytes(dims, layout, num_splits, path)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def gqla_expand_cache(dims, layout, latent, W_uk, W_uv, k_pool, v_pool, tail_tokens=0, dev_status=None,
                      stream=None):
    """Expand every cached token (or, with tail_tokens > 0, only each
    sequence's last tail_tokens) into the per-group pools: K rows
    [c_KV W_uk^g ; k_rope], V rows c_KV W_uv^g.  Pools share the latent pool's
    geometry (contiguous or paged through the same block table)."""
    s = lib().gqla_expand_cache(ctypes.byref(dims), ctypes.byref(layout), _ptr(latent), _ptr(W_uk), _ptr(W_uv),
                                _ptr(k_pool), _ptr(v_pool), int(tail_tokens), _ptr(dev_status),
                                _stream(stream, latent.device))
    _check(s, "gqla_expand_cache")


def gqla_append_tokens(dims, layout, new_rows, latent, W_uk=None, W_uv=None, k_pool=None, v_pool=None,
                       dev_status=None, stream=None):
    """Write each sequence's s_q new token rows new_rows [B, s_q, r + d_rope]
    at positions seq_len - s_q .. seq_len - 1: into the latent pool (when
    latent is given) and, expanded, into the per-group pools (when k_pool and
    v_pool are given; W_uk and W_uv are then required).  latent=None expands
    only, reading the rows from new_rows."""
    s = lib().gqla_append_tokens(ctypes.byref(dims), ctypes.byref(layout), _ptr(new_rows), _ptr(latent), _ptr(W_uk),
                                 _ptr(W_uv), _ptr(k_pool), _ptr(v_pool), _ptr(dev_status),
                                 _stream(stream, new_rows.device))
    _check(s, "gqla_append_tokens")


def gqla_decode_absorb(dims, layout, q, latent, W_uk, W_uv, out, lse=None, num_splits=0, workspace=None,
                       dev_status=None, stream=None):
    """Absorb-path decode over the latent pool: q_nope is absorbed into the
    latent space per group, scores run against [c_KV ; k_rope], the latent
    output is up-projected by W_uv.  out [B, s_q, n_h, d_v]; lse [B, s_q, n_h]
    fp32 (natural log) when given.  num_splits 0 takes the library's plan; a
    workspace of gqla_workspace_bytes is allocated when none is passed."""
    if workspace is None:
        workspace = workspace_for(dims, layout, num_splits, GQLA_PATH_ABSORB, q.device)
    s = lib().gqla_decode_absorb(ctypes.byref(dims), ctypes.byref(layout), _ptr(q), _ptr(latent), _ptr(W_uk),
                                 _ptr(W_uv), _ptr(out), _ptr(lse), int(num_splits), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                 _stream(stream, q.device))
    _check(s, "gqla_decode_absorb")


def gqla_decode_gqa(dims, layout, q, k_pool, v_pool, out, lse=None, num_splits=0, workspace=None,
                    dev_status=None, stream=None):
    """GQA-path decode over the expanded per-group pools: each group's m heads
    attend to that group's K/V rows.  Same output, lse, split and workspace
    conventions as gqla_decode_absorb."""
    if workspace is None:
        workspace = workspace_for(dims, layout, num_splits, GQLA_PATH_GQA, q.device)
    s = lib().gqla_decode_gqa(ctypes.byref(dims), ctypes.byref(layout), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                              _ptr(out), _ptr(lse), int(num_splits), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _ptr(dev_status),
                              _stream(stream, q.device))
    _check(s, "gqla_decode_gqa")


def gqla_decode_gqa_noalloc(dims, layout, q, k_pool, v_pool, out, lse=None, num_splits=0, dev_status=None,
                            stream=None):
    """gqla_decode_gqa with its split scratch in the library's own fixed device
    array: no workspace, no allocation (see include/gqla.h for the limit)."""
    s = lib().gqla_decode_gqa_noalloc(ctypes.byref(dims), ctypes.byref(layout), _ptr(q), _ptr(k_pool),
                                      _ptr(v_pool), _ptr(out), _ptr(lse), int(num_splits), _ptr(dev_status),
                                      _stream(stream, q.device))
    _check(s, "gqla_decode_gqa_noalloc")


def gqla_splitkv_combine(o_part, lse_part, out, lse_out=None, stream=None):
    S, rows, D = (int(x) for x in o_part.shape)
    dt = GQLA_F32 if out.dtype == torch.float32 else GQLA_BF16
    s = lib().gqla_splitkv_combine(S, rows, D, _ptr(o_part), _ptr(lse_part), _ptr(out), dt, _ptr(lse_out),
                                   _stream(stream, o_part.device))
    _check(s, "gqla_splitkv_combine")

"""Helpers for the GPU parity tests: run the library, run the oracle on the same bits, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import unstructured_sparse_kv_b200 as M

MAX_ABS = 2e-3   # attention tolerance: fp16 storage, fp32 accumulation
REL_L2 = 1e-3
LSE_ABS = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    """fp16 tensor -> numpy uint16 bit patterns (on the host)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def cache_np(cache: M.CompressedCache):
    bm, vals, offs = cache.views()
    return (bm.cpu().numpy().view(np.uint32), vals.cpu().numpy().view(np.uint16), offs.cpu().numpy().view(np.uint32))


def assert_cache_matches(cache: M.CompressedCache, x_bits_bhld: np.ndarray, L: int, streams=None):
    """Bit-exact check of bitmap, packed values (tokens [0, L)) and every tile offset.

    ``x_bits_bhld`` holds the dense fp16 bits [B, H, >=L, d] (or, with ``streams``, [n, >=L, d]
    for the listed (b, h) streams only).
    """
    bm, vals, offs = cache_np(cache)
    k, cap = cache.keep, cache.capacity
    if streams is None:
        ref = oracle.compress(x_bits_bhld[:, :, :L], k, cap, L)
        assert np.array_equal(bm[:, :, :L], ref["bitmap"][:, :, :L]), "bitmap mismatch"
        assert np.array_equal(vals[:, :, : L * k], ref["values"][:, :, : L * k]), "packed values mismatch"
        assert np.array_equal(offs, ref["tile_offset"]), "tile offsets mismatch"
        return
    for i, (b, h) in enumerate(streams):
        ref = oracle.compress(x_bits_bhld[i][None, None, :L], k, cap, L)
        assert np.array_equal(bm[b, h, :L], ref["bitmap"][0, 0, :L]), ("bitmap", b, h)
        assert np.array_equal(vals[b, h, : L * k], ref["values"][0, 0, : L * k]), ("values", b, h)
        assert np.array_equal(offs[b, h], ref["tile_offset"][0, 0]), ("offsets", b, h)


def assert_attn_close(out_gpu: torch.Tensor, o_ref: np.ndarray, lse_gpu=None, lse_ref=None, tag=""):
    a = out_gpu.detach().float().cpu().numpy().astype(np.float64)
    diff = np.abs(a - o_ref)
    max_abs = float(diff.max())
    rel = float(np.linalg.norm(a - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{tag}: max-abs {max_abs:.3g}, rel-L2 {rel:.3g}"
    if lse_gpu is not None:
        l = lse_gpu.detach().cpu().numpy().astype(np.float64)
        err = float(np.abs(l - lse_ref).max())
        assert err <= LSE_ABS, f"{tag}: lse max-abs {err:.3g}"
    return max_abs, rel


def oracle_attention(q, K_bits, V_bits, kK, kV, seq_len, scale):
    """Oracle output for full caches given as dense fp16 bits [B, Hkv, >=L, d]."""
    Lmax = int(max(seq_len))
    kp = oracle.prune(K_bits[:, :, :Lmax], kK)
    vp = oracle.prune(V_bits[:, :, :Lmax], kV)
    return oracle.attention(bits(q) if isinstance(q, torch.Tensor) else q, kp, vp, seq_len, scale)

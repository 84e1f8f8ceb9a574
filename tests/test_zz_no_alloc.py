"""The allocation-free decode attention entry point, called through the C ABI.

mustafar_decode_attn_noalloc serves callers that cannot hand the library a workspace (their
device memory is reserved up front, or a plugin interface gives them only inputs and outputs):
it keeps the split-K scratch in a fixed array inside the library.  Its results must match
mustafar_decode_attn, which takes a caller workspace, within the attention tolerance used by
the other tests, on two calls in a row (the second call reuses the scratch the first one left).
This file is named so that pytest collects it last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import unstructured_sparse_kv_b200 as M
from tests import gpu_util as U
from unstructured_sparse_kv_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _noalloc(lib, q, kc, vc, seq, max_len, out, lse, num_splits=0):
    return lib.mustafar_decode_attn_noalloc(C.c_void_p(q.data_ptr()), q.shape[1], C.byref(kc.struct),
                                            C.byref(vc.struct), C.c_void_p(seq.data_ptr()), max_len, 1.0,
                                            C.c_void_p(out.data_ptr()), C.c_void_p(lse.data_ptr()), num_splits, None,
                                            C.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(a, b, la, lb):
    ref = b.float().cpu().numpy().astype(np.float64)
    U.assert_attn_close(a, ref, la, lb.cpu().numpy().astype(np.float64), tag="noalloc vs workspace entry point")


@pytest.mark.parametrize("B,Hq,Hkv,L,num_splits", [(2, 8, 2, 700, 0), (8, 32, 8, 4160, 0), (1, 32, 8, 3000, 9)])
def test_noalloc_matches_workspace_entry_point_twice(B, Hq, Hkv, L, num_splits):
    lib = M.load()
    cap = ((L + 63) // 64) * 64
    K = synth.keys(B, Hkv, L, 128, 31, DEV, capacity=cap)
    V = synth.values(B, Hkv, L, 128, 31, DEV, capacity=cap)
    kc, vc = M.CompressedCache(B, Hkv, cap, 0.7), M.CompressedCache(B, Hkv, cap, 0.5)
    M.mustafar_compress(K, L, 0.7, kc)
    M.mustafar_compress(V, L, 0.5, vc)
    seq = synth.seq_lens(B, L, True, 3).to(DEV)
    for call in range(2):  # two calls in a row share the scratch
        q = synth.queries(B, Hq, 128, 31, DEV, step=call)
        ref_out, ref_lse = M.mustafar_decode_attn(q, kc, vc, seq, L, 1.0, num_splits=num_splits)
        out = torch.empty_like(q)
        lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
        st = _noalloc(lib, q, kc, vc, seq, L, out, lse, num_splits)
        assert st == 0, lib.mustafar_last_error().decode()
        torch.cuda.synchronize()
        _close(out, ref_out, lse, ref_lse)


@pytest.mark.parametrize("pattern_k,pattern_v", [("channel", "channel"), ("channel", "2:4"), ("2:4", "2:4")])
def test_noalloc_variants_match_workspace_entry_point(pattern_k, pattern_v):
    # the other cache formats go through the same allocation-free entry point
    lib = M.load()
    B, Hq, Hkv, L, cap = 4, 32, 8, 1000, 1024
    K = synth.keys(B, Hkv, L, 128, 37, DEV, capacity=cap)
    V = synth.values(B, Hkv, L, 128, 37, DEV, capacity=cap)
    sk = 0.5 if pattern_k == "2:4" else 0.7
    sv = 0.5 if pattern_v == "2:4" else 0.7
    kc = M.CompressedCache(B, Hkv, cap, sk, pattern=pattern_k)
    vc = M.CompressedCache(B, Hkv, cap, sv, pattern=pattern_v)
    M.mustafar_compress(K, L, sk, kc)
    M.mustafar_compress(V, L, sv, vc)
    seq = synth.seq_lens(B, L, True, 5).to(DEV)
    q = synth.queries(B, Hq, 128, 37, DEV)
    ref_out, ref_lse = M.mustafar_decode_attn(q, kc, vc, seq, L, 1.0)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
    st = _noalloc(lib, q, kc, vc, seq, L, out, lse)
    assert st == 0, lib.mustafar_last_error().decode()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)  # the same kernel and plan


def test_noalloc_rejects_a_plan_beyond_its_scratch():
    lib = M.load()
    B, Hq, Hkv, L = 8, 32, 8, 4096
    kc, vc = M.CompressedCache(B, Hkv, L, 0.7), M.CompressedCache(B, Hkv, L, 0.7)
    q = torch.zeros(B, Hq, 128, dtype=torch.float16, device=DEV)
    seq = torch.full((B,), L, dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
    st = _noalloc(lib, q, kc, vc, seq, L, out, lse, num_splits=128)  # 64 streams x 128 splits: 36 MB > 16 MiB
    assert st == 5  # MUSTAFAR_ERR_WORKSPACE
    assert "scratch" in lib.mustafar_last_error().decode()


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_noalloc_automatic_plan_fits_its_scratch(G):
    # the automatic plan at a batch whose streams fill a whole wave of CTAs, for every supported group size:
    # its split-K scratch must fit the fixed array, so the call is accepted and matches the workspace call
    lib = M.load()
    Hkv, L = 8, 2048
    B = 32
    Hq = G * Hkv
    cap = L
    K = synth.keys(B, Hkv, L, 128, 41, DEV)
    V = synth.values(B, Hkv, L, 128, 41, DEV)
    kc, vc = M.CompressedCache(B, Hkv, cap, 0.7), M.CompressedCache(B, Hkv, cap, 0.7)
    M.mustafar_compress(K, L, 0.7, kc)
    M.mustafar_compress(V, L, 0.7, vc)
    seq = torch.full((B,), L, dtype=torch.int32, device=DEV)
    q = synth.queries(B, Hq, 128, 41, DEV)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
    st = _noalloc(lib, q, kc, vc, seq, L, out, lse)
    assert st == 0, lib.mustafar_last_error().decode()
    torch.cuda.synchronize()
    ref_out, ref_lse = M.mustafar_decode_attn(q, kc, vc, seq, L, 1.0)
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


def test_noalloc_call_allocates_no_device_memory():
    # the property the entry point exists for: a warm call leaves the device's free memory unchanged
    # (torch's caching allocator is not involved: the call only gets raw pointers)
    lib = M.load()
    B, Hq, Hkv, L = 8, 32, 8, 4096
    K = synth.keys(B, Hkv, L, 128, 43, DEV)
    V = synth.values(B, Hkv, L, 128, 43, DEV)
    kc, vc = M.CompressedCache(B, Hkv, L, 0.7), M.CompressedCache(B, Hkv, L, 0.7)
    M.mustafar_compress(K, L, 0.7, kc)
    M.mustafar_compress(V, L, 0.7, vc)
    del K, V
    seq = torch.full((B,), L, dtype=torch.int32, device=DEV)
    q = synth.queries(B, Hq, 128, 43, DEV)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
    assert _noalloc(lib, q, kc, vc, seq, L, out, lse) == 0  # first call: loads the device code if needed
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert _noalloc(lib, q, kc, vc, seq, L, out, lse) == 0
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before

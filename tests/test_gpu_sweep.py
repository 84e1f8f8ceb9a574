"""The decode-attention sweep at every one of its 90 points, against the oracle.

Sweep: K and V sparsity {0, 0.3, 0.5, 0.7, 0.9} x batch {1, 8, 32} x context {4096, 32768,
131072} x head shape {MHA 32 q / 32 kv heads (Llama-2-7B-like), GQA 32 / 8 (Llama-3-8B-like)},
head_dim 128, synthetic caches as everywhere else.  Each point runs at full size on the GPU:
both caches are compressed and decode attention runs over all streams with the automatic plan.
The oracle (too slow for every stream of the large points) checks sampled (batch row, kv head)
streams: the bitmap, packed values and tile offsets of both caches bit for bit, and the
attention output and log-sum-exp of the stream's q heads within the attention tolerance.
Dense fp16 attention on the same inputs is compared at a subset of these points in
test_gpu_parity.py.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import unstructured_sparse_kv_b200 as M
from tests import gpu_util as U
from unstructured_sparse_kv_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
D = 128

SPARSITY = (0.0, 0.3, 0.5, 0.7, 0.9)
BATCH = (1, 8, 32)
CONTEXT = (4096, 32768, 131072)
HEADS = ((32, 32), (32, 8))  # (q heads, kv heads)
POINTS = list(itertools.product(HEADS, BATCH, CONTEXT, SPARSITY))
assert len(POINTS) == 90


def _streams(index, B, Hkv, L):
    """Sampled streams of a point: one seeded pick, plus the last stream below the longest context."""
    rng = np.random.default_rng(7000 + index)
    picks = {(int(rng.integers(B)), int(rng.integers(Hkv)))}
    if L < 131072:
        picks.add((B - 1, Hkv - 1))
    return sorted(picks)


def _compress_keeping(kind, B, Hkv, L, s, seed, streams):
    """Generate one dense cache on the GPU, compress it, and keep only the sampled streams' bits on the host."""
    x = (synth.keys if kind == "K" else synth.values)(B, Hkv, L, D, seed, DEV)
    c = M.CompressedCache(B, Hkv, L, s)
    M.mustafar_compress(x, L, s, c)
    host = {bh: U.bits(x[bh[0], bh[1]]) for bh in streams}
    del x
    return c, host


def _check_stream(cache, x_bits, b, h, L):
    """Bit-exact bitmap / values / offsets of stream (b, h); returns the oracle's pruned tensor."""
    k = cache.keep
    ref = oracle.compress(x_bits[None, None], k, L, L)
    bm, vals, offs = cache.views()
    assert np.array_equal(bm[b, h].cpu().numpy().view(np.uint32), ref["bitmap"][0, 0]), ("bitmap", b, h)
    assert np.array_equal(vals[b, h].cpu().numpy().view(np.uint16), ref["values"][0, 0]), ("values", b, h)
    assert np.array_equal(offs[b, h].cpu().numpy().view(np.uint32), ref["tile_offset"][0, 0]), ("offsets", b, h)
    return oracle.decompress(ref["bitmap"], ref["values"], k, L, D)


@pytest.mark.parametrize("index", range(len(POINTS)),
                         ids=[f"{'mha' if hkv == 32 else 'gqa'}-b{B}-L{L}-s{s}" for (_, hkv), B, L, s in POINTS])
def test_sweep_point(index):
    (Hq, Hkv), B, L, s = POINTS[index]
    G = Hq // Hkv
    seed = 3000 + index
    streams = _streams(index, B, Hkv, L)
    kc, kbits = _compress_keeping("K", B, Hkv, L, s, seed, streams)
    vc, vbits = _compress_keeping("V", B, Hkv, L, s, seed, streams)
    assert kc.keep == oracle.keep_count(D, s) and kc.nbytes() == B * Hkv * oracle.compressed_bytes(L, kc.keep, L, D)
    q = synth.queries(B, Hq, D, seed, DEV)
    seq = torch.full((B,), L, dtype=torch.int32, device=DEV)
    out, lse = M.mustafar_decode_attn(q, kc, vc, seq, L, 1.0)
    torch.cuda.synchronize()
    for b, h in streams:
        kp = _check_stream(kc, kbits[(b, h)], b, h, L)
        vp = _check_stream(vc, vbits[(b, h)], b, h, L)
        heads = slice(h * G, (h + 1) * G)
        o_ref, l_ref = oracle.attention(U.bits(q[b:b + 1, heads]), kp, vp, [L], 1.0)
        U.assert_attn_close(out[b:b + 1, heads], o_ref, lse[b:b + 1, heads], l_ref,
                            tag=f"sweep point {POINTS[index]} stream ({b}, {h})")
    del kc, vc
    torch.cuda.empty_cache()

"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Compressed caches (bitmap, packed values, tile offsets) must be bit-exact; attention
outputs within max-abs 2e-3 and relative L2 1e-3 of the float64 oracle, lse within 1e-3.
Sizes span several 16-token chunks and 64-token tiles with ragged tails; the workload
shapes (batch 1..32, context up to 128k, MHA and GQA, sparsity 0..0.9) are checked at
full size, with the oracle run on sampled (batch, kv head) streams where the full
tensor would take it too long.
"""
import math

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


@pytest.fixture(scope="module", autouse=True)
def _lib():
    M.load()


def _setup(B, Hq, Hkv, L, cap, sK, sV, seed, seq=None):
    K = synth.keys(B, Hkv, L, D, seed, DEV, capacity=cap)
    V = synth.values(B, Hkv, L, D, seed, DEV, capacity=cap)
    q = synth.queries(B, Hq, D, seed, DEV)
    kc = M.CompressedCache(B, Hkv, cap, sK)
    vc = M.CompressedCache(B, Hkv, cap, sV)
    M.mustafar_compress(K, L, sK, kc)
    M.mustafar_compress(V, L, sV, vc)
    seq = torch.full((B,), L, dtype=torch.int32) if seq is None else seq
    return K, V, q, kc, vc, seq


def _attend(q, kc, vc, seq, max_len, scale=1.0, splits=0):
    return M.mustafar_decode_attn(q, kc, vc, seq.to(DEV), max_len, scale, num_splits=splits)


# ------------------------------------------------------------------------------------ compress / append
TIE_ROWS = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x03FF, 0x3C00, 0xBC00, 0x4000, 0xC000, 0x7BFF, 0xFBFF],
                    dtype=np.uint16)


@pytest.mark.parametrize("s", [0.0, 0.1, 0.3, 0.5, 0.7, 0.9, 0.995])
def test_compress_bit_exact_strided_with_ties(s):
    B, H, L, cap = 2, 3, 200, 256
    rng = np.random.default_rng(5)
    x = synth.keys(B, H, L, D, 42, "cpu").permute(0, 2, 1, 3).contiguous()  # [B, L, H, d] storage
    xb = x.view(torch.int16).numpy().view(np.uint16).copy()
    xb[0, 3, 1] = rng.choice(TIE_ROWS, D)
    xb[1, 77, 2] = 0x3C00                      # all equal
    xb[1, 78, 0] = 0                           # all +0
    xb[0, 150, 0, :64] = 0x8000                # -0 and ties with +0
    xb[0, 151, 1, 5] = 0x7C00                  # +inf / NaN patterns rank by bits
    xb[0, 151, 1, 9] = 0x7E00
    xdev = torch.from_numpy(xb.view(np.int16)).view(torch.float16).to(DEV)
    view = xdev.permute(0, 2, 1, 3)            # [B, H, L, d] strided view
    c = M.CompressedCache(B, H, cap, s)
    M.mustafar_compress(view, L, s, c)
    U.assert_cache_matches(c, np.ascontiguousarray(xb.transpose(0, 2, 1, 3)), L)


def test_compress_leaves_slots_beyond_L_untouched():
    B, H, L, cap = 1, 2, 100, 192
    x = synth.values(B, H, cap, D, 3, DEV)
    c = M.CompressedCache(B, H, cap, 0.7)
    c.bitmap.fill_(-1)
    c.values.fill_(0x1234)
    M.mustafar_compress(x, L, 0.7, c)
    bm, vals, _ = U.cache_np(c)
    assert (bm[:, :, L:] == 0xFFFFFFFF).all() and (vals[:, :, L * c.keep:] == 0x1234).all()
    U.assert_cache_matches(c, U.bits(x), L)


def test_compress_empty_writes_offsets_only():
    c = M.CompressedCache(2, 2, 128, 0.5)
    c.tile_offset.fill_(-1)
    x = torch.zeros(2, 2, 128, D, dtype=torch.float16, device=DEV)
    M.mustafar_compress(x, 0, 0.5, c)
    _, _, offs = U.cache_np(c)
    assert (offs == np.array([0, 64 * 64], dtype=np.uint32)).all()
    assert int(c.bitmap.abs().sum()) == 0


def test_append_across_tile_boundaries_matches_oracle():
    B, H, cap, k_s = 3, 2, 256, 0.7
    L0 = 60
    full = synth.keys(B, H, 140, D, 9, DEV, capacity=cap)
    c = M.CompressedCache(B, H, cap, k_s)
    M.mustafar_compress(full, L0, k_s, c)
    for t in range(L0, 140):
        pos = torch.full((B,), t, dtype=torch.int32, device=DEV)
        M.mustafar_append(full[:, :, t], pos, c)  # strided [B, H, d] slice
    U.assert_cache_matches(c, U.bits(full), 140)


def test_append_rows_at_different_positions_and_out_of_range():
    B, H, cap = 4, 2, 128
    c = M.CompressedCache(B, H, cap, 0.5)
    x = synth.step_tokens(B, H, D, 11, 0, DEV)[0]
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pos = torch.tensor([0, 63, 64, cap], dtype=torch.int32, device=DEV)  # the last row is out of range
    M.mustafar_append(x, pos, c, err=err)
    assert int(err.item()) & M.DEVERR_POS_RANGE
    bm, vals, _ = U.cache_np(c)
    xb = U.bits(x)
    k = c.keep
    for b, p in enumerate([0, 63, 64]):
        ref = oracle.compress(xb[b][None, :, None, :], k, 64)
        assert np.array_equal(bm[b, :, p], ref["bitmap"][0, :, 0])
        assert np.array_equal(vals[b, :, p * k:(p + 1) * k], ref["values"][0, :, :k])
    assert (bm[3] == 0).all() and (vals[3] == 0).all()


# ------------------------------------------------------------------------------------ decode attention
@pytest.mark.parametrize("B,Hq,Hkv,L,sK,sV,splits,ragged", [
    (2, 8, 2, 200, 0.7, 0.7, 0, True),
    (2, 8, 2, 200, 0.7, 0.5, 3, True),
    (3, 4, 4, 77, 0.5, 0.9, 1, True),      # MHA (G = 1)
    (1, 32, 2, 300, 0.3, 0.7, 0, False),   # G = 16
    (2, 8, 1, 1, 0.7, 0.7, 0, False),      # one token
    (2, 12, 4, 129, 0.0, 0.0, 2, True),    # sparsity 0: plain attention
    (1, 8, 8, 1000, 0.995, 0.995, 0, False),  # keep = 1
    (2, 8, 2, 200, 0.25, 0.0, 0, True),    # keeps 96 and 128: runs staged token by token
    (2, 8, 2, 150, 0.25, 0.7, 2, True),    # one cache staged token by token, one in a single copy
    (2, 8, 2, 213, 0.5, 0.5, 3, True),     # keep 64 in both caches: staged in 4-token groups
    (1, 32, 2, 170, 0.0, 0.25, 0, False),  # G = 16 with both caches staged token by token
    (2, 8, 2, 200, 0.9, 0.9, 0, True),     # keep 13: few kept values per token
    (2, 12, 4, 129, 0.85, 0.9, 3, True),   # keeps 20 and 13, G = 3, forced splits
    (1, 32, 2, 300, 0.9, 0.8, 0, True),    # G = 16 with keeps 13 and 26
    (2, 8, 2, 150, 0.9, 0.7, 0, True),     # keeps 13 and 39
])
def test_decode_small_cases(B, Hq, Hkv, L, sK, sV, splits, ragged):
    cap = ((L + 63) // 64) * 64
    seq = synth.seq_lens(B, L, ragged, 1)
    K, V, q, kc, vc, seq = _setup(B, Hq, Hkv, L, cap, sK, sV, 100 + B + L, seq)
    scale = 1.0 / math.sqrt(D) if sK == 0 else 1.0
    out, lse = _attend(q, kc, vc, seq, L, scale, splits)
    o_ref, l_ref = U.oracle_attention(q, U.bits(K), U.bits(V), kc.keep, vc.keep, seq.numpy(), scale)
    U.assert_attn_close(out, o_ref, lse, l_ref, tag=f"B{B} Hq{Hq} Hkv{Hkv} L{L}")


def test_split_count_invariance():
    B, Hq, Hkv, L = 2, 32, 8, 2000
    K, V, q, kc, vc, seq = _setup(B, Hq, Hkv, L, 2048, 0.7, 0.7, 7)
    outs = [_attend(q, kc, vc, seq, L, 1.0, s) for s in (1, 2, 5, 31, 0)]
    o_ref, l_ref = U.oracle_attention(q, U.bits(K), U.bits(V), kc.keep, vc.keep, seq.numpy(), 1.0)
    for o, l in outs:
        U.assert_attn_close(o, o_ref, l, l_ref, tag="splits")
        assert float((o.float() - outs[0][0].float()).abs().max()) <= 2e-3


@pytest.mark.parametrize("B,Hq,Hkv,L,ragged", [(8, 32, 8, 1024, True), (8, 32, 8, 256, False), (8, 128, 8, 256, True)])
def test_one_cluster_per_stream_plans(B, Hq, Hkv, L, ragged):
    """Shapes whose automatic plan gives every stream the same whole number C of CTAs with all B x Hkv
    clusters resident (B200: C = 8 at 8 x 8 kv heads x 1024 tokens, 2 at 256 tokens with 4 or 16 q heads
    per kv head): those CTAs form one thread-block cluster per stream and merge in
    distributed shared memory.  Ragged rows (one of them empty) and a fused decode step too; the
    ticket plan (a forced split count) on the same caches must agree with the oracle as well."""
    keep = oracle.keep_count(D, 0.7)
    assert M.mustafar_decode_plan_cluster(B, Hq, Hkv, L, keep, oracle.keep_count(D, 0.5)) >= 2
    K, V, q, kc, vc, _ = _setup(B, Hq, Hkv, L, L, 0.7, 0.5, 61)
    seq = synth.seq_lens(B, L, ragged, 61)
    if ragged:
        seq[B // 2] = 0
    rows = (seq > 0).nonzero().flatten()  # the oracle defines no output for an empty row
    o_ref, l_ref = U.oracle_attention(q[rows], U.bits(K)[rows], U.bits(V)[rows], kc.keep, vc.keep,
                                      seq[rows].numpy(), 1.0)
    for splits, tag in ((0, f"cluster plan B{B} G{Hq // Hkv} ragged={ragged}"), (31, "ticket plan")):
        out, lse = _attend(q, kc, vc, seq, L, splits=splits)
        U.assert_attn_close(out[rows.to(DEV)], o_ref, lse[rows.to(DEV)], l_ref, tag=tag)
        if ragged:
            assert float(out[B // 2].abs().max()) == 0.0 and torch.isinf(lse[B // 2]).all() and (lse[B // 2] < 0).all()
    # one fused step that rewrites the last token of every row (position L - 1), so that the step
    # attends over L tokens under the same cluster plan
    kn, vn = synth.step_tokens(B, Hkv, D, 61, 0, DEV)
    pos = torch.full((B,), L - 1, dtype=torch.int32, device=DEV)
    out, lse = M.mustafar_decode_step(q, kn, vn, pos, kc, vc, L, 1.0)
    K[:, :, L - 1], V[:, :, L - 1] = kn, vn
    o_ref, l_ref = U.oracle_attention(q, U.bits(K), U.bits(V), kc.keep, vc.keep, [L] * B, 1.0)
    U.assert_attn_close(out, o_ref, lse, l_ref, tag="cluster plan fused step")


def test_cluster_plan_replays_from_a_cuda_graph():
    """A cluster launch recorded in a CUDA graph (after one eager call of the shape, as for every
    plan) replays bit-identically to the eager call."""
    B, Hq, Hkv, L = 8, 32, 8, 1024
    keep = oracle.keep_count(D, 0.7)
    assert M.mustafar_decode_plan_cluster(B, Hq, Hkv, L, keep, keep) >= 2
    K, V, q, kc, vc, seq = _setup(B, Hq, Hkv, L, L, 0.7, 0.7, 67)
    seq = seq.to(DEV)
    ref_out, ref_lse = M.mustafar_decode_attn(q, kc, vc, seq, L, 1.0)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
    ws = torch.zeros(M.mustafar_decode_workspace_bytes(B, Hq, Hkv, L), dtype=torch.uint8, device=DEV)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        M.mustafar_decode_attn(q, kc, vc, seq, L, 1.0, out=out, lse=lse, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        M.mustafar_decode_attn(q, kc, vc, seq, L, 1.0, out=out, lse=lse, workspace=ws)
    out.zero_()
    lse.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    del g


@pytest.mark.parametrize("kind", ["per-head", "2:4", "channel", "keep-64 skewed staging"])
def test_cache_variants_under_a_cluster_plan(kind):
    """The other cache formats at a shape whose plan is one 8-CTA cluster per stream for uniform caches
    (batch 8 x 8 kv heads x 1024 tokens): the variants share the plan, the range split and the cluster
    merge.  Ragged rows, one of them empty."""
    B, Hq, Hkv, L = 8, 32, 8, 1024
    K = synth.keys(B, Hkv, L, D, 91, DEV)
    V = synth.values(B, Hkv, L, D, 91, DEV)
    Kb, Vb = U.bits(K), U.bits(V)
    if kind == "per-head":
        sK, sV = [0.5, 0.6, 0.7, 0.8, 0.9, 0.7, 0.6, 0.8], [0.8, 0.6, 0.7, 0.9, 0.8, 0.7, 0.6, 0.5]
        kc, vc = M.CompressedCache(B, Hkv, L, sK), M.CompressedCache(B, Hkv, L, sV)
        M.mustafar_compress(K, L, 0.0, kc)
        M.mustafar_compress(V, L, 0.0, vc)
        kp, vp = oracle.prune_heads(Kb, kc.head_keep), oracle.prune_heads(Vb, vc.head_keep)
    elif kind == "2:4":
        kc, vc = M.CompressedCache(B, Hkv, L, 0.5, pattern="2:4"), M.CompressedCache(B, Hkv, L, 0.5, pattern="2:4")
        M.mustafar_compress(K, L, 0.5, kc)
        M.mustafar_compress(V, L, 0.5, vc)
        kp, vp = oracle.prune_24(Kb), oracle.prune_24(Vb)
    elif kind == "channel":
        kc, vc = M.CompressedCache(B, Hkv, L, 0.7, pattern="channel"), M.CompressedCache(B, Hkv, L, 0.7)
        M.mustafar_compress(K, L, 0.7, kc)
        M.mustafar_compress(V, L, 0.7, vc)
        kp, vp = oracle.prune_channel(Kb, 0.7), oracle.prune(Vb, oracle.keep_count(D, 0.7))
    else:
        keep = oracle.keep_count(D, 0.5)
        assert keep == 64 and M.mustafar_decode_plan_cluster(B, Hq, Hkv, L, keep, keep) >= 2
        kc, vc = M.CompressedCache(B, Hkv, L, 0.5), M.CompressedCache(B, Hkv, L, 0.5)
        M.mustafar_compress(K, L, 0.5, kc)
        M.mustafar_compress(V, L, 0.5, vc)
        kp, vp = oracle.prune(Kb, keep), oracle.prune(Vb, keep)
    q = synth.queries(B, Hq, D, 91, DEV)
    seq = synth.seq_lens(B, L, True, 91)
    seq[0] = L
    seq[3] = 0
    out, lse = M.mustafar_decode_attn(q, kc, vc, seq.to(DEV), L, 0.088)
    rows = (seq > 0).nonzero().flatten()
    o_ref, l_ref = oracle.attention(U.bits(q[rows]), kp[rows.numpy()], vp[rows.numpy()], seq[rows].numpy(), 0.088)
    U.assert_attn_close(out[rows.to(DEV)], o_ref, lse[rows.to(DEV)], l_ref, tag=f"{kind} caches, cluster plan")
    assert float(out[3].abs().max()) == 0.0 and torch.isinf(lse[3]).all()


@pytest.mark.parametrize("splits", [0, 2])
def test_batches_beyond_the_row_cache(splits):
    """More than 128 batch rows: rows from 128 on are read from global memory by the range search, the
    stream steps and the row reports (the first 128 come from the shared row cache), and the fused step
    reads their positions from global memory too.  Ragged rows, empty rows on both sides of 128."""
    B, Hq, Hkv, L, cap = 300, 8, 1, 100, 128
    K, V, q, kc, vc, _ = _setup(B, Hq, Hkv, L, cap, 0.7, 0.5, 131)
    seq = synth.seq_lens(B, L, True, 131)
    seq[[5, 127, 128, 200, 299]] = 0
    rows = (seq > 0).nonzero().flatten()
    out, lse = _attend(q, kc, vc, seq, L, 1.0, splits)
    o_ref, l_ref = U.oracle_attention(q[rows], U.bits(K)[rows], U.bits(V)[rows], kc.keep, vc.keep,
                                      seq[rows].numpy(), 1.0)
    U.assert_attn_close(out[rows.to(DEV)], o_ref, lse[rows.to(DEV)], l_ref, tag=f"{B} rows, splits {splits}")
    empty = (seq == 0).nonzero().flatten().to(DEV)
    assert float(out[empty].abs().max()) == 0.0 and torch.isinf(lse[empty]).all()
    # one fused step, each row appending at its own position (an empty row at position 3)
    pos = seq.clone()
    pos[pos == 0] = 3
    posd = pos.to(DEV)
    kn, vn = synth.step_tokens(B, Hkv, D, 131, 0, DEV)
    out, lse = M.mustafar_decode_step(q, kn, vn, posd, kc, vc, L + 1, 1.0, num_splits=splits)
    every = torch.arange(B, device=DEV)
    K[every, :, posd.long()] = kn
    V[every, :, posd.long()] = vn
    o_ref, l_ref = U.oracle_attention(q, U.bits(K), U.bits(V), kc.keep, vc.keep, (pos + 1).numpy(), 1.0)
    U.assert_attn_close(out, o_ref, lse, l_ref, tag=f"{B} rows, fused step, splits {splits}")


def test_decode_step_with_few_kept_values():
    """Fused steps on caches with few kept values per token (s = 0.9, keep 13), rows at their own
    positions."""
    B, Hq, Hkv, L, cap = 4, 32, 8, 700, 768
    K, V, q, kc, vc, _ = _setup(B, Hq, Hkv, L, cap, 0.9, 0.9, 141)
    pos = synth.seq_lens(B, L, True, 141)
    posd = pos.to(DEV)
    every = torch.arange(B, device=DEV)
    for st in range(2):
        qs = synth.queries(B, Hq, D, 141, DEV, step=st + 1)
        kn, vn = synth.step_tokens(B, Hkv, D, 141, st, DEV)
        out, lse = M.mustafar_decode_step(qs, kn, vn, posd, kc, vc, L + 2, 1.0)
        K[every, :, posd.long()] = kn
        V[every, :, posd.long()] = vn
        o_ref, l_ref = U.oracle_attention(qs, U.bits(K), U.bits(V), kc.keep, vc.keep, (pos + 1).numpy(), 1.0)
        U.assert_attn_close(out, o_ref, lse, l_ref, tag=f"keep 13, fused step {st}")
        pos = pos + 1
        posd = pos.to(DEV)


def test_seq_len_zero_and_beyond_capacity():
    B, Hq, Hkv, L, cap = 3, 8, 2, 64, 64
    K, V, q, kc, vc, _ = _setup(B, Hq, Hkv, L, cap, 0.5, 0.5, 21)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    seq = torch.tensor([0, 64, 500], dtype=torch.int32, device=DEV)
    out, lse = M.mustafar_decode_attn(q, kc, vc, seq, 500, 1.0, err=err)
    assert int(err.item()) & M.DEVERR_LEN_RANGE
    assert float(out[0].abs().max()) == 0.0 and torch.isinf(lse[0]).all() and (lse[0] < 0).all()
    o_ref, l_ref = U.oracle_attention(q[1:], U.bits(K)[1:], U.bits(V)[1:], kc.keep, vc.keep, [64, 64], 1.0)
    U.assert_attn_close(out[1:], o_ref, lse[1:], l_ref, tag="clamped")


def test_dense_baseline_matches_oracle_and_sdpa():
    B, Hq, Hkv, L, cap = 2, 32, 8, 700, 704
    K = synth.keys(B, Hkv, L, D, 5, DEV, capacity=cap)
    V = synth.values(B, Hkv, L, D, 5, DEV, capacity=cap)
    q = synth.queries(B, Hq, D, 5, DEV)
    seq = torch.tensor([L, 333], dtype=torch.int32)
    for splits in (1, 0):
        out, lse = M.mustafar_dense_decode_attn(q, K, V, seq.to(DEV), L, 1.0, num_splits=splits)
        o_ref, l_ref = oracle.attention(U.bits(q), U.bits(K), U.bits(V), seq.numpy(), 1.0)
        U.assert_attn_close(out, o_ref, lse, l_ref, tag="dense")
    Kr = K[:1, :, :L].repeat_interleave(Hq // Hkv, dim=1).float()
    Vr = V[:1, :, :L].repeat_interleave(Hq // Hkv, dim=1).float()
    sd = torch.nn.functional.scaled_dot_product_attention(q[:1, :, None].float(), Kr, Vr, scale=1.0)[:, :, 0]
    assert float((sd - out[:1].float()).abs().max()) < 2e-3


# ------------------------------------------------------------------------------------ fused decode step
def _row_cache_matches(cache, x_bits_bhld, lens):
    """Per-row bit-exact check: row b's first lens[b] tokens against the oracle's compression."""
    bm, vals, _ = U.cache_np(cache)
    k, cap = cache.keep, cache.capacity
    for b, Lb in enumerate(lens):
        ref = oracle.compress(x_bits_bhld[b:b + 1, :, :Lb], k, cap, Lb)
        assert np.array_equal(bm[b, :, :Lb], ref["bitmap"][0, :, :Lb]), ("bitmap", b)
        assert np.array_equal(vals[b, :, :Lb * k], ref["values"][0, :, :Lb * k]), ("values", b)


@pytest.mark.parametrize("splits", [0, 1, 3])
def test_decode_step_ragged_positions_match_oracle(splits):
    # rows at different positions; appends cross 16-token chunks, a 64-token tile and split
    # boundaries, and overwrite slots that the prefill compression had filled with other tokens
    B, Hq, Hkv, cap, steps = 3, 8, 2, 256, 20
    L0 = [100, 15, 60]
    K0 = synth.keys(B, Hkv, max(L0), D, 31, DEV, capacity=cap)
    V0 = synth.values(B, Hkv, max(L0), D, 31, DEV, capacity=cap)
    kc, vc = M.CompressedCache(B, Hkv, cap, 0.7), M.CompressedCache(B, Hkv, cap, 0.5)
    M.mustafar_compress(K0, max(L0), 0.7, kc)
    M.mustafar_compress(V0, max(L0), 0.5, vc)
    Kt, Vt = K0.clone(), V0.clone()  # the dense truth each row's cache must hold
    vbuf = torch.zeros(B, Hkv, 2 * D, dtype=torch.float16, device=DEV)  # strided v_new
    rows = torch.arange(B, device=DEV)
    for st in range(steps):
        pos = torch.tensor([l + st for l in L0], dtype=torch.int32, device=DEV)
        kn, vn = synth.step_tokens(B, Hkv, D, 31, st, DEV)
        vbuf[:, :, D:] = vn
        Kt[rows, :, pos.long()] = kn
        Vt[rows, :, pos.long()] = vn
        qs = synth.queries(B, Hq, D, 31, DEV, step=st)
        out, lse = M.mustafar_decode_step(qs, kn, vbuf[:, :, D:], pos, kc, vc, max(L0) + steps, 1.0,
                                          num_splits=splits)
        if st in (0, 1, 4, 5, 19):
            lens = (pos + 1).cpu().numpy()
            o_ref, l_ref = U.oracle_attention(qs, U.bits(Kt), U.bits(Vt), kc.keep, vc.keep, lens, 1.0)
            U.assert_attn_close(out, o_ref, lse, l_ref, tag=f"step {st} splits {splits}")
    final = [l + steps for l in L0]
    _row_cache_matches(kc, U.bits(Kt), final)
    _row_cache_matches(vc, U.bits(Vt), final)


def test_decode_step_same_bits_as_append_then_attend():
    B, Hq, Hkv, L0, cap = 8, 32, 8, 500, 640
    K, V, q, kc, vc, _ = _setup(B, Hq, Hkv, L0, cap, 0.7, 0.7, 77)
    kc2, vc2 = M.CompressedCache(B, Hkv, cap, 0.7), M.CompressedCache(B, Hkv, cap, 0.7)
    for a, b in ((kc, kc2), (vc, vc2)):
        b.bitmap.copy_(a.bitmap)
        b.values.copy_(a.values)
        b.tile_offset.copy_(a.tile_offset)
    for st in range(3):
        kn, vn = synth.step_tokens(B, Hkv, D, 77, st, DEV)
        pos = torch.full((B,), L0 + st, dtype=torch.int32, device=DEV)
        qs = synth.queries(B, Hq, D, 77, DEV, step=st)
        o1, l1 = M.mustafar_decode_step(qs, kn, vn, pos, kc, vc, cap, 1.0)
        M.mustafar_append(kn, pos, kc2)
        M.mustafar_append(vn, pos, vc2)
        o2, l2 = M.mustafar_decode_attn(qs, kc2, vc2, pos + 1, cap, 1.0)
        assert torch.equal(o1, o2) and torch.equal(l1, l2), f"step {st}"
    for a, b in ((kc, kc2), (vc, vc2)):
        assert torch.equal(a.bitmap, b.bitmap) and torch.equal(a.values, b.values)


def test_prepared_decode_step_matches_direct_calls():
    # the prepared call runs the same C entry point on buffers whose contents change between steps
    B, Hq, Hkv, L0, cap = 2, 8, 2, 70, 128
    K, V, q, kc, vc, _ = _setup(B, Hq, Hkv, L0, cap, 0.7, 0.5, 91)
    kc2, vc2 = M.CompressedCache(B, Hkv, cap, 0.7), M.CompressedCache(B, Hkv, cap, 0.5)
    for a, b in ((kc, kc2), (vc, vc2)):
        b.bitmap.copy_(a.bitmap)
        b.values.copy_(a.values)
        b.tile_offset.copy_(a.tile_offset)
    qb, knb, vnb = torch.empty_like(q), torch.empty(B, Hkv, D, dtype=torch.float16, device=DEV), \
        torch.empty(B, Hkv, D, dtype=torch.float16, device=DEV)
    posb = torch.empty(B, dtype=torch.int32, device=DEV)
    call, out_p, lse_p = M.prepare_decode_step(qb, knb, vnb, posb, kc2, vc2, cap, 0.5)
    for st in range(5):
        kn, vn = synth.step_tokens(B, Hkv, D, 91, st, DEV)
        qs = synth.queries(B, Hq, D, 91, DEV, step=st)
        pos = torch.full((B,), L0 + st, dtype=torch.int32, device=DEV)
        o1, l1 = M.mustafar_decode_step(qs, kn, vn, pos, kc, vc, cap, 0.5)
        qb.copy_(qs), knb.copy_(kn), vnb.copy_(vn), posb.copy_(pos)
        call()
        assert torch.equal(o1, out_p) and torch.equal(l1, lse_p), f"step {st}"
    assert torch.equal(kc.values, kc2.values) and torch.equal(vc.bitmap, vc2.bitmap)


def test_captured_decode_loop_matches_eager_steps():
    # a graph of 6 fused steps (one launch each) replayed gives the eager calls' bits
    B, Hq, Hkv, L0, cap, steps = 2, 8, 2, 90, 128, 6
    K = synth.keys(B, Hkv, L0, D, 93, DEV, capacity=cap)
    V = synth.values(B, Hkv, L0, D, 93, DEV, capacity=cap)
    caches = []
    for _ in range(2):
        kc, vc = M.CompressedCache(B, Hkv, cap, 0.7), M.CompressedCache(B, Hkv, cap, 0.7)
        M.mustafar_compress(K, L0, 0.7, kc)
        M.mustafar_compress(V, L0, 0.7, vc)
        caches.append((kc, vc))
    q = torch.stack([synth.queries(B, Hq, D, 93, DEV, step=i) for i in range(steps)])
    toks = [synth.step_tokens(B, Hkv, D, 93, i, DEV) for i in range(steps)]
    kn = torch.stack([t[0] for t in toks])
    vn = torch.stack([t[1] for t in toks])
    pos = torch.stack([torch.full((B,), L0 + i, dtype=torch.int32, device=DEV) for i in range(steps)])
    out = torch.empty(steps, B, Hq, D, dtype=torch.float16, device=DEV)
    lse = torch.empty(steps, B, Hq, dtype=torch.float32, device=DEV)
    g = M.capture_decode_steps(q, kn, vn, pos, caches[0][0], caches[0][1], cap, 0.5, out, lse)
    g.replay()
    torch.cuda.synchronize()
    for i in range(steps):
        o, l = M.mustafar_decode_step(q[i], kn[i], vn[i], pos[i], caches[1][0], caches[1][1], cap, 0.5)
        assert torch.equal(o, out[i]) and torch.equal(l, lse[i]), f"step {i}"
    for a, b in zip(caches[0], caches[1]):
        assert torch.equal(a.bitmap, b.bitmap) and torch.equal(a.values, b.values)


def test_decode_step_out_of_range_positions():
    B, Hq, Hkv, L, cap = 3, 8, 2, 64, 64
    K, V, q, kc, vc, _ = _setup(B, Hq, Hkv, L, cap, 0.5, 0.5, 23)
    bm0, vals0 = kc.bitmap.clone(), kc.values.clone()
    kn, vn = synth.step_tokens(B, Hkv, D, 23, 0, DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    pos = torch.tensor([-1, cap, 20], dtype=torch.int32, device=DEV)
    out, lse = M.mustafar_decode_step(q, kn, vn, pos, kc, vc, cap, 1.0, err=err)
    assert int(err.item()) & M.DEVERR_POS_RANGE
    assert float(out[0].abs().max()) == 0.0 and torch.isinf(lse[0]).all() and (lse[0] < 0).all()
    assert torch.equal(kc.bitmap[:2], bm0[:2]) and torch.equal(kc.values[:2], vals0[:2])  # rows 0, 1: no append
    Kt, Vt = K.clone(), V.clone()
    Kt[2, :, 20] = kn[2]
    Vt[2, :, 20] = vn[2]
    o_ref, l_ref = U.oracle_attention(q[1:], U.bits(Kt)[1:], U.bits(Vt)[1:], kc.keep, vc.keep, [cap, 21], 1.0)
    U.assert_attn_close(out[1:], o_ref, lse[1:], l_ref, tag="clamped step")
    _row_cache_matches(kc, U.bits(Kt), [cap, cap, cap])
    # max_len only sizes the plan: a row longer than it is still attended in full, without a flag
    err.zero_()
    kn2, vn2 = synth.step_tokens(B, Hkv, D, 23, 1, DEV)
    pos = torch.tensor([5, 6, 60], dtype=torch.int32, device=DEV)
    out, lse = M.mustafar_decode_step(q, kn2, vn2, pos, kc, vc, 16, 1.0, err=err)
    assert int(err.item()) == 0
    for b, p in enumerate([5, 6, 60]):
        Kt[b, :, p] = kn2[b]
        Vt[b, :, p] = vn2[b]
    o_ref, l_ref = U.oracle_attention(q, U.bits(Kt), U.bits(Vt), kc.keep, vc.keep, [6, 7, 61], 1.0)
    U.assert_attn_close(out, o_ref, lse, l_ref, tag="row longer than max_len")


# ------------------------------------------------------------------------------------ keep count per kv head
def _heads_cache_matches(cache, x_bits, L, streams=None):
    """Bit-exact check of a per-head cache against the oracle, tokens [0, L) of every (b, h)."""
    B, H, cap = cache.batch, cache.num_kv_heads, cache.capacity
    hk = cache.head_keep
    ref = oracle.compress_heads(x_bits[:, :, :L], hk, cap, L)
    bm = cache.bitmap.view(B, H, cap, 4).cpu().numpy().view(np.uint32)
    offs = cache.tile_offset.view(B, H, cap // 64).cpu().numpy().view(np.uint32)
    vals = cache.values.cpu().numpy().view(np.uint16)
    assert np.array_equal(bm[:, :, :L], ref["bitmap"][:, :, :L]), "bitmap"
    assert np.array_equal(offs, ref["tile_offset"]), "tile offsets"
    for b in range(B):
        for h in range(H):
            base = oracle.value_base_heads(b, h, hk, cap)
            assert cache.value_base(b, h) == base
            assert np.array_equal(vals[base:base + L * hk[h]], ref["values"][base:base + L * hk[h]]), (b, h)


def test_per_head_compress_and_append_bit_exact():
    B, H, L0, L1, cap = 2, 4, 150, 160, 192
    hs = [0.0, 0.3, 0.7, 0.9]
    x = synth.keys(B, H, L1, D, 61, DEV, capacity=cap)
    c = M.CompressedCache(B, H, cap, hs)
    assert c.head_keep == [128, 90, 39, 13] and c.keep == 128
    M.mustafar_compress(x, L0, 0.0, c)  # the sparsity argument is not used by a per-head cache
    for t in range(L0, L1):
        M.mustafar_append(x[:, :, t], torch.full((B,), t, dtype=torch.int32, device=DEV), c)
    _heads_cache_matches(c, U.bits(x), L1)


@pytest.mark.parametrize("splits", [0, 3])
def test_per_head_decode_attn_and_step(splits):
    B, Hq, Hkv, L, cap = 3, 16, 4, 200, 256
    sK, sV = [0.5, 0.7, 0.9, 0.3], [0.7, 0.5, 0.7, 0.0]
    K = synth.keys(B, Hkv, cap, D, 62, DEV)
    V = synth.values(B, Hkv, cap, D, 62, DEV)
    kc, vc = M.CompressedCache(B, Hkv, cap, sK), M.CompressedCache(B, Hkv, cap, sV)
    M.mustafar_compress(K, L, 0.0, kc)
    M.mustafar_compress(V, L, 0.0, vc)
    q = synth.queries(B, Hq, D, 62, DEV)
    seq = synth.seq_lens(B, L, True, 62)
    out, lse = M.mustafar_decode_attn(q, kc, vc, seq.to(DEV), L, 1.0, num_splits=splits)
    Kb, Vb = U.bits(K), U.bits(V)
    kp, vp = oracle.prune_heads(Kb[:, :, :L], kc.head_keep), oracle.prune_heads(Vb[:, :, :L], vc.head_keep)
    o_ref, l_ref = oracle.attention(U.bits(q), kp, vp, seq.numpy(), 1.0)
    U.assert_attn_close(out, o_ref, lse, l_ref, tag=f"per-head decode, splits {splits}")
    # fused steps with fresh tokens, each row at its own position (overwriting prefill slots of
    # the shorter rows with different tokens)
    pos = seq.clone().to(DEV)
    rows = torch.arange(B, device=DEV)
    for st in range(2):
        qs = synth.queries(B, Hq, D, 62, DEV, step=st + 1)
        kn, vn = synth.step_tokens(B, Hkv, D, 62, st, DEV)
        K[rows, :, pos.long()] = kn
        V[rows, :, pos.long()] = vn
        out, lse = M.mustafar_decode_step(qs, kn, vn, pos, kc, vc, L + 2, 1.0, num_splits=splits)
        lens = (pos + 1).cpu().numpy()
        Lm = int(lens.max())
        Kb, Vb = U.bits(K), U.bits(V)
        kp = oracle.prune_heads(Kb[:, :, :Lm], kc.head_keep)
        vp = oracle.prune_heads(Vb[:, :, :Lm], vc.head_keep)
        o_ref, l_ref = oracle.attention(U.bits(qs), kp, vp, lens, 1.0)
        U.assert_attn_close(out, o_ref, lse, l_ref, tag=f"per-head step {st}")
        pos += 1
    # cache rows now hold tokens [0, seq + 2) of K / V
    fin = (seq + 2).numpy()
    for cache, xb in ((kc, Kb), (vc, Vb)):
        for b in range(B):
            ref = oracle.compress_heads(xb[b:b + 1, :, :fin[b]], cache.head_keep, cap, int(fin[b]))
            vals = cache.values.cpu().numpy().view(np.uint16)
            for h, k in enumerate(cache.head_keep):
                base = oracle.value_base_heads(b, h, cache.head_keep, cap)
                rb = oracle.value_base_heads(0, h, cache.head_keep, cap)
                assert np.array_equal(vals[base:base + fin[b] * k], ref["values"][rb:rb + fin[b] * k]), (b, h)


def test_per_head_llama3_gqa_b8_ctx4096_mean_s07():
    # per-head sparsities spread around 0.7 (their keep counts average the uniform s = 0.7 keep)
    B, Hq, Hkv, L = 8, 32, 8, 4096
    sK = [0.5, 0.6, 0.7, 0.8, 0.9, 0.7, 0.6, 0.8]
    sV = sK[::-1]
    K = synth.keys(B, Hkv, L, D, 1005, DEV)
    V = synth.values(B, Hkv, L, D, 1005, DEV)
    kc, vc = M.CompressedCache(B, Hkv, L, sK), M.CompressedCache(B, Hkv, L, sV)
    M.mustafar_compress(K, L, 0.0, kc)
    M.mustafar_compress(V, L, 0.0, vc)
    q = synth.queries(B, Hq, D, 1005, DEV)
    seq = torch.full((B,), L, dtype=torch.int32)
    out, lse = M.mustafar_decode_attn(q, kc, vc, seq.to(DEV), L, 1.0)
    rows = [0, 3, 7]
    Kb, Vb = U.bits(K[rows]), U.bits(V[rows])
    kp, vp = oracle.prune_heads(Kb, kc.head_keep), oracle.prune_heads(Vb, vc.head_keep)
    o_ref, l_ref = oracle.attention(U.bits(q[rows]), kp, vp, [L] * len(rows), 1.0)
    U.assert_attn_close(out[rows], o_ref, lse[rows], l_ref, tag="per-head b8 ctx4096")


# ------------------------------------------------------------------------------------ 2:4 comparison pattern
def test_24_compress_append_bit_exact():
    B, H, L0, L1, cap = 2, 3, 130, 140, 192
    rng = np.random.default_rng(71)
    x = synth.keys(B, H, L1, D, 71, "cpu").permute(0, 2, 1, 3).contiguous()  # [B, L, H, d] storage
    xb = x.view(torch.int16).numpy().view(np.uint16).copy()
    xb[0, 3, 1] = rng.choice(TIE_ROWS, D)
    xb[1, 77, 2] = 0x3C00
    xb[0, 100, 0, :64] = 0x8000
    xdev = torch.from_numpy(xb.view(np.int16)).view(torch.float16).to(DEV)
    view = xdev.permute(0, 2, 1, 3)
    c = M.CompressedCache(B, H, cap, 0.5, pattern="2:4")
    M.mustafar_compress(view, L0, 0.5, c)
    for t in range(L0, L1):
        M.mustafar_append(view[:, :, t], torch.full((B,), t, dtype=torch.int32, device=DEV), c)
    ref = oracle.compress_24(np.ascontiguousarray(xb.transpose(0, 2, 1, 3))[:, :, :L1], cap, L1)
    bm, vals, offs = U.cache_np(c)
    assert np.array_equal(bm[:, :, :L1], ref["bitmap"][:, :, :L1])
    assert np.array_equal(vals[:, :, :L1 * 64], ref["values"][:, :, :L1 * 64])
    assert np.array_equal(offs, ref["tile_offset"])


@pytest.mark.parametrize("splits", [0, 2])
def test_24_decode_attn_and_step(splits):
    B, Hq, Hkv, L, cap = 2, 8, 2, 300, 320
    K = synth.keys(B, Hkv, cap, D, 72, DEV)
    V = synth.values(B, Hkv, cap, D, 72, DEV)
    kc = M.CompressedCache(B, Hkv, cap, 0.5, pattern="2:4")
    vc = M.CompressedCache(B, Hkv, cap, 0.5, pattern="2:4")
    M.mustafar_compress(K, L, 0.5, kc)
    M.mustafar_compress(V, L, 0.5, vc)
    q = synth.queries(B, Hq, D, 72, DEV)
    seq = synth.seq_lens(B, L, True, 72)
    out, lse = M.mustafar_decode_attn(q, kc, vc, seq.to(DEV), L, 1.0, num_splits=splits)
    Kb, Vb = U.bits(K), U.bits(V)
    o_ref, l_ref = oracle.attention(U.bits(q), oracle.prune_24(Kb[:, :, :L]), oracle.prune_24(Vb[:, :, :L]),
                                    seq.numpy(), 1.0)
    U.assert_attn_close(out, o_ref, lse, l_ref, tag=f"2:4 decode splits {splits}")
    pos = seq.clone().to(DEV)
    rows = torch.arange(B, device=DEV)
    kn, vn = synth.step_tokens(B, Hkv, D, 72, 0, DEV)
    K[rows, :, pos.long()] = kn
    V[rows, :, pos.long()] = vn
    out, lse = M.mustafar_decode_step(q, kn, vn, pos, kc, vc, L + 1, 1.0, num_splits=splits)
    lens = (pos + 1).cpu().numpy()
    Kb, Vb = U.bits(K), U.bits(V)
    o_ref, l_ref = oracle.attention(U.bits(q), oracle.prune_24(Kb[:, :, :L + 1]), oracle.prune_24(Vb[:, :, :L + 1]),
                                    lens, 1.0)
    U.assert_attn_close(out, o_ref, lse, l_ref, tag=f"2:4 fused step splits {splits}")
    for cache, xb in ((kc, Kb), (vc, Vb)):
        bm, vals, _ = U.cache_np(cache)
        for b in range(B):
            ref = oracle.compress_24(xb[b:b + 1, :, :lens[b]], cap, int(lens[b]))
            assert np.array_equal(bm[b, :, :lens[b]], ref["bitmap"][0, :, :lens[b]])
            assert np.array_equal(vals[b, :, :lens[b] * 64], ref["values"][0, :, :lens[b] * 64])


def test_24_llama3_gqa_b8_ctx4096():
    B, Hq, Hkv, L = 8, 32, 8, 4096
    K = synth.keys(B, Hkv, L, D, 1007, DEV)
    V = synth.values(B, Hkv, L, D, 1007, DEV)
    kc = M.CompressedCache(B, Hkv, L, 0.5, pattern="2:4")
    vc = M.CompressedCache(B, Hkv, L, 0.5, pattern="2:4")
    M.mustafar_compress(K, L, 0.5, kc)
    M.mustafar_compress(V, L, 0.5, vc)
    q = synth.queries(B, Hq, D, 1007, DEV)
    out, lse = M.mustafar_decode_attn(q, kc, vc, torch.full((B,), L, dtype=torch.int32, device=DEV), L, 1.0)
    rows = [1, 6]
    streams = [(1, 0), (6, 5)]
    Kb, Vb = U.bits(K), U.bits(V)
    bm, vals, _ = U.cache_np(kc)
    for b, h in streams:
        ref = oracle.compress_24(Kb[b:b + 1, h:h + 1], L, L)
        assert np.array_equal(bm[b, h], ref["bitmap"][0, 0]) and np.array_equal(vals[b, h], ref["values"][0, 0])
    o_ref, l_ref = oracle.attention(U.bits(q[rows]), oracle.prune_24(Kb[rows]), oracle.prune_24(Vb[rows]),
                                    [L] * len(rows), 1.0)
    U.assert_attn_close(out[rows], o_ref, lse[rows], l_ref, tag="2:4 b8 ctx4096")


# ------------------------------------------------------------------------------------ channel-wise direction
def _channel_matches(cache, x_bits, lens):
    """Row b of a channel-wise cache against the oracle's compression of its first lens[b] tokens:
    bitmaps, the whole packed value run of every window, tile offsets and the window copy."""
    bm, vals, offs = U.cache_np(cache)
    win = cache.window_view().cpu().numpy().view(np.uint16)
    for b, Lb in enumerate(lens):
        ref = oracle.compress_channel(x_bits[b:b + 1, :, :Lb], cache.sparsity, cache.capacity, int(Lb))
        assert ref["keep"] == cache.keep
        assert np.array_equal(bm[b, :, :Lb], ref["bitmap"][0, :, :Lb]), ("bitmap", b)
        assert np.array_equal(vals[b], ref["values"][0]), ("values", b)
        assert np.array_equal(offs[b], ref["tile_offset"][0]), ("offsets", b)
        r = int(Lb) % 16
        assert np.array_equal(win[b, :, :r], ref["window"][0, :, :r]), ("window", b)


@pytest.mark.parametrize("s", [0.0, 0.3, 0.7, 0.9375])
def test_channel_compress_append_bit_exact(s):
    B, H, L0, L1, cap = 2, 3, 37, 100, 128
    rng = np.random.default_rng(81)
    x = synth.keys(B, H, L1, D, 81, "cpu").permute(0, 2, 1, 3).contiguous()  # [B, L, H, d] storage: strided
    xb = x.view(torch.int16).numpy().view(np.uint16).copy()
    xb[0, 16:32, 1] = rng.choice(TIE_ROWS, (16, D))  # a whole window of ties
    xb[1, 40:48, 2] = 0x3C00                          # equal magnitudes across tokens
    xb[0, 50, 0, :64] = 0x8000
    xdev = torch.from_numpy(xb.view(np.int16)).view(torch.float16).to(DEV)
    view = xdev.permute(0, 2, 1, 3)
    truth = np.ascontiguousarray(xb.transpose(0, 2, 1, 3))
    c = M.CompressedCache(B, H, cap, s, pattern="channel")
    M.mustafar_compress(view, L0, s, c)
    _channel_matches(c, truth, [L0] * B)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    for t in range(L0, L1):  # crosses the window edges at 48, 64, 80, 96
        M.mustafar_append(view[:, :, t], torch.full((B,), t, dtype=torch.int32, device=DEV), c, err=err)
        if t in (47, 48, 63, 77):
            _channel_matches(c, truth, [t + 1] * B)
    _channel_matches(c, truth, [L1] * B)
    assert int(err.item()) == 0
    # a full prefill of the same tokens gives the same bytes
    c2 = M.CompressedCache(B, H, cap, s, pattern="channel")
    M.mustafar_compress(view, L1, s, c2)
    assert torch.equal(c.bitmap, c2.bitmap) and torch.equal(c.values, c2.values)
    assert torch.equal(c.tile_offset, c2.tile_offset)


def test_channel_compress_empty_and_full_capacity():
    B, H, cap = 1, 2, 64
    x = synth.keys(B, H, cap, D, 82, DEV)
    c = M.CompressedCache(B, H, cap, 0.7, pattern="channel")
    M.mustafar_compress(x, 0, 0.7, c)
    assert not c.bitmap.any() and not c.values.any() and not c.window.any()
    assert c.tile_offset.tolist() == [0] * H
    M.mustafar_compress(x, cap, 0.7, c)
    _channel_matches(c, U.bits(x), [cap])
    assert not c.window.any()  # 64 tokens: no incomplete window


def test_channel_append_out_of_range_skips_row():
    B, H, L, cap = 2, 2, 20, 64
    x = synth.keys(B, H, L + 1, D, 83, DEV, capacity=cap)
    c = M.CompressedCache(B, H, cap, 0.7, pattern="channel")
    M.mustafar_compress(x, L, 0.7, c)
    before = (c.bitmap.clone(), c.values.clone(), c.window.clone())
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    M.mustafar_append(x[:, :, L].contiguous(), torch.tensor([-1, cap], dtype=torch.int32, device=DEV), c, err=err)
    assert int(err.item()) & M.DEVERR_POS_RANGE
    assert torch.equal(c.bitmap, before[0]) and torch.equal(c.values, before[1]) and torch.equal(c.window, before[2])


@pytest.mark.parametrize("v_pat,splits", [("channel", 0), ("topk", 0), ("channel", 3)])
def test_channel_decode_attn_ragged_lengths(v_pat, splits):
    # the caches hold 300 tokens; rows attend over fewer, so their last chunk ends inside a window
    # that was pruned with more tokens (its runs are read by popcount prefixes)
    B, Hq, Hkv, L, cap = 3, 8, 2, 300, 320
    sK, sV = 0.7, 0.5
    K = synth.keys(B, Hkv, L, D, 84, DEV, capacity=cap)
    V = synth.values(B, Hkv, L, D, 84, DEV, capacity=cap)
    kc = M.CompressedCache(B, Hkv, cap, sK, pattern="channel")
    vc = M.CompressedCache(B, Hkv, cap, sV, pattern=v_pat)
    M.mustafar_compress(K, L, sK, kc)
    M.mustafar_compress(V, L, sV, vc)
    q = synth.queries(B, Hq, D, 84, DEV)
    seq = torch.tensor([L, 203, 17], dtype=torch.int32)
    out, lse = M.mustafar_decode_attn(q, kc, vc, seq.to(DEV), L, 0.088, num_splits=splits)
    Kb, Vb = U.bits(K)[:, :, :L], U.bits(V)[:, :, :L]
    kp = oracle.prune_channel(Kb, sK)
    vp = oracle.prune_channel(Vb, sV) if v_pat == "channel" else oracle.prune(Vb, oracle.keep_count(D, sV))
    o_ref, l_ref = oracle.attention(U.bits(q), kp, vp, seq.numpy(), 0.088)
    U.assert_attn_close(out, o_ref, lse, l_ref, tag=f"channel K, {v_pat} V, splits {splits}")


@pytest.mark.parametrize("v_pat", ["channel", "2:4"])
def test_channel_decode_step_ragged_rows(v_pat):
    # rows move through their windows at different phases: row b skips its first lag[b] steps
    # (an out-of-range slot: no append, the row attends over nothing), then appends in order
    B, Hq, Hkv, L0, cap, steps = 3, 8, 2, 40, 128, 30
    lag = [0, 5, 11]
    sK, sV = 0.7, 0.5
    K = synth.keys(B, Hkv, L0, D, 85, DEV, capacity=cap)
    V = synth.values(B, Hkv, L0, D, 85, DEV, capacity=cap)
    kc = M.CompressedCache(B, Hkv, cap, sK, pattern="channel")
    vc = M.CompressedCache(B, Hkv, cap, sV, pattern=v_pat)
    M.mustafar_compress(K, L0, sK, kc)
    M.mustafar_compress(V, L0, sV, vc)
    lens = [L0] * B
    for st in range(steps):
        p = [L0 + st - lag[b] if st >= lag[b] else -1 for b in range(B)]
        kn, vn = synth.step_tokens(B, Hkv, D, 85, st, DEV)
        for b in range(B):
            if p[b] >= 0:
                K[b, :, p[b]] = kn[b]
                V[b, :, p[b]] = vn[b]
                lens[b] = p[b] + 1
        qs = synth.queries(B, Hq, D, 85, DEV, step=st)
        pos = torch.tensor(p, dtype=torch.int32, device=DEV)
        out, lse = M.mustafar_decode_step(qs, kn, vn, pos, kc, vc, L0 + steps, 1.0)
        if st in (0, 7, 8, 12, 29):
            live = [b for b in range(B) if p[b] >= 0]
            Kb, Vb = U.bits(K), U.bits(V)
            o_ref, l_ref = [], []
            for b in live:
                kp = oracle.prune_channel(Kb[b:b + 1, :, :lens[b]], sK)
                vp = (oracle.prune_channel(Vb[b:b + 1, :, :lens[b]], sV) if v_pat == "channel"
                      else oracle.prune_24(Vb[b:b + 1, :, :lens[b]]))
                o, l = oracle.attention(U.bits(qs[b:b + 1]), kp, vp, [lens[b]], 1.0)
                o_ref.append(o)
                l_ref.append(l)
            U.assert_attn_close(out[live], np.concatenate(o_ref), lse[live], np.concatenate(l_ref),
                                tag=f"channel step {st}")
    _channel_matches(kc, U.bits(K), lens)
    if v_pat == "channel":
        _channel_matches(vc, U.bits(V), lens)


def test_channel_decode_gqa16():
    # G = 16 (two row tiles of q heads) over channel-wise K and V caches, ragged rows
    B, Hq, Hkv, L, cap = 2, 32, 2, 181, 192
    K = synth.keys(B, Hkv, L, D, 87, DEV, capacity=cap)
    V = synth.values(B, Hkv, L, D, 87, DEV, capacity=cap)
    kc = M.CompressedCache(B, Hkv, cap, 0.7, pattern="channel")
    vc = M.CompressedCache(B, Hkv, cap, 0.5, pattern="channel")
    M.mustafar_compress(K, L, 0.7, kc)
    M.mustafar_compress(V, L, 0.5, vc)
    q = synth.queries(B, Hq, D, 87, DEV)
    seq = torch.tensor([L, 100], dtype=torch.int32)
    out, lse = M.mustafar_decode_attn(q, kc, vc, seq.to(DEV), L, 0.088)
    Kb, Vb = U.bits(K)[:, :, :L], U.bits(V)[:, :, :L]
    o_ref, l_ref = oracle.attention(U.bits(q), oracle.prune_channel(Kb, 0.7), oracle.prune_channel(Vb, 0.5),
                                    seq.numpy(), 0.088)
    U.assert_attn_close(out, o_ref, lse, l_ref, tag="channel G=16")


def test_channel_decode_step_same_bits_as_append_then_attend():
    B, Hq, Hkv, L0, cap = 4, 32, 8, 250, 320
    K = synth.keys(B, Hkv, L0, D, 86, DEV, capacity=cap)
    V = synth.values(B, Hkv, L0, D, 86, DEV, capacity=cap)
    caches = []
    for _ in range(2):
        kc = M.CompressedCache(B, Hkv, cap, 0.7, pattern="channel")
        vc = M.CompressedCache(B, Hkv, cap, 0.7, pattern="channel")
        M.mustafar_compress(K, L0, 0.7, kc)
        M.mustafar_compress(V, L0, 0.7, vc)
        caches.append((kc, vc))
    (kc, vc), (kc2, vc2) = caches
    for st in range(8):
        kn, vn = synth.step_tokens(B, Hkv, D, 86, st, DEV)
        pos = torch.full((B,), L0 + st, dtype=torch.int32, device=DEV)
        qs = synth.queries(B, Hq, D, 86, DEV, step=st)
        o1, l1 = M.mustafar_decode_step(qs, kn, vn, pos, kc, vc, cap, 1.0)
        M.mustafar_append(kn, pos, kc2)
        M.mustafar_append(vn, pos, vc2)
        o2, l2 = M.mustafar_decode_attn(qs, kc2, vc2, pos + 1, cap, 1.0)
        assert torch.equal(o1, o2) and torch.equal(l1, l2), f"step {st}"
    for a, b in ((kc, kc2), (vc, vc2)):
        assert torch.equal(a.bitmap, b.bitmap) and torch.equal(a.values, b.values) and torch.equal(a.window, b.window)


def test_channel_llama3_gqa_b8_ctx4096_s07():
    B, Hq, Hkv, L, cap = 8, 32, 8, 4096, 4160
    K = synth.keys(B, Hkv, L, D, 1009, DEV, capacity=cap)
    V = synth.values(B, Hkv, L, D, 1009, DEV, capacity=cap)
    kc = M.CompressedCache(B, Hkv, cap, 0.7, pattern="channel")
    vc = M.CompressedCache(B, Hkv, cap, 0.7, pattern="channel")
    M.mustafar_compress(K, L, 0.7, kc)
    M.mustafar_compress(V, L, 0.7, vc)
    q = synth.queries(B, Hq, D, 1009, DEV)
    out, lse = M.mustafar_decode_attn(q, kc, vc, torch.full((B,), L, dtype=torch.int32, device=DEV), L, 0.088)
    rows = [2, 7]
    Kb, Vb = U.bits(K)[:, :, :L], U.bits(V)[:, :, :L]
    bm, vals, _ = U.cache_np(kc)
    for b, h in ((2, 1), (7, 6)):
        ref = oracle.compress_channel(Kb[b:b + 1, h:h + 1], 0.7, cap, L)
        assert np.array_equal(bm[b, h], ref["bitmap"][0, 0]) and np.array_equal(vals[b, h], ref["values"][0, 0])
    o_ref, l_ref = oracle.attention(U.bits(q[rows]), oracle.prune_channel(Kb[rows], 0.7),
                                    oracle.prune_channel(Vb[rows], 0.7), [L] * len(rows), 0.088)
    U.assert_attn_close(out[rows], o_ref, lse[rows], l_ref, tag="channel b8 ctx4096")
    # one fused step opens a new window (a lone token keeps every channel)
    kn, vn = synth.step_tokens(B, Hkv, D, 1009, 0, DEV)
    pos = torch.full((B,), L, dtype=torch.int32, device=DEV)
    out, lse = M.mustafar_decode_step(q, kn, vn, pos, kc, vc, L + 1, 0.088)
    K[:, :, L], V[:, :, L] = kn, vn
    Kb, Vb = U.bits(K)[:, :, :L + 1], U.bits(V)[:, :, :L + 1]
    o_ref, l_ref = oracle.attention(U.bits(q[rows]), oracle.prune_channel(Kb[rows], 0.7),
                                    oracle.prune_channel(Vb[rows], 0.7), [L + 1] * len(rows), 0.088)
    U.assert_attn_close(out[rows], o_ref, lse[rows], l_ref, tag="channel b8 ctx4096 fused step")


# ------------------------------------------------------------------------------------ the workload shapes
def test_llama3_gqa_b1_ctx1024_s05():
    B, Hq, Hkv, L = 1, 32, 8, 1024
    K, V, q, kc, vc, seq = _setup(B, Hq, Hkv, L, L, 0.5, 0.5, 1001)
    U.assert_cache_matches(kc, U.bits(K), L)
    U.assert_cache_matches(vc, U.bits(V), L)
    out, lse = _attend(q, kc, vc, seq, L)
    o_ref, l_ref = U.oracle_attention(q, U.bits(K), U.bits(V), kc.keep, vc.keep, seq.numpy(), 1.0)
    U.assert_attn_close(out, o_ref, lse, l_ref, tag="b1 ctx1024")


@pytest.mark.parametrize("fused", [False, True])
def test_llama3_gqa_b8_ctx4096_s07_64_decode_steps(fused):
    B, Hq, Hkv, L0, steps = 8, 32, 8, 4096, 64
    cap = L0 + steps
    K, V, q, kc, vc, _ = _setup(B, Hq, Hkv, L0, cap, 0.7, 0.7, 1002)
    saved = {}
    for st in range(steps):
        kn, vn = synth.step_tokens(B, Hkv, D, 1002, st, DEV)
        K[:, :, L0 + st] = kn
        V[:, :, L0 + st] = vn
        pos = torch.full((B,), L0 + st, dtype=torch.int32, device=DEV)
        qs = synth.queries(B, Hq, D, 1002, DEV, step=st)
        if fused:
            out, lse = M.mustafar_decode_step(qs, kn, vn, pos, kc, vc, cap, 1.0)
        else:
            M.mustafar_append(kn, pos, kc)
            M.mustafar_append(vn, pos, vc)
            out, lse = M.mustafar_decode_attn(qs, kc, vc, pos + 1, cap, 1.0)
        if st in (0, 1, 31, 63):
            saved[st] = (qs.clone(), out.clone(), lse.clone())
    Kb, Vb = U.bits(K), U.bits(V)
    U.assert_cache_matches(kc, Kb, cap)
    U.assert_cache_matches(vc, Vb, cap)
    kp, vp = oracle.prune(Kb, kc.keep), oracle.prune(Vb, vc.keep)
    for st, (qs, out, lse) in saved.items():
        o_ref, l_ref = oracle.attention(U.bits(qs), kp, vp, [L0 + st + 1] * B, 1.0)
        U.assert_attn_close(out, o_ref, lse, l_ref, tag=f"decode step {st}")


def test_mistral_gqa_b4_ctx32k_sk07_sv05():
    B, Hq, Hkv, L = 4, 32, 8, 32768
    K, V, q, kc, vc, seq = _setup(B, Hq, Hkv, L, L, 0.7, 0.5, 1003)
    streams = [(0, 0), (1, 3), (2, 7), (3, 5)]
    Kb, Vb = U.bits(K), U.bits(V)
    U.assert_cache_matches(kc, np.stack([Kb[b, h] for b, h in streams]), L, streams)
    U.assert_cache_matches(vc, np.stack([Vb[b, h] for b, h in streams]), L, streams)
    out, lse = _attend(q, kc, vc, seq, L)
    o_ref, l_ref = U.oracle_attention(q, Kb, Vb, kc.keep, vc.keep, seq.numpy(), 1.0)
    U.assert_attn_close(out, o_ref, lse, l_ref, tag="b4 ctx32k")


@pytest.mark.parametrize("s", [0.3, 0.5, 0.7])
def test_prefill_compress_b8_16k_h8(s):
    B, L, H = 8, 16384, 8
    g = torch.Generator(device=DEV)
    g.manual_seed(1004)
    x = torch.randn(B, L, H, D, generator=g, device=DEV).to(torch.float16)  # [B, L, H, d] storage
    c = M.CompressedCache(B, H, L, s)
    M.mustafar_compress(x.permute(0, 2, 1, 3), L, s, c)
    streams = [(0, 0), (3, 4), (7, 7)]
    xb = U.bits(x)
    U.assert_cache_matches(c, np.stack([xb[b, :, h] for b, h in streams]), L, streams)
    assert c.nbytes() == B * H * oracle.compressed_bytes(L, c.keep, L, D)


SWEEP_POINTS = [  # (Hq, Hkv, B, L, s)
    (32, 8, 1, 4096, 0.0), (32, 32, 8, 4096, 0.3), (32, 8, 32, 4096, 0.5), (32, 32, 1, 32768, 0.7),
    (32, 8, 8, 32768, 0.9), (32, 32, 1, 131072, 0.5), (32, 8, 32, 131072, 0.7), (32, 32, 32, 131072, 0.7),
]


@pytest.mark.parametrize("Hq,Hkv,B,L,s", SWEEP_POINTS)
def test_sweep_points_sampled(Hq, Hkv, B, L, s):
    """Full-size sweep points; the oracle checks sampled (b, kv head) streams and their q heads."""
    K, V, q, kc, vc, seq = _setup(B, Hq, Hkv, L, L, s, s, 2000 + B + Hkv + int(10 * s))
    out, lse = _attend(q, kc, vc, seq, L)
    dense, _ = M.mustafar_dense_decode_attn(q, K, V, seq.to(DEV), L, 1.0)
    rng = np.random.default_rng(B * L)
    picks = sorted({(0, 0), (B - 1, Hkv - 1)} | {(int(rng.integers(B)), int(rng.integers(Hkv))) for _ in range(2)})
    G = Hq // Hkv
    for b, h in picks:
        Kb, Vb = U.bits(K[b, h]), U.bits(V[b, h])
        U.assert_cache_matches(kc, Kb[None], L, [(b, h)])
        U.assert_cache_matches(vc, Vb[None], L, [(b, h)])
        qb = U.bits(q[b:b + 1, h * G:(h + 1) * G])
        o_ref, l_ref = U.oracle_attention(qb, Kb[None, None], Vb[None, None], kc.keep, vc.keep, [L], 1.0)
        U.assert_attn_close(out[b:b + 1, h * G:(h + 1) * G], o_ref, lse[b:b + 1, h * G:(h + 1) * G], l_ref,
                            tag=f"sweep b{b} h{h}")
        d_ref, _ = oracle.attention(qb, Kb[None, None], Vb[None, None], [L], 1.0)
        U.assert_attn_close(dense[b:b + 1, h * G:(h + 1) * G], d_ref, tag=f"dense b{b} h{h}")
    del K, V, kc, vc
    torch.cuda.empty_cache()

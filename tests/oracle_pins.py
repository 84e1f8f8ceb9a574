"""Checks that pin the oracle to the pages and to mathematics, not to itself.

Each ``pin_*`` takes an oracle namespace ``O`` (the real ``oracle`` package, or a
mutant built by ``test_oracle_mutants.py``) and raises ``AssertionError`` when the
oracle disagrees with the fact it checks.  Facts used:

* hand-derived fixtures under ``tests/golden/`` (selection, bitmap bit order,
  value order, keep-count rounding, a two-token attention with logits 0 and ln 3);
* brute-force rank counting on tiny tie-heavy inputs;
* the threshold invariant of a top-k selection and popcount == k;
* decompress(compress(x)) == prune(x) and the closed-form compressed size;
* attention at sparsity 0 against torch's float64 ``scaled_dot_product_attention``;
* L = 1 gives o = V~_0 exactly; softmax weights sum to 1; token-permutation
  invariance; a GQA group with equal queries gives equal outputs.
* per-head keep counts: with one keep for every head the per-head layout equals the uniform
  one byte for byte; the streams tile the value array exactly; brute-force ranks and popcounts
  per head; round trip to the per-head pruned cache; append == compress.
* 2:4 pattern: a hand-derived 32-channel fixture (selection, bitmap word, packed values);
  exactly 2 of every 4 channels; brute-force ranks per group; round trip; append == compress.
* channel-wise direction: a hand-derived fixture (window counts, a partial window with ties, a
  full window with a tie at the keep boundary); counts and pairwise dominance per (window,
  channel); a full window equals brute-force token ranks of the transposed window; the window
  slots and the round trip; sparsity 0 equals the token format with k = d; append == compress.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# fp16 bit patterns with many ties: zeros of both signs, smallest/largest
# subnormals, 1, 2, the largest finite value, of both signs.
TIE_HEAVY = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x03FF, 0x3C00, 0xBC00, 0x4000, 0xC000,
                      0x7BFF, 0xFBFF], dtype=np.uint16)


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _d32_vector():
    g = _load("select_d32.json")
    spec = g["x_hex_by_channel"]
    x = np.zeros(32, dtype=np.uint16)
    for c in range(32):
        if str(c) in spec:
            x[c] = int(spec[str(c)], 16)
        elif c % 2 == 1:
            x[c] = int(spec["odd_11_to_31"], 16)
        else:
            x[c] = int(spec["even_12_to_30"], 16)
    return x, g


def rand_bits(rng, shape, tie_heavy=False):
    if tie_heavy:
        return rng.choice(TIE_HEAVY, size=shape).astype(np.uint16)
    x = rng.standard_normal(shape).astype(np.float16)
    return x.view(np.uint16)


# ----------------------------------------------------------------------------- selection
def pin_golden_selection(O):
    x, g = _d32_vector()
    for case in g["cases"]:
        k = case["k"]
        mask = O.select_sort(x[None, :], k)[0]
        words = O.bitmap_words(mask[None, :])[0]
        assert int(words[0]) == int(case["bitmap_hex"], 16), (k, hex(int(words[0])))
        comp = O.compress(x[None, None, None, :], k, 64)
        vals = comp["values"][0, 0, :k]
        if isinstance(case["values_hex"], list):
            assert [int(v) for v in vals] == [int(h, 16) for h in case["values_hex"]], k
        else:
            keep = [c for c in range(32) if (int(case["bitmap_hex"], 16) >> c) & 1]
            assert [int(v) for v in vals] == [int(x[c]) for c in keep], k
        assert int(comp["bitmap"][0, 0, 0, 0]) == int(case["bitmap_hex"], 16)


def pin_golden_keep_count(O):
    for case in _load("keep_count.json")["cases"]:
        assert O.keep_count(case["d"], case["s"]) == case["k"], case


def pin_bruteforce_selection(O):
    rng = np.random.default_rng(11)
    for d in (32, 128):
        for tie in (True, False):
            x = rand_bits(rng, (6, d), tie_heavy=tie)
            for k in (1, 2, d // 3, d // 2, d - 1, d):
                a = O.select_sort(x, k)
                b = O.select_rank_bruteforce(x, k)
                assert np.array_equal(a, b), (d, tie, k)
    # exhaustive: every 6-channel pattern over a 3-symbol alphabet {+0, -0, 1.0} padded to 32
    alphabet = np.array([0x0000, 0x8000, 0x3C00], dtype=np.uint16)
    idx = np.indices((3,) * 6).reshape(6, -1).T
    xs = np.zeros((idx.shape[0], 32), dtype=np.uint16)
    xs[:, :6] = alphabet[idx]
    xs[:, 6:] = 0x3800  # 0.5 fills the rest
    for k in (1, 3, 26, 27, 29):
        assert np.array_equal(O.select_sort(xs, k), O.select_rank_bruteforce(xs, k)), k


def pin_threshold_invariant(O):
    rng = np.random.default_rng(12)
    for tie in (True, False):
        x = rand_bits(rng, (64, 128), tie_heavy=tie)
        m = (x & 0x7FFF).astype(np.int64)
        for k in (1, 13, 39, 64, 90, 127, 128):
            mask = O.select_sort(x, k)
            assert (mask.sum(axis=1) == k).all()
            for r in range(x.shape[0]):
                kept, pruned = m[r][mask[r]], m[r][~mask[r]]
                if pruned.size == 0:
                    continue
                assert kept.min() >= pruned.max(), "a pruned element outranks a kept one"
                edge = kept.min()
                if pruned.max() == edge:
                    ki = np.nonzero(mask[r] & (m[r] == edge))[0]
                    pi = np.nonzero(~mask[r] & (m[r] == edge))[0]
                    assert ki.max() < pi.min(), "tie not resolved toward the lower channel"


# ----------------------------------------------------------------------------- format
def pin_roundtrip_and_popcount(O):
    rng = np.random.default_rng(13)
    B, H, L, d, cap = 2, 3, 150, 128, 192
    x = rand_bits(rng, (B, H, L, d))
    x[0, 0, 5] = rand_bits(rng, (d,), tie_heavy=True)
    for k in (128, 90, 64, 39, 13, 1):
        comp = O.compress(x, k, cap)
        words = comp["bitmap"][:, :, :L]
        pop = np.vectorize(lambda w: bin(int(w)).count("1"))(words).sum(axis=-1)
        assert (pop == k).all()
        dec = O.decompress(comp["bitmap"], comp["values"], k, L, d)
        assert np.array_equal(dec, O.prune(x, k))
        # pruned positions hold +0, kept positions hold the input bits exactly
        mask = O.bitmap_to_mask(words, d)
        assert np.array_equal(dec[mask], x[mask]) and (dec[~mask] == 0).all()
        # tile offsets = popcount prefix sums at every 64-token boundary = 64*i*k
        prefix = np.concatenate([[0], np.cumsum(pop[0, 0])])
        for i in range(cap // 64):
            expect = prefix[64 * i] if 64 * i <= L else 64 * i * k
            assert int(comp["tile_offset"][0, 0, i]) == expect == 64 * i * k


def pin_compressed_size(O):
    # closed form per stream: 16 B bitmap + 2k B values per token, 4 B per 64-token tile
    cases = [(4096, 39, 4160, 4096 * (16 + 78) + 4 * 65), (16384, 90, 16384, 16384 * 196 + 4 * 256),
             (1024, 64, 1024, 1024 * 144 + 4 * 16), (1, 128, 64, 16 + 256 + 4)]
    for L, k, cap, expect in cases:
        assert O.compressed_bytes(L, k, cap, 128) == expect
    rng = np.random.default_rng(14)
    x = rand_bits(rng, (1, 1, 130, 128))
    comp = O.compress(x, 39, 192)
    used = 130 * 16 + 130 * 39 * 2 + comp["tile_offset"].nbytes
    assert used == O.compressed_bytes(130, 39, 192, 128)
    # the pages' ratios (45% of dense at 70% sparsity, 65% at 50%) are upper bounds for this format
    for s, bound in ((0.7, 0.45), (0.5, 0.65)):
        k = O.keep_count(128, s)
        ratio = O.compressed_bytes(16384, k, 16384, 128) / (16384 * 256)
        assert ratio < bound, (s, ratio)


# ----------------------------------------------------------------------------- attention
def _sdpa_f64(q, K, V, scale, G):
    # q [B,Hq,d], K/V [B,Hkv,L,d] float64 -> [B,Hq,d]
    qt = torch.from_numpy(q)[:, :, None, :]
    Kt = torch.from_numpy(K).repeat_interleave(G, dim=1)
    Vt = torch.from_numpy(V).repeat_interleave(G, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    return o[:, :, 0, :].numpy()


def pin_dense_limit_sdpa(O):
    rng = np.random.default_rng(15)
    B, Hq, Hkv, L, d = 2, 8, 2, 77, 128
    q = rand_bits(rng, (B, Hq, d))
    K = rand_bits(rng, (B, Hkv, L, d))
    V = rand_bits(rng, (B, Hkv, L, d))
    k = O.keep_count(d, 0.0)
    kc, vc = O.compress(K, k, 128), O.compress(V, k, 128)
    seq = np.full(B, L)
    o, lse = O.attention_over_compressed(q, kc, vc, seq, 0.37, d)
    f = lambda b: b.view(np.float16).astype(np.float64)
    ref = _sdpa_f64(f(q), f(K), f(V), 0.37, Hq // Hkv)
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)
    z = 0.37 * np.einsum("bgjd,bgld->bgjl", f(q).reshape(B, Hkv, Hq // Hkv, d), f(K))
    lse_ref = torch.logsumexp(torch.from_numpy(z), dim=-1).numpy().reshape(B, Hq)
    assert np.allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def pin_golden_attention(O):
    g = _load("attention_tiny.json")
    d = 32
    q = np.zeros((1, 1, d), np.float16); q[0, 0, 0] = 1; q[0, 0, 1] = 1
    K = np.zeros((1, 1, 2, d), np.float16)
    K[0, 0, 0, 4:7] = 5
    K[0, 0, 1, 0], K[0, 0, 1, 1], K[0, 0, 1, 2], K[0, 0, 1, 3] = 1, 0.5, 2, 2
    V = np.zeros((1, 1, 2, d), np.float16)
    V[0, 0, 0, :] = 1; V[0, 0, 0, :3] = 4
    V[0, 0, 1, :] = 0.5; V[0, 0, 1, :3] = 8
    scale = float(np.float32(math.log(3)))
    kc = O.compress(K.view(np.uint16), 3, 64)
    vc = O.compress(V.view(np.uint16), 3, 64)
    o, lse = O.attention_over_compressed(q.view(np.uint16), kc, vc, [2], scale, d)
    e = g["expected"]
    assert np.allclose(o[0, 0, :3], e["o_c0_c2"], atol=e["tol"])
    assert np.allclose(o[0, 0, 3:], e["o_other"], atol=e["tol"])
    assert abs(lse[0, 0] - e["lse"]) < e["tol"]


def pin_attention_invariants(O):
    rng = np.random.default_rng(16)
    B, Hq, Hkv, L, d = 2, 8, 2, 70, 128
    G = Hq // Hkv
    K = rand_bits(rng, (B, Hkv, L, d))
    V = rand_bits(rng, (B, Hkv, L, d))
    q = rand_bits(rng, (B, Hq, d))
    k = 39
    kp, vp = O.prune(K, k), O.prune(V, k)
    # L = 1: the output is the single pruned value row, exactly
    o1, lse1 = O.attention(q, kp, vp, [1, 1], 1.0)
    f = lambda b: b.view(np.float16).astype(np.float64)
    for b in range(B):
        for hq in range(Hq):
            assert np.array_equal(o1[b, hq], f(vp[b, hq // G, 0]))
    # weights sum to one: with V~ replaced by all-ones rows, o == 1 everywhere
    ones = np.full_like(vp, 0x3C00)
    o_ones, _ = O.attention(q, kp, ones, [L, L - 5], 0.8)
    assert np.allclose(o_ones, 1.0, rtol=0, atol=1e-13)
    # token permutation invariance
    perm = rng.permutation(L)
    oa, la = O.attention(q, kp, vp, [L, L], 0.8)
    ob, lb = O.attention(q, kp[:, :, perm], vp[:, :, perm], [L, L], 0.8)
    assert np.allclose(oa, ob, rtol=1e-12, atol=1e-13) and np.allclose(la, lb, rtol=1e-12)
    # equal queries inside a GQA group give equal outputs; different kv heads differ
    qg = q.copy()
    for g_ in range(Hkv):
        qg[:, g_ * G:(g_ + 1) * G] = q[:, g_ * G][:, None]
    og, _ = O.attention(qg, kp, vp, [L, L], 0.8)
    for g_ in range(Hkv):
        for j in range(1, G):
            assert np.array_equal(og[:, g_ * G + j], og[:, g_ * G])
    assert not np.allclose(og[:, 0], og[:, G])
    # q head hq reads kv head hq // G: zeroing kv head 1's values changes only heads G..2G-1
    vz = vp.copy(); vz[:, 1] = 0
    oz, _ = O.attention(q, kp, vz, [L, L], 0.8)
    assert np.array_equal(oz[:, :G], oa[:, :G]) and np.allclose(oz[:, G:2 * G], 0)


def pin_append_equals_compress(O):
    rng = np.random.default_rng(17)
    B, H, L, d, cap, k = 2, 2, 70, 128, 128, 39
    x = rand_bits(rng, (B, H, L + 3, d))
    full = O.compress(x, k, cap, L + 3)
    part = O.compress(x, k, cap, L)
    for s in range(3):
        O.append(part, x[:, :, L + s], np.full(B, L + s))
    for key in ("bitmap", "values", "tile_offset"):
        assert np.array_equal(full[key], part[key]), key


# ----------------------------------------------------------------------------- keep count per head
def pin_heads_layout(O):
    rng = np.random.default_rng(19)
    B, H, L, d, cap = 2, 4, 100, 128, 128
    x = rand_bits(rng, (B, H, L, d))
    x[1, 2, 7] = rand_bits(rng, (d,), tie_heavy=True)
    # one keep count for every head: the per-head layout is the uniform layout, byte for byte
    for k in (39, 64):
        u, p = O.compress(x, k, cap), O.compress_heads(x, [k] * H, cap)
        assert np.array_equal(p["values"], u["values"].reshape(-1))
        assert np.array_equal(p["bitmap"], u["bitmap"]) and np.array_equal(p["tile_offset"], u["tile_offset"])
    hk = [13, 128, 1, 64]
    c = O.compress_heads(x, hk, cap)
    # the streams' value ranges tile the array exactly, batch-major then head order
    spans = [(O.value_base_heads(b, h, hk, cap), O.value_base_heads(b, h, hk, cap) + cap * hk[h])
             for b in range(B) for h in range(H)]
    assert spans[0][0] == 0 and spans[-1][1] == c["values"].size == B * cap * sum(hk)
    assert all(a[1] == nxt[0] for a, nxt in zip(spans, spans[1:]))
    # every token of head h keeps exactly hk[h] channels, chosen by the brute-force rank rule
    pop = np.vectorize(lambda w: bin(int(w)).count("1"))(c["bitmap"][:, :, :L]).sum(-1)
    for h, k in enumerate(hk):
        assert (pop[:, h] == k).all()
        mask = O.bitmap_to_mask(c["bitmap"][:, h:h + 1, :4], d)
        assert np.array_equal(mask, O.select_rank_bruteforce(x[:, h:h + 1, :4], k))
        assert all(int(c["tile_offset"][b, h, i]) == 64 * i * k for b in range(B) for i in range(cap // 64))
    # round trip: the packed values put back by the bitmap give the per-head pruned cache
    dec = O.decompress_heads(c, L, d)
    assert np.array_equal(dec, O.prune_heads(x, hk))
    assert all(np.array_equal(dec[:, h:h + 1], O.prune(x[:, h:h + 1], k)) for h, k in enumerate(hk))


def pin_heads_append_equals_compress(O):
    rng = np.random.default_rng(23)
    B, H, L, d, cap, hk = 2, 3, 62, 128, 128, [90, 13, 39]
    x = rand_bits(rng, (B, H, L + 3, d))
    full = O.compress_heads(x, hk, cap, L + 3)
    part = O.compress_heads(x, hk, cap, L)
    for s in range(3):
        O.append_heads(part, x[:, :, L + s], np.full(B, L + s))
    for key in ("bitmap", "values", "tile_offset"):
        assert np.array_equal(full[key], part[key]), key


# ----------------------------------------------------------------------------- 2:4 comparison pattern
def pin_golden_24(O):
    g = _load("select_24.json")
    x = np.array([int(h, 16) for h in g["x_hex_by_channel"]], dtype=np.uint16).reshape(1, 1, 1, 32)
    mask = O.select_24(x)[0, 0, 0]
    assert np.flatnonzero(mask).tolist() == g["kept_channels"]
    assert int(O.bitmap_words(mask[None])[0, 0]) == int(g["bitmap_word_hex"], 16)
    comp = O.compress_24(x, 64)
    assert comp["k"] == 16
    assert comp["values"][0, 0, :16].tolist() == [int(h, 16) for h in g["packed_values_hex"]]


def pin_24_structure(O):
    rng = np.random.default_rng(29)
    B, H, L, d, cap = 2, 2, 70, 128, 128
    x = rand_bits(rng, (B, H, L, d))
    x[0, 1, 3] = rand_bits(rng, (d,), tie_heavy=True)
    x[1, 0, 9] = 0x3C00  # every magnitude equal
    mask = O.select_24(x)
    groups = mask.reshape(B, H, L, d // 4, 4)
    assert (groups.sum(-1) == 2).all()  # exactly two of every four, so d/2 per token
    # brute-force ranks inside each group (independent of the sort-based selection)
    xg = x.reshape(B, H, L, d // 4, 4)
    assert np.array_equal(groups, O.select_rank_bruteforce(xg, 2))
    comp = O.compress_24(x, cap)
    assert comp["k"] == d // 2
    dec = O.decompress(comp["bitmap"], comp["values"], d // 2, L, d)
    assert np.array_equal(dec, O.prune_24(x))
    assert np.array_equal(O.bitmap_to_mask(comp["bitmap"][:, :, :L], d), mask)
    part = O.compress_24(x, cap, L - 2)
    for s in range(2):
        O.append_24(part, x[:, :, L - 2 + s], np.full(B, L - 2 + s))
    for key in ("bitmap", "values", "tile_offset"):
        assert np.array_equal(comp[key], part[key]), key


# ----------------------------------------------------------------------------- channel-wise direction
def _channel_partial_fixture():
    g = _load("select_channel.json")["partial_window"]
    x = np.zeros((1, 1, 4, 32), dtype=np.uint16)
    for t in range(4):
        for c in range(32):
            x[0, 0, t, c] = int(g["x_hex_by_token_and_class"][t][c % 4], 16)
    return x, g


def pin_golden_channel(O):
    g = _load("select_channel.json")
    for case in g["window_counts"]["cases"]:
        F = O.window_prune_count(case["s"])
        assert F == case["F"], case
        assert O.window_keep(case["n"], F) == case["window_keep"], case
    for case in g["window_counts"]["keep_count_channel"]:
        assert O.keep_count_channel(case["d"], case["s"]) == case["keep"], case
    # a partial window: selection with ties, bitmap words, token-major packing, the dense copy
    x, p = _channel_partial_fixture()
    c = O.compress_channel(x, p["s"], 64)
    assert [int(w) for w in c["bitmap"][0, 0, :4, 0]] == [int(h, 16) for h in p["bitmap_words_hex"]]
    expect = []
    for t, grp in enumerate(p["packed_values_hex_per_token_group"]):
        assert 8 * len(grp) == p["values_per_token"][t]
        expect += [int(h, 16) for h in grp] * 8
    assert c["values"][0, 0, :64].tolist() == expect
    assert not c["values"][0, 0, 64:].any()
    assert np.array_equal(c["window"][0, 0, :4], x[0, 0])
    # a full window: the tie at the keep boundary goes to the lower token
    f = g["full_window"]
    t = np.arange(16)
    col = np.where(t % 2 == 1, -(t % 5), t % 5).astype(np.float16).view(np.uint16)
    xf = np.repeat(col[:, None], 32, axis=1)[None, None]
    cf = O.compress_channel(xf, f["s"], 64)
    assert cf["keep"] == f["keep"]
    words = cf["bitmap"][0, 0, :16, 0]
    assert np.flatnonzero(words).tolist() == f["kept_tokens"]
    assert all(int(words[i]) == 0xFFFFFFFF for i in f["kept_tokens"])
    assert cf["values"][0, 0, :16 * f["keep"]].tolist() == sum([[int(h, 16)] * 32 for h in f["kept_value_hex"]], [])
    assert not cf["window"].any()  # 16 tokens: no incomplete window


def pin_channel_selection_rules(O):
    """Counts per (window, channel) and the dominance rule, by brute force over token pairs."""
    rng = np.random.default_rng(31)
    for s in (0.7, 0.5, 0.3, 0.9375, 0.0):
        F = O.window_prune_count(s)
        for T, ties in ((16, False), (37, True), (5, True)):
            x = rand_bits(rng, (2, T, 8), tie_heavy=ties)
            mask = O.select_channel(x, F)
            m = O.magnitude_key(x)
            for t0 in range(0, T, 16):
                n = min(16, T - t0)
                for b in range(2):
                    for c in range(8):
                        kept = [t0 + i for i in range(n) if mask[b, t0 + i, c]]
                        drop = [t0 + i for i in range(n) if not mask[b, t0 + i, c]]
                        assert len(kept) == O.window_keep(n, F)
                        for i in kept:
                            for j in drop:
                                assert m[b, i, c] > m[b, j, c] or (m[b, i, c] == m[b, j, c] and i < j)
        # a full window is a token-wise selection of the transposed window (brute-force ranks)
        x = rand_bits(rng, (3, 16, 8), tie_heavy=True)
        assert np.array_equal(np.swapaxes(O.select_channel(x, F), -1, -2),
                              O.select_rank_bruteforce(np.swapaxes(x, -1, -2), 16 - F))


def pin_channel_layout_roundtrip(O):
    rng = np.random.default_rng(37)
    B, H, L, d, cap = 2, 3, 70, 128, 128
    x = rand_bits(rng, (B, H, L, d))
    x[1, 2, 40:56] = rand_bits(rng, (16, d), tie_heavy=True)
    for s in (0.7, 0.3):
        F = O.window_prune_count(s)
        c = O.compress_channel(x, s, cap)
        keep = c["keep"]
        assert keep * 16 == d * (16 - F)
        dec = O.decompress_channel(c, L, d)
        assert np.array_equal(dec, O.prune_channel(x, s))
        # every window's values fill its slot from the start: a full window exactly, the last one
        # d * window_keep(n) of its 16 * keep
        bits = O.bitmap_to_mask(c["bitmap"][:, :, :L], d)
        for t0 in range(0, L, 16):
            n = min(16, L - t0)
            per_ch = bits[:, :, t0:t0 + n].sum(axis=2)
            assert (per_ch == O.window_keep(n, F)).all()
            used = d * O.window_keep(n, F)
            assert used <= 16 * keep and (n < 16 or used == 16 * keep)
            # the packed run is exactly the window's kept entries, token by token
            for b in range(B):
                for h in range(H):
                    assert np.array_equal(c["values"][b, h, t0 * keep:t0 * keep + used],
                                          x[b, h, t0:t0 + n][bits[b, h, t0:t0 + n]])
        assert all(int(c["tile_offset"][b, h, i]) == 64 * i * keep
                   for b in range(B) for h in range(H) for i in range(cap // 64))
        assert np.array_equal(c["window"][:, :, :L % 16], x[:, :, L - L % 16:L])
    # nothing pruned: the channel-wise cache is the token format with k = d, byte for byte
    c0, t0c = O.compress_channel(x, 0.0, cap), O.compress(x, d, cap)
    for key in ("bitmap", "values", "tile_offset"):
        assert np.array_equal(c0[key], t0c[key]), key


def pin_channel_append_equals_compress(O):
    rng = np.random.default_rng(41)
    B, H, d, cap = 2, 2, 128, 128
    x = rand_bits(rng, (B, H, 70, d))
    for s, L0 in ((0.7, 37), (0.5, 16), (0.3, 0)):
        part = O.compress_channel(x, s, cap, L0)
        for p in range(L0, 70):  # crosses the window edges at 48 and 64
            O.append_channel(part, x[:, :, p], np.full(B, p))
            if p in (47, 50, 69):
                full = O.compress_channel(x, s, cap, p + 1)
                for key in ("bitmap", "values", "tile_offset"):
                    assert np.array_equal(full[key], part[key]), (s, p, key)
                r = (p + 1) % 16
                assert np.array_equal(full["window"][:, :, :r], part["window"][:, :, :r])


ALL_PINS = [pin_golden_selection, pin_golden_keep_count, pin_bruteforce_selection, pin_threshold_invariant,
            pin_roundtrip_and_popcount, pin_compressed_size, pin_dense_limit_sdpa, pin_golden_attention,
            pin_attention_invariants, pin_append_equals_compress, pin_heads_layout, pin_heads_append_equals_compress,
            pin_golden_24, pin_24_structure, pin_golden_channel, pin_channel_selection_rules,
            pin_channel_layout_roundtrip, pin_channel_append_equals_compress]


def failing_pins(O):
    bad = []
    for pin in ALL_PINS:
        try:
            pin(O)
        except Exception:  # a mutant may also crash; that counts as caught
            bad.append(pin.__name__)
    return bad

"""Plain CPU oracle for Mustafar's hot path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this module.  The product path (the CUDA library and its binding) never
does; it shares no code, table or helper with this file.

What it computes, and from which passage:

* Per-token magnitude pruning of the Key and Value caches to an unstructured
  sparsity (MUSTAFAR summary, atlas.scime.ai, "Approach"; Mustafar abstract,
  catalyzex author page): every (token, kv head) vector of ``d`` channels keeps
  its ``k`` largest-magnitude elements and zeroes the rest.
* A bitmap-based compressed format (same two passages): a bitmap marks the kept
  positions, the kept fp16 values are packed, and per-tile offsets locate them.
  The pages give no layout; this oracle follows the library's own choices, which
  are written out in ``keep_count``, ``compress`` and ``compressed_bytes`` below.
* Channel-wise magnitude pruning, the other pruning direction the README names
  (Part II, the K/V [t/c] naming): each channel is pruned across the tokens of
  16-token windows; the readings it takes are written out above ``WINDOW`` below.
* Decode attention over the pruned caches (the abstract: the kernel computes
  "directly over compressed caches"): the exact result it must reach is plain
  softmax attention over the pruned K and V, computed here in float64.

Readings where the pages are silent (each is listed in the design notes):
keep-count ``k = d - floor(s*d)``; magnitude key = fp16 bits with the sign bit
cleared; ties go to the lower channel index; kept values are packed in
ascending channel order; bit ``c % 32`` of 32-bit word ``c // 32`` marks channel
``c``; tiles are 64 tokens with 32-bit offsets counted in elements; every token,
including the newest, is pruned; the new decode token attends to itself; q head
``hq`` reads kv head ``hq // (Hq/Hkv)``.

Arrays of fp16 numbers are passed as their raw bits (``np.uint16``) so that both
sides see identical inputs and the compressed bytes can be compared exactly.
"""
from __future__ import annotations

import math

import numpy as np

TILE_TOKENS = 64
WORD_BITS = 32


# --------------------------------------------------------------------------------------
# keep count and magnitude key
# --------------------------------------------------------------------------------------
def keep_count(d: int, sparsity: float) -> int:
    """Number of channels a token keeps: ``d - floor(s*d)``.

    Sparsity s is the fraction pruned (README, Part II: a setting of 0.5 prunes half the channels).
    ``s`` arrives as a 32-bit float (as it does through the library's C call) and
    the product is formed in double, so the target sparsity is never exceeded.
    """
    s = float(np.float32(sparsity))
    if not (0.0 <= s < 1.0):
        raise ValueError("sparsity must lie in [0, 1)")
    return int(d - math.floor(s * d))


def magnitude_key(x_bits: np.ndarray) -> np.ndarray:
    """|x| ordering key of fp16 bit patterns: the 15 low bits (sign cleared).

    For finite fp16 numbers this integer order equals the order of |x|; +0 and -0
    share key 0.  Inf and NaN patterns rank above every finite value.
    """
    return (np.asarray(x_bits, dtype=np.uint16) & np.uint16(0x7FFF)).astype(np.int32)


# --------------------------------------------------------------------------------------
# selection (per-token magnitude pruning)
# --------------------------------------------------------------------------------------
def select_sort(x_bits: np.ndarray, k: int) -> np.ndarray:
    """Boolean kept-mask over the last axis: the ``k`` largest keys, lower channel first on ties.

    Implemented as a stable sort of the negated keys: equal keys keep their
    channel order, so the first ``k`` positions of the sorted order are the kept set.
    """
    m = magnitude_key(x_bits)
    d = m.shape[-1]
    order = np.argsort(0x7FFF - m, axis=-1, kind="stable")
    keep_idx = order[..., :k]
    mask = np.zeros(m.shape, dtype=bool)
    np.put_along_axis(mask, keep_idx, True, axis=-1)
    assert mask.shape[-1] == d
    return mask


def select_rank_bruteforce(x_bits: np.ndarray, k: int) -> np.ndarray:
    """Same selection by rank counting, for tiny inputs only.

    rank(c) = #{j : m_j > m_c} + #{j < c : m_j == m_c}; channel c is kept iff rank(c) < k.
    """
    m = magnitude_key(x_bits)
    flat = m.reshape(-1, m.shape[-1])
    out = np.zeros(flat.shape, dtype=bool)
    d = flat.shape[1]
    for r in range(flat.shape[0]):
        row = flat[r]
        for c in range(d):
            rank = 0
            for j in range(d):
                if row[j] > row[c] or (row[j] == row[c] and j < c):
                    rank += 1
            out[r, c] = rank < k
    return out.reshape(m.shape)


def prune(x_bits: np.ndarray, k: int) -> np.ndarray:
    """Pruned fp16 bits: kept elements keep their exact bits (sign, -0 included), the rest become +0."""
    x = np.asarray(x_bits, dtype=np.uint16)
    return np.where(select_sort(x, k), x, np.uint16(0)).astype(np.uint16)


# --------------------------------------------------------------------------------------
# bitmap format
# --------------------------------------------------------------------------------------
def bitmap_words(mask: np.ndarray) -> np.ndarray:
    """Pack a [..., d] kept-mask into [..., d/32] uint32 words, channel c -> bit c%32 of word c//32."""
    d = mask.shape[-1]
    assert d % WORD_BITS == 0
    m = mask.reshape(mask.shape[:-1] + (d // WORD_BITS, WORD_BITS)).astype(np.uint64)
    weights = (np.uint64(1) << np.arange(WORD_BITS, dtype=np.uint64))
    return (m * weights).sum(axis=-1).astype(np.uint32)


def bitmap_to_mask(words: np.ndarray, d: int) -> np.ndarray:
    """Inverse of ``bitmap_words``."""
    w = np.asarray(words, dtype=np.uint32).astype(np.uint64)
    bits = (w[..., None] >> np.arange(WORD_BITS, dtype=np.uint64)) & np.uint64(1)
    return bits.reshape(w.shape[:-1] + (d,)).astype(bool)


def compress(x_bits: np.ndarray, k: int, capacity: int, L: int | None = None) -> dict:
    """Compress tokens [0, L) of a dense cache ``[B, H, T, d]`` (fp16 bits) into the bitmap format.

    Output arrays, one stream per (b, h), sized for ``capacity`` tokens:

    * ``bitmap``  uint32 [B, H, capacity, d/32] - kept positions of each token;
    * ``values``  uint16 [B, H, capacity*k]     - kept fp16 bits, ascending channel,
      token t's run starting at element t*k;
    * ``tile_offset`` uint32 [B, H, capacity/64] - element offset of each 64-token
      tile's first value within its stream (the popcount prefix sum).

    Slots of tokens >= L are left zero here; the library leaves them untouched.
    """
    x = np.asarray(x_bits, dtype=np.uint16)
    B, H, T, d = x.shape
    L = T if L is None else L
    assert capacity % TILE_TOKENS == 0 and L <= capacity and L <= T
    return _compress_mask(x, select_sort(x[:, :, :L], k), k, capacity, L)


def _compress_mask(x: np.ndarray, mask: np.ndarray, k: int, capacity: int, L: int) -> dict:
    """The bitmap format of tokens [0, L) of ``x`` given their kept-mask (k kept per token)."""
    B, H, T, d = x.shape
    bitmap = np.zeros((B, H, capacity, d // WORD_BITS), dtype=np.uint32)
    bitmap[:, :, :L] = bitmap_words(mask)
    values = np.zeros((B, H, capacity * k), dtype=np.uint16)
    kept = x[:, :, :L][mask].reshape(B, H, L * k)  # boolean indexing walks channels in ascending order
    values[:, :, : L * k] = kept
    counts = np.zeros((B, H, capacity), dtype=np.int64)
    counts[:, :, :L] = mask.sum(axis=-1)
    # prefix sums over the tokens before each tile; tokens >= L are counted as full (k) so that the
    # offsets of not-yet-written tiles equal their final value (the closed form 64*i*k).
    counts[:, :, L:] = k
    starts = np.concatenate([np.zeros((B, H, 1), np.int64), np.cumsum(counts, axis=-1)[..., :-1]], axis=-1)
    tile_offset = starts[:, :, ::TILE_TOKENS].astype(np.uint32)
    return {"bitmap": bitmap, "values": values, "tile_offset": tile_offset, "k": k, "L": L}


def decompress(bitmap: np.ndarray, values: np.ndarray, k: int, L: int, d: int) -> np.ndarray:
    """Dense fp16 bits [B, H, L, d] rebuilt from the bitmap and packed values (pruned positions are +0)."""
    mask = bitmap_to_mask(bitmap[:, :, :L], d)
    B, H = mask.shape[:2]
    out = np.zeros((B, H, L, d), dtype=np.uint16)
    out[mask] = np.asarray(values, dtype=np.uint16)[:, :, : L * k].reshape(-1)
    return out


def compressed_bytes(L: int, k: int, capacity: int, d: int = 128) -> int:
    """Closed-form bytes of one stream: bitmap d/8 B per token, 2k B of values per token, 4 B per tile."""
    return (d // 8) * L + 2 * k * L + 4 * (capacity // TILE_TOKENS)


def append(cache: dict, x_new_bits: np.ndarray, pos: np.ndarray) -> None:
    """Prune + compress one new token per (b, h) into slot ``pos[b]`` (in place).

    The same per-token pruning as the prefill path, applied to the token the
    decode step produces (the abstract: pruning and compression at runtime).
    """
    k = cache["k"]
    x = np.asarray(x_new_bits, dtype=np.uint16)  # [B, H, d]
    B, H, d = x.shape
    mask = select_sort(x, k)
    words = bitmap_words(mask)
    for b in range(B):
        p = int(pos[b])
        cache["bitmap"][b, :, p] = words[b]
        for h in range(H):
            cache["values"][b, h, p * k:(p + 1) * k] = x[b, h][mask[b, h]]


# --------------------------------------------------------------------------------------
# 2:4 semi-structured pruning (the comparison pattern)
# --------------------------------------------------------------------------------------
# The pages compare against 2:4 semi-structured sparsity (MUSTAFAR summary, atlas.scime.ai,
# "Experimental setup": baselines).  Reading: every group of 4 consecutive channels of a
# (token, kv head) vector keeps its 2 largest-magnitude elements (same key, ties to the lower
# channel), so every token keeps exactly d/2 channels (sparsity 0.5) and the result is stored in
# the same bitmap format.
GROUP = 4
GROUP_KEEP = 2


def select_24(x_bits: np.ndarray) -> np.ndarray:
    """Kept-mask of 2:4 pruning over the last axis: the top 2 of each group of 4 consecutive channels."""
    x = np.asarray(x_bits, dtype=np.uint16)
    d = x.shape[-1]
    groups = x.reshape(x.shape[:-1] + (d // GROUP, GROUP))
    return select_sort(groups, GROUP_KEEP).reshape(x.shape)


def prune_24(x_bits: np.ndarray) -> np.ndarray:
    x = np.asarray(x_bits, dtype=np.uint16)
    return np.where(select_24(x), x, np.uint16(0)).astype(np.uint16)


def compress_24(x_bits: np.ndarray, capacity: int, L: int | None = None) -> dict:
    """2:4-pruned tokens [0, L) of a dense cache [B, H, T, d] in the bitmap format (k = d/2)."""
    x = np.asarray(x_bits, dtype=np.uint16)
    B, H, T, d = x.shape
    L = T if L is None else L
    assert capacity % TILE_TOKENS == 0 and L <= capacity and L <= T
    return _compress_mask(x, select_24(x[:, :, :L]), d // 2, capacity, L)


def append_24(cache: dict, x_new_bits: np.ndarray, pos: np.ndarray) -> None:
    """2:4-prune + compress one new token per (b, h) into slot pos[b] (in place)."""
    k = cache["k"]
    x = np.asarray(x_new_bits, dtype=np.uint16)  # [B, H, d]
    B, H, d = x.shape
    mask = select_24(x)
    words = bitmap_words(mask)
    for b in range(B):
        p = int(pos[b])
        cache["bitmap"][b, :, p] = words[b]
        for h in range(H):
            cache["values"][b, h, p * k:(p + 1) * k] = x[b, h][mask[b, h]]


# --------------------------------------------------------------------------------------
# a keep count per kv head
# --------------------------------------------------------------------------------------
# The pages prune every head to the same sparsity and name per-head allocation as the open
# next step (MUSTAFAR summary, atlas.scime.ai, "Limitations").  With a keep count head_keep[h]
# per kv head, each (token, head h) vector is pruned exactly as above with k = head_keep[h]; the
# library's layout puts the streams batch-major, head h's packed values right after those of the
# heads before it.
def value_base_heads(b: int, h: int, head_keep, capacity: int) -> int:
    """First element of stream (b, h)'s packed values: capacity * (b * sum(k) + sum(k[:h]))."""
    return capacity * (b * int(sum(head_keep)) + int(sum(head_keep[:h])))


def prune_heads(x_bits: np.ndarray, head_keep) -> np.ndarray:
    """Pruned fp16 bits of a dense cache [B, H, T, d]: head h keeps head_keep[h] channels per token."""
    x = np.asarray(x_bits, dtype=np.uint16)
    return np.concatenate([prune(x[:, h:h + 1], int(k)) for h, k in enumerate(head_keep)], axis=1)


def compress_heads(x_bits: np.ndarray, head_keep, capacity: int, L: int | None = None) -> dict:
    """``compress`` with a keep count per kv head: bitmap [B, H, capacity, d/32] and tile_offset
    [B, H, capacity/64] as before (offsets 64*i*head_keep[h]); ``values`` is one flat uint16 array of
    B * capacity * sum(head_keep) elements, stream (b, h) at ``value_base_heads(b, h, ...)``."""
    x = np.asarray(x_bits, dtype=np.uint16)
    B, H, T, d = x.shape
    L = T if L is None else L
    parts = [compress(x[:, h:h + 1], int(k), capacity, L) for h, k in enumerate(head_keep)]
    values = np.zeros(B * capacity * int(sum(head_keep)), dtype=np.uint16)
    for h, k in enumerate(head_keep):
        for b in range(B):
            base = value_base_heads(b, h, head_keep, capacity)
            values[base:base + capacity * int(k)] = parts[h]["values"][b, 0]
    return {"bitmap": np.concatenate([c["bitmap"] for c in parts], axis=1), "values": values,
            "tile_offset": np.concatenate([c["tile_offset"] for c in parts], axis=1),
            "head_keep": [int(k) for k in head_keep], "L": L}


def decompress_heads(cache: dict, L: int, d: int) -> np.ndarray:
    """Dense fp16 bits [B, H, L, d] rebuilt from a per-head compressed cache."""
    hk = cache["head_keep"]
    B, H, cap = cache["bitmap"].shape[:3]
    out = []
    for h, k in enumerate(hk):
        vals = np.stack([cache["values"][value_base_heads(b, h, hk, cap):value_base_heads(b, h, hk, cap) + cap * k]
                         for b in range(B)])[:, None]
        out.append(decompress(cache["bitmap"][:, h:h + 1], vals, k, L, d))
    return np.concatenate(out, axis=1)


def append_heads(cache: dict, x_new_bits: np.ndarray, pos: np.ndarray) -> None:
    """``append`` for a per-head cache: the new token of (b, h) keeps head_keep[h] channels."""
    hk = cache["head_keep"]
    x = np.asarray(x_new_bits, dtype=np.uint16)  # [B, H, d]
    B, H, d = x.shape
    cap = cache["bitmap"].shape[2]
    for h, k in enumerate(hk):
        mask = select_sort(x[:, h], k)
        words = bitmap_words(mask)
        for b in range(B):
            p = int(pos[b])
            cache["bitmap"][b, h, p] = words[b]
            base = value_base_heads(b, h, hk, cap) + p * k
            cache["values"][base:base + k] = x[b, h][mask[b]]


# --------------------------------------------------------------------------------------
# channel-wise magnitude pruning (the Kc_Mag / Vc_Mag direction)
# --------------------------------------------------------------------------------------
# The README (Part II, the K/V [t/c] naming) names a channel-wise pruning direction next to the
# token-wise one and says no more.  Reading: each channel of a kv head is pruned across tokens,
# over consecutive windows of WINDOW tokens counted from token 0.  A full window prunes
# F = floor(s*WINDOW) of its tokens per channel (s as a float32, product in double, as in
# ``keep_count``) and keeps the WINDOW - F of largest magnitude (same key; ties go to the lower
# token index); a window of n < WINDOW tokens (the newest tokens of a row) prunes floor(n*F/WINDOW).
# Storage reuses the token bitmap format: bit c of token t marks a kept (t, c); the kept values of
# a window are packed token after token, each token's in ascending channel order, and window j of
# a stream starts at element j*WINDOW*keep, keep = (d/WINDOW)*(WINDOW - F) being the stream's values
# per token slot (so tile i of 64 tokens starts at 64*i*keep, as in the token format).  A dense copy
# of each stream's last, incomplete window is kept beside the cache, because an appended token
# changes which of that window's entries are kept.
WINDOW = 16


def window_prune_count(sparsity: float) -> int:
    """F = floor(s * WINDOW): tokens a full window prunes in every channel."""
    s = float(np.float32(sparsity))
    if not (0.0 <= s < 1.0):
        raise ValueError("sparsity must lie in [0, 1)")
    return int(math.floor(s * WINDOW))


def window_keep(n: int, F: int) -> int:
    """Tokens a window of n tokens keeps in every channel: n - floor(n*F/WINDOW)."""
    return n - (n * F) // WINDOW


def keep_count_channel(d: int, sparsity: float) -> int:
    """Values per token slot of a channel-wise cache: (d/WINDOW) * (WINDOW - F)."""
    return (d // WINDOW) * (WINDOW - window_prune_count(sparsity))


def select_channel(x_bits: np.ndarray, F: int) -> np.ndarray:
    """Kept-mask of channel-wise pruning of [..., T, d]: in every window of tokens, every channel
    keeps its ``window_keep(n, F)`` largest keys, the lower token first on ties."""
    x = np.asarray(x_bits, dtype=np.uint16)
    T = x.shape[-2]
    mask = np.zeros(x.shape, dtype=bool)
    for t0 in range(0, T, WINDOW):
        n = min(WINDOW, T - t0)
        win = np.swapaxes(x[..., t0:t0 + n, :], -1, -2)  # [..., d, n]: a channel's tokens on the last axis
        mask[..., t0:t0 + n, :] = np.swapaxes(select_sort(win, window_keep(n, F)), -1, -2)
    return mask


def prune_channel(x_bits: np.ndarray, sparsity: float) -> np.ndarray:
    """Channel-wise pruned fp16 bits of [..., T, d] (pruned entries become +0)."""
    x = np.asarray(x_bits, dtype=np.uint16)
    return np.where(select_channel(x, window_prune_count(sparsity)), x, np.uint16(0)).astype(np.uint16)


def compress_channel(x_bits: np.ndarray, sparsity: float, capacity: int, L: int | None = None) -> dict:
    """Channel-wise pruned tokens [0, L) of a dense cache [B, H, T, d] in the bitmap format.

    ``bitmap`` [B, H, capacity, d/32] and ``tile_offset`` [B, H, capacity/64] (= 64*i*keep) as in
    ``compress``; ``values`` [B, H, capacity*keep] with window j at element j*WINDOW*keep;
    ``window`` [B, H, WINDOW, d]: tokens [WINDOW*floor(L/WINDOW), L) in slots 0.. (the rest zero).
    """
    x = np.asarray(x_bits, dtype=np.uint16)
    B, H, T, d = x.shape
    L = T if L is None else L
    assert capacity % TILE_TOKENS == 0 and L <= capacity and L <= T
    F = window_prune_count(sparsity)
    keep = keep_count_channel(d, sparsity)
    mask = select_channel(x[:, :, :L], F)
    bitmap = np.zeros((B, H, capacity, d // WORD_BITS), dtype=np.uint32)
    bitmap[:, :, :L] = bitmap_words(mask)
    values = np.zeros((B, H, capacity * keep), dtype=np.uint16)
    for b in range(B):
        for h in range(H):
            for t0 in range(0, L, WINDOW):
                n = min(WINDOW, L - t0)
                kept = x[b, h, t0:t0 + n][mask[b, h, t0:t0 + n]]  # token-major, channels ascending
                values[b, h, t0 * keep:t0 * keep + kept.size] = kept
    tile_offset = np.broadcast_to(np.arange(capacity // TILE_TOKENS, dtype=np.int64) * TILE_TOKENS * keep,
                                  (B, H, capacity // TILE_TOKENS)).astype(np.uint32)
    window = np.zeros((B, H, WINDOW, d), dtype=np.uint16)
    r = L % WINDOW
    window[:, :, :r] = x[:, :, L - r:L]
    return {"bitmap": bitmap, "values": values, "tile_offset": tile_offset, "window": window, "F": F,
            "keep": keep, "L": L}


def decompress_channel(cache: dict, L: int, d: int) -> np.ndarray:
    """Dense fp16 bits [B, H, L, d] rebuilt from a channel-wise cache (pruned positions are +0)."""
    mask = bitmap_to_mask(cache["bitmap"][:, :, :L], d)
    B, H = mask.shape[:2]
    keep = cache["keep"]
    out = np.zeros((B, H, L, d), dtype=np.uint16)
    for b in range(B):
        for h in range(H):
            for t0 in range(0, L, WINDOW):
                m = mask[b, h, t0:t0 + WINDOW]
                cnt = int(m.sum())
                blk = np.zeros(m.shape, dtype=np.uint16)
                blk[m] = cache["values"][b, h, t0 * keep:t0 * keep + cnt]
                out[b, h, t0:t0 + m.shape[0]] = blk
    return out


def append_channel(cache: dict, x_new_bits: np.ndarray, pos: np.ndarray) -> None:
    """Append one new token per (b, h) at slot pos[b] of a channel-wise cache (in place).

    The token joins its window's dense copy; the window (tokens WINDOW*floor(p/WINDOW) .. p) is
    pruned again as a window of p % WINDOW + 1 tokens, and its bitmaps and packed values are
    rewritten.  Appends must come in token order.
    """
    x = np.asarray(x_new_bits, dtype=np.uint16)  # [B, H, d]
    B, H, d = x.shape
    F, keep = cache["F"], cache["keep"]
    for b in range(B):
        p = int(pos[b])
        t0, r = p - p % WINDOW, p % WINDOW
        cache["window"][b, :, r] = x[b]
        dense = cache["window"][b, :, :r + 1]  # [H, r+1, d]
        mask = select_channel(dense, F)
        cache["bitmap"][b, :, t0:p + 1] = bitmap_words(mask)
        for h in range(H):
            kept = dense[h][mask[h]]
            cache["values"][b, h, t0 * keep:t0 * keep + kept.size] = kept


# --------------------------------------------------------------------------------------
# attention over the pruned caches
# --------------------------------------------------------------------------------------
def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def attention(q_bits: np.ndarray, kp_bits: np.ndarray, vp_bits: np.ndarray, seq_len, scale: float):
    """Softmax attention of one decode query per (b, q head) over the pruned caches, in float64.

    q ``[B, Hq, d]``; K~/V~ ``[B, Hkv, >=L_b, d]`` (pruned fp16 bits); ``seq_len[b]`` tokens per row.
    For q head hq the kv head is g = hq // (Hq/Hkv).  z_t = scale * q . K~_t,
    p = softmax(z), o = sum_t p_t V~_t, lse = log sum_t exp(z_t).
    Returns (o [B, Hq, d] float64, lse [B, Hq] float64).
    """
    q = f16_to_f64(q_bits)
    B, Hq, d = q.shape
    Hkv = kp_bits.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        Lb = int(seq_len[b])
        K = f16_to_f64(kp_bits[b, :, :Lb])  # [Hkv, L, d]
        V = f16_to_f64(vp_bits[b, :, :Lb])
        for hq in range(Hq):
            g = hq // G
            z = scale * (K[g] @ q[b, hq])
            zmax = z.max()
            e = np.exp(z - zmax)
            ssum = e.sum()
            out[b, hq] = (e / ssum) @ V[g]
            lse[b, hq] = zmax + math.log(ssum)
    return out, lse


def attention_over_compressed(q_bits, kc: dict, vc: dict, seq_len, scale: float, d: int):
    """Attention read back from the compressed caches (decompress, then ``attention``)."""
    Lmax = int(max(seq_len))
    kp = decompress(kc["bitmap"], kc["values"], kc["k"], Lmax, d)
    vp = decompress(vc["bitmap"], vc["values"], vc["k"], Lmax, d)
    return attention(q_bits, kp, vp, seq_len, scale)

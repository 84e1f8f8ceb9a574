"""Plant plausible mistakes in copies of the oracle and check that some pin catches each one.

Mistakes are planted in the oracle only, on the CPU.
"""
import builtins
import types

import numpy as np
import pytest

import oracle.mustafar_oracle as real
from tests import oracle_pins as P


def _mutant(**overrides):
    ns = types.SimpleNamespace(**{n: getattr(real, n) for n in dir(real) if not n.startswith("__")})
    for name, fn in overrides.items():
        setattr(ns, name, fn)
    # rebind functions that call each other so they see the overrides
    def compress(x_bits, k, capacity, L=None):
        x = np.asarray(x_bits, dtype=np.uint16)
        B, H, T, d = x.shape
        L = T if L is None else L
        mask = ns.select_sort(x[:, :, :L], k)
        bitmap = np.zeros((B, H, capacity, d // 32), dtype=np.uint32)
        bitmap[:, :, :L] = ns.bitmap_words(mask)
        values = np.zeros((B, H, capacity * k), dtype=np.uint16)
        values[:, :, : L * k] = x[:, :, :L][mask].reshape(B, H, L * k)
        starts = np.arange(capacity // 64, dtype=np.int64) * 64 * k
        return {"bitmap": bitmap, "values": values,
                "tile_offset": np.broadcast_to(starts, (B, H, capacity // 64)).astype(np.uint32), "k": k, "L": L}
    if "compress" not in overrides:
        ns.compress = compress
    def prune(x_bits, k):
        x = np.asarray(x_bits, dtype=np.uint16)
        return np.where(ns.select_sort(x, k), x, np.uint16(0)).astype(np.uint16)
    if "prune" not in overrides:
        ns.prune = prune
    def decompress(bitmap, values, k, L, d):
        mask = ns.bitmap_to_mask(bitmap[:, :, :L], d)
        out = np.zeros(mask.shape, dtype=np.uint16)
        out[mask] = np.asarray(values)[:, :, : L * k].reshape(-1)
        return out
    if "decompress" not in overrides:
        ns.decompress = decompress
    def attention_over_compressed(q_bits, kc, vc, seq_len, scale, d):
        Lmax = int(max(seq_len))
        return ns.attention(q_bits, ns.decompress(kc["bitmap"], kc["values"], kc["k"], Lmax, d),
                            ns.decompress(vc["bitmap"], vc["values"], vc["k"], Lmax, d), seq_len, scale)
    ns.attention_over_compressed = attention_over_compressed
    def append(cache, x_new_bits, pos):
        k = cache["k"]
        x = np.asarray(x_new_bits, dtype=np.uint16)
        mask = ns.select_sort(x, k)
        words = ns.bitmap_words(mask)
        for b in range(x.shape[0]):
            p = int(pos[b])
            cache["bitmap"][b, :, p] = words[b]
            for h in range(x.shape[1]):
                cache["values"][b, h, p * k:(p + 1) * k] = x[b, h][mask[b, h]]
    if "append" not in overrides:
        ns.append = append
    # per-head functions, rebound so that they call the (possibly mutated) namespace
    def prune_heads(x_bits, head_keep):
        x = np.asarray(x_bits, dtype=np.uint16)
        return np.concatenate([ns.prune(x[:, h:h + 1], int(k)) for h, k in enumerate(head_keep)], axis=1)
    if "prune_heads" not in overrides:
        ns.prune_heads = prune_heads
    def compress_heads(x_bits, head_keep, capacity, L=None):
        x = np.asarray(x_bits, dtype=np.uint16)
        B, H, T, d = x.shape
        parts = [ns.compress(x[:, h:h + 1], int(k), capacity, L) for h, k in enumerate(head_keep)]
        values = np.zeros(B * capacity * int(sum(head_keep)), dtype=np.uint16)
        for h, k in enumerate(head_keep):
            for b in range(B):
                base = ns.value_base_heads(b, h, head_keep, capacity)
                values[max(base, 0):max(base, 0) + capacity * int(k)] = parts[h]["values"][b, 0][: max(0, min(
                    capacity * int(k), values.size - max(base, 0)))]
        return {"bitmap": np.concatenate([c["bitmap"] for c in parts], axis=1), "values": values,
                "tile_offset": np.concatenate([c["tile_offset"] for c in parts], axis=1),
                "head_keep": [int(k) for k in head_keep], "L": parts[0]["L"]}
    ns.compress_heads = compress_heads
    def decompress_heads(cache, L, d):
        hk = cache["head_keep"]
        B, H, cap = cache["bitmap"].shape[:3]
        out = []
        for h, k in enumerate(hk):
            vals = np.stack([cache["values"][ns.value_base_heads(b, h, hk, cap):][: cap * k] for b in range(B)])
            out.append(ns.decompress(cache["bitmap"][:, h:h + 1], vals[:, None], k, L, d))
        return np.concatenate(out, axis=1)
    ns.decompress_heads = decompress_heads
    def append_heads(cache, x_new_bits, pos):
        hk = cache["head_keep"]
        x = np.asarray(x_new_bits, dtype=np.uint16)
        cap = cache["bitmap"].shape[2]
        for h, k in enumerate(hk):
            mask = ns.select_sort(x[:, h], k)
            words = ns.bitmap_words(mask)
            for b in range(x.shape[0]):
                p = int(pos[b])
                cache["bitmap"][b, h, p] = words[b]
                base = ns.value_base_heads(b, h, hk, cap) + p * k
                cache["values"][base:base + k] = x[b, h][mask[b]]
    ns.append_heads = append_heads
    # 2:4 functions, rebound to the namespace's select_24 / select_sort
    if "select_24" not in overrides:
        def select_24(x_bits):
            x = np.asarray(x_bits, dtype=np.uint16)
            d = x.shape[-1]
            return ns.select_sort(x.reshape(x.shape[:-1] + (d // 4, 4)), 2).reshape(x.shape)
        ns.select_24 = select_24
    def prune_24(x_bits):
        x = np.asarray(x_bits, dtype=np.uint16)
        return np.where(ns.select_24(x), x, np.uint16(0)).astype(np.uint16)
    ns.prune_24 = prune_24
    def compress_24(x_bits, capacity, L=None):
        x = np.asarray(x_bits, dtype=np.uint16)
        B, H, T, d = x.shape
        L = T if L is None else L
        mask = ns.select_24(x[:, :, :L])
        k = d // 2
        bitmap = np.zeros((B, H, capacity, d // 32), dtype=np.uint32)
        bitmap[:, :, :L] = ns.bitmap_words(mask)
        values = np.zeros((B, H, capacity * k), dtype=np.uint16)
        values[:, :, : L * k] = x[:, :, :L][mask].reshape(B, H, -1)[:, :, : L * k]
        starts = np.arange(capacity // 64, dtype=np.int64) * 64 * k
        return {"bitmap": bitmap, "values": values,
                "tile_offset": np.broadcast_to(starts, (B, H, capacity // 64)).astype(np.uint32), "k": k, "L": L}
    ns.compress_24 = compress_24
    def append_24(cache, x_new_bits, pos):
        k = cache["k"]
        x = np.asarray(x_new_bits, dtype=np.uint16)
        mask = ns.select_24(x)
        words = ns.bitmap_words(mask)
        for b in range(x.shape[0]):
            p = int(pos[b])
            cache["bitmap"][b, :, p] = words[b]
            for h in range(x.shape[1]):
                v = x[b, h][mask[b, h]]
                cache["values"][b, h, p * k:p * k + v.size] = v[:k]
    ns.append_24 = append_24
    # channel-wise functions: the real code, its global names looked up in the namespace
    glb = vars(ns)
    glb["__builtins__"] = builtins
    for name in ("window_prune_count", "window_keep", "keep_count_channel", "select_channel", "prune_channel",
                 "compress_channel", "decompress_channel", "append_channel"):
        if name not in overrides:
            fn = getattr(real, name)
            setattr(ns, name, types.FunctionType(fn.__code__, glb, name, fn.__defaults__))
    return ns


def sel_ascending(x_bits, k):           # wrong sign: keeps the smallest magnitudes
    m = real.magnitude_key(x_bits)
    order = np.argsort(m, axis=-1, kind="stable")[..., :k]
    mask = np.zeros(m.shape, bool); np.put_along_axis(mask, order, True, axis=-1); return mask


def sel_high_index_ties(x_bits, k):     # wrong tie rule: higher channel wins
    m = real.magnitude_key(x_bits)[..., ::-1]
    order = np.argsort(0x7FFF - m, axis=-1, kind="stable")[..., :k]
    mask = np.zeros(m.shape, bool); np.put_along_axis(mask, order, True, axis=-1); return mask[..., ::-1]


def sel_signed(x_bits, k):              # compares signed values instead of magnitudes
    v = np.asarray(x_bits, np.uint16).view(np.float16).astype(np.float64)
    order = np.argsort(-v, axis=-1, kind="stable")[..., :k]
    mask = np.zeros(v.shape, bool); np.put_along_axis(mask, order, True, axis=-1); return mask


def words_msb_first(mask):              # wrong bit order inside a word
    return real.bitmap_words(np.flip(mask.reshape(mask.shape[:-1] + (-1, 32)), -1).reshape(mask.shape))


def keep_round(d, s):                   # rounds (1-s)*d instead of d - floor(s*d)
    return int(round((1 - float(np.float32(s))) * d))


def size_no_offsets(L, k, capacity, d=128):
    return (d // 8) * L + 2 * k * L


def size_bits_as_bytes(L, k, capacity, d=128):
    return d * L + 2 * k * L + 4 * (capacity // 64)


def attn_no_scale(q, kp, vp, seq_len, scale):
    return real.attention(q, kp, vp, seq_len, 1.0)


def attn_wrong_group(q_bits, kp_bits, vp_bits, seq_len, scale):   # hq % Hkv instead of hq // G
    B, Hq, d = q_bits.shape
    Hkv = kp_bits.shape[1]
    perm = np.array([(hq % Hkv) * (Hq // Hkv) + hq // Hkv for hq in range(Hq)])
    inv = np.argsort(perm)
    o, l = real.attention(q_bits[:, perm], kp_bits, vp_bits, seq_len, scale)
    return o[:, inv], l[:, inv]


def attn_unnormalised(q, kp, vp, seq_len, scale):
    o, l = real.attention(q, kp, vp, seq_len, scale)
    return o * np.exp(l)[..., None] / np.exp(l).mean(), l


def attn_drop_last(q, kp, vp, seq_len, scale):      # attends over one token too few
    return real.attention(q, kp, vp, [max(1, int(s) - 1) for s in seq_len], scale)


def attn_lse_log2(q, kp, vp, seq_len, scale):
    o, l = real.attention(q, kp, vp, seq_len, scale)
    return o, l / np.log(2)


def prune_negzero(x_bits, k):           # pruned slots written as -0 instead of +0
    x = np.asarray(x_bits, np.uint16)
    return np.where(real.select_sort(x, k), x, np.uint16(0x8000)).astype(np.uint16)


def base_next_head(b, h, head_keep, capacity):      # stream starts after its own head's values
    return capacity * (b * int(sum(head_keep)) + int(sum(head_keep[:h + 1])))


def base_head_major(b, h, head_keep, capacity):     # head-major instead of batch-major streams
    return capacity * (int(sum(head_keep[:h])) * 2 + b * int(head_keep[h]))


def prune_heads_max(x_bits, head_keep):             # every head pruned with the largest keep
    x = np.asarray(x_bits, dtype=np.uint16)
    return np.concatenate([real.prune(x[:, h:h + 1], int(max(head_keep))) for h in range(x.shape[1])], axis=1)


def sel24_strided(x_bits):            # groups of channels c, c+d/4, c+d/2, c+3d/4 instead of 4 neighbours
    x = np.asarray(x_bits, np.uint16)
    d = x.shape[-1]
    g = np.swapaxes(x.reshape(x.shape[:-1] + (4, d // 4)), -1, -2)
    m = real.select_sort(g, 2)
    return np.swapaxes(m, -1, -2).reshape(x.shape)


def sel24_groups_of_8(x_bits):         # 4 of every 8 instead of 2 of every 4
    x = np.asarray(x_bits, np.uint16)
    d = x.shape[-1]
    return real.select_sort(x.reshape(x.shape[:-1] + (d // 8, 8)), 4).reshape(x.shape)


def selch_high_ties(x_bits, F):          # channel-wise ties go to the later token
    x = np.asarray(x_bits, np.uint16)
    return real.select_channel(x[..., ::-1, :], F)[..., ::-1, :] if x.shape[-2] % 16 == 0 else \
        _selch_windows(x, F, lambda w, k: real.select_sort(w[..., ::-1], k)[..., ::-1])


def _selch_windows(x, F, select):
    T = x.shape[-2]
    mask = np.zeros(x.shape, bool)
    for t0 in range(0, T, 16):
        n = min(16, T - t0)
        w = np.swapaxes(x[..., t0:t0 + n, :], -1, -2)
        mask[..., t0:t0 + n, :] = np.swapaxes(select(w, real.window_keep(n, F)), -1, -2)
    return mask


def selch_from_end(x_bits, F):           # windows counted back from the newest token
    x = np.asarray(x_bits, np.uint16)
    return _selch_windows(x[..., ::-1, :], F, lambda w, k: real.select_sort(w[..., ::-1], k)[..., ::-1])[..., ::-1, :]


def selch_over_channels(x_bits, F):      # prunes across the channels of a token (the token direction)
    x = np.asarray(x_bits, np.uint16)
    d = x.shape[-1]
    return real.select_sort(x, d - (d * F) // 16)


def wkeep_ceil(n, F):                    # rounds the pruned count up
    return n - -(-n * F // 16)


def keepch_token_rule(d, s):             # token-wise keep count instead of (d/16)*(16-F)
    return real.keep_count(d, s)


def compress_channel_major(x_bits, sparsity, capacity, L=None):   # a window's values channel by channel
    c = real.compress_channel(x_bits, sparsity, capacity, L)
    x = np.asarray(x_bits, np.uint16)
    keep, L = c["keep"], c["L"]
    mask = real.bitmap_to_mask(c["bitmap"][:, :, :L], x.shape[-1])
    for b in range(x.shape[0]):
        for h in range(x.shape[1]):
            for t0 in range(0, L, 16):
                xm = x[b, h, t0:t0 + 16][:L - t0].T
                kept = xm[mask[b, h, t0:t0 + 16][:L - t0].T]
                c["values"][b, h, t0 * keep:t0 * keep + kept.size] = kept
    return c


def append_channel_no_window(cache, x_new_bits, pos):   # forgets to keep the window's dense copy
    saved = cache["window"].copy()
    real.append_channel(cache, x_new_bits, pos)
    x = np.asarray(x_new_bits, np.uint16)
    for b in range(x.shape[0]):
        p = int(pos[b])
        cache["window"][b] = saved[b]
        if p % 16 == 0:
            cache["window"][b] = 0


def append_channel_new_only(cache, x_new_bits, pos):    # prunes the new token alone, old bits kept
    x = np.asarray(x_new_bits, np.uint16)
    for b in range(x.shape[0]):
        p = int(pos[b])
        r = p % 16
        cache["window"][b, :, r] = x[b]
        mask = real.select_channel(cache["window"][b, :, :r + 1], cache["F"])
        cache["bitmap"][b, :, p] = real.bitmap_words(mask[:, r])
        t0, keep = p - r, cache["keep"]
        for h in range(x.shape[1]):
            old = real.bitmap_to_mask(cache["bitmap"][b, h, t0:p + 1], x.shape[-1])
            dense = cache["window"][b, h, :r + 1]
            kept = dense[old]
            cache["values"][b, h, t0 * keep:t0 * keep + kept.size] = kept


MUTANTS = {
    "channel ties to later token": dict(select_channel=selch_high_ties),
    "channel windows from the end": dict(select_channel=selch_from_end),
    "channel pruned across channels": dict(select_channel=selch_over_channels),
    "channel window count rounded up": dict(window_keep=wkeep_ceil),
    "channel keep by the token rule": dict(keep_count_channel=keepch_token_rule),
    "channel values channel-major": dict(compress_channel=compress_channel_major),
    "channel append keeps no window": dict(append_channel=append_channel_no_window),
    "channel append prunes new token only": dict(append_channel=append_channel_new_only),
    "2:4 strided groups": dict(select_24=sel24_strided),
    "2:4 as 4:8": dict(select_24=sel24_groups_of_8),
    "per-head base after own head": dict(value_base_heads=base_next_head),
    "per-head streams head-major": dict(value_base_heads=base_head_major),
    "per-head prune with max keep": dict(prune_heads=prune_heads_max),
    "select ascending": dict(select_sort=sel_ascending),
    "ties to higher index": dict(select_sort=sel_high_index_ties),
    "signed compare": dict(select_sort=sel_signed),
    "bitmap msb first": dict(bitmap_words=words_msb_first),
    "keep count rounded": dict(keep_count=keep_round),
    "size without offsets": dict(compressed_bytes=size_no_offsets),
    "bitmap counted in bytes": dict(compressed_bytes=size_bits_as_bytes),
    "scale dropped": dict(attention=attn_no_scale),
    "wrong gqa mapping": dict(attention=attn_wrong_group),
    "softmax not normalised": dict(attention=attn_unnormalised),
    "last token dropped": dict(attention=attn_drop_last),
    "lse in log2": dict(attention=attn_lse_log2),
    "pruned slots -0": dict(prune=prune_negzero),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    caught = P.failing_pins(_mutant(**MUTANTS[name]))
    assert caught, f"no pin catches the planted mistake '{name}'"


def test_unmutated_copy_passes():
    assert P.failing_pins(_mutant()) == []

"""The C-ABI library on the host: it loads, exports every declared symbol, and its
host-side queries and argument checks behave (no kernel launch, no GPU needed)."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import oracle
import unstructured_sparse_kv_b200 as M
from unstructured_sparse_kv_b200 import _lib
from unstructured_sparse_kv_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "mustafar.h")).read()
    return sorted(set(re.findall(r"MUSTAFAR_API[^;(]*?\b(mustafar_\w+)\s*\(", text, flags=re.S)))


def test_header_lists_the_binding_symbols():
    assert declared_symbols() == sorted(_lib.ABI_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.mustafar_abi_version() == 5


def test_keep_count_matches_oracle(lib):
    for d in (32, 64, 128, 256):
        for s in np.concatenate([np.linspace(0, 0.999, 97), [0.1, 0.3, 0.7, 0.9, 0.995]]):
            assert M.mustafar_keep_count(d, float(s)) == oracle.keep_count(d, float(s)), (d, s)
    for bad in (-0.01, 1.0, 2.0, float("nan")):
        assert lib.mustafar_keep_count(128, bad) == -1
    assert lib.mustafar_keep_count(100, 0.5) == -1


def test_cache_sizes_match_closed_form(lib):
    for (Bt, H, cap, s) in [(8, 8, 4160, 0.7), (1, 8, 1024, 0.5), (4, 8, 32768, 0.3), (32, 32, 131072, 0.0)]:
        nb, nv, no = M.mustafar_cache_sizes(Bt, H, 128, cap, s)
        k = oracle.keep_count(128, s)
        per_stream = oracle.compressed_bytes(cap, k, cap, 128)
        assert nb + nv + no == Bt * H * per_stream
        assert nb == Bt * H * cap * 16 and no == Bt * H * (cap // 64) * 4
    with pytest.raises(M.MustafarError):
        M.mustafar_cache_sizes(1, 1, 128, 100, 0.5)  # capacity not a multiple of 64


def _cache(batch=2, heads=2, cap=128, keep=39, bitmap=0x1000, values=0x2000, offs=0x3000, d=128):
    return _lib.CacheT(batch, heads, d, cap, keep, bitmap, values, offs)


def _status(lib, fn, *args):
    st = getattr(lib, fn)(*args)
    return st, lib.mustafar_last_error().decode()


def test_compress_argument_checks(lib):
    ok = _cache()
    cases = [
        (dict(c=None), 1, "NULL"),
        (dict(c=_cache(keep=40)), 1, "keep"),
        (dict(c=_cache(cap=100)), 1, "multiple of 64"),
        (dict(c=_cache(d=64, keep=20)), 2, "128"),
        (dict(c=_cache(bitmap=0x1004)), 3, "alignment"),
        (dict(L=129), 1, "capacity"),
        (dict(s=1.0), 1, "sparsity"),
        (dict(x=0x5002), 3, "multiples of 8"),
        (dict(st=12), 3, "multiples of 8"),
        (dict(x=None), 1, "NULL"),
    ]
    for over, want, msg in cases:
        a = dict(x=0x5000, sb=4096, sh=2048, st=128, L=64, s=0.7, c=ok)
        a.update(over)
        cref = C.byref(a["c"]) if a["c"] is not None else None
        st, err = _status(lib, "mustafar_compress", a["x"], a["sb"], a["sh"], a["st"], a["L"], a["s"], cref, None, None)
        assert st == want and msg in err, (over, st, err)


def test_append_and_decode_argument_checks(lib):
    c = _cache()
    st, err = _status(lib, "mustafar_append", 0x5000, 256, 128, None, C.byref(c), None, None)
    assert st == 1 and "pos" in err
    st, err = _status(lib, "mustafar_append", 0x5000, 256, 100, 0x6000, C.byref(c), None, None)
    assert st == 3
    kc, vc = _cache(), _cache(heads=4)
    st, err = _status(lib, "mustafar_decode_attn", 0x7000, 8, C.byref(kc), C.byref(vc), 0x6000, 64, 1.0, 0x8000,
                      None, None, 0, 0, None, None)
    assert st == 1 and "disagree" in err
    vc = _cache()
    st, err = _status(lib, "mustafar_decode_attn", 0x7000, 5, C.byref(kc), C.byref(vc), 0x6000, 64, 1.0, 0x8000,
                      None, None, 0, 0, None, None)
    assert st == 1 and "multiple" in err
    st, err = _status(lib, "mustafar_decode_attn", 0x7000, 2 * 17, C.byref(kc), C.byref(vc), 0x6000, 64, 1.0,
                      0x8000, None, None, 0, 0, None, None)
    assert st == 2 and "16" in err
    st, err = _status(lib, "mustafar_decode_attn", 0x7008, 8, C.byref(kc), C.byref(vc), 0x6000, 64, 1.0, 0x8000,
                      None, None, 0, 0, None, None)
    assert st == 3
    st, err = _status(lib, "mustafar_decode_attn", 0x7000, 8, C.byref(kc), C.byref(vc), 0x6000, 64,
                      float("inf"), 0x8000, None, None, 0, 0, None, None)
    assert st == 1 and "scale" in err
    st, err = _status(lib, "mustafar_dense_decode_attn", 0x7000, 8, 0x9000, 0xA000, 2, 2, 128, 100, 0x6000, 64,
                      1.0, 0x8000, None, None, 0, 0, None, None)
    assert st == 1 and "16" in err


def test_decode_step_argument_checks(lib):
    kc, vc = _cache(), _cache()
    base = dict(q=0x7000, hq=8, kn=0x5000, ksb=256, ksh=128, vn=0x5800, vsb=256, vsh=128, pos=0x6000, L=64)

    def call(**over):
        a = dict(base, **over)
        return _status(lib, "mustafar_decode_step", a["q"], a["hq"], a["kn"], a["ksb"], a["ksh"], a["vn"], a["vsb"],
                       a["vsh"], a["pos"], C.byref(kc), C.byref(vc), a["L"], 1.0, 0x8000, None, None, 0, 0, None,
                       None)
    for over, want, msg in [(dict(kn=None), 1, "k_new"), (dict(pos=None), 1, "pos must be non-NULL"), (dict(pos=0x6002), 3, "pos needs"),
                            (dict(vn=0x5808), 3, "multiples of 8"), (dict(ksh=100), 3, "multiples of 8"),
                            (dict(vsb=-256), 1, "negative"), (dict(hq=5), 1, "multiple"), (dict(L=0), 1, "max_len")]:
        st, err = call(**over)
        assert st == want and msg in err, (over, st, err)


def test_per_head_keep_checks_and_sizes(lib):
    keeps = (C.c_int32 * 2)(39, 64)
    c = _cache(keep=64)
    c.head_keep = C.cast(keeps, C.c_void_p).value
    for kwargs, want, msg in [(dict(keep=39), 1, "largest head_keep"), ]:
        bad = _cache(**kwargs)
        bad.head_keep = c.head_keep
        st, err = _status(lib, "mustafar_append", 0x5000, 256, 100, 0x6000, C.byref(bad), None, None)
        assert st == want and msg in err, (st, err)
    zero = (C.c_int32 * 2)(39, 0)
    bad = _cache(keep=39)
    bad.head_keep = C.cast(zero, C.c_void_p).value
    st, err = _status(lib, "mustafar_append", 0x5000, 256, 100, 0x6000, C.byref(bad), None, None)
    assert st == 1 and "head_keep[1]" in err
    many = _cache(heads=129)
    many.head_keep = C.cast((C.c_int32 * 129)(*([39] * 129)), C.c_void_p).value
    st, err = _status(lib, "mustafar_append", 0x5000, 256, 100, 0x6000, C.byref(many), None, None)
    assert st == 2 and "128" in err
    # sizes: bitmap and offsets as for a uniform cache, values 2 * B * cap * sum(head_keep)
    B, H, cap, hk = 3, 4, 192, [13, 39, 64, 128]
    nb, nv, no = M.mustafar_cache_sizes_per_head(B, H, cap, hk)
    assert (nb, nv, no) == (B * H * cap * 16, 2 * B * cap * sum(hk), B * H * (cap // 64) * 4)
    with pytest.raises(M.MustafarError):
        M.mustafar_cache_sizes_per_head(B, H, cap, [13, 39, 64, 129])
    # a uniform head_keep gives exactly the uniform sizes
    assert M.mustafar_cache_sizes_per_head(B, H, cap, [39] * H) == M.mustafar_cache_sizes(B, H, 128, cap, 0.7)


def test_pattern_checks(lib):
    # every call stops in host validation (stride 100 is deliberately misaligned): nothing launches
    c = _cache(keep=64)
    c.pattern = 1
    st, err = _status(lib, "mustafar_append", 0x5000, 256, 100, 0x6000, C.byref(c), None, None)
    assert st == 3  # a valid 2:4 descriptor passes the pattern checks
    bad = _cache(keep=39)
    bad.pattern = 1
    st, err = _status(lib, "mustafar_append", 0x5000, 256, 100, 0x6000, C.byref(bad), None, None)
    assert st == 1 and "2:4" in err
    bad = _cache(keep=64)
    bad.pattern = 7
    st, err = _status(lib, "mustafar_append", 0x5000, 256, 100, 0x6000, C.byref(bad), None, None)
    assert st == 1 and "pattern" in err
    with pytest.raises(ValueError):
        M.CompressedCache(1, 1, 64, 0.7, pattern="2:4", device="cpu")


def test_workspace_query(lib):
    # sparse kernel: 256-byte-rounded ticket counters (one per stream), then two partial
    # (m[16], l[16], o[G][128]) fp32 slots per CTA; num_splits = s asks for s CTAs per stream
    def sparse_bytes(ctas, G=4, streams=64):
        return ((streams * 4 + 255) // 256) * 256 + 2 * ctas * (32 + G * 128) * 4
    n1 = M.mustafar_decode_workspace_bytes(8, 32, 8, 4160, num_splits=1)
    n4 = M.mustafar_decode_workspace_bytes(8, 32, 8, 4160, num_splits=4)
    assert n1 == sparse_bytes(64)
    assert n4 == max(sparse_bytes(256), 256 + 8 * 32 * 4 * 2 * 4 + 8 * 32 * 4 * 128 * 4)
    assert M.mustafar_decode_workspace_bytes(8, 32, 8, 4160) >= n1
    with pytest.raises(M.MustafarError):
        M.mustafar_decode_workspace_bytes(8, 30, 8, 4160)


def test_channel_keep_count_sizes_and_checks(lib):
    for d in (32, 128, 256):
        for s in np.concatenate([np.linspace(0, 0.999, 61), [0.3, 0.5, 0.7, 0.75, 0.9375]]):
            assert M.mustafar_keep_count_channel(d, float(s)) == oracle.keep_count_channel(d, float(s)), (d, s)
    assert lib.mustafar_keep_count_channel(128, 1.0) == -1 and lib.mustafar_keep_count_channel(100, 0.5) == -1
    B, H, cap = 3, 4, 192
    nb, nv, no, nw = M.mustafar_cache_sizes_channel(B, H, 128, cap, 0.7)
    assert (nb, nv, no, nw) == (B * H * cap * 16, 2 * B * H * cap * 40, B * H * (cap // 64) * 4, B * H * 16 * 128 * 2)
    # descriptor checks stop in host validation (stride 100 is misaligned: nothing launches)
    good = _cache(keep=40)
    good.pattern, good.window = 2, 0x4000
    st, err = _status(lib, "mustafar_append", 0x5000, 256, 100, 0x6000, C.byref(good), None, None)
    assert st == 3  # a valid channel-wise descriptor passes the pattern checks
    for change, want, msg in [(dict(window=None), 1, "window"), (dict(window=0x4008), 3, "window"),
                              (dict(keep=39), 1, "multiple of head_dim/16")]:
        bad = _cache(keep=40)
        bad.pattern, bad.window = 2, 0x4000
        for k, v in change.items():
            setattr(bad, k, v)
        st, err = _status(lib, "mustafar_append", 0x5000, 256, 100, 0x6000, C.byref(bad), None, None)
        assert st == want and msg in err, (change, st, err)
    # compress: keep must follow the channel rule for that sparsity
    st, err = _status(lib, "mustafar_compress", 0x5000, 4096, 2048, 128, 64, 0.7, C.byref(_cache(keep=40)), None, None)
    assert st == 1 and "keep_count(" in err
    ch = _cache(keep=48)
    ch.pattern, ch.window = 2, 0x4000
    st, err = _status(lib, "mustafar_compress", 0x5000, 4096, 2048, 128, 64, 0.7, C.byref(ch), None, None)
    assert st == 1 and "keep_count_channel" in err
    with pytest.raises(ValueError):
        M.CompressedCache(1, 2, 64, [0.5, 0.7], pattern="channel", device="cpu")


def test_channel_cache_cannot_pair_with_per_head(lib):
    # rejected in host validation, before any plan or launch
    kc = _cache(keep=40)
    kc.pattern, kc.window = 2, 0x4000
    keeps = (C.c_int32 * 2)(39, 64)
    vc = _cache(keep=64)
    vc.head_keep = C.cast(keeps, C.c_void_p).value
    st, err = _status(lib, "mustafar_decode_attn", 0x7000, 8, C.byref(kc), C.byref(vc), 0x6000, 64, 1.0, 0x8000,
                      None, 0x9000, 1 << 20, 0, None, None)
    assert st == 2 and "per-head" in err, (st, err)


def test_24_cache_cannot_have_head_keep(lib):
    keeps = (C.c_int32 * 2)(64, 64)
    c = _cache(keep=64)
    c.pattern = 1
    c.head_keep = C.cast(keeps, C.c_void_p).value
    st, err = _status(lib, "mustafar_append", 0x5000, 256, 100, 0x6000, C.byref(c), None, None)
    assert st == 1 and "2:4" in err, (st, err)



def test_plan_queries_reject_invalid_shapes(lib):
    # shape checks come before any device query, so they answer without a GPU
    plan_cluster = lib.mustafar_decode_plan_cluster
    assert plan_cluster(8, 24, 8, 128, 1024, 39, 39) == -1   # 3 q heads per kv head
    assert plan_cluster(8, 36, 8, 128, 1024, 39, 39) == -1   # q heads not a multiple of kv heads
    assert plan_cluster(8, 32, 8, 64, 1024, 39, 39) == -1    # head_dim other than 128
    assert plan_cluster(8, 32, 8, 128, 0, 39, 39) == -1      # no context
    assert plan_cluster(8, 32, 8, 128, 1024, 0, 39) == -1    # keep out of range
    assert plan_cluster(8, 32, 8, 128, 1024, 39, 129) == -1
    assert plan_cluster(0, 32, 8, 128, 1024, 39, 39) == -1   # no batch
    assert plan_cluster(8, 512, 8, 128, 1024, 39, 39) == -1  # 64 q heads per kv head
    assert lib.mustafar_decode_plan_splits(8, 8, 64, 1024, 39, 39, 0) == -1
    with pytest.raises(M.MustafarError):
        M.mustafar_decode_plan_cluster(8, 24, 8, 1024, 39, 39)

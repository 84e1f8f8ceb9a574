"""ctypes binding of libmustafar.so: argument marshalling only.

Every step of the path runs inside the library's CUDA kernels; these wrappers
turn torch tensors into pointers, shapes and a stream handle, call the C entry
point of the same name, and raise on a non-OK status.  There is no fallback:
if the library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmustafar.so")

MUSTAFAR_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "MISALIGNED", 4: "CUDA", 5: "WORKSPACE"}
DEVERR_POS_RANGE = 0x1
DEVERR_LEN_RANGE = 0x2
HEAD_DIM = 128
PATTERN_TOPK = 0   # per-token top-keep pruning (the method)
PATTERN_2_4 = 1    # 2:4 semi-structured pruning (the comparison pattern)
PATTERN_CHANNEL = 2  # channel-wise pruning over 16-token windows
WINDOW_TOKENS = 16

# every symbol include/mustafar.h declares
ABI_SYMBOLS = (
    "mustafar_keep_count", "mustafar_cache_sizes", "mustafar_compress", "mustafar_append",
    "mustafar_decode_workspace_bytes", "mustafar_decode_attn", "mustafar_dense_decode_attn",
    "mustafar_decode_plan_splits", "mustafar_decode_plan_cluster", "mustafar_status_string", "mustafar_last_error",
    "mustafar_abi_version",
    "mustafar_decode_attn_noalloc", "mustafar_decode_step", "mustafar_cache_sizes_per_head",
    "mustafar_keep_count_channel", "mustafar_cache_sizes_channel",
)


class MustafarError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class CacheT(C.Structure):
    """Mirror of mustafar_cache_t."""
    _fields_ = [("batch", C.c_int32), ("num_kv_heads", C.c_int32), ("head_dim", C.c_int32),
                ("capacity", C.c_int32), ("keep", C.c_int32), ("bitmap", C.c_void_p),
                ("values", C.c_void_p), ("tile_offset", C.c_void_p), ("head_keep", C.c_void_p),
                ("pattern", C.c_int32), ("window", C.c_void_p)]


_lib = None


def load() -> C.CDLL:
    """Load libmustafar.so (built in-tree by ``unstructured_sparse_kv_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libmustafar.so is not built ({LIB_PATH}); run `python -m unstructured_sparse_kv_b200.build`")
    lib = C.CDLL(LIB_PATH)
    i32, i64, f32, vp, sz = C.c_int32, C.c_int64, C.c_float, C.c_void_p, C.c_size_t
    P = C.POINTER
    sig = {
        "mustafar_keep_count": (i32, [i32, f32]),
        "mustafar_keep_count_channel": (i32, [i32, f32]),
        "mustafar_cache_sizes_channel": (i32, [i32, i32, i32, i32, f32, P(sz), P(sz), P(sz), P(sz)]),
        "mustafar_cache_sizes": (i32, [i32, i32, i32, i32, f32, P(sz), P(sz), P(sz)]),
        "mustafar_cache_sizes_per_head": (i32, [i32, i32, i32, i32, vp, P(sz), P(sz), P(sz)]),
        "mustafar_compress": (i32, [vp, i64, i64, i64, i32, f32, P(CacheT), vp, vp]),
        "mustafar_append": (i32, [vp, i64, i64, vp, P(CacheT), vp, vp]),
        "mustafar_decode_workspace_bytes": (i32, [i32, i32, i32, i32, i32, i32, P(sz)]),
        "mustafar_decode_attn": (i32, [vp, i32, P(CacheT), P(CacheT), vp, i32, f32, vp, vp, vp, sz, i32, vp, vp]),
        "mustafar_dense_decode_attn": (i32, [vp, i32, vp, vp, i32, i32, i32, i32, vp, i32, f32, vp, vp, vp, sz,
                                             i32, vp, vp]),
        "mustafar_decode_plan_splits": (i32, [i32, i32, i32, i32, i32, i32, i32]),
        "mustafar_decode_plan_cluster": (i32, [i32, i32, i32, i32, i32, i32, i32]),
        "mustafar_status_string": (C.c_char_p, [i32]),
        "mustafar_last_error": (C.c_char_p, []),
        "mustafar_abi_version": (i32, []),
        "mustafar_decode_attn_noalloc": (i32, [vp, i32, P(CacheT), P(CacheT), vp, i32, f32, vp, vp, i32, vp, vp]),
        "mustafar_decode_step": (i32, [vp, i32, vp, i64, i64, vp, i64, i64, vp, P(CacheT), P(CacheT), i32, f32, vp,
                                       vp, vp, sz, i32, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != MUSTAFAR_OK:
        raise MustafarError(status, load().mustafar_last_error().decode())


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _cuda_f16(t: torch.Tensor, name: str):
    if not (t.is_cuda and t.dtype == torch.float16):
        raise TypeError(f"{name} must be a CUDA float16 tensor")


# ------------------------------------------------------------------------------------------- queries
def mustafar_keep_count(head_dim: int, sparsity: float) -> int:
    k = load().mustafar_keep_count(head_dim, sparsity)
    if k < 0:
        raise ValueError("head_dim must be a positive multiple of 32 and sparsity in [0, 1)")
    return k


def mustafar_keep_count_channel(head_dim: int, sparsity: float) -> int:
    """Values per token slot of a channel-wise cache: (head_dim/16) * (16 - floor(16*s))."""
    k = load().mustafar_keep_count_channel(head_dim, sparsity)
    if k < 0:
        raise ValueError("head_dim must be a positive multiple of 32 and sparsity in [0, 1)")
    return k


def mustafar_cache_sizes_channel(batch, num_kv_heads, head_dim, capacity, sparsity):
    """(bitmap_bytes, values_bytes, offset_bytes, window_bytes) of a channel-wise cache."""
    a, b, c, w = C.c_size_t(), C.c_size_t(), C.c_size_t(), C.c_size_t()
    _check(load().mustafar_cache_sizes_channel(batch, num_kv_heads, head_dim, capacity, sparsity, C.byref(a),
                                               C.byref(b), C.byref(c), C.byref(w)))
    return a.value, b.value, c.value, w.value


def mustafar_cache_sizes(batch, num_kv_heads, head_dim, capacity, sparsity):
    a, b, c = C.c_size_t(), C.c_size_t(), C.c_size_t()
    _check(load().mustafar_cache_sizes(batch, num_kv_heads, head_dim, capacity, sparsity,
                                       C.byref(a), C.byref(b), C.byref(c)))
    return a.value, b.value, c.value


def mustafar_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, max_len, num_splits=0, head_dim=HEAD_DIM):
    n = C.c_size_t()
    _check(load().mustafar_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_len,
                                                  num_splits, C.byref(n)))
    return n.value


def mustafar_decode_plan_splits(batch, num_kv_heads, max_len, keep_k, keep_v, dense=False, head_dim=HEAD_DIM):
    s = load().mustafar_decode_plan_splits(batch, num_kv_heads, head_dim, max_len, keep_k, keep_v, int(dense))
    if s < 1:
        raise MustafarError(1, "invalid shapes for the split plan")
    return s


def mustafar_decode_plan_cluster(batch, num_q_heads, num_kv_heads, max_len, keep_k, keep_v, head_dim=HEAD_DIM):
    """CTAs per thread-block cluster of the automatic plan (0: ticket merge through the workspace)."""
    c = load().mustafar_decode_plan_cluster(batch, num_q_heads, num_kv_heads, head_dim, max_len, keep_k, keep_v)
    if c < 0:
        raise MustafarError(1, "invalid shapes for the decode plan")
    return c


# ------------------------------------------------------------------------------------------- caches
def mustafar_cache_sizes_per_head(batch, num_kv_heads, capacity, head_keep, head_dim=HEAD_DIM):
    """(bitmap_bytes, values_bytes, offset_bytes) of a cache with keep count head_keep[h] per kv head."""
    arr = (C.c_int32 * len(head_keep))(*head_keep)
    nb, nv, no = C.c_size_t(), C.c_size_t(), C.c_size_t()
    _check(load().mustafar_cache_sizes_per_head(batch, num_kv_heads, head_dim, capacity, C.cast(arr, C.c_void_p),
                                                C.byref(nb), C.byref(nv), C.byref(no)))
    return nb.value, nv.value, no.value


class CompressedCache:
    """Caller-owned device arrays of one compressed cache (K or V) plus its C descriptor.

    ``sparsity`` is one value for every kv head, or a sequence with one sparsity per kv head
    (then head h keeps ``mustafar_keep_count(head_dim, sparsity[h])`` channels per token).
    ``pattern="2:4"`` selects 2:4 semi-structured pruning instead (sparsity 0.5, one value), and
    ``pattern="channel"`` channel-wise pruning over 16-token windows (one sparsity; the cache then
    also holds ``window``, the dense copy of each stream's newest incomplete window)."""

    def __init__(self, batch: int, num_kv_heads: int, capacity: int, sparsity, head_dim: int = HEAD_DIM,
                 device="cuda", pattern: str = "topk"):
        self.batch, self.num_kv_heads, self.head_dim, self.capacity = batch, num_kv_heads, head_dim, capacity
        if pattern not in ("topk", "2:4", "channel"):
            raise ValueError("pattern must be 'topk', '2:4' or 'channel'")
        if pattern == "channel" and isinstance(sparsity, (list, tuple)):
            raise ValueError("a channel-wise cache has one sparsity for every head")
        if pattern == "2:4" and (isinstance(sparsity, (list, tuple)) or float(sparsity) != 0.5):
            raise ValueError("a 2:4 cache has sparsity 0.5 for every head")
        self.pattern = pattern
        self._head_keep_arr = None
        if isinstance(sparsity, (list, tuple)):
            if len(sparsity) != num_kv_heads:
                raise ValueError("one sparsity per kv head expected")
            self.head_sparsity = [float(x) for x in sparsity]
            self.head_keep = [mustafar_keep_count(head_dim, x) for x in self.head_sparsity]
            self.sparsity = None
            self.keep = max(self.head_keep)
            nb, nv, no = mustafar_cache_sizes_per_head(batch, num_kv_heads, capacity, self.head_keep, head_dim)
            self._head_keep_arr = (C.c_int32 * num_kv_heads)(*self.head_keep)
        elif pattern == "channel":
            self.sparsity = float(sparsity)
            self.keep = mustafar_keep_count_channel(head_dim, sparsity)
            self.head_keep = [self.keep] * num_kv_heads
            self.head_sparsity = None
            nb, nv, no, nw = mustafar_cache_sizes_channel(batch, num_kv_heads, head_dim, capacity, sparsity)
        else:
            self.sparsity = float(sparsity)
            self.keep = mustafar_keep_count(head_dim, sparsity)
            self.head_keep = [self.keep] * num_kv_heads
            self.head_sparsity = None
            nb, nv, no = mustafar_cache_sizes(batch, num_kv_heads, head_dim, capacity, sparsity)
        self.bitmap = torch.zeros(nb // 4, dtype=torch.int32, device=device)
        self.values = torch.zeros(nv // 2, dtype=torch.int16, device=device)
        self.tile_offset = torch.zeros(no // 4, dtype=torch.int32, device=device)
        self.window = (torch.zeros(nw // 2, dtype=torch.int16, device=device) if pattern == "channel" else None)
        hk = C.cast(self._head_keep_arr, C.c_void_p).value if self._head_keep_arr is not None else None
        code = {"topk": PATTERN_TOPK, "2:4": PATTERN_2_4, "channel": PATTERN_CHANNEL}[pattern]
        self._struct = CacheT(batch, num_kv_heads, head_dim, capacity, self.keep, self.bitmap.data_ptr(),
                              self.values.data_ptr(), self.tile_offset.data_ptr(), hk, code,
                              self.window.data_ptr() if self.window is not None else None)

    @property
    def struct(self) -> CacheT:
        return self._struct

    @property
    def per_head(self) -> bool:
        return self._head_keep_arr is not None

    def nbytes(self) -> int:
        extra = self.window.numel() * 2 if self.window is not None else 0
        return self.bitmap.numel() * 4 + self.values.numel() * 2 + self.tile_offset.numel() * 4 + extra

    def value_base(self, b: int, h: int) -> int:
        """Element index where stream (b, h)'s packed values start."""
        return self.capacity * (b * sum(self.head_keep) + sum(self.head_keep[:h]))

    def stream_values(self, b: int, h: int) -> torch.Tensor:
        """The capacity * head_keep[h] packed values of stream (b, h) (int16 view)."""
        base = self.value_base(b, h)
        return self.values[base:base + self.capacity * self.head_keep[h]]

    def views(self):
        """(bitmap [B,H,cap,d/32] int32, values [B,H,cap*k] int16, tile_offset [B,H,cap/64] int32);
        uniform caches only (per-head caches: ``stream_values``)."""
        if self.per_head:
            raise ValueError("values of a per-head cache have no [B, H, cap*k] view; use stream_values")
        B, H, cap, d = self.batch, self.num_kv_heads, self.capacity, self.head_dim
        return (self.bitmap.view(B, H, cap, d // 32), self.values.view(B, H, cap * self.keep),
                self.tile_offset.view(B, H, cap // 64))

    def window_view(self):
        """window [B, H, 16, d] int16 of a channel-wise cache."""
        if self.window is None:
            raise ValueError("only a channel-wise cache has a window")
        return self.window.view(self.batch, self.num_kv_heads, WINDOW_TOKENS, self.head_dim)


# ------------------------------------------------------------------------------------------- calls
def mustafar_compress(x: torch.Tensor, L: int, sparsity: float, cache: CompressedCache, err=None, stream=None):
    """Prune + compress tokens [0, L) of ``x`` ([B, H, T, d] fp16, d contiguous) into ``cache``."""
    _cuda_f16(x, "x")
    if x.dim() != 4 or x.stride(3) != 1:
        raise ValueError("x must be [B, H, T, d] with contiguous channels")
    if tuple(x.shape[:2]) != (cache.batch, cache.num_kv_heads) or x.shape[3] != cache.head_dim or x.shape[2] < L:
        raise ValueError("x shape does not match the cache")
    _check(load().mustafar_compress(_ptr(x), x.stride(0), x.stride(1), x.stride(2), L, sparsity,
                                    C.byref(cache.struct), _ptr(err), _stream(stream)))


def mustafar_append(x: torch.Tensor, pos: torch.Tensor, cache: CompressedCache, err=None, stream=None):
    """Prune + compress one token per (b, kv head) (``x`` [B, H, d] fp16) into slot ``pos[b]``."""
    _cuda_f16(x, "x")
    if x.dim() != 3 or x.stride(2) != 1 or tuple(x.shape) != (cache.batch, cache.num_kv_heads, cache.head_dim):
        raise ValueError("x must be [B, H, d] with contiguous channels, matching the cache")
    if not (pos.is_cuda and pos.dtype == torch.int32 and pos.numel() == cache.batch):
        raise ValueError("pos must be a CUDA int32 tensor of length batch")
    _check(load().mustafar_append(_ptr(x), x.stride(0), x.stride(1), _ptr(pos), C.byref(cache.struct), _ptr(err),
                                  _stream(stream)))


def _decode_outputs(q, out, lse, want_lse):
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device)
    return out, lse


def mustafar_decode_attn(q: torch.Tensor, k: CompressedCache, v: CompressedCache, seq_len: torch.Tensor,
                         max_len: int, scale: float, out=None, lse=None, workspace=None, num_splits: int = 0,
                         err=None, stream=None, want_lse: bool = True):
    """Sparse decode attention over compressed caches; returns (out [B,Hq,d] fp16, lse [B,Hq] fp32)."""
    _cuda_f16(q, "q")
    if not q.is_contiguous() or q.dim() != 3:
        raise ValueError("q must be a contiguous [B, Hq, d] tensor")
    out, lse = _decode_outputs(q, out, lse, want_lse)
    if workspace is None:
        workspace = torch.zeros(mustafar_decode_workspace_bytes(q.shape[0], q.shape[1], k.num_kv_heads, max_len,
                                                                num_splits), dtype=torch.uint8, device=q.device)
    _check(load().mustafar_decode_attn(_ptr(q), q.shape[1], C.byref(k.struct), C.byref(v.struct), _ptr(seq_len),
                                       max_len, scale, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                                       num_splits, _ptr(err), _stream(stream)))
    return out, lse


def mustafar_dense_decode_attn(q: torch.Tensor, k_dense: torch.Tensor, v_dense: torch.Tensor, seq_len: torch.Tensor,
                               max_len: int, scale: float, out=None, lse=None, workspace=None, num_splits: int = 0,
                               err=None, stream=None, want_lse: bool = True):
    """Dense fp16 decode attention (baseline) over [B, Hkv, cap, d] caches."""
    for t, n in ((q, "q"), (k_dense, "k_dense"), (v_dense, "v_dense")):
        _cuda_f16(t, n)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, Hkv, cap, d = k_dense.shape
    out, lse = _decode_outputs(q, out, lse, want_lse)
    if workspace is None:
        workspace = torch.zeros(mustafar_decode_workspace_bytes(B, q.shape[1], Hkv, max_len, num_splits),
                                dtype=torch.uint8, device=q.device)
    _check(load().mustafar_dense_decode_attn(_ptr(q), q.shape[1], _ptr(k_dense), _ptr(v_dense), B, Hkv, d, cap,
                                             _ptr(seq_len), max_len, scale, _ptr(out), _ptr(lse), _ptr(workspace),
                                             workspace.numel(), num_splits, _ptr(err), _stream(stream)))
    return out, lse


def mustafar_decode_attn_noalloc(q: torch.Tensor, k: CompressedCache, v: CompressedCache, seq_len: torch.Tensor,
                                 max_len: int, scale: float, out=None, lse=None, num_splits: int = 0, err=None,
                                 stream=None, want_lse: bool = True):
    """Sparse decode attention for callers that cannot allocate: same result as
    ``mustafar_decode_attn``, with the split-K scratch kept in the library's own fixed device
    array (shared by every call, so calls must not overlap on the GPU)."""
    _cuda_f16(q, "q")
    if not q.is_contiguous() or q.dim() != 3:
        raise ValueError("q must be a contiguous [B, Hq, d] tensor")
    out, lse = _decode_outputs(q, out, lse, want_lse)
    _check(load().mustafar_decode_attn_noalloc(_ptr(q), q.shape[1], C.byref(k.struct), C.byref(v.struct),
                                               _ptr(seq_len), max_len, scale, _ptr(out), _ptr(lse), num_splits,
                                               _ptr(err), _stream(stream)))
    return out, lse


class PreparedCall:
    """One library call whose arguments were checked and marshalled once.  Calling it runs the C
    entry point again with the same buffers, shapes and stream (the buffers' contents may change
    between calls); a serving loop that reuses its buffers saves the per-call Python marshalling."""

    def __init__(self, fn, args, keep_alive):
        self._fn, self._args, self._keep = fn, args, keep_alive

    def __call__(self) -> None:
        _check(self._fn(*self._args))


def _step_args(q, k_new, v_new, pos, k, v, max_len, scale, out, lse, workspace, num_splits, err, stream, want_lse):
    _cuda_f16(q, "q")
    if not q.is_contiguous() or q.dim() != 3:
        raise ValueError("q must be a contiguous [B, Hq, d] tensor")
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        _cuda_f16(t, n)
        if t.dim() != 3 or t.stride(2) != 1 or tuple(t.shape) != (k.batch, k.num_kv_heads, k.head_dim):
            raise ValueError(f"{n} must be [B, Hkv, d] with contiguous channels, matching the cache")
    if not (pos.is_cuda and pos.dtype == torch.int32 and pos.numel() == k.batch):
        raise ValueError("pos must be a CUDA int32 tensor of length batch")
    out, lse = _decode_outputs(q, out, lse, want_lse)
    if workspace is None:
        workspace = torch.zeros(mustafar_decode_workspace_bytes(q.shape[0], q.shape[1], k.num_kv_heads, max_len,
                                                                num_splits), dtype=torch.uint8, device=q.device)
    args = (_ptr(q), q.shape[1], _ptr(k_new), k_new.stride(0), k_new.stride(1), _ptr(v_new), v_new.stride(0),
            v_new.stride(1), _ptr(pos), C.byref(k.struct), C.byref(v.struct), max_len, scale, _ptr(out), _ptr(lse),
            _ptr(workspace), workspace.numel(), num_splits, _ptr(err), _stream(stream))
    return args, out, lse, (q, k_new, v_new, pos, k, v, out, lse, workspace, err)


def prepare_decode_step(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, pos: torch.Tensor,
                        k: CompressedCache, v: CompressedCache, max_len: int, scale: float, out=None, lse=None,
                        workspace=None, num_splits: int = 0, err=None, stream=None, want_lse: bool = True):
    """``mustafar_decode_step`` with its arguments marshalled once: returns (call, out, lse), where
    ``call()`` runs the step again on the same buffers (fill q, k_new, v_new and pos in place)."""
    args, out, lse, keep = _step_args(q, k_new, v_new, pos, k, v, max_len, scale, out, lse, workspace, num_splits,
                                      err, stream, want_lse)
    return PreparedCall(load().mustafar_decode_step, args, keep), out, lse


def mustafar_decode_step(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, pos: torch.Tensor,
                         k: CompressedCache, v: CompressedCache, max_len: int, scale: float, out=None, lse=None,
                         workspace=None, num_splits: int = 0, err=None, stream=None, want_lse: bool = True):
    """One decode step in one launch: compress ``k_new``/``v_new`` ([B, Hkv, d] fp16) into slot
    ``pos[b]`` of the caches, then attend over the ``pos[b] + 1`` tokens ``[0, pos[b]]``.
    Returns (out [B,Hq,d] fp16, lse [B,Hq] fp32); ``max_len`` bounds ``pos[b] + 1``."""
    args, out, lse, _ = _step_args(q, k_new, v_new, pos, k, v, max_len, scale, out, lse, workspace, num_splits, err,
                                   stream, want_lse)
    _check(load().mustafar_decode_step(*args))
    return out, lse


def capture_decode_steps(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, pos: torch.Tensor,
                         k: CompressedCache, v: CompressedCache, max_len: int, scale: float, out: torch.Tensor,
                         lse: torch.Tensor, workspace: torch.Tensor = None, num_splits: int = 0):
    """A multi-step decode loop as one CUDA graph: step i runs ``mustafar_decode_step`` on
    ``q[i]``, ``k_new[i]``, ``v_new[i]``, ``pos[i]`` (leading step axis) and writes ``out[i]``,
    ``lse[i]``.  Returns the captured ``torch.cuda.CUDAGraph``; each ``replay()`` runs every step
    again, in order, on whatever the input tensors then hold (the graph keeps their addresses).
    One warm-up step runs eagerly first (plans and kernel attributes are set outside capture), so
    the caches already hold step 0's token when the function returns."""
    steps = q.shape[0]
    if not all(t.shape[0] == steps for t in (k_new, v_new, pos, out, lse)):
        raise ValueError("q, k_new, v_new, pos, out and lse need the same number of steps")
    if workspace is None:
        workspace = torch.zeros(mustafar_decode_workspace_bytes(q.shape[1], q.shape[2], k.num_kv_heads, max_len,
                                                                num_splits), dtype=torch.uint8, device=q.device)
    stream = torch.cuda.Stream(device=q.device)
    stream.wait_stream(torch.cuda.current_stream(q.device))
    with torch.cuda.stream(stream):
        mustafar_decode_step(q[0], k_new[0], v_new[0], pos[0], k, v, max_len, scale, out=out[0], lse=lse[0],
                             workspace=workspace, num_splits=num_splits, stream=stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(steps):
                mustafar_decode_step(q[i], k_new[i], v_new[i], pos[i], k, v, max_len, scale, out=out[i], lse=lse[i],
                                     workspace=workspace, num_splits=num_splits, stream=stream)
    torch.cuda.current_stream(q.device).wait_stream(stream)
    graph._mustafar_keep = (q, k_new, v_new, pos, k, v, out, lse, workspace)
    return graph


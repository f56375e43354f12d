"""Python binding of the B200 hybrid GQA attention library (libhyb_attn.so).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/hyb_attn.h.  PyTorch supplies
device memory and streams.  There is no fallback: if the shared library is
missing or the device is not a B200, calls raise.

Functions keep the C names:
    hyb_kv_cache_init, hyb_kv_append, hyb_attn_prefill, hyb_attn_decode,
    hyb_attn_prefill_workspace_size, hyb_attn_decode_workspace_size,
    hyb_device_error, hyb_launch_count
plus the KVCache helper that allocates a layer's cache with torch.
"""
from __future__ import annotations

import ctypes
import os

import torch

SLIDING = 0
FULL = 1
N_Q_HEADS = 16
N_KV_HEADS = 4
HEAD_DIM = 256
WINDOW = 512
N_LAYERS = 36

KV_BF16 = 0
KV_FP8 = 1
DEV_ERR_CAPACITY = 1
DEV_ERR_TIMEOUT = 2
DEV_ERR_PAGE = 4
DEV_ERR_BOUNDS = 8      # debug build only: an index outside its buffer, access skipped
BUILD_DEBUG_BOUNDS = 1  # hyb_build_flags() bit of the debug build

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libhyb_attn.so")
# the -DHYB_DEBUG_BOUNDS build (device-side index checks); load(DEBUG_LIB_PATH) instead of load()
DEBUG_LIB_PATH = os.path.join(_PKG, "_lib", "libhyb_attn_debug.so")

EXPORTED = (
    "hyb_kv_cache_init", "hyb_kv_append", "hyb_attn_prefill_workspace_size", "hyb_attn_prefill",
    "hyb_attn_decode_workspace_size", "hyb_attn_decode", "hyb_device_error", "hyb_last_error",
    "hyb_launch_count", "hyb_profile_events", "hyb_profile_pairs_used", "hyb_attn_decode_noalloc",
    "hyb_selftest_wait_timeout", "hyb_linear", "hyb_attn_layer_prefill_workspace_size", "hyb_attn_layer_prefill",
    "hyb_attn_layer_decode_workspace_size", "hyb_attn_layer_decode", "hyb_attn_decode_partial",
    "hyb_attn_decode_merge", "hyb_attn_prefill_cache_workspace_size", "hyb_attn_layer_prefill_cache_workspace_size",
    "hyb_build_flags",
)


def layer_type(i: int) -> int:
    """Layer i is full attention iff i % 4 == 3 (3 sliding + 1 full, x9); past the schedule: full."""
    if i >= N_LAYERS:
        return FULL
    return FULL if i % 4 == 3 else SLIDING


class HybError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"hyb status {status}: {msg}")
        self.status = status


class _Cache(ctypes.Structure):
    _fields_ = [
        ("type", ctypes.c_int32), ("batch", ctypes.c_int32), ("capacity", ctypes.c_int64),
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("len", ctypes.c_void_p),
        ("head", ctypes.c_void_p), ("tag", ctypes.c_void_p),
        ("kv_dtype", ctypes.c_int32), ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
        ("page_size", ctypes.c_int32), ("max_pages", ctypes.c_int32), ("n_pages", ctypes.c_int64),
        ("block_table", ctypes.c_void_p),
    ]


_lib = None


def load(path: str = LIB_PATH):
    """Loads the shared library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with __graft_entry__.build() "
                           "or python full_gqa_attention_partial_b200/build.py")
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    pc = ctypes.POINTER(_Cache)
    lib.hyb_kv_cache_init.argtypes = [pc, vp, vp]
    lib.hyb_kv_append.argtypes = [pc, vp, vp, i64, vp, i32, vp]
    lib.hyb_attn_prefill_workspace_size.argtypes = [i32, i32, i32, i32]
    lib.hyb_attn_prefill_workspace_size.restype = sz
    lib.hyb_attn_prefill.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i64, i64, vp, pc, vp, sz, vp]
    lib.hyb_attn_decode_workspace_size.argtypes = [i32, i32, i64]
    lib.hyb_attn_decode_workspace_size.restype = sz
    lib.hyb_attn_decode.argtypes = [vp, vp, vp, pc, i32, i64, vp, vp, sz, vp]
    lib.hyb_attn_decode_noalloc.argtypes = [vp, vp, vp, pc, i32, i64, vp, vp]
    lib.hyb_attn_decode_noalloc.restype = ctypes.c_int
    lib.hyb_device_error.argtypes = [ctypes.POINTER(i32), i32, vp]
    lib.hyb_last_error.restype = ctypes.c_char_p
    lib.hyb_launch_count.restype = ctypes.c_uint64
    lib.hyb_build_flags.restype = ctypes.c_int32
    lib.hyb_profile_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), i32]
    lib.hyb_profile_events.restype = ctypes.c_int
    lib.hyb_profile_pairs_used.restype = i32
    lib.hyb_selftest_wait_timeout.argtypes = [vp]
    lib.hyb_linear.argtypes = [vp, i64, vp, i64, vp, i64, i32, i32, i32, vp]
    lib.hyb_attn_layer_prefill_workspace_size.argtypes = [i32, i32, i32, i32]
    lib.hyb_attn_layer_prefill_workspace_size.restype = sz
    lib.hyb_attn_layer_prefill.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, vp, pc, vp, sz, vp]
    lib.hyb_attn_layer_decode_workspace_size.argtypes = [i32, i32, i64]
    lib.hyb_attn_layer_decode_workspace_size.restype = sz
    lib.hyb_attn_layer_decode.argtypes = [vp, vp, vp, vp, pc, i32, i64, vp, vp, sz, vp]
    lib.hyb_attn_decode_partial.argtypes = [vp, vp, pc, i32, i64, vp, vp, vp, sz, vp]
    lib.hyb_attn_decode_merge.argtypes = [vp, vp, i64, i64, i32, i32, vp, vp, vp]
    lib.hyb_attn_prefill_cache_workspace_size.argtypes = [pc, i32]
    lib.hyb_attn_prefill_cache_workspace_size.restype = sz
    lib.hyb_attn_layer_prefill_cache_workspace_size.argtypes = [pc, i32]
    lib.hyb_attn_layer_prefill_cache_workspace_size.restype = sz
    for name in ("hyb_kv_cache_init", "hyb_kv_append", "hyb_attn_prefill", "hyb_attn_decode",
                 "hyb_device_error"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _check(status: int):
    if status != 0:
        raise HybError(status, load().hyb_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _row_stride(t: torch.Tensor, heads: int, name: str) -> int:
    """Token stride (elements) of a [B, T, heads, 256] bf16 view whose rows are laid out densely per token."""
    if t.dtype != torch.bfloat16 or t.dim() != 4 or t.shape[2] != heads or t.shape[3] != HEAD_DIM:
        raise ValueError(f"{name} must be bf16 [B, T, {heads}, 256], got {tuple(t.shape)} {t.dtype}")
    B, T = t.shape[:2]
    if t.stride(3) != 1 or t.stride(2) != HEAD_DIM:
        raise ValueError(f"{name}: heads must be dense 256-element rows")
    rs = t.stride(1) if T > 1 else max(t.stride(1), heads * HEAD_DIM)
    if B > 1 and t.stride(0) != T * rs:
        raise ValueError(f"{name}: batch stride must equal T * token stride")
    return rs


# ---------------------------------------------------------------------------
# KV cache
# ---------------------------------------------------------------------------
class KVCache:
    """One layer's KV cache for `batch` sequences (memory from torch).

    Full layers: linear cache of `capacity` tokens.  Sliding layers: 512-slot
    ring; `head0` gives each sequence's starting write slot.  kv_dtype KV_FP8
    stores e4m3 codes (uint8) with one fp32 scale per (token, KV head) row.

    Paged full layers: `page_size` > 0 (a multiple of 64), a pool of `n_pages`
    pages (k / v [n_pages, 4, page_size, 256], scales [n_pages, 4, page_size])
    and `block_table`, a device int32 [batch, max_pages] tensor owned by the
    caller: token i of sequence b sits in pool page block_table[b, i //
    page_size], row i % page_size; capacity = max_pages * page_size.
    """

    def __init__(self, layer_type: int, batch: int, capacity: int = WINDOW, device="cuda", head0=None,
                 stream=None, kv_dtype: int = 0, page_size: int = 0, n_pages: int = 0, block_table=None):
        paged = page_size > 0
        if paged:
            if block_table is None or block_table.dtype != torch.int32 or block_table.dim() != 2 \
                    or not block_table.is_contiguous() or block_table.shape[0] != batch:
                raise ValueError("a paged cache needs a contiguous int32 block_table [batch, max_pages]")
            cap = int(page_size) * block_table.shape[1]
        else:
            cap = WINDOW if layer_type == SLIDING else int(capacity)
        self.layer_type = layer_type
        self.batch = batch
        self.capacity = cap
        self.kv_dtype = kv_dtype
        self.page_size = int(page_size)
        self.block_table = block_table
        lead, rows = (int(n_pages), int(page_size)) if paged else (batch, cap)
        et = torch.uint8 if kv_dtype == KV_FP8 else torch.bfloat16
        self.k = torch.empty(lead, N_KV_HEADS, rows, HEAD_DIM, dtype=et, device=device)
        self.v = torch.empty(lead, N_KV_HEADS, rows, HEAD_DIM, dtype=et, device=device)
        self.len = torch.empty(batch, dtype=torch.int32, device=device)
        self.head = torch.empty(batch, dtype=torch.int32, device=device)
        self.tag = torch.empty(batch, WINDOW, dtype=torch.int32, device=device)
        self.k_scale = self.v_scale = None
        if kv_dtype == KV_FP8:
            self.k_scale = torch.empty(lead, N_KV_HEADS, rows, dtype=torch.float32, device=device)
            self.v_scale = torch.empty(lead, N_KV_HEADS, rows, dtype=torch.float32, device=device)
        self.c = _Cache(layer_type, batch, cap, self.k.data_ptr(), self.v.data_ptr(), self.len.data_ptr(),
                        self.head.data_ptr(), self.tag.data_ptr(), kv_dtype,
                        _ptr(self.k_scale), _ptr(self.v_scale),
                        self.page_size, block_table.shape[1] if paged else 0, int(n_pages) if paged else 0,
                        _ptr(block_table))
        hyb_kv_cache_init(self, head0, stream)

    @property
    def ref(self):
        return ctypes.byref(self.c)


def hyb_kv_cache_init(cache: KVCache, head0=None, stream=None):
    h0 = None
    if head0 is not None:
        arr = (ctypes.c_int32 * cache.batch)(*[int(x) for x in head0])
        h0 = ctypes.cast(arr, ctypes.c_void_p)
    _check(load().hyb_kv_cache_init(cache.ref, h0, _stream(stream)))


def hyb_kv_append(cache: KVCache, k: torch.Tensor, v: torch.Tensor, pos=None, stream=None):
    """Appends k/v [B, T, 4, 256] (views into fused qkv rows allowed) to the cache."""
    rs = _row_stride(k, N_KV_HEADS, "k")
    if _row_stride(v, N_KV_HEADS, "v") != rs:
        raise ValueError("k and v must share the token stride")
    T = k.shape[1]
    _check(load().hyb_kv_append(cache.ref, _ptr(k), _ptr(v), rs, _ptr(pos), T, _stream(stream)))


def hyb_attn_prefill_workspace_size(layer_type: int, B: int, T: int, with_cache: bool) -> int:
    return int(load().hyb_attn_prefill_workspace_size(layer_type, B, T, 1 if with_cache else 0))


def hyb_attn_decode_workspace_size(layer_type: int, B: int, max_len: int) -> int:
    return int(load().hyb_attn_decode_workspace_size(layer_type, B, max_len))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def hyb_attn_prefill(q, k, v, gate, pos, layer_type: int, out=None, cache: KVCache | None = None,
                     workspace=None, stream=None):
    """Prefill attention.  q [B,T,16,256], k/v [B,T,4,256], gate [B,T,16] or None,
    pos [B,T] int32 or None.  Returns out [B,T,16,256] bf16."""
    qs = _row_stride(q, N_Q_HEADS, "q")
    ks = _row_stride(k, N_KV_HEADS, "k")
    if _row_stride(v, N_KV_HEADS, "v") != ks:
        raise ValueError("k and v must share the token stride")
    B, T = q.shape[:2]
    if gate is not None and (gate.dtype != torch.bfloat16 or not gate.is_contiguous()
                             or tuple(gate.shape) != (B, T, N_Q_HEADS)):
        raise ValueError("gate must be contiguous bf16 [B, T, 16]")
    if pos is not None and (pos.dtype != torch.int32 or not pos.is_contiguous() or tuple(pos.shape) != (B, T)):
        raise ValueError("pos must be contiguous int32 [B, T]")
    if out is None:
        out = torch.empty(B, T, N_Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=q.device)
    need = hyb_attn_prefill_workspace_size(layer_type, B, T, False) if cache is None else \
        hyb_attn_prefill_cache_workspace_size(cache, T)
    if workspace is None and need > 0:
        workspace = alloc_workspace(need, q.device)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hyb_attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(pos), layer_type, B, T, qs, ks,
                                   _ptr(out), None if cache is None else cache.ref, _ptr(workspace), wsz,
                                   _stream(stream)))
    return out


HIDDEN = 2560


def hyb_attn_layer_decode_workspace_size(layer_type: int, B: int, max_len: int) -> int:
    return int(load().hyb_attn_layer_decode_workspace_size(layer_type, B, max_len))


def hyb_attn_prefill_cache_workspace_size(cache: "KVCache", T: int) -> int:
    return int(load().hyb_attn_prefill_cache_workspace_size(cache.ref, T))


def hyb_attn_layer_prefill_cache_workspace_size(cache: "KVCache", T: int) -> int:
    return int(load().hyb_attn_layer_prefill_cache_workspace_size(cache.ref, T))


def hyb_attn_layer_prefill_workspace_size(layer_type: int, B: int, T: int, with_cache: bool) -> int:
    return int(load().hyb_attn_layer_prefill_workspace_size(layer_type, B, T, 1 if with_cache else 0))


def hyb_attn_layer_prefill(hidden, w_qkv, w_gate, w_o, pos, layer_type: int, out=None,
                           cache: KVCache | None = None, workspace=None, stream=None):
    """One attention layer for prefill: q_k_v_proj, gate projection, attention,
    o_proj.  hidden bf16 [B,T,2560] contiguous; w_qkv [6144,2560], w_gate
    [16,2560] or None, w_o [2560,4096] (Linear weight layout); pos [B,T] int32
    or None.  Returns out bf16 [B,T,2560]."""
    if hidden.dtype != torch.bfloat16 or not hidden.is_contiguous() or hidden.shape[-1] != HIDDEN:
        raise ValueError("hidden must be contiguous bf16 [B, T, 2560]")
    for name, w, shape in (("w_qkv", w_qkv, (6144, HIDDEN)), ("w_o", w_o, (HIDDEN, N_Q_HEADS * HEAD_DIM)),
                           ("w_gate", w_gate, (N_Q_HEADS, HIDDEN))):
        if w is not None and (w.dtype != torch.bfloat16 or not w.is_contiguous() or tuple(w.shape) != shape):
            raise ValueError(f"{name} must be contiguous bf16 {list(shape)}")
    B, T = hidden.shape[:2]
    if pos is not None and (pos.dtype != torch.int32 or not pos.is_contiguous() or tuple(pos.shape) != (B, T)):
        raise ValueError("pos must be contiguous int32 [B, T]")
    if out is None:
        out = torch.empty(B, T, HIDDEN, dtype=torch.bfloat16, device=hidden.device)
    need = hyb_attn_layer_prefill_workspace_size(layer_type, B, T, False) if cache is None else \
        hyb_attn_layer_prefill_cache_workspace_size(cache, T)
    if workspace is None:
        workspace = alloc_workspace(need, hidden.device)
    wsz = workspace.numel() * workspace.element_size()
    _check(load().hyb_attn_layer_prefill(_ptr(hidden), _ptr(w_qkv), _ptr(w_gate), _ptr(w_o), _ptr(pos), layer_type,
                                         B, T, _ptr(out), None if cache is None else cache.ref, _ptr(workspace), wsz,
                                         _stream(stream)))
    return out


def hyb_attn_layer_decode(hidden, w_qkv, w_gate, w_o, cache: KVCache, max_len: int = 0, out=None, workspace=None,
                          stream=None):
    """One attention layer for a decode step: hidden bf16 [B,2560] (one new token
    per sequence); appends the token's K/V to `cache` and attends.  Returns
    out bf16 [B,2560]."""
    if hidden.dtype != torch.bfloat16 or not hidden.is_contiguous() or tuple(hidden.shape) != (cache.batch, HIDDEN):
        raise ValueError("hidden must be contiguous bf16 [B, 2560]")
    for name, w, shape in (("w_qkv", w_qkv, (6144, HIDDEN)), ("w_o", w_o, (HIDDEN, N_Q_HEADS * HEAD_DIM)),
                           ("w_gate", w_gate, (N_Q_HEADS, HIDDEN))):
        if w is not None and (w.dtype != torch.bfloat16 or not w.is_contiguous() or tuple(w.shape) != shape):
            raise ValueError(f"{name} must be contiguous bf16 {list(shape)}")
    B = cache.batch
    if out is None:
        out = torch.empty(B, HIDDEN, dtype=torch.bfloat16, device=hidden.device)
    lt = cache.layer_type
    need = hyb_attn_layer_decode_workspace_size(lt, B, max_len or cache.capacity)
    if workspace is None:
        workspace = alloc_workspace(need, hidden.device)
    wsz = workspace.numel() * workspace.element_size()
    _check(load().hyb_attn_layer_decode(_ptr(hidden), _ptr(w_qkv), _ptr(w_gate), _ptr(w_o), cache.ref, lt, max_len,
                                        _ptr(out), _ptr(workspace), wsz, _stream(stream)))
    return out



def _check_decode_args(q, gate, pos, cache: "KVCache", out=None):
    """Host-side checks of a decode call's tensors against the cache.

    The kernels launch one block row per cache sequence and read q / pos and
    write out for every one of them, so a q, pos or out with fewer rows than
    cache.batch would be read or written out of bounds: reject it here."""
    if q.dtype != torch.bfloat16 or not q.is_contiguous() or q.dim() != 3 \
            or tuple(q.shape[1:]) != (N_Q_HEADS, HEAD_DIM):
        raise ValueError("q must be contiguous bf16 [B, 16, 256]")
    B = q.shape[0]
    if B != cache.batch:
        raise ValueError(f"q has {B} sequences, the cache {cache.batch}")
    if gate is not None and (gate.dtype != torch.bfloat16 or not gate.is_contiguous()
                             or tuple(gate.shape) != (B, N_Q_HEADS)):
        raise ValueError("gate must be contiguous bf16 [B, 16]")
    if pos is not None and (pos.dtype != torch.int32 or not pos.is_contiguous() or tuple(pos.shape) != (B,)):
        raise ValueError("pos must be contiguous int32 [B]")
    if out is not None and (out.dtype != torch.bfloat16 or not out.is_contiguous()
                            or tuple(out.shape) != (B, N_Q_HEADS, HEAD_DIM)):
        raise ValueError("out must be contiguous bf16 [B, 16, 256]")
    return B


def hyb_attn_decode(q, gate, cache: KVCache, pos=None, max_len: int = 0, out=None, workspace=None,
                    stream=None):
    """One decode step.  q [B,16,256] contiguous (B = cache.batch), gate [B,16] or None,
    pos int32 [B] or None.  Returns out [B,16,256]."""
    _check_decode_args(q, gate, pos, cache, out)
    if out is None:
        out = torch.empty_like(q)
    ml = max_len if max_len else cache.capacity
    if workspace is None:
        workspace = alloc_workspace(hyb_attn_decode_workspace_size(cache.layer_type, cache.batch, ml), q.device)
    wsz = workspace.numel() * workspace.element_size()
    _check(load().hyb_attn_decode(_ptr(q), _ptr(gate), _ptr(pos), cache.ref, cache.layer_type, max_len,
                                  _ptr(out), _ptr(workspace), wsz, _stream(stream)))
    return out


def hyb_attn_decode_noalloc(q, gate, cache: KVCache, pos=None, max_len: int = 0, out=None, stream=None):
    """hyb_attn_decode without a workspace: for callers that may not allocate
    device memory while decoding.  The split partials go to a fixed 4 MiB
    scratch inside the library, shared by all calls (calls that overlap on
    the GPU race on it).  `out` should be preallocated by such callers; when
    it is None a tensor is allocated here for convenience."""
    _check_decode_args(q, gate, pos, cache, out)
    if out is None:
        out = torch.empty_like(q)
    _check(load().hyb_attn_decode_noalloc(_ptr(q), _ptr(gate), _ptr(pos), cache.ref, cache.layer_type, max_len,
                                          _ptr(out), _stream(stream)))
    return out


def hyb_attn_decode_partial(q, cache: KVCache, pos=None, max_len: int = 0, part_o=None, part_lse=None,
                            workspace=None, stream=None):
    """Attention of q [B,16,256] over the keys of `cache` only, ungated: returns
    (part_o fp32 [B,16,256] normalised over these keys, part_lse fp32 [B,16] =
    log2 sum_j exp(q.k_j / 16)).  pos: int32 [B] query positions in the whole
    sequence (None: len - 1 of this cache)."""
    B = _check_decode_args(q, None, pos, cache)
    if part_o is None:
        part_o = torch.empty(B, N_Q_HEADS, HEAD_DIM, dtype=torch.float32, device=q.device)
    if part_lse is None:
        part_lse = torch.empty(B, N_Q_HEADS, dtype=torch.float32, device=q.device)
    if part_o.dtype != torch.float32 or not part_o.is_contiguous() or tuple(part_o.shape) != (B, N_Q_HEADS, HEAD_DIM):
        raise ValueError("part_o must be contiguous fp32 [B, 16, 256]")
    if part_lse.dtype != torch.float32 or not part_lse.is_contiguous() or tuple(part_lse.shape) != (B, N_Q_HEADS):
        raise ValueError("part_lse must be contiguous fp32 [B, 16]")
    need = hyb_attn_decode_workspace_size(cache.layer_type, B, max_len or cache.capacity)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    wsz = workspace.numel() * workspace.element_size()
    _check(load().hyb_attn_decode_partial(_ptr(q), _ptr(pos), cache.ref, cache.layer_type, max_len, _ptr(part_o),
                                          _ptr(part_lse), _ptr(workspace), wsz, _stream(stream)))
    return part_o, part_lse


def hyb_attn_decode_merge(part_o, part_lse, gate=None, out=None, stream=None):
    """Merges partials part_o fp32 [P,B,16,256] / part_lse fp32 [P,B,16]
    (e.g. all-gathered from P GPUs), applies the gate (bf16 [B,16] or None);
    returns bf16 [B,16,256]."""
    if part_o.dtype != torch.float32 or not part_o.is_contiguous() or part_o.dim() != 4 \
            or tuple(part_o.shape[2:]) != (N_Q_HEADS, HEAD_DIM):
        raise ValueError("part_o must be contiguous fp32 [P, B, 16, 256]")
    P, B = part_o.shape[:2]
    if part_lse.dtype != torch.float32 or not part_lse.is_contiguous() or tuple(part_lse.shape) != (P, B, N_Q_HEADS):
        raise ValueError("part_lse must be contiguous fp32 [P, B, 16]")
    if gate is not None and (gate.dtype != torch.bfloat16 or not gate.is_contiguous()
                             or tuple(gate.shape) != (B, N_Q_HEADS)):
        raise ValueError("gate must be contiguous bf16 [B, 16]")
    if out is None:
        out = torch.empty(B, N_Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=part_o.device)
    _check(load().hyb_attn_decode_merge(_ptr(part_o), _ptr(part_lse), 0, 0, P, B, _ptr(gate), _ptr(out),
                                        _stream(stream)))
    return out


def decode_record_floats(B: int) -> int:
    """Floats in one partial record: output [B,16,256] then lse [B,16]."""
    return B * N_Q_HEADS * (HEAD_DIM + 1)


def record_views(rec: torch.Tensor, B: int):
    """(part_o [B,16,256], part_lse [B,16]) views into one fp32 partial record."""
    n = B * N_Q_HEADS * HEAD_DIM
    return rec[:n].view(B, N_Q_HEADS, HEAD_DIM), rec[n:n + B * N_Q_HEADS].view(B, N_Q_HEADS)


def hyb_attn_decode_merge_records(records, B: int, gate=None, out=None, stream=None):
    """Merges P partial records (fp32 [P, B*16*257]: each part's output, then
    its lse), e.g. one all-gather of the per-GPU records; returns bf16 [B,16,256]."""
    rf = decode_record_floats(B)
    if records.dtype != torch.float32 or not records.is_contiguous() or records.dim() != 2 \
            or records.shape[1] != rf:
        raise ValueError(f"records must be contiguous fp32 [P, {rf}]")
    if gate is not None and (gate.dtype != torch.bfloat16 or not gate.is_contiguous()
                             or tuple(gate.shape) != (B, N_Q_HEADS)):
        raise ValueError("gate must be contiguous bf16 [B, 16]")
    if out is None:
        out = torch.empty(B, N_Q_HEADS, HEAD_DIM, dtype=torch.bfloat16, device=records.device)
    base = records.data_ptr()
    _check(load().hyb_attn_decode_merge(ctypes.c_void_p(base), ctypes.c_void_p(base + 4 * B * N_Q_HEADS * HEAD_DIM),
                                        rf, rf, records.shape[0], B, _ptr(gate), _ptr(out), _stream(stream)))
    return out


def hyb_device_error(clear: bool = True, stream=None) -> int:
    flags = ctypes.c_int32(0)
    _check(load().hyb_device_error(ctypes.byref(flags), 1 if clear else 0, _stream(stream)))
    return int(flags.value)


def hyb_linear(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor = None, stream=None) -> torch.Tensor:
    """y = x @ w.T on the tensor cores: x bf16 [..., K] (unit stride along K),
    w bf16 [N, K] (Linear weight layout); returns bf16 [..., N]."""
    K = x.shape[-1]
    N = w.shape[0]
    x2 = x.reshape(-1, K)
    if x2.stride(-1) != 1:
        x2 = x2.contiguous()
    if w.stride(-1) != 1:
        w = w.contiguous()
    M = x2.shape[0]
    if out is None:
        out = torch.empty(*x.shape[:-1], N, dtype=torch.bfloat16, device=x.device)
    y2 = out.view(-1, N)
    _check(load().hyb_linear(_ptr(x2), x2.stride(0), _ptr(w), w.stride(0), _ptr(y2), y2.stride(0), M, N, K,
                             _stream(stream)))
    return out


def hyb_selftest_wait_timeout(stream=None) -> None:
    """Runs the failure-path self-test kernel (a wait that times out); the
    error word then holds DEV_ERR_TIMEOUT (read it with hyb_device_error)."""
    _check(load().hyb_selftest_wait_timeout(_stream(stream)))


def hyb_launch_count() -> int:
    return int(load().hyb_launch_count())


def hyb_build_flags() -> int:
    """BUILD_DEBUG_BOUNDS when the loaded library is the index-checking debug build, else 0."""
    return int(load().hyb_build_flags())


class KernelTimer:
    """Brackets the next `n` attention-kernel launches with CUDA events.

    Uses hyb_profile_events: the library records events[2i] / events[2i+1]
    on the launch stream right before / after the i-th prefill-attention or
    decode split-KV kernel launch.
    """

    def __init__(self, n: int):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n)]
        for e in self.events:   # torch creates the CUDA event lazily, on first record
            e.record()
        torch.cuda.synchronize()
        self._arr = (ctypes.c_void_p * (2 * n))(*[e.cuda_event for e in self.events])
        self.n = n

    def __enter__(self):
        _check(load().hyb_profile_events(self._arr, self.n))
        return self

    def __exit__(self, *exc):
        self.used = int(load().hyb_profile_pairs_used())
        _check(load().hyb_profile_events(None, 0))
        return False

    def times_ms(self):
        torch.cuda.synchronize()
        return [self.events[2 * i].elapsed_time(self.events[2 * i + 1]) for i in range(self.used)]

"""Host-side tests of the C-ABI library that need no GPU.

* the shared library loads and exports every function include/hyb_attn.h
  declares;
* argument checks that run before any CUDA call return the documented
  status codes;
* workspace-size arithmetic.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hyb_attn.h")


@pytest.fixture(scope="module")
def hyb():
    import full_gqa_attention_partial_b200 as hyb
    from full_gqa_attention_partial_b200 import build
    build.build()
    hyb.load()
    return hyb


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hyb_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for fn in ("hyb_attn_prefill", "hyb_attn_decode", "hyb_kv_append", "hyb_kv_cache_init"):
        assert fn in names


def test_library_exports_every_declared_symbol(hyb):
    lib = ctypes.CDLL(hyb.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(_declared_functions()) <= set(hyb.EXPORTED) | {"hyb_last_error"}


def test_debug_bounds_build(hyb):
    """The -DHYB_DEBUG_BOUNDS twin is built beside the library, exports the
    same boundary and says what it is; the normal build says it is not."""
    assert os.path.exists(hyb.DEBUG_LIB_PATH)
    dbg = ctypes.CDLL(hyb.DEBUG_LIB_PATH)
    for name in _declared_functions():
        assert hasattr(dbg, name), name
    dbg.hyb_build_flags.restype = ctypes.c_int32
    assert dbg.hyb_build_flags() == hyb.BUILD_DEBUG_BOUNDS
    assert hyb.hyb_build_flags() == 0


def _cache(hyb, lt=0, batch=1, cap=512, null_k=False):
    c = hyb._Cache(lt, batch, cap, 0 if null_k else 0x1000, 0x2000, 0x3000, 0x4000, 0x5000)
    return c


def test_argument_checks_before_any_cuda_call(hyb):
    lib = hyb.load()
    vp = ctypes.c_void_p
    A = vp(0x10000)
    # null q
    assert lib.hyb_attn_prefill(None, A, A, None, None, 0, 1, 8, 4096, 1024, A, None, None, 0, None) == -1
    # bad layer type
    assert lib.hyb_attn_prefill(A, A, A, None, None, 7, 1, 8, 4096, 1024, A, None, None, 0, None) == -1
    # T = 0
    assert lib.hyb_attn_prefill(A, A, A, None, None, 0, 1, 0, 4096, 1024, A, None, None, 0, None) == -1
    # misaligned q
    assert lib.hyb_attn_prefill(vp(0x10008), A, A, None, None, 0, 1, 8, 4096, 1024, A, None, None, 0,
                                None) == -3
    # q row stride not a multiple of 8 / too small
    assert lib.hyb_attn_prefill(A, A, A, None, None, 0, 1, 8, 4100, 1024, A, None, None, 0, None) == -3
    assert lib.hyb_attn_prefill(A, A, A, None, None, 0, 1, 8, 1024, 1024, A, None, None, 0, None) == -3
    # workspace missing / too small
    assert lib.hyb_attn_prefill(A, A, A, None, None, 0, 1, 8, 4096, 1024, A, None, None, 0, None) == -1
    assert lib.hyb_attn_prefill(A, A, A, None, None, 0, 1, 8, 4096, 1024, A, None, vp(0x20000), 16,
                                None) == -4
    msg = lib.hyb_last_error().decode()
    assert "workspace" in msg
    # cache problems
    c = _cache(hyb, lt=0, cap=100)
    assert lib.hyb_kv_append(ctypes.byref(c), A, A, 1024, None, 4, None) == -2      # sliding cap != 512
    c = _cache(hyb, lt=1, cap=1024, null_k=True)
    assert lib.hyb_kv_append(ctypes.byref(c), A, A, 1024, None, 4, None) == -1      # null k buffer
    c = _cache(hyb, lt=1, cap=1024)
    assert lib.hyb_kv_append(ctypes.byref(c), A, A, 1024, None, 0, None) == -1      # T = 0
    assert lib.hyb_kv_append(ctypes.byref(c), A, A, 1000, None, 4, None) == -3      # stride
    # cache type vs layer type; batch mismatch; T beyond a full cache's capacity
    assert lib.hyb_attn_prefill(A, A, A, None, None, 0, 1, 8, 4096, 1024, A, ctypes.byref(c), None, 0,
                                None) == -2
    assert lib.hyb_attn_prefill(A, A, A, None, None, 1, 2, 8, 4096, 1024, A, ctypes.byref(c), None, 0,
                                None) == -2
    assert lib.hyb_attn_prefill(A, A, A, None, None, 1, 1, 2048, 4096, 1024, A, ctypes.byref(c), None, 0,
                                None) == -2
    # decode: max_len beyond capacity, layer type mismatch
    assert lib.hyb_attn_decode(A, None, None, ctypes.byref(c), 1, 4096, A, A, 1 << 20, None) == -2
    assert lib.hyb_attn_decode(A, None, None, ctypes.byref(c), 0, 0, A, A, 1 << 20, None) == -2


def test_workspace_sizes(hyb):
    # cache-less prefill holds the rotated keys: B * T * 4 heads * 256 * 2 bytes
    assert hyb.hyb_attn_prefill_workspace_size(hyb.FULL, 2, 1000, False) == 2 * 1000 * 2048
    assert hyb.hyb_attn_prefill_workspace_size(hyb.FULL, 2, 1000, True) == 0
    # sliding chunk: context K and V of 511 + T rows, plus the rotated copy of the queries
    assert hyb.hyb_attn_prefill_workspace_size(hyb.SLIDING, 1, 8192, True) == 2 * (511 + 8192) * 2048 + 8192 * 8192
    assert hyb.hyb_attn_prefill_workspace_size(hyb.SLIDING, 2, 1000, False) == 2 * 1000 * (2048 + 8192)
    # decode: B * 16 * splits * (256 + 1) floats, rounded up
    for lt, B, L in ((hyb.FULL, 1, 1 << 20), (hyb.FULL, 16, 131073), (hyb.SLIDING, 16, 512)):
        n = hyb.hyb_attn_decode_workspace_size(lt, B, L)
        assert n >= B * 16 * 257 * 4 and n % 4 == 0


def test_layer_schedule_binding(hyb):
    types = [hyb.layer_type(i) for i in range(36)]
    assert types.count(hyb.FULL) == 9 and types[3] == hyb.FULL and types[35] == hyb.FULL


def test_paged_cache_checks_before_any_cuda_call(hyb):
    """A paged cache (full layers only) must have a page size that is a
    multiple of 64, capacity = max_pages x page_size, a pool and an aligned
    block table; every violation returns before anything is enqueued."""
    lib = hyb.load()
    A = ctypes.c_void_p(0x10000)

    def paged(lt=1, page=128, max_pages=8, cap=None, n_pages=16, table=0x6000):
        cap = page * max_pages if cap is None else cap
        return hyb._Cache(lt, 2, cap, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0, None, None,
                          page, max_pages, n_pages, table)

    def append(c):
        return lib.hyb_kv_append(ctypes.byref(c), A, A, 1024, None, 4, None)

    assert append(paged(lt=0, cap=512, page=64, max_pages=8)) == -1      # a sliding ring cannot be paged
    assert append(paged(page=96)) == -2                                   # not a multiple of 64
    assert append(paged(cap=1000)) == -2                                  # capacity != max_pages x page
    assert append(paged(max_pages=0, cap=0)) == -1                        # no table entries
    assert append(paged(n_pages=0)) == -1                                 # empty pool
    assert append(paged(table=0)) == -1                                   # no block table
    assert append(paged(table=0x6002)) == -3                              # misaligned block table
    assert append(hyb._Cache(1, 2, 1024, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0, None, None,
                             -64, 0, 0, None)) == -1                      # negative page size
    assert "page" in lib.hyb_last_error().decode()


def test_partial_and_merge_checks_before_any_cuda_call(hyb):
    lib = hyb.load()
    A = ctypes.c_void_p(0x10000)
    c = _cache(hyb, lt=1, cap=1024)
    # partial: output buffers required and aligned
    assert lib.hyb_attn_decode_partial(A, None, ctypes.byref(c), 1, 0, None, A, A, 1 << 20, None) == -1
    assert lib.hyb_attn_decode_partial(A, None, ctypes.byref(c), 1, 0, ctypes.c_void_p(0x10004), A, A, 1 << 20,
                                       None) == -3
    assert lib.hyb_attn_decode_partial(A, None, ctypes.byref(c), 0, 0, A, A, A, 1 << 20, None) == -2   # type
    # merge: null buffers, non-positive counts, misalignment
    assert lib.hyb_attn_decode_merge(None, A, 0, 0, 2, 1, None, A, None) == -1
    assert lib.hyb_attn_decode_merge(A, A, 0, 0, 0, 1, None, A, None) == -1
    assert lib.hyb_attn_decode_merge(A, A, 0, 0, 2, -1, None, A, None) == -1
    assert lib.hyb_attn_decode_merge(A, A, 4095, 0, 2, 1, None, A, None) == -2               # stride below a part
    assert lib.hyb_attn_decode_merge(A, A, 0, 15, 2, 1, None, A, None) == -2
    assert lib.hyb_attn_decode_merge(A, ctypes.c_void_p(0x10002), 0, 0, 2, 1, None, A, None) == -3
    assert lib.hyb_attn_decode_merge(A, A, 0, 0, 2, 1, ctypes.c_void_p(0x10001), A, None) == -3
    assert lib.hyb_attn_decode_merge(A, A, 0, 0, 1 << 20, 1 << 10, None, A, None) == -4      # > 2^31 elements


def test_header_is_plain_c_and_links(hyb, tmp_path):
    """A C99 program that includes only the header links against the library
    and gets the documented status back from a call that fails its checks
    (no CUDA device is touched)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include "hyb_attn.h"
int main(void) {
  hyb_kv_cache c = {0};
  c.type = HYB_SLIDING; c.batch = 1; c.capacity = 100;          /* a ring must hold 512 */
  c.k = (void*)0x1000; c.v = (void*)0x2000; c.len = (int32_t*)0x3000;
  c.head = (int32_t*)0x4000; c.tag = (int32_t*)0x5000;
  hyb_status s = hyb_kv_append(&c, (void*)0x10000, (void*)0x10000, 1024, NULL, 4, NULL);
  printf("%d %s\n", (int)s, hyb_last_error());
  return s == HYB_ESHAPE ? 0 : 1;
}
''')
    exe = tmp_path / "abi"
    lib_dir = os.path.dirname(hyb.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", str(exe), "-L", lib_dir, "-lhyb_attn", "-Wl,-rpath," + lib_dir])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "512" in r.stdout


def test_workspace_sizes_cover_every_grid(hyb):
    """For random batch sizes and lengths the decode workspace holds the
    partials of the larger of the bf16 and FP8 split grids (B x 16 x splits x
    (256 + 1) floats), and the whole-layer sizes exceed the attention's."""
    import random
    rnd = random.Random(3)
    for _ in range(200):
        lt = rnd.choice([hyb.SLIDING, hyb.FULL])
        B = rnd.randint(1, 64)
        L = rnd.randint(1, 1 << 21)
        n = hyb.hyb_attn_decode_workspace_size(lt, B, L)
        assert n % 256 == 0 or n % 4 == 0
        rows = B * 16
        splits = (n - ((rows * 4 + 255) // 256) * 256) // (rows * 256 * 4)
        assert splits >= 1
        assert hyb.hyb_attn_layer_decode_workspace_size(lt, B, L) > n
        T = rnd.randint(1, 40000)
        # the layer call holds the fused q|k|v rows and the attention output besides the attention's scratch
        # (minus the rotated query copy, which the layer's pre-rotated queries do not need)
        attn = hyb.hyb_attn_prefill_workspace_size(lt, B, T, True) - (B * T * 16 * 256 * 2 if lt == hyb.SLIDING else 0)
        assert hyb.hyb_attn_layer_prefill_workspace_size(lt, B, T, True) >= attn + B * T * (6144 + 4096) * 2


class _FakeCache:
    """Stands in for a KVCache in the binding's host-side checks (no device memory)."""

    def __init__(self, batch, layer_type=0, capacity=512):
        self.batch, self.layer_type, self.capacity = batch, layer_type, capacity

    @property
    def ref(self):   # reaching the library would mean a check was skipped
        raise AssertionError("the call got past the binding's checks")


@pytest.mark.parametrize("fn", ["hyb_attn_decode", "hyb_attn_decode_noalloc", "hyb_attn_decode_partial"])
def test_decode_wrappers_reject_shape_mismatches_before_any_launch(hyb, fn):
    import torch
    call = getattr(hyb, fn)
    cache = _FakeCache(batch=3)
    bf = torch.bfloat16

    def go(q, gate=None, pos=None, out=None):
        if fn == "hyb_attn_decode_partial":
            return call(q, cache, pos=pos)
        return call(q, gate, cache, pos=pos, out=out)

    good_q = torch.zeros(3, 16, 256, dtype=bf)
    bad = [
        dict(q=torch.zeros(2, 16, 256, dtype=bf)),                       # fewer sequences than the cache
        dict(q=torch.zeros(4, 16, 256, dtype=bf)),                       # more sequences than the cache
        dict(q=torch.zeros(3, 16, 256, dtype=torch.float16)),            # wrong dtype
        dict(q=torch.zeros(3, 256, 16, dtype=bf).transpose(1, 2)),       # not contiguous
        dict(q=good_q, pos=torch.zeros(2, dtype=torch.int32)),           # pos too short
        dict(q=good_q, pos=torch.zeros(3, dtype=torch.int64)),           # pos not int32
        dict(q=good_q, pos=torch.zeros(6, dtype=torch.int32)[::2]),      # pos not contiguous
    ]
    if fn != "hyb_attn_decode_partial":
        bad += [
            dict(q=good_q, gate=torch.zeros(2, 16, dtype=bf)),               # gate too short
            dict(q=good_q, out=torch.zeros(2, 16, 256, dtype=bf)),           # out too short
            dict(q=good_q, out=torch.zeros(3, 16, 256, dtype=torch.float32)),  # out not bf16
        ]
    for kw in bad:
        with pytest.raises(ValueError):
            go(**kw)


def _wave_fill_splits(full: bool, B: int, max_len: int, fp8: bool) -> int:
    """The decode grid's split count as documented: the smallest count whose
    CTAs (B x 4 KV heads x splits) fill whole waves of CTA slots (148 SMs; two
    FP8 CTAs per SM), else the first within 5 % of the best fill, else the best
    fill; full layers take at most one split per 512 keys (and 1024), ring
    layers at most 8 (one 64-key stage each)."""
    keys = max_len if full else 512
    s_max = max(keys // 512, 1) if full else 8
    sms = 2 * 148 if fp8 else 148
    best, best_eff, first95 = 1, 0.0, 0
    for s in range(1, min(s_max, 1024) + 1):
        ctas = B * 4 * s
        waves = -(-ctas // sms)
        eff = ctas / (waves * sms)
        if eff >= 0.999:
            return s
        if eff >= 0.95 and first95 == 0:
            first95 = s
        if eff > best_eff + 1e-9:
            best_eff, best = eff, s
    return first95 or best


def test_decode_grid_fills_whole_waves(hyb):
    """The split count behind hyb_attn_decode_workspace_size (the larger of the
    bf16 and FP8 grids) is the wave-filling one: 74 FP8 / 37 bf16 splits for a
    batch-1 1M-token full layer (296 / 148 CTAs, one wave each), and the same
    rule for random batches and lengths."""
    import random

    def splits_of(lt, B, L):
        n = hyb.hyb_attn_decode_workspace_size(lt, B, L)
        rows = B * 16
        s = (n - ((rows * 4 + 255) // 256) * 256) // (rows * 256 * 4)
        assert n == rows * s * 256 * 4 + ((rows * s * 4 + 255) // 256) * 256
        return s

    assert splits_of(hyb.FULL, 1, 1 << 20) == 74
    assert _wave_fill_splits(True, 1, 1 << 20, False) == 37
    rnd = random.Random(11)
    for _ in range(300):
        lt = rnd.choice([hyb.SLIDING, hyb.FULL])
        B = rnd.randint(1, 64)
        L = rnd.randint(1, 1 << 21)
        full = lt == hyb.FULL
        want = max(_wave_fill_splits(full, B, L, False), _wave_fill_splits(full, B, L, True))
        assert splits_of(lt, B, L) == want, (lt, B, L)

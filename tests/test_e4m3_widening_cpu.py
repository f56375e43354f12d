"""The kernels' e4m3 -> bf16 widening, checked on the CPU against the two
formats' definitions.

The FP8 paths widen e4m3 codes (sign bit 7, exponent bits 6-3 with bias 7,
mantissa bits 2-0; exponent 0 is subnormal, m 2^-9; S.1111.111 is NaN) to
bf16 (sign bit 15, exponent bits 14-7 with bias 127, mantissa bits 6-0) by
integer moves: a byte permute places each code in a 16-bit half with its
sign copied over the high byte, a shift by 4 and a mask clear the rest.  The
result is the code's value times 2^-120, exactly.

This test takes every permute selector the kernel sources use (the single-word
helpers of common.cuh and each two-word selector written in the kernels),
emulates the byte permute from its definition (selector nibble: bits 0-2 pick
byte 0-7 of {a, b}, bit 3 replaces the byte by copies of its sign bit) and
checks, for every finite code in each selected byte position, that the two
bf16 halves equal the e4m3 values times 2^-120.  A wrong selector (a byte
that does not carry its own sign copy, a swapped half) or a wrong shift or
mask fails here.
"""
import glob
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "full_gqa_attention_partial_b200", "csrc")


def prmt(a: int, b: int, sel: int) -> int:
    """Byte permute, default mode: bytes 0-3 from a, 4-7 from b."""
    src = [(a >> (8 * i)) & 0xFF for i in range(4)] + [(b >> (8 * i)) & 0xFF for i in range(4)]
    out = 0
    for i in range(4):
        n = (sel >> (4 * i)) & 0xF
        byte = src[n & 7]
        if n & 8:
            byte = 0xFF if byte & 0x80 else 0x00
        out |= byte << (8 * i)
    return out


def e4m3_value(code: int) -> float:
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def bf16_value(h: int) -> float:
    s = -1.0 if h & 0x8000 else 1.0
    e = (h >> 7) & 0xFF
    m = h & 0x7F
    assert e != 0xFF
    if e == 0:
        return s * m / 128.0 * 2.0 ** -126
    return s * (1.0 + m / 128.0) * 2.0 ** (e - 127)


def widen(a: int, b: int, sel: int):
    w = ((prmt(a, b, sel) << 4) & 0xFFFFFFFF) & 0x87F087F0
    return bf16_value(w & 0xFFFF), bf16_value(w >> 16)


def _sources():
    return {os.path.basename(p): open(p, encoding="utf-8").read()
            for p in glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))}


def used_selectors():
    """(name, selector, two_words) for every widening selector in the kernel sources."""
    src = _sources()
    common = src["common.cuh"]
    # the single-word helpers: e4m3_bXY_bf16x2(w) { return e4m3_pair_bf16x2<0x....u>(w); }
    single = re.findall(r"e4m3_(b\d\d)_bf16x2\(uint32_t w\) \{ return e4m3_pair_bf16x2<0x([0-9A-Fa-f]+)u>\(w\); \}", common)
    out = [(name, int(sel, 16), False) for name, sel in single]
    # the widening itself must be the permute, the shift by 4 and the mask tested here
    assert common.count("(prmt(w, 0u, SEL) << 4) & 0x87F087F0u") == 1
    assert common.count("(prmt(a, b, SEL) << 4) & 0x87F087F0u") == 1
    for fname, text in sorted(src.items()):
        for sel in sorted(set(re.findall(r"e4m3_pair2_bf16x2<0x([0-9A-Fa-f]+)u>", text))):
            out.append((f"{fname}:pair2", int(sel, 16), True))
    return out


FINITE = [c for c in range(256) if c not in (0x7F, 0xFF)]


def test_every_used_selector_is_found():
    sels = used_selectors()
    names = {n for n, _, two in sels if not two}
    assert {"b01", "b23", "b02", "b13"} <= names
    assert any(two for _, _, two in sels), "the decode's two-word selectors"


@pytest.mark.parametrize("name,sel,two_words", used_selectors())
def test_widening_is_exact_for_every_code(name, sel, two_words):
    n = [(sel >> (4 * i)) & 0xF for i in range(4)]
    # each half: one code byte and, above it, copies of that byte's sign
    assert n[1] == (n[0] | 8) and n[3] == (n[2] | 8), hex(sel)
    if not two_words:
        assert n[0] < 4 and n[2] < 4, "a single-word selector reads the word's own bytes"
    lo_byte, hi_byte = n[0] & 7, n[2] & 7
    scale = 2.0 ** -120
    rng = np.random.default_rng(sel)
    for c in FINITE:
        # the code in each selected position, random bytes everywhere else
        for pos, other_pos in ((lo_byte, hi_byte), (hi_byte, lo_byte)):
            c2 = int(rng.choice(FINITE))
            bytes8 = [int(x) for x in rng.integers(0, 256, 8)]
            bytes8[pos] = c
            if other_pos != pos:
                bytes8[other_pos] = c2
            a = sum(bytes8[i] << (8 * i) for i in range(4))
            b = sum(bytes8[4 + i] << (8 * i) for i in range(4))
            lo, hi = widen(a, b, sel)
            assert lo == e4m3_value(bytes8[lo_byte]) * scale, (name, hex(sel), c)
            assert hi == e4m3_value(bytes8[hi_byte]) * scale, (name, hex(sel), c)


def test_natural_and_paired_orders():
    """The single-word helpers' byte choices: b01 / b23 in order, b02 / b13 interleaved."""
    want = {"b01": (0, 1), "b23": (2, 3), "b02": (0, 2), "b13": (1, 3)}
    for name, sel, two in used_selectors():
        if not two:
            assert ((sel & 0xF) & 7, ((sel >> 8) & 0xF) & 7) == want[name], name

"""The index-checking debug build (libhyb_attn_debug.so, -DHYB_DEBUG_BOUNDS)
on in-range work: in a child process that loads it instead of the normal
library, random cache paths (both layer types, bf16 and FP8, paged and ring
caches) and plain prefills match the oracle with the error word clear, so no
check fires on a valid call and the checks change no result."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import numpy as np, torch
import full_gqa_attention_partial_b200 as hyb
hyb.load(hyb.DEBUG_LIB_PATH)
import oracle as O
from full_gqa_attention_partial_b200 import synth
import test_fuzz_gpu as F
res = {{"flags": hyb.hyb_build_flags()}}
for seed in range(6):
    F.test_random_cache_path(hyb, seed)
for (B, T) in ((2, 300), (1, 700)):
    x = synth.prefill_inputs(B, T, seed=11, device="cuda")
    for lt in (O.SLIDING, O.FULL):
        out = hyb.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], x["pos"], lt)
        torch.cuda.synchronize()
        ref = O.prefill(F.f64(x["q"]), F.f64(x["k"]), F.f64(x["v"]), F.f64(x["gate"]), x["pos"].cpu().numpy(), lt)
        F.check(out, ref, f"prefill B={{B}} T={{T}} lt={{lt}}")
res["dev_err"] = hyb.hyb_device_error()
print(json.dumps(res))
"""


def test_debug_build_in_range_matches_oracle(lib):
    assert os.path.exists(lib.DEBUG_LIB_PATH), "build the library first (it builds the debug twin too)"
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["flags"] == lib.BUILD_DEBUG_BOUNDS
    assert res["dev_err"] == 0

"""The projection GEMM (hyb_linear) against the fp64 oracle: ragged M and N
tiles, a K that is not a multiple of the 64-wide K block, strided rows, the
model's q_k_v_proj / gate / o_proj shapes; and the few-row kernel that takes
M <= 16 with K a multiple of 512 (decode steps): M = 1 .. 16, every
split-K cluster size from 1 to 8, an N that leaves a partial 32-feature
block, strided rows and an output view."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


def f64(t):
    return t.detach().float().cpu().double().numpy()


def make(M, N, K, seed, ldx=None):
    g = torch.Generator(device="cuda").manual_seed(seed)
    ldx = ldx or K
    xbuf = torch.randn(M, ldx, generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g, device="cuda") / K ** 0.5).to(torch.bfloat16)
    return xbuf[:, :K], w


def check(y, x, w, what, rows=None):
    xs = f64(x) if rows is None else f64(x[rows])
    ref = O.linear(xs, f64(w))
    got = f64(y) if rows is None else f64(y[rows])
    assert np.all(np.isfinite(got)), what
    max_abs = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"


@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (300, 264, 200), (257, 520, 136), (1024, 768, 2560)])
def test_linear_small_and_ragged(lib, M, N, K):
    x, w = make(M, N, K, seed=M + N + K)
    y = lib.hyb_linear(x, w)
    torch.cuda.synchronize()
    check(y, x, w, f"linear {M}x{N}x{K}")


def test_linear_strided_rows_and_output_view(lib):
    M, N, K = 640, 384, 320
    x, w = make(M, N, K, seed=3, ldx=K + 72)            # rows of a wider buffer
    ybuf = torch.full((M, N + 64), 7.0, dtype=torch.bfloat16, device="cuda")
    lib.hyb_linear(x, w, out=ybuf[:, :N])
    torch.cuda.synchronize()
    check(ybuf[:, :N], x, w, "strided linear")
    assert torch.all(ybuf[:, N:] == 7.0)                 # nothing written past N


@pytest.mark.parametrize("name,N,K", [("q_k_v_proj", 6144, 2560), ("gate", 16, 2560), ("o_proj", 2560, 4096)])
def test_linear_model_shapes_T32768(lib, name, N, K):
    M = 32768
    x, w = make(M, N, K, seed=N + K)
    y = lib.hyb_linear(x, w)
    torch.cuda.synchronize()
    rng = np.random.default_rng(N)
    rows = np.unique(np.concatenate([np.arange(0, 300), np.arange(M - 300, M), rng.choice(M, 600, replace=False)]))
    check(y, x, w, f"{name} at T=32768", rows=torch.as_tensor(rows, device="cuda"))


def test_linear_rejects_bad_shapes(lib):
    x = torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(8, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.HybError):
        lib.hyb_linear(x, w)                               # K = 12 is not a multiple of 8


@pytest.mark.parametrize("M,N,K", [(1, 8, 512), (3, 40, 1024), (16, 264, 1536), (7, 6144, 2560), (16, 16, 2560),
                                   (16, 2560, 4096), (5, 96, 3584), (11, 200, 2048)])
def test_linear_few_rows(lib, M, N, K):
    x, w = make(M, N, K, seed=7 * M + N + K)
    y = lib.hyb_linear(x, w)
    torch.cuda.synchronize()
    check(y, x, w, f"few-row linear {M}x{N}x{K}")
    assert lib.hyb_device_error() == 0


def test_linear_few_rows_strided_and_view(lib):
    M, N, K = 12, 72, 1024
    x, w = make(M, N, K, seed=5, ldx=K + 40)
    ybuf = torch.full((M, N + 24), 7.0, dtype=torch.bfloat16, device="cuda")
    lib.hyb_linear(x, w, out=ybuf[:, :N])
    torch.cuda.synchronize()
    check(ybuf[:, :N], x, w, "strided few-row linear")
    assert torch.all(ybuf[:, N:] == 7.0)

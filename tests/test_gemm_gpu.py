"""Tensor-core (tcgen05) GEMM and its epilogues against the fp64 definition.

Inputs are bf16-rounded on the host; the reference is the float64 matrix
product of those rounded values (the oracle's contraction primitive), then
the epilogue written out element-wise.
"""

import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

from gpt_decoder_lm_b200 import binding as gb  # noqa: E402
from scipy.special import erf  # noqa: E402

TC2, SKINNY, TC, SIMT_BF16, SIMT_F32 = 4, 3, 2, 1, 0


def bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).bfloat16().float().numpy().astype(np.float64)


def dev_bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda().bfloat16()


def dev_f32(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()


def gelu(x):
    return x * 0.5 * (1 + erf(x / math.sqrt(2)))


def gelu_grad(x):
    return 0.5 * (1 + erf(x / math.sqrt(2))) + x * np.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)


def operands(M, N, K, ak, bk, seed):
    rng = np.random.default_rng(seed)
    A = bf16_round(rng.standard_normal((M, K)))
    B = bf16_round(rng.standard_normal((N, K)))
    Ad = dev_bf16(A if ak else A.T)
    Bd = dev_bf16(B if bk else B.T)
    lda = K if ak else M
    ldb = K if bk else N
    return A, B, Ad, Bd, lda, ldb


def acc_tol(K):
    """Bound on the fp32-accumulation error of K bf16 products, relative to
    the largest entry: the tensor core's fp32 accumulator loses precision at
    a rate that adds up linearly over K (measured about 1.45e-9 K on B200),
    so the bound is 3e-9 K, and never below 2e-6 for short K."""
    return max(2e-6, 3e-9 * K)


def run(backend, M, N, K, Ad, lda, ak, Bd, ldb, bk, kind, **kw):
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = gb.test_gemm(backend, M, N, K, Ad, lda, ak, Bd, ldb, bk, kind,
                      stream=torch.cuda.current_stream().cuda_stream, flags=flags, **kw)
    assert gb.STATUS[st] == "GPT_OK", gb.STATUS[st]
    assert int(flags.item()) == 0


LAYOUTS = [(1, 1), (1, 0), (0, 0)]   # forward (TN), dX (B MN-major), dW (both MN-major)
SHAPES = [(128, 128, 64), (256, 384, 192), (200, 328, 136), (1024, 2304, 256), (4096, 1024, 128), (64, 96, 520)]


@pytest.mark.parametrize("backend", [TC, TC2], ids=["tc", "tc2"])
@pytest.mark.parametrize("ak,bk", LAYOUTS, ids=["tn", "b_mn", "ab_mn"])
@pytest.mark.parametrize("M,N,K", SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in SHAPES])
def test_tc_gemm_store_f32(M, N, K, ak, bk, backend):
    A, B, Ad, Bd, lda, ldb = operands(M, N, K, ak, bk, M + N + K)
    out = torch.full((M, N), float("nan"), device="cuda")
    run(backend, M, N, K, Ad, lda, ak, Bd, ldb, bk, 6, out=out, ldo=N)
    ref = A @ B.T
    got = out.double().cpu().numpy()
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < 2e-6, err


@pytest.mark.parametrize("backend,M", [(TC, 384), (TC2, 384), (SIMT_BF16, 384), (SKINNY, 12), (SKINNY, 5)],
                         ids=["tc", "tc2", "simt", "skinny12", "skinny5"])
def test_epilogues(backend, M):
    N, K = 512, 256
    rng = np.random.default_rng(7)
    A, B, Ad, Bd, lda, ldb = operands(M, N, K, 1, 1, 3)
    D = A @ B.T
    bias = rng.standard_normal(N).astype(np.float32)
    bias_d = dev_f32(bias)
    # 1: bias
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    run(backend, M, N, K, Ad, lda, 1, Bd, ldb, 1, 1, out=out, ldo=N, bias=bias_d)
    np.testing.assert_allclose(out.double().cpu().numpy(), D + bias, rtol=1e-2, atol=0.06)
    # 2: bias + GELU: derivative at the pre-activation (kept for backward) and activation
    out2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    run(backend, M, N, K, Ad, lda, 1, Bd, ldb, 1, 2, act=0, out=out, out2=out2, ldo=N, bias=bias_d)
    h = D + bias
    # GELU' has slope ~0.4 near 0: the fp32 pre-activation's bf16-level error moves it by ~0.01
    np.testing.assert_allclose(out.double().cpu().numpy(), gelu_grad(h), rtol=1e-2, atol=0.02)
    np.testing.assert_allclose(out2.double().cpu().numpy(), gelu(h), rtol=1e-2, atol=0.06)
    run(backend, M, N, K, Ad, lda, 1, Bd, ldb, 1, 2, act=1, out=out, out2=out2, ldo=N, bias=bias_d)
    np.testing.assert_allclose(out2.double().cpu().numpy(), np.maximum(h, 0), rtol=1e-2, atol=0.06)
    far = np.abs(h) > 0.1  # the ReLU derivative is a step: compare away from the kink
    np.testing.assert_array_equal(out.double().cpu().numpy()[far], (h > 0).astype(np.float64)[far])
    # 3: residual add (fp32)
    res = rng.standard_normal((M, N)).astype(np.float32)
    res_in = dev_f32(res)
    res_out = torch.empty_like(res_in)
    run(backend, M, N, K, Ad, lda, 1, Bd, ldb, 1, 3, ldo=N, bias=bias_d, res_in=res_in, res_out=res_out)
    np.testing.assert_allclose(res_out.double().cpu().numpy(), res + D + bias, rtol=1e-5, atol=1e-4)
    # 4: activation backward: the accumulator times a saved derivative
    dd = bf16_round(gelu_grad(rng.standard_normal((M, N))))
    aux = dev_bf16(dd)
    run(backend, M, N, K, Ad, lda, 1, Bd, ldb, 1, 4, act=0, out=out, ldo=N, aux=aux)
    np.testing.assert_allclose(out.double().cpu().numpy(), D * dd, rtol=1e-2, atol=0.06)
    # 5: fp32 accumulate
    acc0 = rng.standard_normal((M, N)).astype(np.float32)
    acc = dev_f32(acc0)
    run(backend, M, N, K, Ad, lda, 1, Bd, ldb, 1, 5, out=acc, ldo=N)
    np.testing.assert_allclose(acc.double().cpu().numpy(), acc0 + D, rtol=1e-5, atol=1e-4)


SKINNY_SHAPES = [(1, 16, 32), (5, 200, 96), (8, 1000, 64), (12, 2304, 768), (12, 768, 3072), (16, 3072, 768),
                 (12, 50304, 768), (9, 40, 4096)]


@pytest.mark.parametrize("M,N,K", SKINNY_SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in SKINNY_SHAPES])
def test_skinny_gemm_store_f32(M, N, K):
    """The decoding-step GEMM (at most 16 rows): every row count of an 8-row
    tile pair, ragged N, each K split of the warps, the GPT-2 124M shapes."""
    A, B, Ad, Bd, lda, ldb = operands(M, N, K, 1, 1, M * 7 + N + K)
    out = torch.full((M, N), float("nan"), device="cuda")
    run(SKINNY, M, N, K, Ad, lda, 1, Bd, ldb, 1, 6, out=out, ldo=N)
    ref = A @ B.T
    got = out.double().cpu().numpy()
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < 2e-6, err


def test_skinny_gemm_pitches():
    """Row pitches wider than the rows (lda, ldb, ldo) and a strided output,
    as the decoding step writes into the key / value cache."""
    M, N, K = 12, 2304, 768
    rng = np.random.default_rng(4)
    A = bf16_round(rng.standard_normal((M, K)))
    B = bf16_round(rng.standard_normal((N, K)))
    Ad = dev_bf16(np.concatenate([A, np.zeros((M, 64))], 1))
    Bd = dev_bf16(np.concatenate([B, np.ones((N, 32))], 1))
    out = torch.full((M, 3 * N), float("nan"), device="cuda")
    run(SKINNY, M, N, K, Ad, K + 64, 1, Bd, K + 32, 1, 6, out=out, ldo=3 * N)
    got = out.double().cpu().numpy()
    err = np.abs(got[:, :N] - A @ B.T).max() / np.abs(A @ B.T).max()
    assert err < 2e-6, err
    assert np.isnan(got[:, N:]).all()


def test_skinny_gemm_unsupported():
    A, B, Ad, Bd, lda, ldb = operands(17, 64, 64, 1, 1, 1)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty((17, 64), device="cuda")
    st = gb.test_gemm(SKINNY, 17, 64, 64, Ad, lda, 1, Bd, ldb, 1, 6, out=out, ldo=64,
                      stream=torch.cuda.current_stream().cuda_stream, flags=flags)
    assert gb.STATUS[st] == "GPT_ERR_UNSUPPORTED"
    st = gb.test_gemm(SKINNY, 8, 64, 48, Ad, lda, 1, Bd, ldb, 1, 6, out=out, ldo=64,
                      stream=torch.cuda.current_stream().cuda_stream, flags=flags)
    assert gb.STATUS[st] == "GPT_ERR_UNSUPPORTED"  # K not a multiple of 32


@pytest.mark.parametrize("backend", [TC, TC2], ids=["tc", "tc2"])
@pytest.mark.parametrize("splits", [2, 5])
def test_tc_split_k_accumulate(splits, backend):
    M, N, K = 256, 384, 4096      # dW-like: both operands MN-major, long contraction
    A, B, Ad, Bd, lda, ldb = operands(M, N, K, 0, 0, 11)
    acc0 = np.random.default_rng(2).standard_normal((M, N)).astype(np.float32)
    acc = dev_f32(acc0)
    partial = torch.empty((splits, M, N), device="cuda")
    run(backend, M, N, K, Ad, lda, 0, Bd, ldb, 0, 5, out=acc, ldo=N, split_k=splits, partial=partial)
    ref = acc0 + A @ B.T
    err = np.abs(acc.double().cpu().numpy() - ref).max() / np.abs(ref).max()
    # fp32 accumulation over K = 4096 products: rounding grows like sqrt(K) * 2^-24
    assert err < 1e-5, err


def test_tc_matches_simt_bitwise_close():
    M, N, K = 512, 768, 768
    A, B, Ad, Bd, lda, ldb = operands(M, N, K, 1, 0, 5)
    o1 = torch.empty((M, N), device="cuda")
    o2 = torch.empty((M, N), device="cuda")
    run(TC, M, N, K, Ad, lda, 1, Bd, ldb, 0, 6, out=o1, ldo=N)
    run(SIMT_BF16, M, N, K, Ad, lda, 1, Bd, ldb, 0, 6, out=o2, ldo=N)
    ref = A @ B.T
    for o in (o1, o2):
        assert np.abs(o.double().cpu().numpy() - ref).max() / np.abs(ref).max() < 2e-6


def test_gelu_epilogue_accuracy_fp32():
    # fp32 operands on the CUDA-core GEMM: the GELU and GELU' epilogues against
    # scipy's erf to well inside the fp32-mode gradient bound
    M, N, K = 64, 256, 64
    rng = np.random.default_rng(9)
    A = rng.standard_normal((M, K)).astype(np.float32)
    B = (rng.standard_normal((N, K)) * 0.4).astype(np.float32)
    D = A.astype(np.float64) @ B.astype(np.float64).T
    out = torch.empty((M, N), device="cuda")
    out2 = torch.empty((M, N), device="cuda")
    run(SIMT_F32, M, N, K, dev_f32(A), K, 1, dev_f32(B), K, 1, 2, act=0, out=out, out2=out2, ldo=N)
    np.testing.assert_allclose(out2.double().cpu().numpy(), gelu(D), rtol=1e-5, atol=2e-6)
    np.testing.assert_allclose(out.double().cpu().numpy(), gelu_grad(D), rtol=1e-5, atol=2e-6)
    dd = gelu_grad(rng.standard_normal((M, N)) * 3).astype(np.float32)
    run(SIMT_F32, M, N, K, dev_f32(A), K, 1, dev_f32(B), K, 1, 4, act=0, out=out, ldo=N, aux=dev_f32(dd))
    np.testing.assert_allclose(out.double().cpu().numpy(), D * dd.astype(np.float64), rtol=1e-5, atol=2e-6)


def bf16_ulp(y):
    """Spacing of bf16 numbers at |y| (7 stored fraction bits against fp32's 23)."""
    return np.spacing(np.abs(np.asarray(y, np.float32))).astype(np.float64) * 2.0 ** 16


@pytest.mark.parametrize("backend", [TC, TC2], ids=["tc", "tc2"])
def test_gelu_epilogue_bf16_half_ulp(backend):
    # Pre-activations known exactly: B selects one column of A per output column
    # (one 1 per row), so the fp32 accumulator holds A's bf16 values unchanged.
    # The two bf16 outputs are then GELU and GELU' of known values rounded once:
    # within half a bf16 ulp of the float64 values, plus 1e-6 (1 + |x|) for the
    # erf approximation (|error| <= 1.5e-7, Abramowitz & Stegun 7.1.26) and the
    # fp32 arithmetic.  A wrong constant or sign moves values by far more and
    # flips roundings near the half-ulp points.
    M, N, K = 512, 256, 64
    rng = np.random.default_rng(21)
    A = rng.uniform(-8.0, 8.0, (M, K))
    A[0, :12] = [0.0, 1.0, -1.0, 0.5, -0.5, 3.0, -3.0, 20.0, -20.0, 100.0, -100.0, 1e-3]
    A = bf16_round(A)
    B = np.zeros((N, K))
    B[np.arange(N), np.arange(N) % K] = 1.0
    x = A @ B.T
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    out2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    run(backend, M, N, K, dev_bf16(A), K, 1, dev_bf16(B), K, 1, 2, act=0, out=out, out2=out2, ldo=N)
    for got, ref in ((out2.double().cpu().numpy(), gelu(x)), (out.double().cpu().numpy(), gelu_grad(x))):
        bound = 0.5 * bf16_ulp(np.maximum(np.abs(ref), np.abs(got))) + 1e-6 * (1.0 + np.abs(x))
        excess = np.abs(got - ref) - bound
        assert excess.max() <= 0.0, (x.flat[excess.argmax()], got.flat[excess.argmax()], ref.flat[excess.argmax()])


# The contractions of the benchmarked step at their own shapes: GPT-2 124M
# (M = 12 x 1024 rows, d 768, 3d 2304, 4d 3072) and GPT-2 XL's layer (M =
# 2 x 1024, d 1600, 3d 4800 and 4d 6400, both ragged against the 256-column
# tile).  (M, N, K) with the layout each one runs in: forward TN, dX with W
# MN-major, dW with both operands MN-major (K = the token count).
FULL_SHAPES = [
    ("qkv_fwd_124m", 12288, 2304, 768, 1, 1), ("fc_dx_124m", 12288, 768, 3072, 1, 0),
    ("fc_dw_124m", 3072, 768, 12288, 0, 0),
    ("qkv_fwd_xl", 2048, 4800, 1600, 1, 1), ("proj_fwd_xl", 2048, 1600, 6400, 1, 1),
    ("qkv_dx_xl", 2048, 1600, 4800, 1, 0), ("fc_dx_xl", 2048, 1600, 6400, 1, 0),
    ("qkv_dw_xl", 4800, 1600, 2048, 0, 0), ("fc_dw_xl", 6400, 1600, 2048, 0, 0),
]


@pytest.mark.parametrize("backend", [TC, TC2], ids=["tc", "tc2"])
@pytest.mark.parametrize("name,M,N,K,ak,bk", FULL_SHAPES, ids=[s[0] for s in FULL_SHAPES])
def test_tc_gemm_full_shapes(name, M, N, K, ak, bk, backend):
    A, B, Ad, Bd, lda, ldb = operands(M, N, K, ak, bk, M + N + K)
    out = torch.full((M, N), float("nan"), device="cuda")
    run(backend, M, N, K, Ad, lda, ak, Bd, ldb, bk, 6, out=out, ldo=N)
    ref = A @ B.T
    got = out.double().cpu().numpy()
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < acc_tol(K), err


@pytest.mark.parametrize("splits", [1, 4])
def test_tc_gemm_dw_split_full_shape(splits):
    # the fc weight gradient of GPT-2 124M (3072 x 768 over 12288 tokens),
    # split-K partials added to an existing fp32 gradient in a fixed order
    M, N, K = 3072, 768, 12288
    A, B, Ad, Bd, lda, ldb = operands(M, N, K, 0, 0, 21)
    acc0 = np.random.default_rng(3).standard_normal((M, N)).astype(np.float32)
    acc = dev_f32(acc0)
    partial = torch.empty((splits, M, N), device="cuda")
    run(TC, M, N, K, Ad, lda, 0, Bd, ldb, 0, 5, out=acc, ldo=N, split_k=splits, partial=partial)
    ref = acc0 + A @ B.T
    err = np.abs(acc.double().cpu().numpy() - ref).max() / np.abs(ref).max()
    assert err < acc_tol(K), err


@pytest.mark.parametrize("layout", ["fwd", "dw"])
def test_tc_gemm_lm_head_sampled(layout):
    # the lm_head at full size: logits [12288, 50304] = x [12288, 768] W^T
    # (forward, TN) and its weight gradient [50304, 768] over 12288 tokens
    # (both operands MN-major, as dlogits and the final norm's output are
    # stored).  Operands are drawn on the device (seeded) and rounded to
    # bf16 there; the float64 reference is formed on the host for 96 sampled
    # output rows.
    gen = torch.Generator(device="cuda").manual_seed(41)
    Mx, V, d = 12288, 50304, 768
    if layout == "fwd":
        M, N, K, ak, bk = Mx, V, d, 1, 1
        Ad = torch.randn((M, K), generator=gen, device="cuda").bfloat16()
        Bd = torch.randn((N, K), generator=gen, device="cuda").bfloat16()
        lda, ldb = K, K
    else:
        M, N, K, ak, bk = V, d, Mx, 0, 0
        Ad = torch.randn((K, M), generator=gen, device="cuda").bfloat16()
        Bd = torch.randn((K, N), generator=gen, device="cuda").bfloat16()
        lda, ldb = M, N
    out = torch.full((M, N), float("nan"), device="cuda")
    run(TC, M, N, K, Ad, lda, ak, Bd, ldb, bk, 6, out=out, ldo=N)
    rng = np.random.default_rng(31)
    rows = np.sort(np.concatenate([rng.choice(M, 94, replace=False), [0, M - 1]]))
    r = torch.from_numpy(rows).cuda()
    a_rows = (Ad[r] if ak else Ad[:, r].t()).double().cpu().numpy()      # [96, K]
    b_all = (Bd if bk else Bd.t()).double().cpu().numpy()                # [N, K]
    ref = a_rows @ b_all.T
    got = out[r].double().cpu().numpy()
    err = np.abs(got - ref).max() / np.abs(ref).max()
    assert err < acc_tol(K), err
    assert not torch.isnan(out).any().item()


@pytest.mark.parametrize("backend", [TC, TC2], ids=["tc", "tc2"])
@pytest.mark.parametrize("M", [384, 200, 12288])
def test_act_bwd_epilogue_column_sums(backend, M):
    # the activation-backward GEMM (dh = (dy W) * act'(h)) also writes the
    # column sums of the stored bf16 dh over each 32-row group (the fc bias
    # gradient's partials): against the sums of the stored values
    N, K = 3072, 768
    rng = np.random.default_rng(13)
    A, B, Ad, Bd, lda, ldb = operands(M, N, K, 1, 0, 17)
    aux = dev_bf16(gelu_grad(rng.standard_normal((M, N))))
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    groups = (M + 31) // 32
    cs = torch.full((groups, N), float("nan"), device="cuda")
    run(backend, M, N, K, Ad, lda, 1, Bd, ldb, 0, 4, act=0, out=out, ldo=N, aux=aux, colsum=cs)
    dh = out.double().cpu().numpy()
    pad = np.zeros((groups * 32, N))
    pad[:M] = dh
    want = pad.reshape(groups, 32, N).sum(axis=1)
    got = cs.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.abs(got - want).max() <= 1e-5 * max(1.0, np.abs(want).max())

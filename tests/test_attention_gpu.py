"""Causal attention kernels (tensor-core and CUDA-core) against the oracle's
attention_fwd / attention_bwd on the same bf16-rounded q, k, v, dO.

Tolerances: O and the gradients are bf16 tensors built from bf16
probabilities, so element errors are a few 2^-8 relative; compared as
rel-L2 <= 2e-2 (the bf16 gradient bound).  LSE is fp32 arithmetic on exact
fp32 scores: |dLSE| <= 1e-3.  Dropout masks are integer and must agree
exactly, which the outputs only show through these bounds.
"""

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import oracle  # noqa: E402
from gpt_decoder_lm_b200 import binding as gb  # noqa: E402
from tests.helpers import rel_l2  # noqa: E402

SEED, COUNTER, LAYER = 1339, 5, 2


def bf(x):
    return torch.from_numpy(np.asarray(x, np.float32)).bfloat16()


def run_case(backend, B, T, H, p, seed=0, qkv_np=None):
    hd = 64
    rng = np.random.default_rng(seed)
    qkv = bf(rng.standard_normal((B, T, 3, H, hd)) if qkv_np is None else qkv_np)
    dout = bf(rng.standard_normal((B, T, H, hd)))
    q, k, v = (qkv.float().numpy().astype(np.float64)[:, :, i].transpose(0, 2, 1, 3) for i in range(3))
    do = dout.float().numpy().astype(np.float64).transpose(0, 2, 1, 3)
    keep = None
    if p > 0:
        bh = np.arange(B * H, dtype=np.uint64).reshape(B, H, 1, 1)
        i = np.arange(T, dtype=np.uint64).reshape(1, 1, T, 1)
        j = np.arange(T, dtype=np.uint64).reshape(1, 1, 1, T)
        elems = (bh * np.uint64(T) + i) * np.uint64(T) + j
        keep = oracle.dropout_keep(SEED, COUNTER, LAYER, 1, elems, p)
    o_ref, pr, lse_ref = oracle.attention_fwd(q, k, v, keep, p)
    dq, dk, dv = oracle.attention_bwd(q, k, v, pr, do, keep, p)

    d_qkv = qkv.cuda()
    d_o = torch.empty((B, T, H, hd), dtype=torch.bfloat16, device="cuda")
    d_lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    d_do = dout.cuda()
    d_dqkv = torch.full((B, T, 3, H, hd), float("nan"), dtype=torch.bfloat16, device="cuda")
    d_dsum = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    rc = gb.test_attention(backend, 0, 1, B, T, H, hd, d_qkv, d_o, d_lse, p=p, seed=SEED, counter=COUNTER,
                           layer=LAYER, stream=st, flags=flags)
    assert gb.STATUS[rc] == "GPT_OK", gb.STATUS[rc]
    # the tensor-core backward also writes the column sums of the stored dqkv
    # per 128-row block (the qkv bias gradient's partials)
    cs = torch.full((B * T // 128, 3 * H * hd), float("nan"), device="cuda") if backend == 1 else None
    rc = gb.test_attention(backend, 1, 1, B, T, H, hd, d_qkv, d_o, d_lse, d_do, d_dqkv, d_dsum, p=p, seed=SEED,
                           counter=COUNTER, layer=LAYER, stream=st, flags=flags, colsum=cs)
    assert gb.STATUS[rc] == "GPT_OK", gb.STATUS[rc]
    if cs is not None:
        stored = d_dqkv.double().cpu().numpy().reshape(B * T // 128, 128, 3 * H * hd).sum(axis=1)
        got = cs.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert np.abs(got - stored).max() <= 1e-5 * max(1.0, np.abs(stored).max())
    assert int(flags.item()) == 0
    o = d_o.float().cpu().numpy().astype(np.float64).transpose(0, 2, 1, 3)
    assert rel_l2(o, o_ref) < 2e-2
    assert np.abs(d_lse.cpu().numpy() - lse_ref).max() < 1e-3
    g = d_dqkv.float().cpu().numpy().astype(np.float64)
    for idx, ref in ((0, dq), (1, dk), (2, dv)):
        got = g[:, :, idx].transpose(0, 2, 1, 3)
        assert np.isfinite(got).all()
        assert rel_l2(got, ref) < 2e-2, (idx, rel_l2(got, ref))
    return o, g


# the last three are the benchmarked shapes: GPT-2 124M (T 1024, 12 heads;
# two batch rows so the longest-block-first order spans several (b, h)) and
# GPT-2 XL (T 1024, 25 heads)
@pytest.mark.parametrize("B,T,H", [(2, 256, 3), (1, 512, 2), (1, 128, 1), (1, 384, 2), (2, 1024, 12),
                                   (1, 1024, 25)])
@pytest.mark.parametrize("p", [0.0, 0.1], ids=["nodrop", "dropout"])
def test_attention_tensor_core(B, T, H, p):
    run_case(1, B, T, H, p)


@pytest.mark.parametrize("p", [0.0, 0.1], ids=["nodrop", "dropout"])
def test_attention_cuda_core_bf16(p):
    run_case(0, 2, 192, 2, p)


def test_tensor_core_matches_cuda_core():
    o1, g1 = run_case(1, 2, 256, 2, 0.0, seed=4)
    o2, g2 = run_case(0, 2, 256, 2, 0.0, seed=4)
    assert rel_l2(o1, o2) < 1e-2 and rel_l2(g1, g2) < 2e-2


def test_attention_rescale_path():
    # Scores that grow by about 10 log2 units per 64-key block: the forward's
    # running maximum is exceeded by more than its rescale threshold in every
    # block, so O and l are rescaled in TMEM each time (the path random inputs
    # of unit scale almost never take).
    B, T, H, hd = 1, 512, 2, 64
    rng = np.random.default_rng(3)
    x = rng.standard_normal((B, T, 3, H, hd))
    u = rng.standard_normal(hd)
    u /= np.linalg.norm(u)
    x[:, :, 0] += 21.0 * u
    x[:, :, 1] += (np.arange(T) / T * 21.0)[None, :, None, None] * u
    run_case(1, B, T, H, 0.0, qkv_np=x)

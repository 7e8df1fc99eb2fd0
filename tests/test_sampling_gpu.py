"""The fused softmax-sample kernel (gpt_sample) and the evaluation loss
(gpt_eval_loss) against the oracle (oracle/sampling.py).

Draws are integers decided by floating point: the kernel takes them in fp32,
the oracle in fp64, on the same (bf16-exact) logits.  Where the uniform
lands within a small relative margin of a boundary of the kept cumulative
distribution, or the nucleus target within that margin of a boundary of the
sorted cumulative mass, either neighbour is correct and the test checks that
the token is kept; everywhere else the tokens must be equal.  Greedy
decoding and the top-k set are exact (comparisons of the same values)."""

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import oracle  # noqa: E402
from oracle import sampling as S  # noqa: E402
from gpt_decoder_lm_b200 import binding as gb  # noqa: E402
from gpt_decoder_lm_b200 import workloads as W  # noqa: E402
from tests.helpers import oracle_config  # noqa: E402

MARGIN = 1e-4


def check_row(z, temperature, top_k, top_p, u, got):
    """True when the row was compared exactly; asserts the token either way."""
    ref = S.sample_row(z, temperature, top_k, top_p, u)
    if temperature <= 0:
        assert got == ref, (got, ref)
        return True
    d = MARGIN
    # the nucleus boundary: the same draw under top_p -/+ MARGIN, else either side is right
    refs = {ref}
    if top_p < 1.0:
        refs |= {S.sample_row(z, temperature, top_k, max(top_p - d, 0.0), u),
                 S.sample_row(z, temperature, top_k, min(top_p + d, 1.0), u)}
    p = S._kept_probs(z, temperature, top_k, top_p)
    c = np.cumsum(p)
    margin = np.min(np.abs(c - u * c[-1])) / c[-1]
    if len(refs) == 1 and margin > d:
        assert got == ref, (got, ref, margin)
        return True
    loose = S._kept_probs(z, temperature, top_k, min(top_p + d, 1.0) if top_p < 1.0 else 1.0)
    assert loose[got] > 0, got
    return False


def run_case(V, rows, dtype, temperature, top_k, top_p, seed):
    rng = np.random.default_rng(seed)
    z = (rng.standard_normal((rows, V)) * 3).astype(np.float32)
    zt = torch.from_numpy(z).to(dtype)
    z64 = zt.float().numpy().astype(np.float64)  # the values the kernel sees
    u = rng.random(rows).astype(np.float32)
    u64 = u.astype(np.float64)
    out = torch.empty(rows, dtype=torch.int32, device="cuda")
    gb.sample(zt.cuda(), temperature, top_k, top_p, torch.from_numpy(u).cuda(), out)
    got = out.cpu().numpy()
    exact = sum(check_row(z64[r], temperature, top_k, top_p, u64[r], int(got[r])) for r in range(rows))
    assert exact >= rows // 4, exact


@pytest.mark.parametrize("temperature,top_k,top_p", [
    (0.0, 0, 1.0), (1.0, 0, 1.0), (0.7, 40, 1.0), (1.3, 0, 0.9), (0.8, 40, 0.9), (1.0, 1, 1.0), (1.0, 5, 0.5),
    (1.0, 0, 0.0), (1.0, 4000, 0.95), (1.0, 5000, 0.9)])
def test_sample_vocab_bf16(temperature, top_k, top_p):
    run_case(50257, 24, torch.bfloat16, temperature, top_k, top_p, seed=int(temperature * 10) + top_k)


@pytest.mark.parametrize("V", [1, 7, 1000, 4097])
def test_sample_small_vocab_fp32(V):
    run_case(V, 16, torch.float32, 0.9, min(3, V), 0.95, seed=V)


@pytest.mark.parametrize("V", [1000, 20000])
def test_sample_top_k_ties(V):
    """Logits on a coarse grid: the k-th largest value is shared by many
    tokens, all of which are kept (a few hundred in shared memory at V = 1000,
    more than it holds at V = 20000)."""
    rows = 16
    rng = np.random.default_rng(V)
    z = rng.integers(0, 4, (rows, V)).astype(np.float32)
    u = rng.random(rows).astype(np.float32)
    out = torch.empty(rows, dtype=torch.int32, device="cuda")
    gb.sample(torch.from_numpy(z).cuda(), 1.0, 5, 0.8, torch.from_numpy(u).cuda(), out)
    got = out.cpu().numpy()
    for r in range(rows):
        ref = S.sample_row(z[r].astype(np.float64), 1.0, 5, 0.8, float(u[r]))
        p = S._kept_probs(z[r].astype(np.float64), 1.0, 5, 0.8)
        assert p[got[r]] > 0, (r, got[r])
        # equal probabilities: the draw is the token whose CDF interval holds u
        # up to rounding of the running sum
        c = np.cumsum(p) / p.sum()
        lo = np.searchsorted(c, u[r] - 1e-5, side="right")
        hi = np.searchsorted(c, u[r] + 1e-5, side="right")
        assert min(lo, ref) <= got[r] <= max(hi, ref), (r, got[r], ref, lo, hi)


def test_sample_frequencies_follow_the_kept_softmax():
    # one row of logits drawn at a grid of uniforms: each token's frequency is
    # its kept, renormalised probability to within 1/rows (plus fp32 slack)
    V, rows = 64, 4096
    rng = np.random.default_rng(11)
    z = (rng.standard_normal(V) * 2).astype(np.float32)
    zt = torch.from_numpy(np.tile(z, (rows, 1))).cuda()
    u = torch.from_numpy(((np.arange(rows) + 0.5) / rows).astype(np.float32)).cuda()
    out = torch.empty(rows, dtype=torch.int32, device="cuda")
    gb.sample(zt, 0.8, 10, 0.9, u, out)
    f = np.bincount(out.cpu().numpy(), minlength=V) / rows
    p = S._kept_probs(z.astype(np.float64), 0.8, 10, 0.9)
    np.testing.assert_allclose(f, p / p.sum(), atol=1.0 / rows + 1e-4)


@pytest.mark.parametrize("precision,tol", [("bf16", 2e-3), ("fp32", 1e-5)])
def test_eval_loss_matches_oracle(precision, tol):
    w = W.CHAR.with_(precision=precision)
    cfg = gb.make_config(w, n_layer=2, batch_size=4, block_size=128)
    m = gb.Model(cfg, seed=w.weight_seed)
    oc = oracle_config(w).with_(n_layer=2, batch_size=4, block_size=128, grad_accum=cfg.grad_accum)
    P = oracle.init_params(oc, w.weight_seed)
    stream = W.token_stream(w, n=1 << 15)
    sd = torch.from_numpy(stream.astype(np.int32)).cuda()
    got = m.eval_loss(sd, 77, 3)
    ref = S.eval_loss(oc, P, stream, 77, 3)
    if precision == "bf16":
        assert abs(got - ref) <= tol, (got, ref)
    else:
        assert abs(got - ref) <= tol * abs(ref), (got, ref)
    m.close()

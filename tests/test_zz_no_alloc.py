"""The allocation-free weight-gradient GEMM (gpt_gemm_dw_accumulate_noalloc)
against the same GEMM run through the caller-scratch entry point.

That entry point serves callers that cannot allocate device memory (plugin or
custom-operator interfaces that only pass inputs and outputs, processes whose
device memory belongs to another allocator, work that must not call
cudaMalloc); its split-K partial sums live in an array inside the library.
Two calls in a row, with different operands and split counts, must each
equal the caller-scratch result on the same inputs bit for bit (the partial
sums are added in a fixed order); the caller-scratch result itself is checked
against the float64 product within the GEMM tests' tolerance (fp32
accumulation over K = 8192: 1e-5 of the largest entry).  This file is collected last and needs nothing from the
other tests, so it also runs alone in a fresh process.
"""

import ctypes as C

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

from gpt_decoder_lm_b200 import binding as gb  # noqa: E402


def _caller_scratch(A, B, base, M, N, K, splits, stream):
    # the same GEMM through the entry point that takes caller-provided scratch
    out = base.clone()
    partial = torch.empty(splits, M, N, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    # backend 5: the kernel and split count the library's cost model picks,
    # which the allocation-free entry point runs too
    st = gb.test_gemm(5, M, N, K, A, M, 0, B, N, 0, 5, 0, out, None, N, None, None, None, None, splits, partial,
                      stream, flags)
    assert gb.STATUS[st] == "GPT_OK" and int(flags.item()) == 0
    return out


def test_noalloc_dw_gemm_matches_caller_scratch_twice():
    lib = gb.lib()
    M, N, K = 768, 768, 8192
    g = torch.Generator(device="cuda").manual_seed(5)
    stream = torch.cuda.current_stream().cuda_stream
    # Two calls in a row with different operands and different split counts:
    # the library's array still holds the first call's partial sums when the
    # second call starts, so a result that leaned on stale contents would
    # differ.  The partial sums are added in a fixed order, so each call must
    # equal the caller-scratch run on the same inputs bit for bit.
    for splits in (4, 3):
        A = torch.randn(K, M, device="cuda", generator=g).bfloat16()   # [K, M]: tokens outermost
        B = torch.randn(K, N, device="cuda", generator=g).bfloat16()
        base = torch.randn(M, N, device="cuda", generator=g)
        ref = _caller_scratch(A, B, base, M, N, K, splits, stream)
        exact = base.double() + A.double().T @ B.double()
        assert (ref.double() - exact).abs().max().item() <= 1e-5 * exact.abs().max().item()
        out = base.clone()
        st = lib.gpt_gemm_dw_accumulate_noalloc(M, N, K, A.data_ptr(), M, B.data_ptr(), N, out.data_ptr(), splits,
                                                 C.c_void_p(stream))
        assert gb.STATUS[st] == "GPT_OK"
        assert torch.equal(out, ref)


def test_noalloc_rejects_sizes_beyond_its_array():
    lib = gb.lib()
    M = N = 2048
    A = torch.zeros(64, M, device="cuda").bfloat16()
    out = torch.zeros(M, N, device="cuda")
    st = lib.gpt_gemm_dw_accumulate_noalloc(M, N, 64, A.data_ptr(), M, A.data_ptr(), N, out.data_ptr(), 2,
                                             C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert gb.STATUS[st] == "GPT_ERR_WORKSPACE_TOO_SMALL"
    assert gb.STATUS[lib.gpt_gemm_dw_accumulate_noalloc(0, N, 64, None, M, None, N, None, 1, None)] == \
        "GPT_ERR_INVALID_ARG"

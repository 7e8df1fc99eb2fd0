"""The C ABI library loads and exports every declared symbol; its pure host
functions agree with the oracle's closed forms.  No device work here."""

import ctypes as C
import math

import pytest

import oracle
from gpt_decoder_lm_b200 import binding as gb
from gpt_decoder_lm_b200 import workloads as W
from tests.helpers import oracle_config


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    return gb.lib()


def test_every_declared_symbol_is_exported(lib):
    names = gb.declared_symbols()
    assert "gpt_train_step" in names and "gpt_test_gemm" in names
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) <= set(gb._PROTOS), set(names) - set(gb._PROTOS)


@pytest.mark.parametrize("w", list(W.ALL.values()), ids=list(W.ALL))
def test_param_count_matches_oracle(lib, w):
    cfg = gb.make_config(w)
    assert gb.param_count(cfg) == oracle.param_count(oracle_config(w))
    assert gb.workspace_bytes(cfg) > 4 * 4 * gb.param_count(cfg)


def test_micro_param_count_4192(lib):
    assert gb.param_count(gb.make_config(W.MICRO)) == 4192


def test_lr_schedules_match_oracle(lib):
    for it in [0, 1, 5, 10, 50, 99, 100, 101, 500, 1099, 1100]:
        assert math.isclose(gb.lr_cosine(6e-4, it, 100, 1100), oracle.lr_cosine(6e-4, it, 100, 1100),
                            rel_tol=1e-6, abs_tol=1e-12)
    for it in [0, 3, 7, 10]:
        assert math.isclose(gb.lr_linear(1e-2, it, 10), oracle.lr_linear(1e-2, it, 10), rel_tol=1e-6, abs_tol=1e-12)


@pytest.mark.parametrize("field,value,status", [
    ("n_head", 5, "GPT_ERR_CONFIG"),           # 384 % 5 != 0
    ("abi_version", 99, "GPT_ERR_CONFIG"),
    ("vocab_size", 1, "GPT_ERR_CONFIG"),
    ("padded_vocab", 70, "GPT_ERR_CONFIG"),
    ("dropout", 1.0, "GPT_ERR_CONFIG"),
    ("precision", 7, "GPT_ERR_CONFIG"),
    ("batch_size", 1000, "GPT_ERR_CONFIG"),    # B*T above the routing limit
    ("zero_world", 65, "GPT_ERR_CONFIG"),      # at most 64 optimiser shards
    ("zero_rank", 1, "GPT_ERR_CONFIG"),        # a rank needs zero_world > rank
])
def test_invalid_configs_rejected_on_host(lib, field, value, status):
    cfg = gb.make_config(W.CHAR)
    setattr(cfg, field, value)
    n = C.c_size_t()
    st = lib.gpt_workspace_bytes(C.byref(cfg), C.byref(n))
    assert gb.STATUS[st] == status
    assert gb.param_count(cfg) == 0


def test_null_arguments(lib):
    assert gb.STATUS[lib.gpt_workspace_bytes(None, None)] == "GPT_ERR_INVALID_ARG"
    out = C.c_void_p()
    cfg = gb.make_config(W.MICRO)
    assert gb.STATUS[lib.gpt_create(C.byref(cfg), 1, None, 0, None, C.byref(out))] == "GPT_ERR_INVALID_ARG"
    assert lib.gpt_param_count(None) == 0
    assert lib.gpt_status_string(0) == b"ok"


@pytest.mark.parametrize("w", [W.GPT2_124M, W.CHAR, W.MICRO], ids=["gpt2_124m", "char", "micro"])
def test_recompute_workspace_saving(lib, w):
    """Activation recompute keeps one layer of the norms' outputs, qkv, the
    attention output and both fc outputs (14 M d operand-type elements per
    layer) instead of L of them; everything else is laid out as before."""
    full = gb.workspace_bytes(gb.make_config(w))
    rc = gb.workspace_bytes(gb.make_config(w, recompute=1))
    M, d, L = w.batch_size * w.block_size, w.n_embd, w.n_layer
    esz = 2 if w.precision == "bf16" else 4
    saved = (L - 1) * 14 * M * d * esz
    assert abs((full - rc) - saved) <= 6 * 256, (full - rc, saved)  # six buffers, 256-byte granules


def test_recompute_flag_validated(lib):
    cfg = gb.make_config(W.CHAR, recompute=2)
    n = C.c_size_t()
    assert gb.STATUS[lib.gpt_workspace_bytes(C.byref(cfg), C.byref(n))] == "GPT_ERR_CONFIG"


@pytest.mark.parametrize("w,over,want", [
    (W.GPT2_124M, {}, gb.GPT_PATH_GEMM_TC | gb.GPT_PATH_ATTN_TC),
    (W.GPT2_XL, {}, gb.GPT_PATH_GEMM_TC | gb.GPT_PATH_ATTN_TC),
    (W.DROPOUT_512, {}, gb.GPT_PATH_GEMM_TC | gb.GPT_PATH_ATTN_TC),
    (W.CHAR, {}, gb.GPT_PATH_GEMM_TC | gb.GPT_PATH_ATTN_TC),
    (W.CHAR, {"block_size": 96}, gb.GPT_PATH_GEMM_TC),          # T not a multiple of 128
    (W.CHAR, {"n_head": 12}, gb.GPT_PATH_GEMM_TC),              # head_dim 32
    (W.MICRO, {}, 0),                                           # fp32 mode
    (W.CHAR.with_(precision="fp32"), {}, 0),
], ids=["gpt2_124m", "gpt2_xl", "dropout_512", "char", "char_T96", "char_hd32", "micro", "char_fp32"])
def test_kernel_paths_follow_the_shape_rule(lib, w, over, want):
    """Which kernels a config runs is a stated rule of the config (bf16: the
    tensor-core GEMM; tensor-core attention at head_dim 64 and T a multiple
    of 128), never a fallback taken at run time."""
    assert gb.kernel_paths(gb.make_config(w, **over)) == want


def test_sharded_moments_shrink_the_workspace(lib):
    """zero_world > 1: the workspace holds the AdamW moments of the rank's
    shard only (the other arenas are unchanged)."""
    full = gb.make_config(W.GPT2_124M)
    n = sum(c for _, c, _ in gb.grad_buckets(full))
    for world in (2, 8):
        for rank in (0, world - 1):
            cfg = gb.make_config(W.GPT2_124M, zero_world=world, zero_rank=rank)
            off, cnt, stride = gb.zero1_shard(cfg, world, rank)
            saved = gb.workspace_bytes(full) - gb.workspace_bytes(cfg)
            assert abs(saved - 8 * (n + 4096 - stride)) <= 1024

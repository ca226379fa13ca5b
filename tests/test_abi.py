"""The C-ABI library: it loads, exports every symbol include/lora_linear.h
declares, and rejects bad arguments on the host before touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lora_linear.h")


@pytest.fixture(scope="module")
def lib():
    from lora_linear_fine_b200 import build
    build.build(quiet=True)
    import lora_linear_fine_b200 as L
    return L


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lora_\w+)\s*\(", text)))


def test_header_declares_expected(lib):
    assert set(declared_functions()) == set(lib.EXPORTED)


def declared_arity():
    """{function: number of parameters} from the header's prototypes."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(lora_\w+)\s*\(([^)]*)\)\s*;", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_bindings_match_header_arity(lib):
    """Every ctypes binding declares as many arguments as the C prototype."""
    lib.lora_linear_abi_version()          # loads the library and its argtypes
    handle = lib._LazyLib._h
    for name, n in declared_arity().items():
        assert len(getattr(handle, name).argtypes) == n, name


def test_library_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(so, name), name


def test_abi_version_and_status_strings(lib):
    assert lib.lora_linear_abi_version() == 1
    for code in range(8):
        assert lib.status_string(code)
    assert lib.status_string(99) == "unknown status"


def test_workspace_size(lib):
    d = lib.make_desc(64, 256, 256, 8, 2.0, "identity")
    assert lib.lora_linear_workspace_size(d, 0) > 0
    assert lib.lora_linear_workspace_size(d, 1) >= lib.lora_linear_workspace_size(d, 0)
    # SwiGLU backward needs the hi/lo dZ buffers: 4 * M * d_out * 2 bytes at least
    d2 = lib.make_desc(64, 256, 256, 8, 2.0, "swiglu")
    assert lib.lora_linear_workspace_size(d2, 1) >= 4 * 64 * 256 * 2
    for bad in [lib.make_desc(64, 256, 256, 12, 2.0, 0), lib.make_desc(64, 250, 256, 8, 2.0, 0),
                lib.make_desc(-1, 256, 256, 8, 2.0, 0), lib.make_desc(64, 256, 256, 8, 2.0, 7),
                lib.make_desc(64, 256, 256, 136, 2.0, 0)]:
        assert lib.lora_linear_workspace_size(bad, 0) == 0
        assert lib.lora_linear_workspace_size(bad, 1) == 0
    # every rank 8..128 in steps of 8 is accepted, every act
    for r in range(0, 129, 8):
        for act in ("identity", "silu", "swiglu"):
            d3 = lib.make_desc(64, 256, 256, r, 2.0, act)
            assert lib.lora_linear_workspace_size(d3, 1) >= lib.lora_linear_workspace_size(d3, 0) > 0


def _fwd(lib, desc, X=16, W=16, A=16, B=16, Y=16, ws=16, ws_bytes=1 << 20, **kw):
    return lib.lora_linear_fwd(desc, X, W, A, B, kw.get("W_up"), kw.get("A_up"), kw.get("B_up"), Y,
                               kw.get("T"), kw.get("Z"), ws, ws_bytes, None)


def test_fwd_rejects_bad_arguments_without_launching(lib):
    ok = lib.make_desc(64, 256, 256, 8, 2.0, "identity")
    assert _fwd(lib, ok, X=None) == 1                 # INVALID_ARG
    assert _fwd(lib, ok, A=None) == 1                 # r > 0 needs A, B
    assert _fwd(lib, ok, X=24) == 2                   # not 16-byte aligned
    assert _fwd(lib, lib.make_desc(64, 252, 256, 8, 2.0, 0)) == 2   # d_in % 8
    assert _fwd(lib, lib.make_desc(64, 256, 256, 12, 2.0, 0)) == 3  # r % 8
    assert _fwd(lib, lib.make_desc(64, 256, 256, 8, 2.0, 5)) == 1   # act
    sw = lib.make_desc(64, 256, 256, 8, 2.0, "swiglu")
    assert _fwd(lib, sw) == 1                         # swiglu needs the up projection
    # an empty batch may pass NULL token tensors: whatever comes back, it is
    # not an argument error (without a GPU the device check answers)
    empty = lib.make_desc(0, 256, 256, 8, 2.0, "identity")
    assert _fwd(lib, empty, X=None, Y=None) not in (1, 2)
    assert _fwd(lib, empty, W=None) == 1              # the weights are still required


def test_bwd_rejects_bad_arguments_without_launching(lib):
    d = lib.make_desc(64, 256, 256, 8, 2.0, "silu")
    # act != identity needs Z_save
    st = lib.lora_linear_bwd(d, 16, 16, 16, 16, 16, None, None, None, 16, None, 16, 16, 16, None, None,
                             16, 1 << 20, None)
    assert st == 1
    st = lib.lora_linear_bwd(d, 16, 16, 16, 16, 16, None, None, None, 16, 16, 16, 16, None, None, None,
                             16, 1 << 20, None)
    assert st == 1                                    # dB missing


def test_no_gpu_means_cuda_error_not_crash(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    ok = lib.make_desc(64, 256, 256, 8, 2.0, "identity")
    assert _fwd(lib, ok) == 6                         # LORA_ERR_CUDA: no device


def test_noalloc_rejects_bad_arguments_before_touching_the_scratch(lib):
    """The no-alloc forward checks its arguments in lora_linear_fwd's order,
    before any device query, symbol lookup or memset."""
    ok = lib.make_desc(64, 256, 256, 8, 2.0, "identity")
    na = lambda desc=ok, X=16, A=16, Y=16: lib.lora_linear_fwd_noalloc(desc, X, 16, A, 16, None, None, None, Y,
                                                                       None, None, None)
    assert na(X=None) == 1                       # INVALID_ARG: X required with M > 0
    assert na(A=None) == 1
    assert na(Y=24) == 2                         # ALIGNMENT
    assert na(desc=lib.make_desc(64, 256, 256, 12, 2.0, 0)) == 3
    raw = lib._LazyLib._h
    assert raw.lora_linear_noalloc_status(None, None) == 1     # out_status NULL


def test_selftest_rejects_bad_arguments_without_launching(lib):
    assert lib.lora_linear_selftest_wait_timeout(None, 1 << 20, 16, None) == 5   # WORKSPACE
    assert lib.lora_linear_selftest_wait_timeout(16, 64, 16, None) == 5          # below the header
    assert lib.lora_linear_selftest_wait_timeout(16, 1 << 20, 5, None) == 1      # INVALID_ARG
    assert lib.lora_linear_selftest_wait_timeout(16, 1 << 20, 31, None) == 1


def test_dropout_and_w4_argument_checks(lib):
    d = lib.make_desc(64, 256, 256, 8, 2.0, "identity")
    assert lib.lora_linear_workspace_size_dropout(d, 1) >= lib.lora_linear_workspace_size_dropout(d, 0) > 0
    # no masked copy of X: with many tokens the dropout workspace is the plain
    # layer's; with few it is the tiled path's, larger than the few-token
    # forward's (which keeps everything on chip)
    many = lib.make_desc(4096, 256, 256, 8, 2.0, "identity")
    assert lib.lora_linear_workspace_size_dropout(many, 0) == lib.lora_linear_workspace_size(many, 0)
    assert lib.lora_linear_workspace_size_dropout(many, 1) == max(lib.lora_linear_workspace_size(many, 0),
                                                                  lib.lora_linear_workspace_size(many, 1))
    assert lib.lora_linear_workspace_size_dropout(d, 0) > lib.lora_linear_workspace_size(d, 0)
    fwd = lambda mask=16, p=0.1, **kw: lib.lora_linear_fwd_dropout(d, 16, 16, 16, 16, None, None, None, mask, None,
                                                                   p, 16, None, None, 16, 1 << 30, None)
    assert fwd(p=1.0) == 1                     # p_drop must be < 1
    assert fwd(p=-0.1) == 1
    assert fwd(mask=None) == 1                 # the mask is required with tokens and an adapter
    sw = lib.make_desc(64, 256, 256, 8, 2.0, "swiglu")
    assert lib.lora_linear_fwd_dropout(sw, 16, 16, 16, 16, 16, 16, 16, 16, None, 0.1, 16, None, None, 16, 1 << 30,
                                       None) == 1   # SwiGLU needs its up projection's mask
    # 4-bit weight: d_in must be a multiple of 64; the codes and scales are required
    assert lib.lora_linear_workspace_size_w4(lib.make_desc(64, 264, 256, 8, 2.0, 0), 0) == 0
    few = lib.make_desc(16, 256, 256, 8, 2.0, "identity")
    many = lib.make_desc(4096, 256, 256, 8, 2.0, "identity")
    assert lib.lora_linear_workspace_size_w4(few, 0) == 256      # the few-token forward reads the codes directly
    assert lib.lora_linear_workspace_size_w4(many, 0) >= lib.lora_linear_workspace_size(many, 0) + 256 * 256 * 2
    w4 = lambda desc, Wq=16, Ws=16: lib.lora_linear_fwd_w4(desc, 16, Wq, Ws, 16, 16, None, None, None, None, 16,
                                                           None, None, 16, 1 << 30, None)
    assert w4(lib.make_desc(64, 264, 256, 8, 2.0, 0)) == 2       # d_in % 64
    assert w4(few, Wq=None) == 1
    assert w4(few, Ws=24) == 2                                     # 16-byte alignment
    assert lib.lora_linear_dequant_w4(16, 16, 256, 100, 16, None) == 2
    assert lib.lora_linear_dequant_w4(None, 16, 256, 128, 16, None) == 1


def test_norm_and_rope_argument_checks(lib):
    """RMSNorm prologue and rotary epilogue: every bad argument is caught on the
    host (these checks come before any device query)."""
    # RMSNorm forward: d % 8, eps, required pointers, alignment
    assert lib.lora_linear_rmsnorm_fwd(16, 16, 4, 100, 1e-6, 16, 16, None) == 2
    assert lib.lora_linear_rmsnorm_fwd(16, 16, 4, 64, -1.0, 16, 16, None) == 1
    assert lib.lora_linear_rmsnorm_fwd(16, 16, 4, 64, float("nan"), 16, 16, None) == 1
    assert lib.lora_linear_rmsnorm_fwd(16, None, 4, 64, 1e-6, 16, 16, None) == 1
    assert lib.lora_linear_rmsnorm_fwd(None, 16, 4, 64, 1e-6, 16, 16, None) == 1
    assert lib.lora_linear_rmsnorm_fwd(24, 16, 4, 64, 1e-6, 16, 16, None) == 2
    assert lib.lora_linear_rmsnorm_fwd(16, 16, 4, 64, 1e-6, 16, 18, None) == 2      # rstd 4-byte aligned
    # RMSNorm backward: the fp32 gradient sum is required and aligned
    assert lib.lora_linear_rmsnorm_bwd(16, 16, 16, None, 4, 64, 16, None) == 1
    assert lib.lora_linear_rmsnorm_bwd(16, 16, 16, 24, 4, 64, 16, None) == 2
    assert lib.lora_linear_rmsnorm_bwd(16, 16, 16, 16, 4, 60, 16, None) == 2
    # rotary projections: identity only, head_dim 64 / 128 dividing d_out, tables aligned
    d = lib.make_desc(256, 512, 256, 8, 2.0, "identity")
    f = lib.lora_linear_workspace_size_rope(d, 0)
    b = lib.lora_linear_workspace_size_rope(d, 1)
    assert b >= f > 0
    assert b >= 2 * 256 * 256 * 2 + 256 * 512 * 2       # fp16 dZ hi + lo and the fp16 copy of W
    assert lib.lora_linear_workspace_size_rope(lib.make_desc(256, 512, 256, 8, 2.0, "silu"), 0) == 0

    def fwd(desc=d, pos=16, cos=16, sin=16, n_pos=32, head_dim=128):
        rope = lib.make_rope_desc(pos, cos, sin, n_pos, head_dim)
        return lib.lora_linear_fwd_rope(desc, rope, 16, 16, 16, 16, 16, None, 16, 1 << 30, None)

    assert fwd(head_dim=96) == 3
    assert fwd(head_dim=32) == 3
    assert fwd(desc=lib.make_desc(256, 512, 192, 8, 2.0, "identity")) == 1   # 192 % 128
    assert fwd(desc=lib.make_desc(256, 512, 256, 8, 2.0, "silu")) == 3
    assert fwd(n_pos=0) == 1
    assert fwd(pos=None) == 1
    assert fwd(cos=24) == 2
    assert fwd(pos=18) == 2
    raw = lib._LazyLib._h
    assert raw.lora_linear_fwd_rope(ctypes.byref(d), None, 16, 16, 16, 16, 16, None, 16, 1 << 30, None) == 1
    rope = lib.make_rope_desc(16, 16, 16, 32, 64)
    bwd = lambda desc=d, rope=rope, dXn=16, acc=0: lib.lora_linear_bwd_rope(desc, rope, 16, 16, 16, 16, 16, None, dXn,
                                                                            acc, 16, 16, 16, 1 << 30, None)
    assert bwd(desc=lib.make_desc(256, 512, 256, 8, 2.0, "swiglu")) == 3
    assert bwd(desc=lib.make_desc(256, 512, 256, 8, 2.0, "silu"), rope=None) == 3   # identity only, rotated or not
    assert bwd(acc=2) == 1
    assert bwd(dXn=None) == 1
    assert bwd(dXn=24) == 2
    assert bwd(rope=lib.make_rope_desc(16, 16, 16, 32, 96)) == 3


def test_cross_entropy_argument_checks(lib):
    """Output projection + cross-entropy: sizes, required pointers and
    alignment are checked on the host before any device query."""
    d = lib.make_ce_desc(64, 256, 1000)
    f = lib.lora_linear_ce_workspace_size(d, 0)
    b = lib.lora_linear_ce_workspace_size(d, 1)
    assert b >= f > 2 * 4 * 64 * 8                     # (max, sum) per token and 128-entry block
    assert b >= 64 * 1000 * 2                          # the chunk's bf16 logit gradient
    assert lib.lora_linear_ce_workspace_size(lib.make_ce_desc(64, 252, 1000), 0) == 0    # d % 8
    assert lib.lora_linear_ce_workspace_size(lib.make_ce_desc(64, 256, 1001), 1) == 0    # V % 8
    assert lib.lora_linear_ce_workspace_size(lib.make_ce_desc(-1, 256, 1000), 0) == 0
    fwd = lambda desc=d, H=16, W=16, lab=16, loss=16, lse=16: lib.lora_linear_ce_fwd(desc, H, W, lab, loss, lse, 16,
                                                                                   1 << 30, None)
    assert fwd(desc=lib.make_ce_desc(64, 252, 1000)) == 2
    assert fwd(desc=lib.make_ce_desc(64, 256, 1004)) == 2       # V % 8: ALIGNMENT
    assert fwd(H=None) == 1
    assert fwd(lab=None) == 1
    assert fwd(loss=None) == 1
    assert fwd(lse=None) == 1
    assert fwd(H=24) == 2
    assert fwd(lab=18) == 2
    # the fused call: the chunk's fp32 logits and bf16 gradient on top of the forward's partials
    assert lib.lora_linear_ce_workspace_size(d, 2) >= f + 64 * 1000 * 6
    both = lambda H=16, dl=16, loss=16, lse=16, dH=16: lib.lora_linear_ce_fwd_bwd(d, H, 16, 16, dl, loss, lse, dH,
                                                                                 16, 1 << 30, None)
    assert both(dl=None) == 1
    assert both(loss=None) == 1
    assert both(lse=None) == 1
    assert both(dH=None) == 1
    assert both(H=None) == 1
    assert both(dH=24) == 2
    assert both(dl=18) == 2
    bwd = lambda H=16, lse=16, dl=16, dH=16: lib.lora_linear_ce_bwd(d, H, 16, 16, lse, dl, dH, 16, 1 << 30, None)
    assert bwd(dl=None) == 1
    assert bwd(dH=None) == 1
    assert bwd(dH=24) == 2
    assert bwd(lse=None) == 1

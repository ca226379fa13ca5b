"""lora_linear_fwd_noalloc: the forward for callers that cannot allocate device
memory (for example a plug-in whose host application owns every device
allocation, or a caller that must not pay for cudaMalloc's synchronisation).
Its scratch is a fixed 16 MiB array inside the library, shared by all calls.

The test calls it through the C ABI twice in a row and compares each result
with the ordinary entry point's (caller-supplied workspace) within the
tolerance the parity tests use, and with the fp64 oracle; after each call it
reads the array's status word back (lora_linear_noalloc_status).  It lives in
a file of its own that pytest collects last, and passes both alone in a fresh
process and after the rest."""
import numpy as np
import pytest

import oracle
import seeded_inputs
from oracle import lora_oracle_c
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu

CASES = [
    (512, 1024, 1024, 8, "identity"),     # rank pass + CTA-pair GEMM
    (300, 512, 768, 64, "silu"),          # rank 64, saved Z
    (16, 1024, 512, 16, "identity"),      # few tokens
]


def _ptr(t):
    return None if t is None else t.data_ptr()


def _noalloc_call_and_check(M, d_in, d_out, r, act, calls=2):
    """Run the no-alloc forward `calls` times on one seeded problem; after each
    call read its status word (expect 0) and compare Y, T (and Z) with the
    ordinary workspace forward within the parity tolerance, and Y, T (and Z)
    with the fp64 oracle."""
    import torch
    import lora_linear_fine_b200 as L
    s = 16.0 / r
    inp = seeded_inputs.make_inputs(M, d_in, d_out, r, act, seed=7, with_grad=False)
    t = {k: G.dev(v) for k, v in inp.items()}
    Y_ref, T_ref, Z_ref = L.forward(t["X"], t["W"], t["A"], t["B"], s, act)
    g = {k: lora_oracle_c.bf16_to_f64(v) for k, v in inp.items()}
    f = lora_oracle_c.lora_forward(g["X"], g["W"], g["A"], g["B"], s, act)
    desc = L.make_desc(M, d_in, d_out, r, s, act)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(calls):
        Y = torch.empty_like(Y_ref)
        T = torch.empty_like(T_ref)
        Z = torch.empty_like(Z_ref) if Z_ref is not None else None
        st = L.lora_linear_fwd_noalloc(desc, _ptr(t["X"]), _ptr(t["W"]), _ptr(t["A"]), _ptr(t["B"]),
                                       None, None, None, _ptr(Y), _ptr(T), _ptr(Z), stream)
        assert st == 0, L.status_string(st)
        st, word = L.lora_linear_noalloc_status(stream)
        assert (st, word) == (0, 0), f"call {call}: status word 0x{word:x}"
        torch.cuda.synchronize()
        res = {"Y": oracle.compare(G.host_f64(Y), G.host_f64(Y_ref)),
               "T": oracle.compare(G.host_f64(T), G.host_f64(T_ref)),
               "Y_vs_oracle": oracle.compare(G.host_f64(Y), f["Y"])}
        res["T_vs_oracle"] = oracle.compare(G.host_f64(T).reshape(f["T"].shape), f["T"])
        if Z is not None:
            res["Z"] = oracle.compare(G.host_f64(Z), G.host_f64(Z_ref))
            res["Z_vs_oracle"] = oracle.compare(G.host_f64(Z).reshape(f["Z"].shape), f["Z"])
        bad = {k: v for k, v in res.items() if not v["ok"]}
        assert not bad, f"call {call}: {bad}"


@pytest.mark.parametrize("M,d_in,d_out,r,act", CASES)
def test_noalloc_forward_matches_workspace_forward_twice(M, d_in, d_out, r, act):
    _noalloc_call_and_check(M, d_in, d_out, r, act)


def test_noalloc_after_a_larger_plan():
    """A large plan (rank 64, split-K partials and saved T regions further into
    the array) followed by a smaller one: the second call must not read what
    the first left behind."""
    _noalloc_call_and_check(512, 1024, 1024, 64, "silu", calls=1)
    _noalloc_call_and_check(300, 512, 768, 8, "identity", calls=1)
    _noalloc_call_and_check(16, 1024, 512, 16, "identity", calls=1)


def test_noalloc_rejects_problems_beyond_the_static_scratch():
    import lora_linear_fine_b200 as L
    # 262144 tokens x rank 64 needs far more than 16 MiB of forward workspace
    desc = L.make_desc(262144, 4096, 4096, 64, 0.25, "identity")
    assert L.lora_linear_workspace_size(desc, 0) > L.NOALLOC_SCRATCH_BYTES
    st = L.lora_linear_fwd_noalloc(desc, 16, 16, 16, 16, None, None, None, 16, None, None, None)
    assert st == 3   # LORA_ERR_UNSUPPORTED, before anything runs

"""The forward GEMM with T = X A^T accumulated inside it when there are more
GEMM tiles than CTA pairs but at most one 256-row block per pair: the
N-tile-0 tile of each row block computes T on the tensor cores during its
main K-loop and publishes bf16(s T); the row block's other tiles, on other
pairs, wait for its flag bits and load that operand for their LoRA K-block.
(The method's adapter input X is read once in the forward: "Liger-Kernel加持！
LlamaPro微调性能大幅提升的秘密", the fused LoRA forward.)

Parity with the fp64 oracle on the same seeded inputs, per element
|err| <= 1e-2 + 1e-2 |ref| and normwise <= 5e-3 on every output, as the other
parity tests; plus the flag protocol's own properties: the workspace header
is zero again after a launch, and back-to-back forwards over different
inputs on one workspace each match their own oracle result."""
import numpy as np
import pytest

import seeded_inputs
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu

CASES = [
    # M, d_in, d_out, r, alpha: row blocks x N tiles > 74 pairs, row blocks <= 74
    (4096, 1024, 4096, 64, 16.0),     # 16 x 16 tiles, rank 64
    (3000, 512, 2000, 40, 16.0),      # ragged M (184-row last block) and N (208-column last tile), RP = 48
    (2048, 1024, 3072, 8, 16.0),      # rank 8: a 16-wide T block
    (74 * 256, 256, 520, 16, 16.0),   # every pair holds a T tile; 8-column last N tile
]


@pytest.mark.parametrize("M,d_in,d_out,r,alpha", CASES)
def test_shared_t_fwd_bwd_parity(M, d_in, d_out, r, alpha):
    s = alpha / r
    inp = seeded_inputs.make_inputs(M, d_in, d_out, r, "identity", seed=21)
    out = G.run_library(inp, M, d_in, d_out, r, s, "identity")
    ref = G.run_oracle(inp, s, "identity")
    G.assert_all_ok(G.compare_all(out, ref, "identity", r))


def _fwd(L, t, desc, ws, M, d_out, r):
    import torch
    p = lambda x: x.data_ptr()
    Y = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((1, M, r), dtype=torch.float32, device="cuda")
    sh = torch.cuda.current_stream().cuda_stream
    st = L.lora_linear_fwd(desc, p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), None, None, None, p(Y), p(T), None,
                           ws.buf.data_ptr(), ws.nbytes, sh)
    assert st == 0, L.status_string(st)
    return Y, T


def test_shared_t_flags_zero_at_rest_and_back_to_back_inputs():
    """Two forwards on one workspace, the second over a different X: each
    matches the oracle for its own inputs (a flag left set by the first
    launch would let the second read the first launch's s T), and the
    256-byte header (status word and flag words) is all zero after each."""
    import lora_linear_fine_b200 as L
    import torch
    M, d_in, d_out, r, s = 4096, 512, 2048, 32, 0.5
    desc = L.make_desc(M, d_in, d_out, r, s, "identity")
    ws = L.Workspace(L.lora_linear_workspace_size(desc, 0))
    for seed in (31, 32):
        inp = seeded_inputs.make_inputs(M, d_in, d_out, r, "identity", seed=seed)
        t = {k: G.dev(v) for k, v in inp.items()}
        Y, T = _fwd(L, t, desc, ws, M, d_out, r)
        torch.cuda.synchronize()
        assert torch.count_nonzero(ws.buf[:256]).item() == 0
        ref = G.run_oracle(inp, s, "identity")
        G.assert_all_ok(G.compare_all({"Y": Y, "T": T, "Z": None}, ref, "identity", r, backward=False))


def test_shared_t_deterministic():
    import lora_linear_fine_b200 as L
    import torch
    M, d_in, d_out, r, s = 3000, 512, 2000, 40, 0.4
    inp = seeded_inputs.make_inputs(M, d_in, d_out, r, "identity", seed=33)
    t = {k: G.dev(v) for k, v in inp.items()}
    desc = L.make_desc(M, d_in, d_out, r, s, "identity")
    ws = L.Workspace(L.lora_linear_workspace_size(desc, 0))
    Y1, T1 = _fwd(L, t, desc, ws, M, d_out, r)
    Y2, T2 = _fwd(L, t, desc, ws, M, d_out, r)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert torch.equal(Y1, Y2) and torch.equal(T1, T2)
    assert not np.isnan(G.host_f64(Y1)).any()

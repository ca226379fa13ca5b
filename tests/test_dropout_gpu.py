"""Parity of dropout on the adapter input with the fp64 oracle
(oracle/dropout_oracle.py) on the same seeded inputs and masks; per element
|err| <= 1e-2 + 1e-2 |ref| and normwise <= 5e-3 on every output."""
import numpy as np
import pytest

import oracle
import seeded_inputs
from oracle import dropout_oracle
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,d_in,d_out,r,act,p_drop", [
    (200, 384, 264, 8, "identity", 0.1),
    (260, 512, 264, 64, "silu", 0.05),
    (136, 256, 392, 8, "swiglu", 0.25),
    (16, 512, 264, 16, "identity", 0.1),      # few tokens: dropout keeps the tiled path
    (256, 512, 520, 128, "identity", 0.3),    # rank 128
    (300, 640, 264, 72, "silu", 0.5),
    # every CTA pair runs several dX tiles, so the epilogue's shared-memory
    # copy of A's columns is refilled between tiles (256 and 128 pair tiles)
    (4096, 4096, 1024, 64, "identity", 0.1),
    (2048, 4096, 512, 8, "silu", 0.1),
])
def test_dropout_fwd_bwd(M, d_in, d_out, r, act, p_drop):
    import lora_linear_fine_b200 as L
    import torch
    s = 16.0 / r
    inp = seeded_inputs.make_inputs(M, d_in, d_out, r, act, seed=9)
    mask = seeded_inputs.draw_mask("mask", M, d_in, p_drop, 9)
    mask_up = seeded_inputs.draw_mask("mask_up", M, d_in, p_drop, 9) if act == "swiglu" else None
    t = {k: G.dev(v) for k, v in inp.items()}
    mk = torch.from_numpy(mask).cuda()
    mk_up = torch.from_numpy(mask_up).cuda() if mask_up is not None else None
    np_ = 2 if act == "swiglu" else 1
    p = lambda x: None if x is None else x.data_ptr()
    desc = L.make_desc(M, d_in, d_out, r, s, act)
    ws = L.Workspace(L.lora_linear_workspace_size_dropout(desc, 1))
    sh = torch.cuda.current_stream().cuda_stream
    Y = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((np_, M, r), dtype=torch.float32, device="cuda")
    Z = torch.empty((np_, M, d_out), dtype=torch.float32, device="cuda") if act != "identity" else None
    st = L.lora_linear_fwd_dropout(desc, p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), p(t.get("W_up")),
                                   p(t.get("A_up")), p(t.get("B_up")), p(mk), p(mk_up), p_drop, p(Y), p(T), p(Z),
                                   ws.buf.data_ptr(), ws.nbytes, sh)
    assert st == 0, L.status_string(st)
    dX = torch.empty((M, d_in), dtype=torch.bfloat16, device="cuda")
    dA = [torch.empty((r, d_in), dtype=torch.float32, device="cuda") for _ in range(np_)]
    dB = [torch.empty((d_out, r), dtype=torch.float32, device="cuda") for _ in range(np_)]
    st = L.lora_linear_bwd_dropout(desc, p(t["dY"]), p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), p(t.get("W_up")),
                                   p(t.get("A_up")), p(t.get("B_up")), p(mk), p(mk_up), p_drop, p(T), p(Z), p(dX),
                                   p(dA[0]), p(dB[0]), p(dA[1]) if np_ == 2 else None,
                                   p(dB[1]) if np_ == 2 else None, ws.buf.data_ptr(), ws.nbytes, sh)
    assert st == 0, L.status_string(st)
    torch.cuda.synchronize()
    assert ws.status() == 0

    g = {k: oracle.bf16_to_f64(v) for k, v in inp.items()}
    m = dropout_oracle.unpack_mask(mask, d_in)
    m_up = dropout_oracle.unpack_mask(mask_up, d_in) if mask_up is not None else None
    ref = dropout_oracle.dropout_backward(g["dY"], g["X"], g["W"], g["A"], g["B"], s, m, p_drop, act,
                                          g.get("W_up"), g.get("A_up"), g.get("B_up"), m_up)
    f = ref["fwd"]
    res = {"Y": oracle.compare(G.host_f64(Y), f["Y"]),
           # T_save holds (X * mask) A^T: the oracle's T = X_d A^T times (1 - p)
           "T": oracle.compare(G.host_f64(T[0]), f["T"] * (1.0 - p_drop)),
           "dX": oracle.compare(G.host_f64(dX), ref["dX"]),
           "dA": oracle.compare(G.host_f64(dA[0]), ref["dA"]),
           "dB": oracle.compare(G.host_f64(dB[0]), ref["dB"])}
    if act != "identity":
        res["Z"] = oracle.compare(G.host_f64(Z[0]), f["Z"])
    if act == "swiglu":
        res["T_up"] = oracle.compare(G.host_f64(T[1]), f["T_up"] * (1.0 - p_drop))
        res["Z_up"] = oracle.compare(G.host_f64(Z[1]), f["Z_up"])
        res["dA_up"] = oracle.compare(G.host_f64(dA[1]), ref["dA_up"])
        res["dB_up"] = oracle.compare(G.host_f64(dB[1]), ref["dB_up"])
    G.assert_all_ok(res)


def test_dropout_all_kept_matches_plain_layer():
    """p = 0 with every element kept: the forward is bit-identical to the
    plain call.  The shape has more 256-row blocks (75) than the 74 CTA pairs
    of a B200, so the plain forward also takes the separate T pass (with at
    most one row block per pair it accumulates T inside the GEMM, a different
    summation order)."""
    import lora_linear_fine_b200 as L
    import torch
    M, d_in, d_out, r = 75 * 256, 512, 512, 16
    inp = seeded_inputs.make_inputs(M, d_in, d_out, r, "identity", seed=10)
    t = {k: G.dev(v) for k, v in inp.items()}
    ones = torch.full((M, d_in // 8), 0xFF, dtype=torch.uint8, device="cuda")
    p = lambda x: None if x is None else x.data_ptr()
    desc = L.make_desc(M, d_in, d_out, r, 1.0, "identity")
    ws = L.Workspace(L.lora_linear_workspace_size_dropout(desc, 1))
    sh = torch.cuda.current_stream().cuda_stream
    Y1 = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
    Y2 = torch.empty_like(Y1)
    T1 = torch.empty((1, M, r), dtype=torch.float32, device="cuda")
    T2 = torch.empty_like(T1)
    assert L.lora_linear_fwd(desc, p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), None, None, None, p(Y1), p(T1),
                             None, ws.buf.data_ptr(), ws.nbytes, sh) == 0
    assert L.lora_linear_fwd_dropout(desc, p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), None, None, None, p(ones),
                                     None, 0.0, p(Y2), p(T2), None, ws.buf.data_ptr(), ws.nbytes, sh) == 0
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2) and torch.equal(T1, T2)


def test_dropout_and_w4_empty_batch():
    """M = 0 through the dropout and 4-bit entry points: no token tensors (NULL),
    no launches but the zero-fill of the adapter gradients."""
    import lora_linear_fine_b200 as L
    import torch
    d_in, d_out, r = 256, 264, 16
    inp = seeded_inputs.make_inputs(8, d_in, d_out, r, "identity", seed=12)
    t = {k: G.dev(v) for k, v in inp.items()}
    Wq, Ws = seeded_inputs.draw_w4("W", d_out, d_in, 12)
    Wq_d, Ws_d = torch.from_numpy(Wq).cuda(), G.dev(Ws)
    sh = torch.cuda.current_stream().cuda_stream
    desc = L.make_desc(0, d_in, d_out, r, 1.0, "identity")
    p = lambda x: x.data_ptr()
    ws = L.Workspace(max(L.lora_linear_workspace_size_dropout(desc, 1), L.lora_linear_workspace_size_w4(desc, 1)))
    for call in ("dropout", "w4"):
        dA = torch.full((r, d_in), float("nan"), device="cuda")
        dB = torch.full((d_out, r), float("nan"), device="cuda")
        if call == "dropout":
            assert L.lora_linear_fwd_dropout(desc, None, p(t["W"]), p(t["A"]), p(t["B"]), None, None, None, None, None,
                                             0.1, None, None, None, ws.buf.data_ptr(), ws.nbytes, sh) == 0
            assert L.lora_linear_bwd_dropout(desc, None, None, p(t["W"]), p(t["A"]), p(t["B"]), None, None, None,
                                             None, None, 0.1, None, None, None, p(dA), p(dB), None, None,
                                             ws.buf.data_ptr(), ws.nbytes, sh) == 0
        else:
            assert L.lora_linear_fwd_w4(desc, None, p(Wq_d), p(Ws_d), p(t["A"]), p(t["B"]), None, None, None, None,
                                        None, None, None, ws.buf.data_ptr(), ws.nbytes, sh) == 0
            assert L.lora_linear_bwd_w4(desc, None, None, p(Wq_d), p(Ws_d), p(t["A"]), p(t["B"]), None, None, None,
                                        None, None, None, None, p(dA), p(dB), None, None, ws.buf.data_ptr(),
                                        ws.nbytes, sh) == 0
        torch.cuda.synchronize()
        assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dB).item() == 0, call
    assert ws.status() == 0

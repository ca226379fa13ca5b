"""Parity of the 4-bit base-weight path ("w4g64") with the fp64 oracle on the
same seeded codes, scales and bf16 inputs.  The expansion to bf16 is an
integer-exact step (a product exact in fp32, then one rounding), so it is
compared bit for bit; the layer uses the per-element and normwise bounds of
the bf16 layer."""
import numpy as np
import pytest

import oracle
import seeded_inputs
from oracle import w4_oracle
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu


def _u8(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _w4_inputs(M, d_in, d_out, r, act, seed):
    inp = seeded_inputs.make_inputs(M, d_in, d_out, r, act, seed=seed)
    inp.pop("W")
    inp.pop("W_up", None)
    w4 = {"Wq": None, "Ws": None}
    w4["Wq"], w4["Ws"] = seeded_inputs.draw_w4("W", d_out, d_in, seed)
    if act == "swiglu":
        w4["Wq_up"], w4["Ws_up"] = seeded_inputs.draw_w4("W_up", d_out, d_in, seed)
    return inp, w4


@pytest.mark.parametrize("d_out,d_in", [(264, 384), (1024, 4096), (8, 64)])
def test_dequant_bit_exact(d_out, d_in):
    import lora_linear_fine_b200 as L
    import torch
    Wq, Ws = seeded_inputs.draw_w4("W", d_out, d_in, 3)
    W = torch.empty((d_out, d_in), dtype=torch.bfloat16, device="cuda")
    Wq_d, Ws_d = _u8(Wq), G.dev(Ws)           # held until the kernel has run
    st = L.lora_linear_dequant_w4(Wq_d.data_ptr(), Ws_d.data_ptr(), d_out, d_in, W.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    got = W.view(torch.int16).cpu().numpy().view(np.uint16)
    ref = w4_oracle.w4_dequant(Wq, Ws)
    ref_bits = (ref.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)   # exact: ref is bf16-valued
    assert np.array_equal(got, ref_bits)


def _run(M, d_in, d_out, r, act, seed, backward):
    import lora_linear_fine_b200 as L
    import torch
    s = 16.0 / r
    inp, w4 = _w4_inputs(M, d_in, d_out, r, act, seed)
    t = {k: G.dev(v) for k, v in inp.items()}
    q = {k: (_u8(v) if k.startswith("Wq") else G.dev(v)) for k, v in w4.items()}
    np_ = 2 if act == "swiglu" else 1
    p = lambda x: None if x is None else x.data_ptr()
    desc = L.make_desc(M, d_in, d_out, r, s, act)
    ws = L.Workspace(L.lora_linear_workspace_size_w4(desc, 1))
    sh = torch.cuda.current_stream().cuda_stream
    Y = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((np_, M, r), dtype=torch.float32, device="cuda")
    Z = torch.empty((np_, M, d_out), dtype=torch.float32, device="cuda") if act != "identity" else None
    st = L.lora_linear_fwd_w4(desc, p(t["X"]), p(q["Wq"]), p(q["Ws"]), p(t["A"]), p(t["B"]), p(q.get("Wq_up")),
                              p(q.get("Ws_up")), p(t.get("A_up")), p(t.get("B_up")), p(Y), p(T), p(Z),
                              ws.buf.data_ptr(), ws.nbytes, sh)
    assert st == 0, L.status_string(st)
    out = {"Y": Y, "T": T, "Z": Z}
    if backward:
        dX = torch.empty((M, d_in), dtype=torch.bfloat16, device="cuda")
        dA = [torch.empty((r, d_in), dtype=torch.float32, device="cuda") for _ in range(np_)]
        dB = [torch.empty((d_out, r), dtype=torch.float32, device="cuda") for _ in range(np_)]
        st = L.lora_linear_bwd_w4(desc, p(t["dY"]), p(t["X"]), p(q["Wq"]), p(q["Ws"]), p(t["A"]), p(t["B"]),
                                  p(q.get("Wq_up")), p(q.get("Ws_up")), p(t.get("A_up")), p(t.get("B_up")), p(T),
                                  p(Z), p(dX), p(dA[0]), p(dB[0]), p(dA[1]) if np_ == 2 else None,
                                  p(dB[1]) if np_ == 2 else None, ws.buf.data_ptr(), ws.nbytes, sh)
        assert st == 0, L.status_string(st)
        out.update(dX=dX, dA=dA[0], dB=dB[0], dA_up=dA[1] if np_ == 2 else None, dB_up=dB[1] if np_ == 2 else None)
    torch.cuda.synchronize()
    assert ws.status() == 0
    g = {k: oracle.bf16_to_f64(v) for k, v in inp.items()}
    ref = w4_oracle.w4_backward(g["dY"], g["X"], w4["Wq"], w4["Ws"], g["A"], g["B"], s, act, w4.get("Wq_up"),
                                w4.get("Ws_up"), g.get("A_up"), g.get("B_up"))
    return out, ref, s


@pytest.mark.parametrize("M,d_in,d_out,r,act", [
    (16, 4096, 4096, 8, "identity"),     # the few-token workload: codes streamed inside the kernel
    (1, 256, 256, 8, "identity"),
    (5, 512, 264, 16, "silu"),
    (33, 1024, 1032, 32, "silu"),
    (64, 768, 520, 64, "identity"),
])
def test_fwd_w4_few_tokens(M, d_in, d_out, r, act):
    out, ref, _ = _run(M, d_in, d_out, r, act, seed=7, backward=False)
    G.assert_all_ok(G.compare_all(out, ref, act, r, backward=False))


@pytest.mark.parametrize("M,d_in,d_out,r,act", [
    (200, 384, 264, 8, "identity"),      # expanded once, then the tiled path
    (260, 512, 264, 64, "silu"),
    (136, 256, 392, 8, "swiglu"),
    (16, 512, 264, 128, "identity"),     # few tokens but r > 64: the tiled path
])
def test_fwd_bwd_w4(M, d_in, d_out, r, act):
    out, ref, _ = _run(M, d_in, d_out, r, act, seed=8, backward=True)
    G.assert_all_ok(G.compare_all(out, ref, act, r, backward=True))


@pytest.mark.parametrize("d_out,d_in", [(264, 384), (4096, 4096)])
def test_tile_bit_exact(d_out, d_in):
    import lora_linear_fine_b200 as L
    import torch
    Wq, _ = seeded_inputs.draw_w4("W", d_out, d_in, 4)
    Wq_d = _u8(Wq)
    Wt = torch.empty(L.lora_linear_w4_tiled_bytes(d_out, d_in), dtype=torch.uint8, device="cuda")
    assert L.lora_linear_w4_tile(Wq_d.data_ptr(), d_out, d_in, Wt.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert np.array_equal(Wt.cpu().numpy(), w4_oracle.w4_tile(Wq))


@pytest.mark.parametrize("M,d_in,d_out,r,act", [
    (16, 4096, 4096, 8, "identity"),
    (5, 512, 264, 16, "silu"),
    (64, 768, 520, 64, "identity"),
])
def test_fwd_w4_tiled_few_tokens(M, d_in, d_out, r, act):
    """The tiled-code forward: parity with the oracle, and bit-identical to the
    row-major-code forward (same kernel, same arithmetic, only the loads differ)."""
    import lora_linear_fine_b200 as L
    import torch
    out, ref, s = _run(M, d_in, d_out, r, act, seed=7, backward=False)
    inp, w4 = _w4_inputs(M, d_in, d_out, r, act, 7)
    t = {k: G.dev(v) for k, v in inp.items()}
    Wq_d, Ws_d = _u8(w4["Wq"]), G.dev(w4["Ws"])
    sh = torch.cuda.current_stream().cuda_stream
    Wt = torch.empty(L.lora_linear_w4_tiled_bytes(d_out, d_in), dtype=torch.uint8, device="cuda")
    assert L.lora_linear_w4_tile(Wq_d.data_ptr(), d_out, d_in, Wt.data_ptr(), sh) == 0
    desc = L.make_desc(M, d_in, d_out, r, s, act)
    ws = L.Workspace(L.lora_linear_workspace_size(desc, 0))
    Y = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((1, M, r), dtype=torch.float32, device="cuda")
    Z = torch.empty((1, M, d_out), dtype=torch.float32, device="cuda") if act != "identity" else None
    st = L.lora_linear_fwd_w4_tiled(desc, t["X"].data_ptr(), Wt.data_ptr(), Ws_d.data_ptr(), t["A"].data_ptr(),
                                    t["B"].data_ptr(), Y.data_ptr(), T.data_ptr(),
                                    Z.data_ptr() if Z is not None else None, ws.buf.data_ptr(), ws.nbytes, sh)
    assert st == 0, L.status_string(st)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert torch.equal(Y, out["Y"]) and torch.equal(T, out["T"])
    G.assert_all_ok(G.compare_all({"Y": Y, "T": T, "Z": Z}, ref, act, r, backward=False))

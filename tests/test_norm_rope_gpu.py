"""Parity of the RMSNorm prologue and rotary-embedding epilogue with the fp64
oracle (oracle/norm_rope_oracle.py) on the same seeded inputs.  x_n is
compared bit for bit (both sides round the exact norm once to bf16); every
other output per element |err| <= 1e-2 + 1e-2 |ref| and normwise <= 5e-3."""
import numpy as np
import pytest

import oracle
import seeded_inputs as S
from oracle import norm_rope_oracle as NR
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu


def _sh():
    import torch
    return torch.cuda.current_stream().cuda_stream


def _bf16_bits(v):
    """bf16-representable float64 values -> their bit patterns."""
    return (np.asarray(v, dtype=np.float64).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _dev_bits(t):
    import torch
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def _norm_inputs(M, d, seed, zero_row):
    X = G.f64(S.draw("X", (M, d), seed, d))
    scale = np.exp2(np.random.default_rng(seed).integers(-8, 9, size=M)).astype(np.float64)   # exact in bf16
    X = X * scale[:, None]
    if zero_row and M > 2:
        X[M // 2] = 0.0
    return S.f64_to_bf16_bits(X), S.draw_norm_weight(d, seed)


@pytest.mark.parametrize("M,d,eps", [(1, 8, 1e-6), (37, 264, 1e-6), (300, 4096, 1e-5), (5, 14336, 0.0),
                                     (129, 512, 3.0)])
def test_rmsnorm_forward_bit_exact(M, d, eps):
    import lora_linear_fine_b200 as L
    import torch
    Xb, gb = _norm_inputs(M, d, 41, zero_row=eps > 0)
    X, g = G.dev(Xb), G.dev(gb)
    Xn = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    rstd = torch.empty(M, dtype=torch.float32, device="cuda")
    assert L.lora_linear_rmsnorm_fwd(X.data_ptr(), g.data_ptr(), M, d, eps, Xn.data_ptr(), rstd.data_ptr(), _sh()) == 0
    torch.cuda.synchronize()
    eps32 = float(np.float32(eps))
    exact, rstd_ref = NR.rms_norm(G.f64(Xb), G.f64(gb), eps32)
    want = _bf16_bits(NR.round_bf16(exact))
    got = _dev_bits(Xn)
    assert np.array_equal(got, want), f"{np.count_nonzero(got != want)} of {got.size} x_n differ"
    assert np.allclose(G.host_f64(rstd), rstd_ref, rtol=1e-6, atol=0)


@pytest.mark.parametrize("M,d,n", [(37, 264, 1), (300, 4096, 3), (129, 512, 2), (4, 8, 4)])
def test_rmsnorm_backward(M, d, n):
    """dx_n: the fp32 sum of n drawn gradients (as the projections' dX GEMMs
    leave it)."""
    import lora_linear_fine_b200 as L
    import torch
    Xb, gb = _norm_inputs(M, d, 42, zero_row=False)
    eps = 1e-6
    X, g = G.dev(Xb), G.dev(gb)
    Xn = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    rstd = torch.empty(M, dtype=torch.float32, device="cuda")
    assert L.lora_linear_rmsnorm_fwd(X.data_ptr(), g.data_ptr(), M, d, eps, Xn.data_ptr(), rstd.data_ptr(), _sh()) == 0
    dXn = sum(G.f64(S.draw("dY", (M, d), 50 + j, d)) for j in range(n)).astype(np.float32)
    dXn_d = torch.from_numpy(dXn).cuda()
    dX = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    assert L.lora_linear_rmsnorm_bwd(X.data_ptr(), g.data_ptr(), rstd.data_ptr(), dXn_d.data_ptr(), M, d,
                                     dX.data_ptr(), _sh()) == 0
    torch.cuda.synchronize()
    dXn = dXn.astype(np.float64)
    ref = NR.rms_norm_backward(dXn, G.f64(Xb), G.f64(gb), float(np.float32(eps)))
    G.assert_all_ok({"dX": oracle.compare(G.host_f64(dX), ref)})


def _rope_call(L, M, d_in, d_out, r, s, t, pos, cos, sin, n_pos, hd, prefill=None):
    """One forward + backward of a rotated projection through the C ABI.  The
    input gradient is fp32; with ``prefill`` it is added to that tensor."""
    import torch
    p = lambda x: None if x is None else x.data_ptr()
    desc = L.make_desc(M, d_in, d_out, r, s, "identity")
    rope = L.make_rope_desc(p(pos), p(cos), p(sin), n_pos, hd)
    ws = L.Workspace(L.lora_linear_workspace_size_rope(desc, 1))
    Y = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((M, r), dtype=torch.float32, device="cuda")
    st = L.lora_linear_fwd_rope(desc, rope, p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), p(Y), p(T),
                                ws.buf.data_ptr(), ws.nbytes, _sh())
    assert st == 0, L.status_string(st)
    dX = (torch.from_numpy(prefill).cuda() if prefill is not None
          else torch.empty((M, d_in), dtype=torch.float32, device="cuda"))
    dA = torch.empty((r, d_in), dtype=torch.float32, device="cuda")
    dB = torch.empty((d_out, r), dtype=torch.float32, device="cuda")
    st = L.lora_linear_bwd_rope(desc, rope, p(t["dY"]), p(t["X"]), p(t["W"]), p(t["A"]), p(t["B"]), p(T), p(dX),
                                0 if prefill is None else 1, p(dA), p(dB), ws.buf.data_ptr(), ws.nbytes, _sh())
    assert st == 0, L.status_string(st)
    torch.cuda.synchronize()
    return {"Y": Y, "T": T, "dX": dX, "dA": dA, "dB": dB}, ws


def _tables_dev(n_pos, hd):
    import torch
    cos, sin = S.rotary_tables(n_pos, hd)
    return cos, sin, torch.from_numpy(cos).cuda(), torch.from_numpy(sin).cuda()


@pytest.mark.parametrize("M,d_in,d_out,r,hd,acc", [
    (200, 384, 256, 8, 128, False),     # CTA-pair GEMM, ragged last tile
    (96, 512, 384, 16, 64, True),       # single-CTA GEMM, two heads per 128 columns; dx added to a prefilled dx_n
    (260, 256, 640, 64, 128, False),    # the last N tile runs past d_out
    (136, 512, 192, 128, 64, True),     # rank 128; d_out not a multiple of 128; added
    (3, 256, 128, 8, 128, False),       # a few tokens still take the tiled GEMM
])
def test_rotated_projection(M, d_in, d_out, r, hd, acc):
    import lora_linear_fine_b200 as L
    import torch
    s = 16.0 / r
    inp = S.make_inputs(M, d_in, d_out, r, "identity", seed=21)
    n_pos = 257
    pos = S.draw_positions(M, n_pos, 21)
    cos, sin, cos_d, sin_d = _tables_dev(n_pos, hd)
    t = {k: G.dev(v) for k, v in inp.items()}
    pre = (np.random.default_rng(5).standard_normal((M, d_in)).astype(np.float32) if acc else None)
    out, ws = _rope_call(L, M, d_in, d_out, r, s, t, torch.from_numpy(pos).cuda(), cos_d, sin_d, n_pos, hd, pre)
    assert ws.status() == 0
    dx = G.host_f64(out["dX"]) - (pre.astype(np.float64) if acc else 0.0)
    g = {k: G.f64(v) for k, v in inp.items()}
    c64, s64 = cos.astype(np.float64), sin.astype(np.float64)
    f = oracle.lora_forward(g["X"], g["W"], g["A"], g["B"], s)
    dZ = NR.apply_rotary_backward(g["dY"], pos, c64, s64, hd)
    b = oracle.lora_linear_branch_backward(dZ, g["X"], g["W"], g["A"], g["B"], f["T"], s)
    G.assert_all_ok({"Y": oracle.compare(G.host_f64(out["Y"]), NR.apply_rotary(f["Z"], pos, c64, s64, hd)),
                     "T": oracle.compare(G.host_f64(out["T"]), f["T"]),
                     "dX": oracle.compare(dx, b["dX"]),
                     "dA": oracle.compare(G.host_f64(out["dA"]), b["dA"]),
                     "dB": oracle.compare(G.host_f64(out["dB"]), b["dB"])})


def test_rotated_projection_position_outside_table():
    """A position outside the table sets status bit 0x2; that token's output
    and gradient pass through unturned, the others are turned as usual."""
    import lora_linear_fine_b200 as L
    import torch
    M, d_in, d_out, r, hd, n_pos = 130, 256, 256, 8, 128, 16
    s = 2.0
    inp = S.make_inputs(M, d_in, d_out, r, "identity", seed=22)
    pos = S.draw_positions(M, n_pos, 22)
    bad = [5, 77]
    pos[5], pos[77] = n_pos, -1
    cos, sin, cos_d, sin_d = _tables_dev(n_pos, hd)
    t = {k: G.dev(v) for k, v in inp.items()}
    out, ws = _rope_call(L, M, d_in, d_out, r, s, t, torch.from_numpy(pos).cuda(), cos_d, sin_d, n_pos, hd)
    assert ws.status() & 0x2
    g = {k: G.f64(v) for k, v in inp.items()}
    c64, s64 = cos.astype(np.float64), sin.astype(np.float64)
    safe = np.where((pos >= 0) & (pos < n_pos), pos, 0)
    f = oracle.lora_forward(g["X"], g["W"], g["A"], g["B"], s)
    Yref = NR.apply_rotary(f["Z"], safe, c64, s64, hd)
    Yref[bad] = f["Z"][bad]
    dZ = NR.apply_rotary_backward(g["dY"], safe, c64, s64, hd)
    dZ[bad] = g["dY"][bad]
    b = oracle.lora_linear_branch_backward(dZ, g["X"], g["W"], g["A"], g["B"], f["T"], s)
    G.assert_all_ok({"Y": oracle.compare(G.host_f64(out["Y"]), Yref),
                     "dX": oracle.compare(G.host_f64(out["dX"]), b["dX"]),
                     "dA": oracle.compare(G.host_f64(out["dA"]), b["dA"]),
                     "dB": oracle.compare(G.host_f64(out["dB"]), b["dB"])})


def _qkv_run(L, M, d, douts, r, hd, eps, Xb, gb, proj_inp, pos, cos_d, sin_d, n_pos):
    """The block through the C ABI: norm, q and k rotated, v plain, backward,
    the norm's backward over the three input gradients."""
    import torch
    p = lambda x: None if x is None else x.data_ptr()
    s = 16.0 / r
    X, g = G.dev(Xb), G.dev(gb)
    Xn = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    rstd = torch.empty(M, dtype=torch.float32, device="cuda")
    assert L.lora_linear_rmsnorm_fwd(p(X), p(g), M, d, eps, p(Xn), p(rstd), _sh()) == 0
    rope = L.make_rope_desc(p(pos), p(cos_d), p(sin_d), n_pos, hd)
    dXn = torch.empty((M, d), dtype=torch.float32, device="cuda")
    outs = []
    for j, (d_out, inp) in enumerate(zip(douts, proj_inp)):
        t = {k: G.dev(v) for k, v in inp.items() if k != "X"}
        desc = L.make_desc(M, d, d_out, r, s, "identity")
        ws = L.Workspace(max(L.lora_linear_workspace_size_rope(desc, 1), L.lora_linear_workspace_size(desc, 1)))
        Y = torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda")
        T = torch.empty((M, r), dtype=torch.float32, device="cuda")
        dA = torch.empty((r, d), dtype=torch.float32, device="cuda")
        dB = torch.empty((d_out, r), dtype=torch.float32, device="cuda")
        args = (p(t["W"]), p(t["A"]), p(t["B"]))
        if j < 2:
            assert L.lora_linear_fwd_rope(desc, rope, p(Xn), *args, p(Y), p(T), ws.buf.data_ptr(), ws.nbytes,
                                          _sh()) == 0
        else:
            assert L.lora_linear_fwd(desc, p(Xn), *args, None, None, None, p(Y), p(T), None, ws.buf.data_ptr(),
                                     ws.nbytes, _sh()) == 0
        # q writes the fp32 dx_n, k and v add to it; v is not rotated
        assert L.lora_linear_bwd_rope(desc, rope if j < 2 else None, p(t["dY"]), p(Xn), *args, p(T), p(dXn),
                                      1 if j else 0, p(dA), p(dB), ws.buf.data_ptr(), ws.nbytes, _sh()) == 0
        outs.append({"Y": Y, "T": T, "dA": dA, "dB": dB, "ws": ws, "t": t})
    dXall = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    assert L.lora_linear_rmsnorm_bwd(p(X), p(g), p(rstd), p(dXn), M, d, p(dXall), _sh()) == 0
    torch.cuda.synchronize()
    for o in outs:
        assert o["ws"].status() == 0
    return Xn, outs, dXall


def _qkv_inputs(M, d, douts, r, seed):
    Xb = S.draw("X", (M, d), seed, d)
    gb = S.draw_norm_weight(d, seed)
    proj = [S.make_inputs(M, d, d_out, r, "identity", seed=seed * 10 + j) for j, d_out in enumerate(douts)]
    return Xb, gb, proj


@pytest.mark.parametrize("M,d,dq,dkv,r,hd", [(264, 512, 512, 128, 8, 64), (130, 256, 256, 256, 16, 128)])
def test_qkv_block(M, d, dq, dkv, r, hd):
    import lora_linear_fine_b200 as L
    import torch
    douts = (dq, dkv, dkv)
    eps = 1e-6
    Xb, gb, proj = _qkv_inputs(M, d, douts, r, 23)
    n_pos = 512
    pos = S.draw_positions(M, n_pos, 23)
    cos, sin, cos_d, sin_d = _tables_dev(n_pos, hd)
    Xn, outs, dX = _qkv_run(L, M, d, douts, r, hd, eps, Xb, gb, proj, torch.from_numpy(pos).cuda(), cos_d, sin_d,
                            n_pos)
    projs = [{k: G.f64(inp[k]) for k in ("W", "A", "B")} for inp in proj]
    dYs = [G.f64(inp["dY"]) for inp in proj]
    ref = NR.qkv_backward(dYs, G.f64(Xb), G.f64(gb), float(np.float32(eps)), projs, 16.0 / r, [True, True, False],
                          pos, cos.astype(np.float64), sin.astype(np.float64), hd)
    f = ref["fwd"]
    assert np.array_equal(_dev_bits(Xn), _bf16_bits(f["Xn"]))
    res = {"dX": oracle.compare(G.host_f64(dX), ref["dX"])}
    for j, name in enumerate("qkv"):
        res["Y_" + name] = oracle.compare(G.host_f64(outs[j]["Y"]), f["Y"][j])
        res["T_" + name] = oracle.compare(G.host_f64(outs[j]["T"]), f["T"][j])
        res["dA_" + name] = oracle.compare(G.host_f64(outs[j]["dA"]), ref["dA"][j])
        res["dB_" + name] = oracle.compare(G.host_f64(outs[j]["dB"]), ref["dB"][j])
    G.assert_all_ok(res)


def test_qkv_block_full_size_sampled():
    """The benchmark's block (M = 16384 tokens of 4 sequences, 4096 -> q 4096,
    k 1024, v 1024, r = 8, head_dim 128) through the same calls bench.py times:
    x_n bit for bit in full; rows of Y and dX sampled (each row depends only
    on its token); T, dA, dB in full."""
    import lora_linear_fine_b200 as L
    import torch
    c = S.CONFIGS["qkv_rmsnorm_rope"]
    M, d, r, hd = c["M"], c["d_in"], c["r"], c["head_dim"]
    douts = (c["d_out"], c["d_kv"], c["d_kv"])
    s = c["alpha"] / r
    Xb, gb, proj = _qkv_inputs(M, d, douts, r, 0)
    n_pos = c["seq_len"]
    pos = S.sequence_positions(M, n_pos)
    cos, sin, cos_d, sin_d = _tables_dev(n_pos, hd)
    Xn, outs, dX = _qkv_run(L, M, d, douts, r, hd, c["eps"], Xb, gb, proj, torch.from_numpy(pos).cuda(), cos_d,
                            sin_d, n_pos)
    eps32 = float(np.float32(c["eps"]))
    X64, g64 = G.f64(Xb), G.f64(gb)
    exact, _ = NR.rms_norm(X64, g64, eps32)
    xn = NR.round_bf16(exact)
    del exact
    assert np.array_equal(_dev_bits(Xn), _bf16_bits(xn))
    rows = np.array(sorted({0, 1, 127, 128, 4095, 4096, M - 1} |
                           set(np.random.default_rng(0).choice(M, 40, replace=False).tolist())))
    c64, s64 = cos.astype(np.float64), sin.astype(np.float64)
    res = {}
    dXn_rows = np.zeros((len(rows), d))
    for j, name in enumerate("qkv"):
        W, A, B = (G.f64(proj[j][k]) for k in ("W", "A", "B"))
        dY = G.f64(proj[j]["dY"])
        T = xn @ A.T
        Zr = xn[rows] @ W.T + s * (T[rows] @ B.T)
        Yr = NR.apply_rotary(Zr, pos[rows], c64, s64, hd) if j < 2 else Zr
        dZ = NR.apply_rotary_backward(dY, pos, c64, s64, hd) if j < 2 else dY
        U = dZ @ B
        res["Y_" + name] = oracle.compare(G.host_f64(outs[j]["Y"])[rows], Yr)
        res["T_" + name] = oracle.compare(G.host_f64(outs[j]["T"]), T)
        res["dA_" + name] = oracle.compare(G.host_f64(outs[j]["dA"]), s * (U.T @ xn))
        res["dB_" + name] = oracle.compare(G.host_f64(outs[j]["dB"]), s * (dZ.T @ T))
        dXn_rows += dZ[rows] @ W + s * (U[rows] @ A)
        del dZ, U, T
    dXr = NR.rms_norm_backward(dXn_rows, X64[rows], g64, eps32)
    res["dX"] = oracle.compare(G.host_f64(dX)[rows], dXr)
    G.assert_all_ok(res)

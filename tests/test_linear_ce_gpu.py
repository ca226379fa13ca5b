"""Parity of the fused output projection + cross-entropy (lora_linear_ce_fwd /
lora_linear_ce_bwd) with the fp64 oracle (oracle/linear_ce_oracle.py) on the
same seeded bf16 inputs: the loss, every token's log-sum-exp and dH, per
element |err| <= 1e-2 + 1e-2 |ref| and normwise <= 5e-3.  Sizes cover ragged
token and vocabulary tails (V not a multiple of the 256-wide tile), the
single-CTA and CTA-pair GEMMs, ignored tokens, a Llama-3-8B vocabulary
(V = 128256, d = 4096) and the benchmark's 8192 tokens."""
import numpy as np
import pytest

import oracle
import seeded_inputs
from oracle import linear_ce_oracle as CE
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu


def _dev_i32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _run(H, W, labels, dloss=1.0):
    import torch
    import lora_linear_fine_b200 as L
    tH, tW, tl = G.dev(H), G.dev(W), _dev_i32(labels)
    loss, lse = L.linear_cross_entropy(tH, tW, tl)
    dl = torch.tensor(dloss, dtype=torch.float32, device="cuda")
    dH = L.linear_cross_entropy_backward(tH, tW, tl, lse, dl)
    torch.cuda.synchronize()
    return float(loss.item()), G.host_f64(lse), G.host_f64(dH)


def _check(H, W, labels, dloss=1.0):
    Hf, Wf = G.f64(H), G.f64(W)
    loss, lse, dH = _run(H, W, labels, dloss)
    ref = CE.linear_ce_backward(Hf, Wf, labels, dloss)
    f = ref["fwd"]
    res = {"loss": oracle.compare(np.array([loss]), np.array([f["loss"] * 1.0])),
           "lse": oracle.compare(lse, f["lse"]),
           "dH": oracle.compare(dH, ref["dH"])}
    G.assert_all_ok(res)
    return res


CASES = [
    # M, d, V
    (64, 256, 1000),        # single CTA, ragged vocabulary tail
    (300, 264, 2048),       # CTA pairs, ragged tokens and hidden size
    (1, 128, 8),            # one token, eight classes
    (257, 512, 32008),      # V = 125 tiles + 8 entries
    (1024, 1024, 4096),
]


@pytest.mark.parametrize("M,d,V", CASES)
def test_ce_parity(M, d, V):
    H, W, labels = seeded_inputs.draw_ce(M, d, V, seed=M + V)
    _check(H, W, labels)


def test_ce_peaked_logits_and_upstream_factor():
    """Logits four times wider (a softmax far from uniform) and d(loss) = 3.5."""
    H, W, labels = seeded_inputs.draw_ce(384, 512, 5000, seed=5, h_scale=4.0)
    _check(H, W, labels, dloss=3.5)


def test_ce_every_token_ignored():
    H, W, labels = seeded_inputs.draw_ce(200, 256, 1000, seed=6)
    labels[:] = -100
    loss, lse, dH = _run(H, W, labels)
    assert loss == 0.0
    assert not np.any(dH)
    f = CE.linear_ce_forward(G.f64(H), G.f64(W), labels)
    G.assert_all_ok({"lse": oracle.compare(lse, f["lse"])})


def test_ce_label_out_of_range_is_flagged_and_ignored():
    """A label >= V sets status bit 0x2 and that token counts as ignored."""
    import torch
    import lora_linear_fine_b200 as L
    M, d, V = 130, 256, 1000
    H, W, labels = seeded_inputs.draw_ce(M, d, V, seed=7)
    bad = labels.copy()
    bad[3] = V + 5
    desc = L.make_ce_desc(M, d, V)
    ws = L.Workspace(L.lora_linear_ce_workspace_size(desc, 1))
    tH, tW, tl = G.dev(H), G.dev(W), _dev_i32(bad)
    loss, lse = L.linear_cross_entropy(tH, tW, tl, workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() & 0x2
    ok = labels.copy()
    ok[3] = -1
    f = CE.linear_ce_forward(G.f64(H), G.f64(W), ok)
    G.assert_all_ok({"loss": oracle.compare(np.array([float(loss.item())]), np.array([f["loss"]]))})


def test_ce_empty_batch():
    import torch
    import lora_linear_fine_b200 as L
    desc = L.make_ce_desc(0, 256, 1000)
    ws = L.Workspace(L.lora_linear_ce_workspace_size(desc, 1))
    W = G.dev(seeded_inputs.draw_ce(1, 256, 1000, seed=8)[1])
    loss = torch.full((), 7.0, dtype=torch.float32, device="cuda")
    dl = torch.ones((), dtype=torch.float32, device="cuda")
    sh = torch.cuda.current_stream().cuda_stream
    assert L.lora_linear_ce_fwd(desc, None, W.data_ptr(), None, loss.data_ptr(), None, ws.buf.data_ptr(), ws.nbytes,
                                sh) == 0
    assert L.lora_linear_ce_bwd(desc, None, W.data_ptr(), None, None, dl.data_ptr(), None, ws.buf.data_ptr(),
                                ws.nbytes, sh) == 0
    torch.cuda.synchronize()
    assert loss.item() == 0.0
    assert ws.status() == 0


def test_ce_deterministic():
    H, W, labels = seeded_inputs.draw_ce(300, 512, 4000, seed=9)
    a = _run(H, W, labels)
    b = _run(H, W, labels)
    assert a[0] == b[0] and np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])


def test_ce_llama3_vocabulary_512_tokens():
    """V = 128256, d = 4096 (the Llama-3-8B output projection), 512 tokens:
    every output in full."""
    H, W, labels = seeded_inputs.draw_ce(512, 4096, 128256, seed=10)
    _check(H, W, labels)


def test_ce_llama3_vocabulary_8192_tokens():
    """The benchmark's size (8192 tokens, one backward chunk): the loss over all
    tokens, lse of every token and dH of sampled rows.  The oracle runs over
    row blocks (each token's logits depend on its own row only); dH rows are
    scaled by 1/N with N counted over the whole batch."""
    M, d, V = 8192, 4096, 128256
    H, W, labels = seeded_inputs.draw_ce(M, d, V, seed=11)
    loss, lse, dH = _run(H, W, labels)
    Hf, Wf = G.f64(H), G.f64(W)
    n_valid = int(np.count_nonzero(labels >= 0))
    lse_ref = np.empty(M)
    tok = np.empty(M)
    for m0 in range(0, M, 1024):
        f = CE.linear_ce_forward(Hf[m0:m0 + 1024], Wf, labels[m0:m0 + 1024])
        lse_ref[m0:m0 + 1024] = f["lse"]
        tok[m0:m0 + 1024] = f["loss_tok"]
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, 255, 256, M - 1], rng.choice(M, 123, replace=False)]))
    sub = labels[rows]
    b = CE.linear_ce_backward(Hf[rows], Wf, sub, dloss=np.count_nonzero(sub >= 0) / n_valid)
    res = {"loss": oracle.compare(np.array([loss]), np.array([tok.sum() / n_valid])),
           "lse": oracle.compare(lse, lse_ref),
           "dH_rows": oracle.compare(dH[rows], b["dH"])}
    G.assert_all_ok(res)


@pytest.mark.parametrize("M,d,V,dloss", [
    (300, 264, 2048, 1.0),       # CTA pairs, ragged tokens and hidden size
    (64, 256, 1000, 0.5),        # single CTA, ragged vocabulary tail, upstream factor
    (8200, 256, 1032, 1.0),      # two chunks (8192 + 8 tokens)
    (512, 4096, 128256, 1.0),    # Llama-3-8B vocabulary
])
def test_ce_fused_forward_backward_matches_separate_calls(M, d, V, dloss):
    """The fused call's loss, lse and dH equal, bit for bit, those of the
    forward followed by the backward (same GEMM, same gradient arithmetic),
    with ignored labels in the batch; and the loss matches the oracle."""
    import torch
    import lora_linear_fine_b200 as L
    H, W, labels = seeded_inputs.draw_ce(M, d, V, seed=3 * M + V)
    tH, tW, tl = G.dev(H), G.dev(W), _dev_i32(labels)
    dl = torch.tensor(dloss, dtype=torch.float32, device="cuda")
    loss1, lse1 = L.linear_cross_entropy(tH, tW, tl)
    dH1 = L.linear_cross_entropy_backward(tH, tW, tl, lse1, dl)
    loss2, lse2, dH2 = L.linear_cross_entropy_fwd_bwd(tH, tW, tl, dl)
    torch.cuda.synchronize()
    assert (labels < 0).any()
    assert torch.equal(loss1, loss2) and torch.equal(lse1, lse2) and torch.equal(dH1, dH2)
    if V <= 32768:
        ref = CE.linear_ce_forward(G.f64(H), G.f64(W), labels)
        G.assert_all_ok({"loss": oracle.compare(np.array([float(loss2.item())]), np.array([ref["loss"] * 1.0]))})

"""Host-side replay of the rotary kernels' index arithmetic (CPU only): the
GEMM epilogue's two passes over a thread's 128 accumulator columns hold whole
pairs (features i and i + head_dim/2 of one head) and together store every
output column once; the gradient kernel's (token, head, 8-pair) items cover
every element once with 16-byte aligned accesses inside the tensor and the
tables.  The formulas restate the layout documented in
lora_linear_fine_b200/csrc/lora_mma.cuh (kMEpiRope) and lora_norm_rope.cuh
(rope_bwd_kernel) for the supported head sizes and ragged shapes."""
import pytest


def epilogue_columns(N, half):
    """Columns each (tile, thread half, pass, part) stores; asserts pairing."""
    written = []
    hd = 2 * half
    for nt in range((N + 255) // 256):
        for h in (0, 1):
            col0 = nt * 256 + h * 128                  # a thread's 128 columns
            for hv in (0, 1):
                c0 = 32 * hv if half == 64 else 64 * hv
                toff = c0 % half
                assert c0 % 32 == 0 and c0 + half + 32 <= 128          # two 32-column TMEM loads inside the 128
                assert toff + 32 <= half and (toff * 4) % 16 == 0      # table reads: in the row, 16-byte aligned
                for e in range(32):
                    a, b = col0 + c0 + e, col0 + c0 + half + e
                    assert a // hd == b // hd                          # one head
                    assert a % hd == toff + e and b % hd == toff + e + half
                for part in (0, 1):
                    cc = c0 + part * half
                    for j in range(0, 32, 8):
                        if col0 + cc + j < N:
                            written.extend(range(col0 + cc + j, col0 + cc + j + 8))
    return written


@pytest.mark.parametrize("N,half", [(128, 64), (256, 64), (640, 64), (4096, 64), (64, 32), (192, 32), (1024, 32)])
def test_epilogue_stores_every_column_once(N, half):
    cols = epilogue_columns(N, half)
    assert sorted(cols) == list(range(N))


@pytest.mark.parametrize("M,N,half,n_pos", [(3, 128, 64, 1), (200, 256, 64, 37), (130, 384, 32, 5), (17, 192, 32, 8)])
def test_gradient_items_cover_every_element_once(M, N, half, n_pos):
    chunks, heads = half // 8, N // (2 * half)
    per_row = heads * chunks
    seen = set()
    for i in range(M * per_row):
        m, rem = divmod(i, per_row)
        head, ch = divmod(rem, chunks)
        a0 = m * N + head * 2 * half + ch * 8
        for base in (a0, a0 + half):
            assert base + 8 <= M * N and (base * 2) % 16 == 0
            span = set(range(base, base + 8))
            assert not (span & seen)
            seen |= span
        for p in (0, n_pos - 1):
            t = p * half + ch * 8
            assert t + 8 <= n_pos * half and (t * 4) % 16 == 0
    assert len(seen) == M * N
    assert M * per_row == M * N // 16          # the launch's item count

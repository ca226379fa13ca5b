"""CPU replay of the forward GEMM's tile schedule (lora_mma_kernel's
mma_tile_coords and the host's choice of a shared T), checking the
properties the shared-T forward relies on, for many shapes:

* the raster visits every (row block, N tile) exactly once;
* with a shared T, tiles 0 .. m_tiles - 1 are the N-tile-0 tiles, one per
  row block, and with units = min(tiles, pairs) each is its unit's first
  tile (unit u takes tiles u, u + units, ...), so its second accumulator
  buffer is free for T;
* every other tile's row block has its T tile on a unit (the flag it waits
  for is set by a resident CTA);
* the flag bits (4 per CTA of each T tile) fit the header's flag words.

The replay restates the index arithmetic of csrc/lora_mma.cuh
(mma_tile_coords) and csrc/lora_linear.cu (set_raster, the shared-T test)."""
import itertools

import pytest

K_TFLAG_WORDS = 19          # lora_mma.cuh kTFlagWords
K_HEADER_WORDS = 256 // 4   # the workspace header
K_TFLAG_WORD0 = 8           # lora_linear.cu kTFlagWord0


def tile_coords(t, m_tiles, n_tiles, group, along_n, shared):
    nt0 = 0
    if shared:
        if t < m_tiles:
            return t, 0
        t -= m_tiles
        n_tiles -= 1
        nt0 = 1
    if along_n:
        per_group = group * m_tiles
        g, idx = divmod(t, per_group)
        return idx % m_tiles, nt0 + g * group + idx // m_tiles
    per_group = group * n_tiles
    g, idx = divmod(t, per_group)
    first_m = g * group
    gm = min(m_tiles - first_m, group)
    return first_m + idx % gm, nt0 + idx // gm


def raster(pair, m_bytes, n_bytes):
    """set_raster: (group, along_n)."""
    if m_bytes <= 64 * 1024 * 1024 and n_bytes > m_bytes:
        return 1, 1
    return (4 if pair else 8), 0


SHAPES = [  # M, d_in, d_out
    (16384, 4096, 4096), (16384, 4096, 1024), (8192, 14336, 4096), (4096, 1024, 4096),
    (3000, 512, 2000), (2048, 1024, 3072), (74 * 256, 256, 520), (18944, 4096, 1024),
    (1000, 4096, 4096), (300, 512, 768), (129, 256, 256), (100, 512, 520),
]


@pytest.mark.parametrize("M,d_in,d_out", SHAPES)
@pytest.mark.parametrize("sms", [148, 132])
def test_shared_t_schedule(M, d_in, d_out, sms):
    pair = M > 128
    m_tiles = -(-M // (256 if pair else 128))
    n_tiles = -(-d_out // 256)
    tiles = m_tiles * n_tiles
    units_max = sms // 2 if pair else sms
    share = tiles > units_max and m_tiles <= units_max       # the host's shared-T test
    units = min(tiles, units_max)
    group, along_n = raster(pair, 2.0 * M * d_in, 2.0 * d_out * d_in)
    seen = [tile_coords(t, m_tiles, n_tiles, group, along_n, share) for t in range(tiles)]
    assert sorted(seen) == sorted(itertools.product(range(m_tiles), range(n_tiles)))
    if not share:
        return
    for t, (mt, nt) in enumerate(seen):
        assert (t < m_tiles) == (nt == 0)
        if t < m_tiles:
            assert mt == t and t < units          # unit t's first tile
    ctas = 2 if pair else 1
    assert m_tiles * ctas * 4 <= 32 * K_TFLAG_WORDS
    assert K_TFLAG_WORD0 + 1 + K_TFLAG_WORDS <= K_HEADER_WORDS


def test_raster_groups_cover_ragged_last_group():
    # 10 row blocks in groups of 4: the last group holds 2 (gm < group)
    seen = [tile_coords(t, 10, 5, 4, 0, False) for t in range(50)]
    assert sorted(seen) == sorted(itertools.product(range(10), range(5)))
    seen = [tile_coords(t, 10, 5, 4, 0, True) for t in range(50)]
    assert sorted(seen) == sorted(itertools.product(range(10), range(5)))

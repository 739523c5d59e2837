"""Host replay of the fused MLP GEMM's schedule and global-memory indexing (gemm_swiglu_quant_kernel
and finalize_u_kernel in csrc/svdq_fused.cuh, host set-up in svdq_gemm_swiglu_quant): for the
GPU tests' shapes and full-size MLPs, at several resident-pair counts, every (row block, column
tile) is computed by exactly one CTA pair; every code, scale and partial-sum write stays inside its
buffer; the L1s' slice and h store coordinates are in range and 128-byte aligned; and every
partial row finalize reads was written. The offsets grow with the row and the column, so each
tile is checked at its first and last row and column."""
import pytest

MAX_SPLITS = 8


def act_sf_offset(m, kb, K):
    """Byte offset of the E4M3 scale of row m, 16-element block kb in the activation scale layout
    (as csrc/svdq_quant.cuh lays it out; also pinned on the GPU through svdq_export_act)."""
    return (((m >> 7) * (K >> 6) + (kb >> 2)) << 9) + ((m & 31) << 4) + (((m >> 5) & 3) << 2) + (kb & 3)


def replay(M, N, r2, max_pairs):
    M_pad = (M + 127) // 128 * 128
    m_tiles = M_pad // 128
    m_pairs = (m_tiles + 1) // 2
    n_tiles = N // 256
    K2 = N // 2
    splits = max(1, min(max_pairs // m_pairs, MAX_SPLITS, n_tiles))
    num_units = m_pairs * splits
    pairs = min(num_units, max_pairs)
    codes_bytes = M_pad * K2 // 2
    sf_bytes = (M_pad // 128) * (K2 // 64) * 512
    scratch_floats = MAX_SPLITS * M_pad * r2
    seen, written = set(), set()
    for pair in range(pairs):
        for unit in range(pair, num_units, pairs):
            m_pair, split = divmod(unit, splits)
            n_beg, n_end = split * n_tiles // splits, (split + 1) * n_tiles // splits
            assert n_end > n_beg
            for n_blk in range(n_beg, n_end):
                assert (m_pair, n_blk) not in seen
                seen.add((m_pair, n_blk))
                x = n_blk * 128                                  # slice / h-store column
                assert x % 64 == 0 and x + 128 <= K2
                for rank in (0, 1):
                    m_blk = 2 * m_pair + rank
                    for rl in (0, 127):
                        row = m_blk * 128 + rl
                        if row >= M_pad:                         # the odd CTA past the last block
                            continue
                        for k in (n_blk * 128, n_blk * 128 + 112):   # first and last 16-column block
                            off = row * (K2 // 2) + k // 2
                            assert 0 <= off and off + 8 <= codes_bytes
                            assert 0 <= act_sf_offset(row, k >> 4, K2) < sf_bytes
            for rank in (0, 1):
                for rl in range(128):
                    row = (2 * m_pair + rank) * 128 + rl
                    if row < M_pad:
                        assert (split * M_pad + row) * r2 + r2 <= scratch_floats
                        written.add((split, row))
    assert len(seen) == m_pairs * n_tiles
    assert all((sp, row) in written for sp in range(splits) for row in range(M_pad))
    return splits, num_units, pairs


@pytest.mark.parametrize("M,N,r2", [(300, 1024, 32), (1024, 6144, 32), (520, 2560, 16), (384, 2048, 64),
                                    (1, 512, 16), (4608, 24576, 32), (16896, 24576, 32), (33280, 24576, 64)])
@pytest.mark.parametrize("max_pairs", [74, 71, 64, 37, 9, 1])
def test_fused_schedule_and_indexing(M, N, r2, max_pairs):
    replay(M, N, r2, max_pairs)


def test_split_choice_fills_the_pairs():
    """At 74 resident pairs the 1024² MLP (M = 4608) splits each row block's 96 column tiles four
    ways: 72 units of 24 tiles; the 2048² one (M = 16896) needs no split."""
    assert replay(4608, 24576, 32, 74) == (4, 72, 72)
    assert replay(16896, 24576, 32, 74) == (1, 66, 66)

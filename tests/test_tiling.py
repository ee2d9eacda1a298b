"""Host-side check of the GEMM tile schedule (mirrors the kernel's tile decode, no GPU).

For the shapes the library runs, every output element of the symmetric
(Gram / polynomial) and plain (update) products must be written exactly once,
directly or by the mirror store; every TMA load must start at an x coordinate
that is a multiple of 64 elements (128 bytes); every store must stay inside
its [rows][pitch] buffer.
"""
import numpy as np
import pytest

BN = 256
KINDS = {"single": (128, 64)}  # (tile rows, column granularity)


def tiles_per_matrix(M, N, sym, kind="single"):
    BM = KINDS[kind][0]
    if sym:
        return sum((M - BM * mb + BN - 1) // BN for mb in range((M + BM - 1) // BM))
    return ((M + BM - 1) // BM) * ((N + BN - 1) // BN)


def decode(M, N, sym, r, kind="single"):
    BM, NG = KINDS[kind]
    if sym:
        mb = 0
        while True:
            cnt = (M - BM * mb + BN - 1) // BN
            if r < cnt:
                break
            r -= cnt
            mb += 1
        m0, n0 = BM * mb, BM * mb + BN * r
    else:
        tn = (N + BN - 1) // BN
        mb = r // tn
        m0, n0 = BM * mb, (r - mb * tn) * BN
    nw = min(BN, (N - n0 + NG - 1) // NG * NG)
    return m0, n0, nw


SHAPES = [(64, 96), (128, 128), (200, 328), (257, 700), (96, 1000), (37, 53), (768, 1536), (768, 3352),
          (2048, 4096), (2048, 8768), (8192, 8192), (1, 1), (130, 260)]


@pytest.mark.parametrize("kind", sorted(KINDS))
@pytest.mark.parametrize("m,n", SHAPES)
def test_symmetric_cover_exactly_once(m, n, kind):
    if m > 2048:
        pytest.skip("large")
    BM, NG = KINDS[kind]
    pitch = (m + 7) // 8 * 8
    hits = np.zeros((m, pitch), np.int32)
    for r in range(tiles_per_matrix(m, m, 1, kind)):
        m0, n0, nw = decode(m, m, 1, r, kind)
        assert n0 % 64 == 0 and nw % NG == 0 and NG <= nw <= 256 and n0 >= m0
        rows = np.arange(m0, min(m0 + BM, m))
        for c in range(0, nw, 32):
            j0 = n0 + c
            if j0 >= m:
                continue
            cols = np.arange(j0, min(j0 + 32, m))
            hits[np.ix_(rows, cols)] += 1
            if j0 >= m0 + BM:  # mirror store
                hits[np.ix_(cols, rows)] += 1
    assert np.all(hits[:, :m] == 1)
    assert np.all(hits[:, m:] == 0)


@pytest.mark.parametrize("kind", sorted(KINDS))
@pytest.mark.parametrize("m,n", SHAPES)
def test_update_cover_exactly_once(m, n, kind):
    if m * n > 2048 * 8768:
        pytest.skip("large")
    BM, NG = KINDS[kind]
    hits = np.zeros((m, n), np.int32)
    for r in range(tiles_per_matrix(m, n, 0, kind)):
        m0, n0, nw = decode(m, n, 0, r, kind)
        assert n0 % 64 == 0 and nw % NG == 0 and nw <= 256
        assert n0 + nw <= (n + NG - 1) // NG * NG
        rows = slice(m0, min(m0 + BM, m))
        hits[rows, n0:min(n0 + nw, n)] += 1
    assert np.all(hits == 1)


def test_reverse_walk_visits_every_matrix_once():
    L, tpm = 5, 7
    seen = []
    for local in range(L * tpm):
        lm, r = divmod(local, tpm)
        seen.append((L - 1 - lm, r))
    assert sorted(seen) == [(l, r) for l in range(L) for r in range(tpm)]
    assert seen[0][0] == L - 1 and seen[-1][0] == 0


@pytest.mark.parametrize("kind", sorted(KINDS))
@pytest.mark.parametrize("m,n", SHAPES)
def test_tma_coordinates_aligned(m, n, kind):
    for sym, N, K in ((1, m, n), (1, m, m), (0, n, m)):
        for r in range(min(tiles_per_matrix(m, N, sym, kind), 4000)):
            m0, n0, nw = decode(m, N, sym, r, kind)
            for kb in range((K + 63) // 64):
                assert (kb * 64 * 2) % 16 == 0  # A / K-major B: x = k
            for c in range(nw // 64):
                x = n0 + 64 * c
                assert (x * 2) % 16 == 0  # MN-major B: x = n
                assert nw % 64 == 0


@pytest.mark.parametrize("m,n", SHAPES)
def test_diagonal_tiles_have_a_inside_b(m, n):
    """Single-CTA symmetric problems: exactly the first tile of each 128-row block starts on the
    diagonal (n0 == m0), and its B box ({64, 256} or, for tiles <= 128 wide, {64, 128}) holds at
    least the 128 rows of the A tile, so the kernel may read A from the first rows of B."""
    BM = KINDS["single"][0]
    firsts = {}
    for r in range(tiles_per_matrix(m, m, 1, "single")):
        m0, n0, nw = decode(m, m, 1, r, "single")
        firsts.setdefault(m0, (n0, nw))
        if n0 == m0:
            assert firsts[m0] == (n0, nw)  # only the block's first tile
            box_rows = 256 if nw > 128 else 128
            assert box_rows >= BM
    assert sorted(firsts) == list(range(0, m, BM))
    assert all(n0 == m0 for m0, (n0, _) in firsts.items())

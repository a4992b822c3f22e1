"""Host restatement of the tiled NNLS factor's bookkeeping (heads whose factor
lives in the workspace): the tile layout, the order in which a solve streams
tiles, the in-place move of a deletion, the blocked solves with inverted
diagonal blocks, and the rule that decides when a cached block inverse is
still valid.  No GPU is involved; the CUDA kernels follow the same rules."""
import numpy as np
import pytest

KSB = 32
SLOT_TILES = 3


def tile_at(I, J):
    return (I * (I + 1) // 2 + J) * KSB * KSB


def tl(r, c):
    return tile_at(r // KSB, c // KSB) + (r % KSB) * KSB + (c % KSB)


def forward_steps(I0, n):
    """(I, J0, nt, diag) in the forward solve's order over rows [32·I0, n)."""
    out, I1 = [], (n - 1) // KSB
    I, J = I0, 0
    while I <= I1:
        diag = J >= I
        out.append((I, I if diag else J, 1 if diag else min(SLOT_TILES, I - J), diag))
        if J >= I:
            I, J = I + 1, 0
        else:
            J += SLOT_TILES
    return out


def backward_steps(n):
    out = []
    I, J = (n - 1) // KSB, -1
    while I >= 0:
        diag = J < 0
        out.append((I, I if diag else J, 1 if diag else min(SLOT_TILES, I - J), diag))
        J = 0 if J < 0 else J + SLOT_TILES
        if J >= I:
            I, J = I - 1, -1
    return out


@pytest.mark.parametrize("t", [1, 31, 32, 33, 100, 257, 1024])
def test_layout_is_a_bijection_with_contiguous_row_blocks(t):
    nb = (t + KSB - 1) // KSB
    pos = {tl(r, c) for r in range(t) for c in range(r + 1)}
    assert len(pos) == t * (t + 1) // 2                       # distinct slots
    assert max(pos) < tile_at(nb, 0)                          # inside the blocks' tiles
    for I in range(nb):                                       # off-diagonal tiles of a row block
        assert tile_at(I, I) - tile_at(I, 0) == I * KSB * KSB  # are one contiguous range
    # fits a t×t region (+1 for alignment) for every t >= 102, enumerated up to
    # 4096 (for t >= 114, nb(nb+1)·512 + 1 <= t²/2 + 48t + 1025 <= t²); 101 does not
    if t >= 102:
        assert tile_at(nb, 0) + 1 <= t * t
    assert all(tile_at((u + KSB - 1) // KSB, 0) + 1 <= u * u for u in range(102, 4097))
    assert tile_at(4, 0) + 1 > 101 * 101


@pytest.mark.parametrize("n", [1, 2, 31, 32, 33, 95, 96, 97, 200, 548])
def test_solves_stream_every_needed_tile_once_in_order(n):
    for I0 in sorted({0, (n - 1) // KSB // 2, (n - 1) // KSB}):
        seen, done_diag = [], set()
        for I, J0, nt, diag in forward_steps(I0, n):
            if diag:
                seen.append((I, I))
                done_diag.add(I)
            else:
                assert I not in done_diag                    # products before the block's diagonal
                assert all(j < I for j in range(J0, J0 + nt)) and nt <= SLOT_TILES
                seen += [(I, j) for j in range(J0, J0 + nt)]
        want = [(I, J) for I in range(I0, (n - 1) // KSB + 1) for J in range(I + 1)]
        assert sorted(seen) == sorted(want) and len(seen) == len(want)
    seen, solved = [], set()
    for I, J0, nt, diag in backward_steps(n):
        if diag:
            assert all(i in solved for i in range(I + 1, (n - 1) // KSB + 1))   # bottom up
            solved.add(I)
            seen.append((I, I))
        else:
            assert I in solved                               # the block's own values first
            seen += [(I, j) for j in range(J0, J0 + nt)]
    want = [(I, J) for I in range((n - 1) // KSB + 1) for J in range(I + 1)]
    assert sorted(seen) == sorted(want) and len(seen) == len(want)


@pytest.mark.parametrize("np_", [2, 33, 64, 97, 130])
def test_deletion_move_reads_every_source_before_it_is_overwritten(np_):
    """The move writes new (r, c) = old (r + 1, c + [c >= q]) over the new
    factor's tiles in storage order, two tiles per chunk, each chunk read
    before written: simulate it on a storage array and compare."""
    for q in sorted({0, 1, 31, 32, np_ // 2, np_ - 2, np_ - 1}):
        if q > np_ - 1:
            continue
        nb = (np_ + KSB - 1) // KSB
        mem = np.full(tile_at(nb, 0), np.nan)
        old = {}
        for r in range(np_):
            for c in range(r + 1):
                v = 1000.0 * r + c
                mem[tl(r, c)] = v
                old[(r, c)] = v
        nbn = (np_ - 1 + KSB - 1) // KSB
        tiles = [(I, J) for I in range(q // KSB, nbn) for J in range(I + 1)]
        for k in range(0, len(tiles), 2):
            chunk = tiles[k:k + 2]
            reads = []
            for (I, J) in chunk:
                for l in range(KSB * KSB):
                    r, c = KSB * I + l // KSB, KSB * J + l % KSB
                    if q <= r < np_ - 1 and c <= r:
                        src = tl(r + 1, c + (c >= q))
                        assert src > tile_at(I, J) + l                 # source after destination
                        reads.append((tile_at(I, J) + l, mem[src]))
            for dst, v in reads:
                mem[dst] = v
        for r in range(np_ - 1):
            for c in range(r + 1):
                orow, ocol = r + (r >= q), c + (c >= q)
                assert mem[tl(r, c)] == old[(orow, ocol)]


def _blocked_solves(L, b, Dinv):
    n = len(b)
    y = b.copy()
    for r0 in range(0, n, KSB):
        r1 = min(n, r0 + KSB)
        y[r0:r1] = Dinv[r0 // KSB][:r1 - r0, :r1 - r0] @ (y[r0:r1] - L[r0:r1, :r0] @ y[:r0])
    x = y.copy()
    for r0 in reversed(range(0, n, KSB)):
        r1 = min(n, r0 + KSB)
        x[r0:r1] = Dinv[r0 // KSB][:r1 - r0, :r1 - r0].T @ x[r0:r1]
        x[:r0] -= L[r0:r1, :r0].T @ x[r0:r1]
    return y, x


def _inverse_by_columns(S, d):
    """The kernel's block inverse: column c by substitution, each finished
    entry's terms added to every later row's sum."""
    X = np.zeros((KSB, KSB))
    for c in range(KSB):
        a = np.zeros(KSB)
        for m in range(c, KSB):
            a[m] = d[m] if m == c else -a[m] * d[m]
            a[m + 1:] += S[m + 1:, m] * a[m]
        X[:, c] = a
    return X


def test_blocked_solves_with_inverted_diagonal_blocks_match_substitution():
    rng = np.random.default_rng(7)
    for n in (1, 32, 45, 100):
        A = rng.standard_normal((n + 20, n))
        G = A.T @ A
        L = np.linalg.cholesky(G)
        b = rng.standard_normal(n)
        Lpad = np.zeros((n + KSB, n + KSB))
        Lpad[:n, :n] = L
        Lpad[n:, :] = 7.0                                     # rows past n: whatever was there
        dpad = np.ones(n + KSB)
        dpad[:n] = 1.0 / np.diag(L)
        Dinv = [_inverse_by_columns(Lpad[r0:r0 + KSB, r0:r0 + KSB], dpad[r0:r0 + KSB]) for r0 in range(0, n, KSB)]
        y, x = _blocked_solves(L, b, Dinv)
        assert np.allclose(y, np.linalg.solve(L, b), rtol=1e-10, atol=1e-12)
        assert np.allclose(x, np.linalg.solve(G, b), rtol=1e-8, atol=1e-10)


def test_cached_inverse_validity_rule():
    """Leading row blocks stay valid until an append lands in them (the block
    holding row np) or a deletion reaches them (every block from the deleted
    position down); a solve over [32·I0, n) revalidates through its last block
    when it starts at or below the valid prefix.  Over a random sequence of
    appends, deletions and solves, every block the rule calls valid holds the
    inverse of the factor's current diagonal block."""
    rng = np.random.default_rng(11)
    tmax = 300
    A = rng.standard_normal((400, tmax))
    order = list(rng.permutation(tmax))
    P, cache, dvalid = [], {}, 0

    def factor():
        return np.linalg.cholesky(A[:, P].T @ A[:, P]) if P else np.zeros((0, 0))

    def solve(I0):
        nonlocal dvalid
        L = factor()
        n = len(P)
        for I in range(I0, (n - 1) // KSB + 1):
            r0 = KSB * I
            blk = L[r0:r0 + KSB, r0:r0 + KSB]
            if I >= dvalid:
                cache[I] = np.linalg.inv(blk)
            assert np.allclose(cache[I], np.linalg.inv(blk), rtol=1e-8, atol=1e-8), (I, dvalid)
        if dvalid >= I0:
            dvalid = max(dvalid, (n - 1) // KSB + 1)

    for step in range(120):
        if order and (not P or rng.random() < 0.7):
            k = min(int(rng.integers(1, 9)), len(order))
            np_old = len(P)
            solve(0)                                          # the append's forward solve
            P += [order.pop() for _ in range(k)]
            dvalid = min(dvalid, np_old // KSB)               # the block holding row np changed
        elif len(P) > 1:
            q = int(rng.integers(0, len(P)))
            order.append(P.pop(q))
            dvalid = min(dvalid, q // KSB)                    # every block from q down changed
        if P:
            solve(int(rng.integers(0, (len(P) - 1) // KSB + 1)))   # forward extension
            solve(0)                                          # backward solve: all blocks

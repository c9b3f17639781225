"""CPU model of the bf16 score kernel's exact top-K selection (no GPU).

hyper.ai summary of arXiv 2607.02980 (HiLS-Attention), section 方法 (Method),
third practical design choice: the K chunks with the largest group score (the
maximum over the GQA group's heads of s^) among the complete chunks before the
chunk-aligned window.  Among equal group scores the smaller chunk is taken
(the oracle's rule, pinned in test_oracle_pins.py).

The kernel reaches that set in two passes over tiles of 64 chunks, each tile
split into two 32-chunk halves held by the two threads of a row:

- pass 1: each half keeps its KT >= K largest scores, sorted.  Candidates
  above the list's current KT-th value (a threshold that only rises and is
  read stale between merges) go to a buffer, merged into the list 32 at a
  time; the warp may merge earlier than a row needs, because another lane's
  buffer filled.  The row threshold is tau = min_{j<K} max(a_j, b_{K-1-j})
  over the halves' lists a and b, and A = the number of scores above tau.
- pass 2: in ascending chunk order (half 0 of a tile before half 1), every
  chunk above tau and the first K - A chunks equal to tau.

These tests run those steps in numpy, with the merge schedule randomised, and
check the result against the oracle's selection on inputs whose scores are
exact (k' = 0, so s^ = b'), with many ties, no ties, and orders that make
every candidate beat the running threshold."""
import numpy as np
import pytest

import oracle

S, TCH, HALF = 64, 64, 32


def kernel_selection(g, ncand, K, KT, extra_tiles, rng):
    """Chosen chunks (ascending) of one row with group scores g[:ncand]."""
    T = (ncand + TCH - 1) // TCH + extra_tiles  # a CTA's tile count follows its last row
    lists = [np.full(KT, -np.inf, np.float32) for _ in range(2)]
    bufs = [[], []]
    for t in range(T):
        for hf in range(2):
            c0 = t * TCH + hf * HALF
            thr = lists[hf][KT - 1]
            bufs[hf] += [g[c] for c in range(c0, min(c0 + HALF, ncand)) if g[c] > thr]
        flush = t == T - 1
        for hf in range(2):
            # a full buffer forces a merge; another lane of the warp may force one at any time
            while bufs[hf] and (len(bufs[hf]) >= HALF or flush or rng.random() < 0.3):
                blk, bufs[hf] = bufs[hf][:HALF], bufs[hf][HALF:]
                lists[hf] = np.sort(np.concatenate([lists[hf], np.array(blk, np.float32)]))[::-1][:KT]
    a, b = lists
    tau = min(max(a[j], b[K - 1 - j]) for j in range(K))
    t_rem = max(0, K - int((a > tau).sum() + (b > tau).sum()))
    chosen = []
    for t in range(T):
        for hf in range(2):
            for c in range(t * TCH + hf * HALF, min(t * TCH + hf * HALF + HALF, ncand)):
                if g[c] > tau:
                    chosen.append(c)
                elif g[c] == tau and t_rem > 0:
                    chosen.append(c)
                    t_rem -= 1
    return chosen


def _b_sum(kind, Hq, C, rng):
    if kind == "ties":  # whole numbers 0..3: most group scores tie
        return rng.integers(0, 4, (1, Hq, C)).astype(np.float32)
    if kind == "distinct":
        return rng.standard_normal((1, Hq, C)).astype(np.float32)
    if kind == "rising":  # every candidate beats all earlier ones: the buffer fills on every tile
        return np.broadcast_to(np.arange(C, dtype=np.float32) * 0.25, (1, Hq, C)).copy()
    if kind == "constant":  # all candidates tie: the first K chunks
        return np.full((1, Hq, C), 1.5, np.float32)
    raise ValueError(kind)


@pytest.mark.parametrize("K,KT", [(8, 16), (32, 32), (48, 64)])
@pytest.mark.parametrize("kind", ["ties", "distinct", "rising", "constant"])
def test_kernel_selection_model_matches_oracle(K, KT, kind):
    Hq, Hkv, W, N = 8, 2, 128, 64 * 200 + 17
    G, C, nw = Hq // Hkv, N // S, W // S
    rng = np.random.default_rng(K * 7 + len(kind))
    b_sum = _b_sum(kind, Hq, C, rng)
    q = rng.standard_normal((1, Hq, N, 128)).astype(np.float32)
    dm = oracle.Dims(B=1, Hq=Hq, Hkv=Hkv, N=N, d=128, S=S, W=W, K=K)
    pos = sorted({0, W + S, K * S + W, N - 1, N - 2} | set(rng.integers(0, N, 120).tolist()))
    rows = [(0, p) for p in pos]
    idx_o, _ = oracle.select(dm, rows, q, k_sum=np.zeros((1, Hq, C, 128)), b_sum=b_sum.astype(np.float64))
    for r, (_, i) in enumerate(rows):
        ncand = max(0, i // S - nw + 1)
        for grp in range(Hkv):
            g = b_sum[0, grp * G:(grp + 1) * G, :].max(axis=0)
            got = kernel_selection(g, ncand, K, KT, extra_tiles=int(rng.integers(0, 3)), rng=rng)
            want = [c for c in idx_o[r, grp].tolist() if c >= 0]
            assert got == want, (kind, i, grp)


def test_tau_formula_is_the_kth_largest_of_the_union():
    """min_{j<K} max(a_j, b_{K-1-j}) over two descending lists equals the K-th
    largest element of their union (the two lists each hold at least K values)."""
    rng = np.random.default_rng(3)
    for _ in range(500):
        K = int(rng.integers(1, 65))
        a = np.sort(rng.integers(-5, 6, K + int(rng.integers(0, 5))).astype(np.float64))[::-1]
        b = np.sort(rng.integers(-5, 6, K + int(rng.integers(0, 5))).astype(np.float64))[::-1]
        tau = min(max(a[j], b[K - 1 - j]) for j in range(K))
        assert tau == np.sort(np.concatenate([a, b]))[::-1][K - 1]

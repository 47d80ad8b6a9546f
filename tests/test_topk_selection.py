"""The candidate floor of the top-k-truncated sampler, checked on a CPU model
of its selection (no GPU; no oracle code: the reference is a brute-force sort).

The kernel splits each row of V logits into NC contiguous slices, one CTA
(256 threads) each; thread t of a CTA sees the float4 groups t, t + 256, ...
of its slice.  A CTA's floor is the K-th largest of its 256 per-thread maxima;
the row's floor F is the largest CTA floor; only values >= F are buffered.
When every buffer and their total fit 2048 entries, rank 0 sorts all of them
once; otherwise each CTA keeps its K best (from its buffer, or from its whole
slice when even that overflowed) and rank 0 merges.  The claim: the K best
that come out, in (value descending, index ascending) order, are exactly the
row's K best in that order, for every row kind and cluster size."""
import numpy as np
import pytest

from block_text_diffusion_b200 import inputs as I

THREADS, CAP = 256, 2048


def brute_topk(row, K):
    return np.lexsort((np.arange(row.size), -row.astype(np.float64)))[:K]


def order(vals, idx):
    return np.lexsort((idx, -vals.astype(np.float64)))


def kernel_selection(row, K, NC):
    V = row.size
    n4 = V // (4 * NC)
    floors, bufs = [], []
    for r in range(NC):
        sl = row[r * n4 * 4:(r + 1) * n4 * 4]
        groups = sl.reshape(n4, 4)
        tmax = np.full(THREADS, -np.inf, dtype=np.float32)
        for t in range(min(THREADS, n4)):
            tmax[t] = groups[t::THREADS].max()
        floors.append(tmax[order(tmax, np.arange(THREADS))[K - 1]])
    F = max(floors)
    for r in range(NC):
        sl = row[r * n4 * 4:(r + 1) * n4 * 4]
        sel = np.nonzero(sl >= F)[0]
        bufs.append((sl[sel], sel + r * n4 * 4, sl))
    counts = [b[0].size for b in bufs]
    if all(c <= CAP for c in counts) and sum(counts) <= CAP:
        v = np.concatenate([b[0] for b in bufs])
        i = np.concatenate([b[1] for b in bufs])
    else:
        vs, is_ = [], []
        for r, (bv, bi, sl) in enumerate(bufs):
            if bv.size > CAP:                      # the CTA's own K best from its whole slice
                o = order(sl, np.arange(sl.size))[:K]
                bv, bi = sl[o], o + r * n4 * 4
            o = order(bv, bi)[:K]
            vs.append(bv[o])
            is_.append(bi[o])
        v, i = np.concatenate(vs), np.concatenate(is_)
    return i[order(v, i)[:K]]


@pytest.mark.parametrize("NC", [1, 2, 8])
@pytest.mark.parametrize("V,rows,kind,scale,K", [
    (1024, 8, "normal", 1.0, 256),
    (1024, 8, "mixed", 3.0, 64),
    (32768, 4, "peaked", 1.0, 64),
    (32768, 4, "ties", 1.0, 200),     # many equal logits across the K-th place
    (32768, 2, "flat", 1.0, 32),      # every logit equal: the K lowest indices
    (32768, 4, "normal", 1.0, 64),
    (4096, 4, "normal", 1.0, 1),
])
def test_candidate_floor_keeps_exactly_the_k_best(NC, V, rows, kind, scale, K):
    l = I.logits(V + rows + K, rows, V, kind, scale)
    for r in range(rows):
        assert np.array_equal(kernel_selection(l[r], K, NC), brute_topk(l[r], K)), (kind, r)

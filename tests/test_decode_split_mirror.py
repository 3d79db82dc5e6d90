"""CPU mirror of the W4A16 decode kernel's work split (the index arithmetic of
w4a16_kernel, restated in Python): clusters of two CTAs own contiguous runs of
whole 32-row tiles, each CTA and each of its 8 warps an even share of the
run's 128-wide k-group units.  Over many shapes and grid sizes every output
tile must be written exactly once -- by the warp that covered it whole, by the
CTA that summed its warps' partials, or by rank 1 after rank 0's partial has
been pushed to it -- and the push and the receive must pair up."""
import pytest

CS, W, SG = 2, 8, 2


def split_at(length, i, log2p):
    return (length * i) >> log2p


def producers(ntiles, G, nclu):
    out = {}
    tq, tr = divmod(ntiles, nclu)
    for cid in range(nclu):
        A = (tq * cid + tr * cid // nclu) * G
        L = (tq * (cid + 1) + tr * (cid + 1) // nclu) * G - A
        pushed, received = [], []
        for rank in range(CS):
            F0, F1 = A + split_at(L, rank, 1), A + split_at(L, rank + 1, 1)
            FL = F1 - F0
            for warp in range(W):                        # the warp's own pass over its units
                f0, f1 = F0 + split_at(FL, warp, 3), F0 + split_at(FL, warp + 1, 3)
                if f1 <= f0:
                    continue
                wt_first, g_first = divmod(f0, G)
                nt, g, left = wt_first, g_first, f1 - f0
                while left > 0:
                    n = min(left, SG, G - g)             # a stage never straddles a tile
                    g, left = g + n, left - n
                    if g == G:
                        if not (nt == wt_first and g_first != 0):
                            out.setdefault(nt, []).append(("warp", cid, rank, warp))
                        g, nt = 0, nt + 1
            if FL == 0:
                continue
            for tt in range(F0 // G, (F1 - 1) // G + 1):  # the CTA's reduction of partial tiles
                tb, te = tt * G, tt * G + G
                takers = [w2 for w2 in range(W)
                          if (lambda a, b: a < b and a < te and b > tb and not (a <= tb and b >= te))(
                              F0 + split_at(FL, w2, 3), F0 + split_at(FL, w2 + 1, 3))]
                if tb >= F0 and te <= F1:
                    if takers:
                        out.setdefault(tt, []).append(("cta", cid, rank))
                elif te > F1:
                    assert rank == 0 and takers
                    pushed.append(tt)
                else:
                    assert rank == 1 and tb < F0
                    received.append(tt)
                    out.setdefault(tt, []).append(("rank1", cid))
        assert pushed == received and len(pushed) <= 1
    return out


@pytest.mark.parametrize("G", [1, 2, 3, 5, 32, 96, 200])
def test_every_tile_written_once(G):
    for ntiles in list(range(1, 24)) + [96, 128, 192, 768, 1600]:
        for nclu in (1, 2, 3, 7, 74, 148):
            if nclu > ntiles:
                continue
            got = producers(ntiles, G, nclu)
            assert sorted(got) == list(range(ntiles))
            assert all(len(v) == 1 for v in got.values()), (ntiles, G, nclu)

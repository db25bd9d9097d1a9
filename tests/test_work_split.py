"""Host-side restatement of the register GEMV's two work splits, checked for coverage and for a
deterministic single reduction of every shared tile (no GPU; the CUDA kernel implements the same
arithmetic in gemv_reg_kernel):
  * CTA-local: CTA c owns tiles [c*T/G, (c+1)*T/G); its NW warps cut the CTA's (tile, window) units
    into runs of ceil(units/NW); a run's first and last tile, when shared, get one partial slot each
    (first / last), and the tile's first contributor sums the contributors' slots in warp order.
  * stream-K: runs of `run` units dealt as run i -> CTA i % G, warp i / G; the runs touching a tile
    are consecutive, one slot per (slice, rank)."""
import itertools

import pytest


def local_split(tiles, nwin, grid, nw):
    covered, slots, owners = {}, {}, {}
    for c in range(grid):
        t_lo, t_hi = c * tiles // grid, (c + 1) * tiles // grid
        ucta = (t_hi - t_lo) * nwin
        lrun = max(1, -(-ucta // nw))
        lbase = t_lo * nwin
        for w in range(nw):
            u0, u1 = lbase + min(w * lrun, ucta), lbase + min(w * lrun + lrun, ucta)
            if u0 == u1:
                continue
            tile0 = u0 // nwin
            for u in range(u0, u1):
                covered[u] = covered.get(u, 0) + 1
            for t in range(tile0, (u1 - 1) // nwin + 1):
                rel0 = t * nwin - lbase
                contributors = (rel0 + nwin - 1) // lrun - rel0 // lrun + 1
                if contributors > 1:
                    slot = (c, w, 0 if t == tile0 else 1)
                    assert slot not in slots, "two tiles share one partial slot"
                    slots[slot] = t
        for t in range(t_lo, t_hi):
            rel0 = t * nwin - lbase
            first, last = rel0 // lrun, (rel0 + nwin - 1) // lrun
            if last > first:
                owners[t] = owners.get(t, 0) + 1
                for w in range(first, last + 1):  # the owner reads warp w's slot for tile t
                    tw0 = (lbase + w * lrun) // nwin
                    assert slots[(c, w, 0 if t == tw0 else 1)] == t
    return covered, slots, owners


@pytest.mark.parametrize("tiles,nwin,grid,nw", [(128, 16, 128, 16), (768, 13, 296, 8), (768, 16, 296, 8),
                                                (128, 48, 128, 16), (128, 39, 128, 16), (5, 7, 5, 16),
                                                (1088, 20, 296, 8), (4748, 13, 296, 8), (10, 1, 10, 16)])
def test_local_split_covers_every_unit_once_and_reduces_each_shared_tile_once(tiles, nwin, grid, nw):
    covered, slots, owners = local_split(tiles, nwin, grid, nw)
    assert sorted(covered) == list(range(tiles * nwin)) and set(covered.values()) == {1}
    shared = set(slots.values())
    assert set(owners) == shared and set(owners.values()) <= {1}


def stream_k_runs(tiles, nwin, grid, nw, run):
    units = tiles * nwin
    runs = []
    for wi in range(grid * nw):
        u0 = min(wi * run, units)
        u1 = min(u0 + run, units)
        if u0 < u1:
            runs.append((wi, u0, u1))
    return runs


@pytest.mark.parametrize("tiles,nwin,grid,nw,run", [(160, 68, 148, 16, 5), (32, 136, 148, 16, 2), (7, 5, 3, 16, 1)])
def test_stream_k_runs_cover_units_and_ranks_are_consecutive(tiles, nwin, grid, nw, run):
    runs = stream_k_runs(tiles, nwin, grid, nw, run)
    covered = list(itertools.chain.from_iterable(range(u0, u1) for _, u0, u1 in runs))
    assert covered == list(range(tiles * nwin))
    for t in range(tiles):
        touching = [wi for wi, u0, u1 in runs if u0 < (t + 1) * nwin and u1 > t * nwin]
        # the kernel's rank of run wi among tile t's runs is wi - (t * nwin) // run: 0, 1, 2, ...
        assert [wi - (t * nwin) // run for wi in touching] == list(range(len(touching)))
        # and the count matches the kernel's contributor formula
        assert len(touching) == ((t * nwin + nwin - 1) // run - (t * nwin) // run + 1)

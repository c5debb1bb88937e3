"""The token phase's CTA-pair tile schedule (host logic of the library, no GPU).

The pair kernel computes, per tile of 256 chunk tokens x 128 hidden units, the forward and
backprop through the fast weights (LaCT analysis, "Nonlinear memory complements local
attention").  Whatever form the launch picks -- weight blocks streamed with every operand
stage, or resident in shared memory for a range of token tiles -- every (head, token tile,
hidden block) tile must be computed exactly once.  ttt_pair_schedule runs the same host code
the launch uses (form and grid choice, and each pair's tile sequence) on given device
capacities.
"""
import itertools

import pytest

from weight_sequence_mixing_b200 import binding


def _check_cover(m_tiles, n_tiles, batches, tiles):
    want = {(z, mt, nt) for z in range(batches) for mt in range(m_tiles) for nt in range(n_tiles)}
    assert len(tiles) == len(want)
    assert set(tiles) == want


GEOMS = list(itertools.product([1, 2, 5, 19, 40], [1, 2, 4, 8], [1, 3, 8], [1, 4, 8], [74, 9, 2]))


@pytest.mark.parametrize("m_tiles,n_tiles,batches,kblocks,cap", GEOMS)
def test_every_tile_once(m_tiles, n_tiles, batches, kblocks, cap):
    resident, pairs, counts, tiles = binding.pair_schedule(m_tiles, n_tiles, batches, kblocks, cap, cap)
    _check_cover(m_tiles, n_tiles, batches, tiles)
    assert sum(counts) == len(tiles) and len(counts) == pairs
    U = m_tiles * batches
    groups = cap // n_tiles
    if resident:
        # d <= 256, a full wave of groups of n_tiles pairs, each pair at least four token tiles
        assert kblocks <= 4 and groups > 0 and U >= 4 * groups and pairs == groups * n_tiles
        assert min(counts) >= 4
        k = 0
        per_pair = []
        for p in range(pairs):
            seq = tiles[k:k + counts[p]]
            k += counts[p]
            # one hidden block per pair, consecutive (head, token tile) positions
            assert {nt for _, _, nt in seq} == {p % n_tiles}
            u = [z * m_tiles + mt for z, mt, _ in seq]
            assert u == list(range(u[0], u[0] + len(u)))
            per_pair.append(u)
        # the pairs of a group walk the same token tiles (each key/value tile crosses HBM once)
        for g in range(groups):
            assert all(per_pair[g * n_tiles + i] == per_pair[g * n_tiles] for i in range(n_tiles))
    else:
        assert not (kblocks <= 4 and groups > 0 and U >= 4 * groups)
        total = m_tiles * n_tiles * batches
        assert pairs == min(total, cap)
        # tile k of pair p is p + k * pairs of the (head, token tile, hidden block) order
        k = 0
        for p in range(pairs):
            for i in range(counts[p]):
                t = p + i * pairs
                assert tiles[k] == (t // (n_tiles * m_tiles), (t // n_tiles) % m_tiles, t % n_tiles)
                k += 1


def test_workload_forms():
    # the million-token scene layer: 512 pair tiles of tokens per chunk and head, h 512, d 256
    resident, pairs, counts, _ = binding.pair_schedule(512, 4, 4, 4, 74, 74)
    assert resident and pairs == 72 and set(counts) == {113, 114}
    # the causal language layer's 2048-token chunks: one or two tiles per pair, streaming
    resident, pairs, _, _ = binding.pair_schedule(8, 2, 8, 4, 74, 74)
    assert not resident and pairs == 74
    # the novel-view layer (d 512): weight blocks too large to keep, streaming
    resident, pairs, _, _ = binding.pair_schedule(128, 8, 2, 8, 74, 74)
    assert not resident and pairs == 74


def test_capacity_edges():
    # no resident pair fits: streaming; a hidden-block group wider than the resident capacity: streaming
    assert binding.pair_schedule(512, 4, 4, 4, 0, 74)[0] is False
    assert binding.pair_schedule(512, 4, 4, 4, 3, 74)[0] is False
    # no pair of either form fits
    with pytest.raises(binding.TTTError):
        binding.pair_schedule(512, 4, 4, 4, 0, 0)
    lib = binding.LIB
    import ctypes
    r, p = ctypes.c_int(), ctypes.c_int()
    counts = (ctypes.c_int * 74)()
    tiles = (ctypes.c_int * 3)()
    inv = binding.TTT_ERR_INVALID_ARG
    # too small a tile buffer, bad geometry
    assert lib.ttt_pair_schedule(4, 2, 1, 4, 74, 74, ctypes.byref(r), ctypes.byref(p), counts, tiles, 1) == inv
    assert lib.ttt_pair_schedule(0, 2, 1, 4, 74, 74, ctypes.byref(r), ctypes.byref(p), counts, tiles, 1) == inv
    assert lib.ttt_pair_schedule(4, 2, 1, 0, 74, 74, ctypes.byref(r), ctypes.byref(p), counts, tiles, 1) == inv

"""Host-side model of the int4 / int8 GEMM's W ring hand-off (sq_gemm.cu, "W ring").

Each cluster c takes the tiles c, c + C, c + 2C, ... (tile = mt + m_tiles * nt).  Its writers
walk those tiles in order.  For tile (mt, nt) they wait until ring_done[nt % R] >= (nt // R) *
m_tiles, then both CTAs add their share to ring_ready[nt % R].  Its consumer (producer, MMA,
epilogue) walks the same tiles in order.  It waits until ring_ready[nt % R] >= (nt // R + 1) * 2
* m_tiles, reads the slot, and adds 1 to ring_done[nt % R] when the tile's MMAs are done.

The counters only grow and every wait is a threshold on one of them, so a process that can move
can still move after any other step.  Hence one schedule that always moves some process settles
whether the system can stall.  The model checks three things: every process finishes, no writer
overwrites a slot that a consumer of its previous tile has not finished, and every consumer
reads a slot holding all shares of its own tile and none of the next one.
"""
import math

import pytest


def ring_slots(M, N, pairs=74):
    """The slot count the library sizes its workspace with (sq_api.cu)."""
    m_tiles, n_tiles = math.ceil(M / 256), math.ceil(N / 256)
    return min(n_tiles, math.ceil(pairs / m_tiles) + 2)


def run_ring(m_tiles, n_tiles, clusters, R, shares_waited=2):
    tiles = m_tiles * n_tiles
    own = [list(range(c, tiles, clusters)) for c in range(min(clusters, tiles))]
    ready = [0] * R
    done = [0] * R
    wpos = [0] * len(own)                     # next tile index of each cluster's writers
    cpos = [0] * len(own)                     # next tile index of each cluster's consumer
    slot_tile = [None] * R                    # W tile whose shares the slot currently holds
    shares = [0] * R                          # shares of slot_tile written so far
    readers = [set() for _ in range(R)]       # (cluster, tile) reading the slot's current tile
    steps = 0
    while True:
        moved = False
        for c in range(len(own)):
            # writers of cluster c: one share per tile (both CTAs), in tile order
            if wpos[c] < len(own[c]):
                t = own[c][wpos[c]]
                nt = t // m_tiles
                s = nt % R
                if done[s] >= (nt // R) * m_tiles:
                    if slot_tile[s] != nt:
                        assert not readers[s], f"slot {s} overwritten while tile {slot_tile[s]} is read"
                        assert slot_tile[s] is None or slot_tile[s] == nt - R, "slot skipped a tile"
                        slot_tile[s], shares[s] = nt, 0
                    shares[s] += 2
                    ready[s] += 2
                    wpos[c] += 1
                    moved = True
            # consumer of cluster c: read the slot, then count the tile as done
            if cpos[c] < len(own[c]):
                t = own[c][cpos[c]]
                nt = t // m_tiles
                s = nt % R
                if (c, t) in readers[s]:
                    readers[s].discard((c, t))
                    done[s] += 1
                    cpos[c] += 1
                    moved = True
                elif ready[s] >= (nt // R + 1) * shares_waited * m_tiles:
                    assert slot_tile[s] == nt and shares[s] == 2 * m_tiles, \
                        f"tile {nt} read from slot {s} holding tile {slot_tile[s]} with {shares[s]} shares"
                    readers[s].add((c, t))
                    moved = True
            steps += 1
        if all(wpos[c] == len(own[c]) and cpos[c] == len(own[c]) for c in range(len(own))):
            return steps
        assert moved, (f"stall: m_tiles={m_tiles} n_tiles={n_tiles} clusters={clusters} R={R} "
                       f"writers at {wpos}, consumers at {cpos}")


@pytest.mark.parametrize("m_tiles", [1, 2, 6, 18, 35])
@pytest.mark.parametrize("n_tiles", [1, 3, 16, 64])
@pytest.mark.parametrize("clusters", [1, 5, 74])
def test_ring_finishes_for_any_slot_count(m_tiles, n_tiles, clusters):
    for R in sorted({1, 2, 3, 7, n_tiles, ring_slots(256 * m_tiles, 256 * n_tiles)}):
        if R <= n_tiles:
            run_ring(m_tiles, n_tiles, clusters, R)


def test_ring_slots_matches_the_documented_shapes():
    assert ring_slots(4480, 16384) == 7       # the bench shape: 18 M tiles, 64 W tiles
    assert ring_slots(1536, 9216) == 15       # 6 M tiles, 36 W tiles
    assert ring_slots(1536, 3072) == 12       # all 12 W tiles
    assert ring_slots(64, 16384) == 64        # one M tile: every W tile in flight
    assert ring_slots(2560, 4096) == 10       # the GPU tests' slot-reuse shape: 10 slots, 16 W tiles


def test_model_detects_a_broken_wait():
    """A consumer that waited for only one CTA's share per cluster (half the count) could read a
    slot whose tile is half written; the model must catch that."""
    with pytest.raises(AssertionError, match="shares"):
        run_ring(6, 16, 74, 10, shares_waited=1)

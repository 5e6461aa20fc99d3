"""The dense kernel's barrier protocol, run as a host model (tests/dense_protocol.py).

Each case is one CTA pair's list of tiles, given by the KV blocks of its two
256-row sub-tiles (0 = no rows or no visible key), run in many random
interleavings of the roles and of the asynchronous work.
"""
import random

import pytest

import dense_protocol as dp

CASES = {
    # a tile whose second sub-tile has no rows, then the end of the list
    "rows_in_one_sub_tile": [(1, 0)],
    # a tile without any visible key (a sequence with no keys)
    "no_keys": [(0, 0)],
    "no_keys_between": [(0, 0), (2, 3), (0, 0), (0, 0), (1, 0), (0, 1)],
    # causal tiles: the second sub-tile sees two more blocks than the first
    "causal_run": [(1, 2), (3, 4), (5, 6), (7, 8)],
    # more tiles than the hand-off ring has slots, short and long mixed
    "long_list": [(3, 5), (0, 0), (1, 2), (4, 4), (0, 1), (2, 2), (0, 0), (6, 8), (1, 0),
                  (2, 0), (9, 9), (1, 1)],
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_protocol_holds_in_random_interleavings(name):
    tiles = CASES[name]
    for seed in range(150):
        dp.run_case(tiles, seed)


def test_protocol_holds_on_random_tile_lists():
    rng = random.Random(7)
    for seed in range(200):
        tiles = [(rng.choice([0, 0, 1, 2, 3, 5]), rng.choice([0, 1, 2, 4, 6]))
                 for _ in range(rng.randint(1, 10))]
        dp.run_case(tiles, seed)


def test_model_catches_a_producer_overtaken_on_q_empty():
    """With q_full counting only the leader's producer (the protocol before
    it counted both), a tile without visible keys lets the MMA warp finish
    with Q and commit q_empty before the peer's producer has checked the
    previous phase; the peer then waits on a parity that names the next
    phase (on the GPU: a wait that never ends)."""
    caught = 0
    for seed in range(200):
        try:
            dp.run_case([(0, 0)], seed, q_full_both=False)
        except dp.ProtocolError as e:
            assert "producer@1" in str(e) and "q_empty" in str(e), e
            caught += 1
    assert caught > 0


def test_model_catches_an_early_next_tile_read():
    """The MMA warp must not wait for the next tile's coordinates before it
    has consumed this tile's K/V blocks: the producer publishes the next
    tile only after issuing this one's loads, and with more blocks than K/V
    slots those loads wait for the MMA warp."""
    with pytest.raises(dp.ProtocolError, match="deadlock"):
        dp.run_case([(5, 6), (1, 1)], 0, early_fetch=True)


def test_protocol_holds_with_two_kv_slots():
    """The 256-wide qk geometry keeps two K/V slots instead of three."""
    rng = random.Random(11)
    for seed in range(150):
        tiles = [(rng.choice([0, 1, 2, 3, 5]), rng.choice([0, 1, 2, 4, 6]))
                 for _ in range(rng.randint(1, 8))]
        dp.run_case(tiles, seed, slots=2)

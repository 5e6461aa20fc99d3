"""The sparse kernel's barrier protocol, run as a host model (tests/sparse_protocol.py).

Each case is one CTA's chunk count, run in many random interleavings of the
roles, of the landing of the gathered rows and of the MMA pipe, with random
rows rescaling O.
"""
import pytest

import sparse_protocol as spp


@pytest.mark.parametrize("nchunks", [0, 1, 2, 3, 4, 7, 12, 32])
def test_protocol_holds_in_random_interleavings(nchunks):
    for seed in range(120):
        spp.run_case(nchunks, seed)


def test_protocol_holds_with_every_row_rescaling():
    for seed in range(60):
        spp.run_case(6, seed, rescale_rate=1.0)


def _fails(**kw) -> bool:
    for seed in range(300):
        try:
            spp.run_case(8, seed, **kw)
        except spp.ProtocolError:
            return True
    return False


def test_model_catches_a_rescale_after_the_wrong_pv():
    assert _fails(stale_pv_wait=True, rescale_rate=0.3)


def test_model_catches_a_slot_freed_before_its_values_are_read():
    assert _fails(free_after_s=True)

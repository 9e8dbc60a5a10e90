"""The prefill kernel's barrier protocol (paired K/V ring stages), run as a CPU model: no deadlock and
no buffer hazard over random interleavings of its roles, dense and block-sparse, for the ring depth
the kernel uses and others; planted protocol slips are caught."""
from tests import prefill_protocol_model as m


def test_protocol_model_clean():
    assert m.check(trials=12) is None


def test_protocol_model_catches_slips():
    caught = m.mutation_check(trials=12)
    missed = [k for k, v in caught.items() if not v]
    assert not missed, f"planted slips not caught: {missed}"


def test_protocol_model_finds_the_one_stage_deadlock():
    """With a single stage the next tile's S waits for a stage that only its own tile's P.V would
    release: the model must report that deadlock (a check that it can find one)."""
    r = m.check(trials=2, rings=[1], geoms=[(1024, 1024, True)])
    assert r is not None and r["error"].startswith("deadlock")

"""Race detection for the tensor-core kernels' barrier protocols (CPU): the
models in protocol_model.py run under many random interleavings without a
hazard or a stuck wait, and each planted protocol mistake is caught."""
import pytest

import protocol_model as pm


def _cases_prefill():
    # equal tile counts (grouped heads), the second tile one longer
    # (consecutive position blocks), and an empty second tile
    for n in range(1, 9):
        yield (n, n)
        yield (n - 1, n)
    yield (3, 0)
    yield (0, 1)


@pytest.mark.parametrize("rope,paged_tail", [(False, False), (True, False), (False, True)])
def test_prefill_protocol_hazard_free(rope, paged_tail):
    for nt in _cases_prefill():
        for seed in range(40):
            pm.prefill(nt, seed, rescale_p=(0.0, 0.3, 1.0)[seed % 3], rope=rope, paged_tail=paged_tail)


@pytest.mark.parametrize("bug", pm.PREFILL_BUGS)
def test_prefill_planted_bug_is_caught(bug):
    with pytest.raises(pm.Hazard):
        for nt in _cases_prefill():
            for seed in range(40):
                pm.prefill(nt, seed, rescale_p=0.5, bug=bug, rope=True, paged_tail=True)


def test_mla_protocol_hazard_free():
    for nt in range(0, 10):
        for tail_partial in (False, True):
            for seed in range(40):
                pm.mla(nt, tail_partial, seed, rescale_p=(0.0, 0.3, 1.0)[seed % 3])


@pytest.mark.parametrize("bug", pm.MLA_BUGS)
def test_mla_planted_bug_is_caught(bug):
    with pytest.raises(pm.Hazard):
        for nt in range(0, 10):
            for tail_partial in (False, True):
                for seed in range(40):
                    pm.mla(nt, tail_partial, seed, rescale_p=0.5, bug=bug)


def _decode_cases():
    import random
    rng = random.Random(7)
    for trial in range(120):
        yield trial, [rng.randint(1, 5) for _ in range(rng.randint(1, 4))]


@pytest.mark.parametrize("fp8", [False, True])
def test_decode_protocol_hazard_free(fp8):
    for seed, units in _decode_cases():
        pm.decode(units, seed, fp8=fp8)


@pytest.mark.parametrize("bug", pm.DECODE_BUGS)
def test_decode_planted_bug_is_caught(bug):
    with pytest.raises(pm.Hazard):
        for seed, units in _decode_cases():
            pm.decode(units, seed, fp8=bug.startswith("conv"), bug=bug)

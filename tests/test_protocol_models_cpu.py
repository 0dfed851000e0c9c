"""The barrier protocols of the forward's unit ring and of the dK / dV
pipeline, checked in random-interleaving models (host only).  Each planted
mistake must be caught within the sampled traces."""
import random

import pytest

from tests import protocol_models as pm


def _dkdv_traces(n, KS, mutation=None):
    rng = random.Random(7)
    failures = 0
    for seed in range(n):
        units = [rng.choice([0, 0, 1, 2, 3, 5, 8]) for _ in range(rng.randint(1, 6))]
        try:
            pm.dkdv_pair(units, seed, KS=KS, mutation=mutation)
        except pm.ProtocolError:
            failures += 1
    return failures


@pytest.mark.parametrize("KS", [2, 3, 4])
def test_dkdv_pair_protocol_holds(KS):
    assert _dkdv_traces(400, KS) == 0


@pytest.mark.parametrize("mutation", ["pd_empty_count", "no_buffer_wait", "no_stage_release", "no_acc_wait"])
def test_dkdv_pair_protocol_mutants_are_caught(mutation):
    assert _dkdv_traces(200, 4, mutation) > 0


def _ring_traces(n, mutation=None):
    rng = random.Random(2)
    failures = 0
    for seed in range(n):
        try:
            pm.unit_ring(rng.randint(0, 30), rng.randint(1, 4), seed, mutation=mutation)
        except pm.ProtocolError:
            failures += 1
    return failures


def test_unit_ring_protocol_holds():
    assert _ring_traces(1500) == 0


@pytest.mark.parametrize("mutation", ["empty_count", "no_empty_wait"])
def test_unit_ring_mutants_are_caught(mutation):
    assert _ring_traces(400, mutation) > 0


def _fwd_traces(n, mutation=None):
    rng = random.Random(11)
    failures = 0
    for seed in range(n):
        units = [rng.choice([0, 1, 1, 2, 3, 5, 9]) for _ in range(rng.randint(1, 6))]
        try:
            pm.fwd_pipeline(units, seed, mutation=mutation)
        except pm.ProtocolError:
            failures += 1
    return failures


def test_forward_pipeline_protocol_holds():
    assert _fwd_traces(600) == 0


@pytest.mark.parametrize("mutation", ["no_q_wait", "no_v_wait", "no_k_wait", "rescale_lag", "o_final_for_empty_units"])
def test_forward_pipeline_mutants_are_caught(mutation):
    assert _fwd_traces(300, mutation) > 0


def _gemm_traces(n, S, mutation=None):
    rng = random.Random(5)
    failures = 0
    for seed in range(n):
        try:
            pm.score_gemm(rng.randint(0, 9), seed, S=S, n_sub=rng.choice([2, 4]), mutation=mutation)
        except pm.ProtocolError:
            failures += 1
    return failures


@pytest.mark.parametrize("S", [2, 3, 4])
def test_score_gemm_protocol_holds(S):
    assert _gemm_traces(1500, S) == 0


@pytest.mark.parametrize("mutation", ["no_stage_wait", "no_acc_wait", "early_release"])
def test_score_gemm_mutants_are_caught(mutation):
    assert _gemm_traces(600, 2, mutation) > 0


def test_staging_ring_protocol_holds():
    for seed in range(800):
        pm.staging_ring(6, seed)


def test_staging_ring_single_tile_is_caught():
    failures = 0
    for seed in range(300):
        try:
            pm.staging_ring(6, seed, mutation="one_tile")
        except pm.ProtocolError:
            failures += 1
    assert failures > 0

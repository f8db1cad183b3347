"""GPU parity of the decode step (kda_decode) against the fp64 oracle.

A decode step is the recurrence for one token per request, so the oracle is
the scan over sequences of length 1 from the requests' states (and, for
several steps, the scan over the steps' tokens). All calls go through the C
ABI via the thin binding. Bars as for the prefill: o max-abs <= 3e-2 and
rel-RMS <= 5e-3, state rel-RMS <= 5e-3.
"""
import numpy as np
import pytest

import kda_inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kimi_delta_attention_26_b200 as m

    return m


def _step_inputs(inp, rows):
    """Device tensors of the tokens `rows` of a packed batch ([B, H, ...])."""
    d = H.to_device(inp)
    return {n: d[n][rows] for n in ("q", "k", "v", "g", "beta")}


def test_decode_batch_matches_oracle(kda, oracle_mod):
    import torch

    inp = kda_inputs.make_inputs([1] * 37, 3, seed=60, random_initial_state=True)
    o_ref, f_ref = oracle_mod.scan_inputs(inp)
    t = _step_inputs(inp, slice(None))
    state = torch.from_numpy(inp.initial_state).cuda()
    out = kda.kda_decode(t["q"], t["k"], t["v"], t["g"], t["beta"], state, scale=inp.scale)
    torch.cuda.synchronize()
    H.assert_parity(out, state, o_ref, f_ref, label="decode B=37 H=3")


def test_decode_steps_equal_the_scan(kda, oracle_mod):
    """40 decode steps of 2 requests from random states equal the oracle's
    scan over the 40 tokens (every step's output and the final state)."""
    import torch

    T, nh = 40, 2
    inp = kda_inputs.make_inputs([T, T], nh, seed=61, random_initial_state=True)
    o_ref, f_ref = oracle_mod.scan_inputs(inp)
    d = H.to_device(inp)
    state = d["initial_state"].clone()
    outs = torch.empty((2 * T, nh, 128), dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        rows = torch.tensor([t, T + t], device="cuda")
        outs[rows] = kda.kda_decode(d["q"][rows], d["k"][rows], d["v"][rows], d["g"][rows], d["beta"][rows],
                                    state, scale=inp.scale)
    torch.cuda.synchronize()
    H.assert_parity(outs, state, o_ref, f_ref, label="decode 40 steps x 2 requests")


def test_decode_state_indices_pool(kda):
    """Requests address slots of a larger pool: only their slots change, and
    the results equal a call on the gathered states, bitwise."""
    import torch

    inp = kda_inputs.make_inputs([1] * 3, 2, seed=62, random_initial_state=True)
    t = _step_inputs(inp, slice(None))
    torch.manual_seed(0)
    pool = 0.1 * torch.randn((6, 2, 128, 128), device="cuda")
    before = pool.clone()
    idx = torch.tensor([4, 0, 2], dtype=torch.int32, device="cuda")
    gathered = pool[idx.long()].clone()
    out_i = kda.kda_decode(t["q"], t["k"], t["v"], t["g"], t["beta"], pool, scale=inp.scale, state_indices=idx)
    out_g = kda.kda_decode(t["q"], t["k"], t["v"], t["g"], t["beta"], gathered, scale=inp.scale)
    torch.cuda.synchronize()
    assert torch.equal(out_i, out_g)
    assert torch.equal(pool[idx.long()], gathered)
    for s in (1, 3, 5):
        assert torch.equal(pool[s], before[s])
    assert kda.device_status(reset=True) == 0


def test_decode_bad_state_index_is_recorded_and_skipped(kda):
    import torch

    kda.device_status(reset=True)
    inp = kda_inputs.make_inputs([1] * 3, 2, seed=63, random_initial_state=True)
    t = _step_inputs(inp, slice(None))
    pool = torch.zeros((3, 2, 128, 128), device="cuda")
    out = torch.full((3, 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    idx = torch.tensor([0, 3, 2], dtype=torch.int32, device="cuda")  # slot 3 is outside the pool
    kda.kda_decode(t["q"], t["k"], t["v"], t["g"], t["beta"], pool, scale=inp.scale, state_indices=idx, out=out)
    torch.cuda.synchronize()
    assert kda.device_status(reset=True) == 4
    assert bool((out[1] == 7.0).all())          # the skipped request's row is untouched
    assert not bool((out[0] == 7.0).all()) and not bool((out[2] == 7.0).all())
    assert bool((pool[1] == 0).all())           # no slot was written for it


def test_decode_strided_views_and_empty_batch(kda):
    """q, k, v as slices of a fused projection and a head-major output give the
    same bits as contiguous tensors; B = 0 runs nothing."""
    import torch

    inp = kda_inputs.make_inputs([1] * 9, 3, seed=64, random_initial_state=True)
    t = _step_inputs(inp, slice(None))
    s0 = torch.from_numpy(inp.initial_state).cuda()
    s1 = s0.clone()
    ref = kda.kda_decode(t["q"], t["k"], t["v"], t["g"], t["beta"], s0, scale=inp.scale)
    fused = torch.cat([t["q"], t["k"], t["v"]], dim=2)
    out_hm = torch.empty((3, 9, 128), dtype=torch.bfloat16, device="cuda").transpose(0, 1)
    o = kda.kda_decode(fused[:, :, :128], fused[:, :, 128:256], fused[:, :, 256:], t["g"], t["beta"], s1,
                       scale=inp.scale, out=out_hm)
    torch.cuda.synchronize()
    assert torch.equal(o, ref) and torch.equal(s0, s1)
    e = torch.empty((0, 3, 128), dtype=torch.bfloat16, device="cuda")
    o = kda.kda_decode(e, e, e, torch.empty((0, 3, 128), device="cuda"), torch.empty((0, 3), device="cuda"), s1,
                       scale=inp.scale)
    assert o.shape == (0, 3, 128)


def test_decode_full_size_workload(kda, oracle_mod):
    """The benchmarked decode step (256 requests, H=32) against the oracle, in full."""
    import torch

    inp = kda_inputs.DECODE.make()
    o_ref, f_ref = oracle_mod.scan_inputs(inp)
    t = _step_inputs(inp, slice(None))
    state = torch.from_numpy(inp.initial_state).cuda()
    out = kda.kda_decode(t["q"], t["k"], t["v"], t["g"], t["beta"], state, scale=inp.scale)
    torch.cuda.synchronize()
    H.assert_parity(out, state, o_ref, f_ref, label="decode B=256 H=32 (full)")
    assert kda.device_status(reset=True) == 0


@pytest.mark.parametrize("fill", [-5.0, 0.0])
def test_decode_gate_extremes_and_no_write(kda, oracle_mod, fill):
    """g at the lower bound or at 0 everywhere; then beta = 0 (the state only
    decays and the output reads it)."""
    import torch

    inp = kda_inputs.make_inputs([1] * 19, 2, seed=65, random_initial_state=True)
    inp.g[:] = fill
    for beta0 in (False, True):
        if beta0:
            inp.beta[:] = 0.0
        o_ref, f_ref = oracle_mod.scan_inputs(inp)
        t = _step_inputs(inp, slice(None))
        state = torch.from_numpy(inp.initial_state).cuda()
        out = kda.kda_decode(t["q"], t["k"], t["v"], t["g"], t["beta"], state, scale=inp.scale)
        torch.cuda.synchronize()
        H.assert_parity(out, state, o_ref, f_ref, label=f"decode g={fill} beta0={beta0}")


def test_decode_reversed_slot_order(kda):
    """A permutation of the pool (request b uses slot B - 1 - b) gives the same
    bits as the identity order on the permuted states."""
    import torch

    inp = kda_inputs.make_inputs([1] * 12, 3, seed=66, random_initial_state=True)
    t = _step_inputs(inp, slice(None))
    s0 = torch.from_numpy(inp.initial_state).cuda()
    pool = s0.flip(0).contiguous()
    idx = torch.arange(11, -1, -1, dtype=torch.int32, device="cuda")
    o1 = kda.kda_decode(t["q"], t["k"], t["v"], t["g"], t["beta"], s0, scale=inp.scale)
    o2 = kda.kda_decode(t["q"], t["k"], t["v"], t["g"], t["beta"], pool, scale=inp.scale, state_indices=idx)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(pool.flip(0), s0)

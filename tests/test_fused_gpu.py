"""GPU parity of kda_fwd_fused (gate preprocessing fused into the prefill)
against the fp64 oracle: ``oracle.preprocess`` (L2 norms, gate from logits
with the lower bound, beta from logits) followed by the scan, on the raw draws
of the input generator. Bars as for kda_fwd.
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


def _raw_device(inp):
    import torch

    d = H.to_device(inp)
    return {
        "q": torch.from_numpy(inp.q_raw).view(torch.bfloat16).cuda(),
        "k": torch.from_numpy(inp.k_raw).view(torch.bfloat16).cuda(),
        "v": d["v"],
        "g": torch.from_numpy(inp.g_logit).cuda(),
        "beta": torch.from_numpy(inp.beta_logit).cuda(),
        "cu_seqlens": d["cu_seqlens"],
        "initial_state": d["initial_state"],
    }


def run_fused(kda, inp, lower_bound=-5.0, **kw):
    import torch

    d = _raw_device(inp)
    out, fin = kda.kda_fwd_fused(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, lower_bound,
                                 cu_seqlens=d["cu_seqlens"], initial_state=d["initial_state"], **kw)
    torch.cuda.synchronize()
    return out, fin


def _check(kda, oracle_mod, inp, label, lower_bound=-5.0, col_ranges=None):
    out, fin = run_fused(kda, inp, lower_bound)
    for a, b in col_ranges or [(0, 128)]:
        o_ref, f_ref = oracle_mod.scan_raw_inputs(inp, lower_bound, col_begin=a, col_end=b)
        H.assert_parity(out, fin, o_ref, f_ref, cols=slice(a, b), label=f"{label} cols {a}-{b}")


@pytest.mark.parametrize("lower_bound", [-5.0, -2.0])
def test_fused_ragged_batch(kda, oracle_mod, lower_bound):
    lens = [1, 15, 16, 17, 0, 63, 100, 300]
    inp = kda_inputs.make_inputs(lens, 3, seed=80, raw=True, random_initial_state=True)
    _check(kda, oracle_mod, inp, f"fused ragged lb={lower_bound}", lower_bound)


def test_fused_time_split(kda, oracle_mod):
    kda.set_time_split(2)
    try:
        inp = kda_inputs.make_inputs([1000], 2, seed=81, raw=True, random_initial_state=True)
        _check(kda, oracle_mod, inp, "fused time split T=1000")
    finally:
        kda.set_time_split(0)


def test_fused_segments_bit_exact_and_zero_query(kda):
    """A sequence gives the same bits alone or packed; a zero raw query row
    (normalised to zero) gives an exactly zero output row."""
    import torch

    lens = [40, 0, 77, 5]
    inp = kda_inputs.make_inputs(lens, 2, seed=82, raw=True, random_initial_state=True)
    inp.q_raw[50, 1, :] = 0
    out, fin = run_fused(kda, inp)
    assert torch.count_nonzero(out[50, 1]) == 0
    cu = inp.cu_seqlens
    for i, L in enumerate(lens):
        a, b = cu[i], cu[i + 1]
        sub = kda_inputs.KDAInputs(
            q=inp.q[a:b], k=inp.k[a:b], v=inp.v[a:b], g=inp.g[a:b], beta=inp.beta[a:b],
            cu_seqlens=np.array([0, L], np.int32), initial_state=inp.initial_state[i:i + 1].copy(),
            scale=inp.scale, seed=inp.seed, q_raw=inp.q_raw[a:b], k_raw=inp.k_raw[a:b],
            g_logit=inp.g_logit[a:b], beta_logit=inp.beta_logit[a:b])
        o_i, f_i = run_fused(kda, sub)
        assert torch.equal(out[a:b], o_i), f"segment {i}: output bits differ"
        assert torch.equal(fin[i], f_i[0]), f"segment {i}: state bits differ"


def test_fused_full_size_kimi_linear_shape(kda, oracle_mod):
    """The Kimi-Linear-shaped workload (T=8192, H=32) from raw draws; the
    oracle checks 8 columns of every 32-column slice."""
    wl = kda_inputs.workload(2)
    inp = wl.make(raw=True)
    _check(kda, oracle_mod, inp, "fused T=8192 H=32", col_ranges=[(8, 16), (40, 48), (72, 80), (104, 112)])
    assert kda.wait_timeouts(reset=True) == 0


def test_fused_heavy_clamp_and_strided_projection(kda, oracle_mod):
    """lower_bound = -0.5 clamps most gates; raw q, k, v as slices of one fused
    projection give the same bits as contiguous tensors."""
    import torch

    inp = kda_inputs.make_inputs([120, 33], 2, seed=83, raw=True, random_initial_state=True)
    _check(kda, oracle_mod, inp, "fused lb=-0.5", lower_bound=-0.5)
    d = _raw_device(inp)
    ref = kda.kda_fwd_fused(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, -0.5, cu_seqlens=d["cu_seqlens"],
                            initial_state=d["initial_state"])
    proj = torch.cat([d["q"], d["k"], d["v"]], dim=2)
    got = kda.kda_fwd_fused(proj[:, :, :128], proj[:, :, 128:256], proj[:, :, 256:], d["g"], d["beta"], inp.scale, -0.5,
                            cu_seqlens=d["cu_seqlens"], initial_state=d["initial_state"])
    torch.cuda.synchronize()
    assert torch.equal(ref[0], got[0]) and torch.equal(ref[1], got[1])


def test_fused_persistent_schedule_bitwise(kda):
    """Fused preprocessing with two persistent clusters taking all the pairs
    gives the bits of one cluster per pair."""
    import torch

    inp = kda_inputs.make_inputs([200, 0, 31, 90, 16, 400], 3, seed=84, raw=True, random_initial_state=True)
    try:
        kda.set_schedule(1)
        ref = run_fused(kda, inp)
        kda.set_schedule(2, 2)
        got = run_fused(kda, inp)
    finally:
        kda.set_schedule(0)
    assert torch.equal(ref[0], got[0]) and torch.equal(ref[1], got[1])

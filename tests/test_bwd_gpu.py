"""GPU parity of kda_bwd (gradients of the prefill) against the fp64 oracle's
reverse-mode derivative (itself pinned by finite differences).

The kernel computes in fp32 from the exact bf16/fp32 inputs, so the bar is
tighter than the forward's: relative RMS <= 1e-4 for every gradient (fp32
rounding over recurrences of a few thousand steps stays near 1e-6..1e-5).
"""
import numpy as np
import pytest

import kda_inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu
GRAD_REL_RMS = 1e-4


@pytest.fixture(scope="module")
def kda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kimi_delta_attention_26_b200 as m

    return m


def _grads(kda, oracle_mod, inp, seed, label, with_dfin=True):
    import torch

    rng = np.random.default_rng(seed)
    T, nh = inp.total_tokens, inp.num_heads
    dout = kda_inputs.f32_to_bf16_bits(rng.standard_normal((T, nh, 128)).astype(np.float32))
    dfin = rng.standard_normal((inp.num_seqs, nh, 128, 128)).astype(np.float32) if with_dfin else None
    d = H.to_device(inp)
    gr = kda.kda_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], torch.from_numpy(dout).view(torch.bfloat16).cuda(),
                     inp.scale, d["cu_seqlens"], d["initial_state"],
                     None if dfin is None else torch.from_numpy(dfin).cuda())
    torch.cuda.synchronize()
    ref = oracle_mod.backward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.scale, dout,
                              inp.initial_state, dfin)
    pairs = [("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dg", "dg"), ("dbeta", "dbeta")]
    if inp.initial_state is not None:
        pairs.append(("dinitial_state", "dinit"))
    worst = {}
    for gname, rname in pairs:
        x = gr[gname].cpu().numpy().astype(np.float64)
        m = H.metrics(x, ref[rname])
        worst[gname] = m["rel_rms"]
        H.REPORT.append({"case": f"{label} {gname}", "o_max_abs": m["max_abs"], "o_rel_rms": m["rel_rms"],
                         "state_rel_rms": None})
        assert np.isfinite(x).all(), f"{label}: non-finite {gname}"
        assert m["rel_rms"] <= GRAD_REL_RMS, f"{label}: {gname} rel-RMS {m}"
    return worst


def test_bwd_ragged_batch(kda, oracle_mod):
    lens = [1, 3, 4, 5, 0, 17, 64, 130]
    inp = kda_inputs.make_inputs(lens, 3, seed=100, random_initial_state=True)
    _grads(kda, oracle_mod, inp, 101, "bwd ragged")


def test_bwd_zero_initial_state_no_final_gradient(kda, oracle_mod):
    inp = kda_inputs.make_inputs([77, 40], 2, seed=102)
    _grads(kda, oracle_mod, inp, 103, "bwd zero-init", with_dfin=False)


def test_bwd_deterministic(kda):
    import torch

    inp = kda_inputs.make_inputs([300, 45], 2, seed=104, random_initial_state=True)
    d = H.to_device(inp)
    dout = torch.randn((inp.total_tokens, 2, 128), device="cuda").bfloat16()
    a = kda.kda_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dout, inp.scale, d["cu_seqlens"], d["initial_state"])
    b = kda.kda_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dout, inp.scale, d["cu_seqlens"], d["initial_state"])
    torch.cuda.synchronize()
    for n in a:
        assert torch.equal(a[n], b[n]), n


def test_bwd_full_size_uniform_varlen(kda, oracle_mod):
    """The uniform-varlen workload (8 x 1024 tokens, H=32, random states) in full."""
    inp = kda_inputs.workload(3).make()
    _grads(kda, oracle_mod, inp, 105, "bwd 8x1024 H=32 (full)")
    assert kda.device_status(reset=True) == 0


@pytest.mark.parametrize("fill", [-5.0, 0.0])
def test_bwd_gate_extremes(kda, oracle_mod, fill):
    inp = kda_inputs.make_inputs([50, 9], 2, seed=106, random_initial_state=True)
    inp.g[:] = fill
    _grads(kda, oracle_mod, inp, 107, f"bwd g={fill}")


def test_bwd_strided_views_bitwise_equal_contiguous(kda):
    """q, k, v as slices of one fused projection and dout as a head-major view
    give the same bits as contiguous tensors."""
    import torch

    inp = kda_inputs.make_inputs([130, 21], 3, seed=108, random_initial_state=True)
    d = H.to_device(inp)
    dout = torch.randn((inp.total_tokens, 3, 128), device="cuda").bfloat16()
    ref = kda.kda_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dout, inp.scale, d["cu_seqlens"], d["initial_state"])
    fused = torch.cat([d["q"], d["k"], d["v"]], dim=2)
    dout_hm = dout.transpose(0, 1).contiguous().transpose(0, 1)
    got = kda.kda_bwd(fused[:, :, :128], fused[:, :, 128:256], fused[:, :, 256:], d["g"], d["beta"], dout_hm,
                      inp.scale, d["cu_seqlens"], d["initial_state"])
    torch.cuda.synchronize()
    for n in ref:
        assert torch.equal(ref[n], got[n]), n

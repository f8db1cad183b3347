"""GPU parity: the CUDA paths against the fp64 oracle on the same seeded inputs.

All calls go through the C ABI (``libkda.so``) via the thin Python binding.
Bars: o max-abs <= 3e-2 and rel-RMS <= 5e-3; final state rel-RMS <= 5e-3;
segment handling bit-exact (a sequence gives the same bits alone or packed).

Every behaviour test runs on each kernel variant: the 16-token path with 32-
and 16-column value slices per CTA, the same with a few persistent clusters
taking all the (sequence, head) pairs round robin, and the 64-token tcgen05
path.
"""
import numpy as np
import pytest

import kda_inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu

# path, value columns per CTA, persistent clusters (0: the default schedule)
VARIANTS = {"p16s32": (16, 32, 0), "p16s16": (16, 16, 0), "p16s32q3": (16, 32, 3), "p16s16q2": (16, 16, 2),
            "p64": (64, 0, 0)}


@pytest.fixture(scope="module")
def kda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kimi_delta_attention_26_b200 as m

    return m


@pytest.fixture(params=list(VARIANTS), ids=list(VARIANTS))
def variant(request, kda):
    """One kernel variant for the test; the library defaults are restored after."""
    path, cols, clusters = VARIANTS[request.param]
    kda.set_path(path)
    kda.set_slice_columns(cols)
    kda.set_schedule(2 if clusters else 0, clusters)
    yield request.param
    kda.set_path(0)
    kda.set_slice_columns(0)
    kda.set_schedule(0)


@pytest.fixture(params=[16, 64], ids=["p16", "p64"])
def path(request, kda):
    kda.set_path(request.param)
    yield request.param
    kda.set_path(0)


def _check(oracle_mod, inp, label, col_ranges=None, **kw):
    out, fin = H.run_gpu(inp, **kw)
    if col_ranges is None:
        o_ref, f_ref = oracle_mod.scan_inputs(inp)
        return H.assert_parity(out, fin, o_ref, f_ref, label=label)
    res = None
    for a, b in col_ranges:
        o_ref, f_ref = oracle_mod.scan_inputs(inp, col_begin=a, col_end=b)
        res = H.assert_parity(out, fin, o_ref, f_ref, cols=slice(a, b), label=f"{label} cols {a}-{b}")
    return res


def test_tiny_config(kda, oracle_mod, variant):
    inp = kda_inputs.workload(1).make()
    _check(oracle_mod, inp, f"tiny T=256 H=2 [{variant}]")


@pytest.mark.parametrize("seed", [0, 1])
def test_ragged_varlen_small(kda, oracle_mod, seed, variant):
    # lengths around the 16- and 64-token chunks, an empty sequence, several
    # chunks, random initial states
    lens = [1, 15, 16, 17, 63, 64, 65, 200, 0, 129, 300]
    inp = kda_inputs.make_inputs(lens, 3, seed=50 + seed, random_initial_state=True)
    _check(oracle_mod, inp, f"ragged seed={seed} [{variant}]")


def test_zero_initial_state_null_equals_zeros(kda, path):
    import torch

    inp = kda_inputs.make_inputs([100, 37], 2, seed=3)
    out_a, fin_a = H.run_gpu(inp)
    inp.initial_state = np.zeros((2, 2, 128, 128), np.float32)
    out_b, fin_b = H.run_gpu(inp)
    assert torch.equal(out_a, out_b) and torch.equal(fin_a, fin_b)


def test_gate_extremes(kda, oracle_mod, variant):
    # g at the lower bound everywhere (fastest decay) and g = 0 (no decay)
    for fill in (-5.0, 0.0):
        inp = kda_inputs.make_inputs([150, 70], 2, seed=8, random_initial_state=True)
        inp.g[:] = fill
        _check(oracle_mod, inp, f"g={fill} [{variant}]")


def test_beta_zero_reads_only_the_decayed_initial_state(kda, oracle_mod, variant):
    # beta = 0: no token writes, so o_t = scale (q_t * exp G_t)^T S_0 and the
    # final state is Diag(exp G_T) S_0 (checked against the oracle's scan)
    inp = kda_inputs.make_inputs([90, 33], 2, seed=19, random_initial_state=True)
    inp.beta[:] = 0.0
    _check(oracle_mod, inp, f"beta=0 [{variant}]")


def test_chunk_boundary_lengths_with_empty_sequences(kda, oracle_mod, variant):
    # every length around 16- and 64-token chunk boundaries, empty sequences between
    lens = [15, 0, 16, 17, 0, 0, 31, 32, 33, 47, 48, 49, 63, 64, 65, 127, 128, 129, 0]
    inp = kda_inputs.make_inputs(lens, 2, seed=21, random_initial_state=True)
    _check(oracle_mod, inp, f"chunk-boundary lengths [{variant}]")


def test_single_token_and_all_empty(kda, oracle_mod, variant):
    import torch

    inp = kda_inputs.make_inputs([1], 4, seed=9, random_initial_state=True)
    _check(oracle_mod, inp, f"T=1 [{variant}]")
    inp = kda_inputs.make_inputs([0, 0, 0], 2, seed=10, random_initial_state=True)
    out, fin = H.run_gpu(inp)
    assert out.numel() == 0
    assert torch.equal(fin.cpu(), torch.from_numpy(inp.initial_state))


def test_segments_bit_exact(kda, variant):
    """A packed batch restricted to one sequence equals that sequence run alone, bitwise."""
    import torch

    lens = [5, 64, 0, 130, 77, 1]
    inp = kda_inputs.make_inputs(lens, 2, seed=11, random_initial_state=True)
    out, fin = H.run_gpu(inp)
    cu = inp.cu_seqlens
    for i, L in enumerate(lens):
        sub = kda_inputs.KDAInputs(
            q=inp.q[cu[i]:cu[i + 1]], k=inp.k[cu[i]:cu[i + 1]], v=inp.v[cu[i]:cu[i + 1]],
            g=inp.g[cu[i]:cu[i + 1]], beta=inp.beta[cu[i]:cu[i + 1]],
            cu_seqlens=np.array([0, L], np.int32), initial_state=inp.initial_state[i:i + 1].copy(),
            scale=inp.scale, seed=inp.seed)
        o_i, f_i = H.run_gpu(sub)
        assert torch.equal(out[cu[i]:cu[i + 1]], o_i), f"segment {i}: output bits differ"
        assert torch.equal(fin[i], f_i[0]), f"segment {i}: state bits differ"


def test_no_cu_seqlens_equals_single_sequence(kda, path):
    import torch

    inp = kda_inputs.make_inputs([333], 2, seed=12, random_initial_state=True)
    d = H.to_device(inp)
    a = kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, d["cu_seqlens"], d["initial_state"])
    b = kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, None, d["initial_state"])
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("t1", [64, 100])
def test_resume_from_final_state(kda, oracle_mod, t1, variant):
    import torch

    inp = kda_inputs.make_inputs([257], 2, seed=13, random_initial_state=True)
    d = H.to_device(inp)
    full_o, full_f = kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, None, d["initial_state"])
    a_o, a_f = kda.kda_fwd(d["q"][:t1].contiguous(), d["k"][:t1].contiguous(), d["v"][:t1].contiguous(),
                           d["g"][:t1].contiguous(), d["beta"][:t1].contiguous(), inp.scale, None, d["initial_state"])
    b_o, b_f = kda.kda_fwd(d["q"][t1:].contiguous(), d["k"][t1:].contiguous(), d["v"][t1:].contiguous(),
                           d["g"][t1:].contiguous(), d["beta"][t1:].contiguous(), inp.scale, None, a_f)
    torch.cuda.synchronize()
    o_ref, f_ref = oracle_mod.scan_inputs(inp)
    H.assert_parity(torch.cat([a_o, b_o]), b_f, o_ref, f_ref, label=f"resume t1={t1} [{variant}]")
    if t1 % 64 == 0:
        # splitting on a chunk boundary changes nothing but the state's fp32 round trip
        assert torch.equal(torch.cat([a_o, b_o]), full_o)
        assert torch.equal(b_f, full_f)


def test_in_place_state_update(kda, variant):
    import torch

    inp = kda_inputs.make_inputs([90, 10], 2, seed=14, random_initial_state=True)
    d = H.to_device(inp)
    o1, f1 = kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, d["cu_seqlens"], d["initial_state"])
    st = d["initial_state"].clone()
    o2, f2 = kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, d["cu_seqlens"], st, final_state=st)
    torch.cuda.synchronize()
    assert f2.data_ptr() == st.data_ptr()
    assert torch.equal(o1, o2) and torch.equal(f1, st)


def test_deterministic(kda, path):
    import torch

    inp = kda_inputs.make_inputs([500, 3, 260], 4, seed=15, random_initial_state=True)
    a = H.run_gpu(inp)
    b = H.run_gpu(inp)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_no_writes_outside_outputs(kda, variant):
    """Guard regions around out and final_state keep their sentinel values."""
    import torch

    inp = kda_inputs.make_inputs([70, 0, 33], 2, seed=16, random_initial_state=True)
    d = H.to_device(inp)
    T, nh = inp.total_tokens, inp.num_heads
    guard = 4096
    ob = torch.full((T * nh * 128 + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    fb = torch.full((3 * nh * 128 * 128 + 2 * guard,), 7.0, dtype=torch.float32, device="cuda")
    out = ob[guard:guard + T * nh * 128].view(T, nh, 128)
    fin = fb[guard:guard + 3 * nh * 128 * 128].view(3, nh, 128, 128)
    kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, d["cu_seqlens"], d["initial_state"],
                out=out, final_state=fin)
    torch.cuda.synchronize()
    for buf in (ob, fb):
        assert bool((buf[:guard] == 7.0).all()) and bool((buf[-guard:] == 7.0).all())


def test_strided_views_bitwise_equal_contiguous(kda, path):
    """q, k, v as slices of one fused [T, H, 384] projection, beta as a column
    of a wider matrix and a head-major output give the same bits as
    contiguous tensors."""
    import torch

    inp = kda_inputs.make_inputs([200, 65], 3, seed=23, random_initial_state=True)
    d = H.to_device(inp)
    ref_o, ref_f = kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, d["cu_seqlens"],
                               d["initial_state"])
    T, nh = inp.total_tokens, inp.num_heads
    fused = torch.cat([d["q"], d["k"], d["v"]], dim=2)               # [T, H, 384]
    bwide = torch.zeros((T, nh, 4), dtype=torch.float32, device="cuda")
    bwide[:, :, 2] = d["beta"]
    out_hm = torch.empty((nh, T, 128), dtype=torch.bfloat16, device="cuda").transpose(0, 1)  # head-major
    o, f = kda.kda_fwd(fused[:, :, :128], fused[:, :, 128:256], fused[:, :, 256:], d["g"], bwide[:, :, 2],
                       inp.scale, d["cu_seqlens"], d["initial_state"], out=out_hm)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o) and torch.equal(f, ref_f)


def test_paths_agree(kda):
    """The two kernels round differently but agree within the parity bar."""
    inp = kda_inputs.make_inputs([700, 129, 64, 3], 3, seed=24, random_initial_state=True)
    res = {}
    for p in (16, 64):
        kda.set_path(p)
        res[p] = H.run_gpu(inp)
    kda.set_path(0)
    o16, f16 = (x.float().cpu().numpy().astype(np.float64) for x in res[16])
    o64, f64 = (x.float().cpu().numpy().astype(np.float64) for x in res[64])
    mo, ms = H.metrics(o64, o16), H.metrics(f64, f16)
    assert mo["max_abs"] <= H.O_MAX_ABS and mo["rel_rms"] <= 2 * H.O_REL_RMS, mo
    assert ms["rel_rms"] <= 2 * H.S_REL_RMS, ms


def test_bad_cu_seqlens_is_recorded(kda, path):
    """A cu_seqlens that is not a non-decreasing partition of [0, T) is
    clamped by the kernel (no access outside the tensors) and recorded in the
    device status word."""
    import torch

    kda.device_status(reset=True)
    inp = kda_inputs.make_inputs([40, 60], 2, seed=25, random_initial_state=True)
    d = H.to_device(inp)
    for bad in ([0, 60, 40], [0, 40, 90], [8, 40, 100]):  # decreasing; past T; not starting at 0
        cu = torch.tensor(bad, dtype=torch.int32, device="cuda")
        kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, cu, d["initial_state"])
        torch.cuda.synchronize()
        assert kda.device_status(reset=True) & 1, bad
    kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, d["cu_seqlens"], d["initial_state"])
    assert kda.device_status(reset=True) == 0


# --------------------------------------------------------------- full sizes
# The five workloads at their full sizes, in the launch configuration the
# bench times; the oracle computes a sample of value columns (columns evolve
# independently, so a column subset is exact) for every token and head. The
# sample has 8 columns in each 32-column slice, so every CTA of a cluster
# (16-token path) is checked.
FULL_COLS = [(8, 16), (40, 48), (72, 80), (104, 112)]


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_full_size_workloads_sampled_columns(kda, oracle_mod, cfg, path):
    inp = kda_inputs.workload(cfg).make()
    _check(oracle_mod, inp, f"config {cfg} [p{path}]", col_ranges=FULL_COLS)


def test_slice_variants_bitwise_equal(kda):
    """Each column's arithmetic does not depend on how many columns a CTA
    holds, so the two 16-token variants give the same bits."""
    import torch

    inp = kda_inputs.make_inputs([700, 129, 64], 3, seed=17, random_initial_state=True)
    res = {}
    kda.set_path(16)
    for cols in (16, 32):
        kda.set_slice_columns(cols)
        res[cols] = H.run_gpu(inp)
    kda.set_slice_columns(0)
    kda.set_path(0)
    o16, f16 = res[16]
    o32, f32 = res[32]
    assert torch.equal(o16, o32) and torch.equal(f16, f32)


@pytest.mark.parametrize("cols", [32, 16])
def test_persistent_schedules_bitwise_equal(kda, oracle_mod, cols):
    """A cluster that runs several (sequence, head) pairs back to back gives
    every pair the same bits as a cluster of its own: one cluster for all
    pairs, a few, and as many as the device holds, on a batch of empty,
    ragged and multi-chunk sequences; the persistent result also meets the
    oracle."""
    import torch

    lens = [0, 300, 17, 1, 64, 0, 129, 1000, 16, 33, 250, 5]
    inp = kda_inputs.make_inputs(lens, 5, seed=40, random_initial_state=True)
    kda.set_path(16)
    kda.set_slice_columns(cols)
    try:
        kda.set_schedule(1)
        ref_o, ref_f = H.run_gpu(inp)
        for cap in (1, 3, 7, 0):
            kda.set_schedule(2, cap)
            o, f = H.run_gpu(inp)
            assert torch.equal(o, ref_o) and torch.equal(f, ref_f), f"{cols} columns, {cap} clusters"
        kda.set_schedule(2, 4)
        _check(oracle_mod, inp, f"persistent 4 clusters s{cols}")
    finally:
        kda.set_schedule(0)
        kda.set_slice_columns(0)
        kda.set_path(0)


def test_persistent_full_size_uniform_varlen_bitwise(kda):
    """The 8 x 1024, H = 32 batch (256 pairs, more than the device holds at
    once): the default schedule (persistent) equals one cluster per pair."""
    import torch

    inp = kda_inputs.workload(3).make()
    kda.set_path(16)
    try:
        kda.set_schedule(1)
        ref = H.run_gpu(inp)
        kda.set_schedule(0)
        got = H.run_gpu(inp)
    finally:
        kda.set_schedule(0)
        kda.set_path(0)
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])


def test_zz_no_wait_timeouts(kda):
    """Every bounded in-kernel wait of this module's runs completed in time."""
    import torch

    torch.cuda.synchronize()
    assert kda.wait_timeouts(reset=True) == 0


# --------------------------------------------------------------- time split
@pytest.fixture
def split_on(kda):
    """The time-split prefill forced on for one sequence (16-token path)."""
    kda.set_path(16)
    kda.set_time_split(2)
    yield
    kda.set_time_split(0)
    kda.set_path(0)


@pytest.mark.parametrize("T,rinit", [(64, True), (300, True), (1000, False), (4097, True)])
def test_time_split_matches_oracle(kda, oracle_mod, split_on, T, rinit):
    inp = kda_inputs.make_inputs([T], 3, seed=30 + T, random_initial_state=rinit)
    _check(oracle_mod, inp, f"time split T={T} init={rinit}")


def test_time_split_in_place_state_and_guards(kda, split_on):
    """The split writes only out and final_state (which may alias the initial state)."""
    import torch

    inp = kda_inputs.make_inputs([777], 2, seed=31, random_initial_state=True)
    d = H.to_device(inp)
    ref_o, ref_f = kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, None, d["initial_state"])
    guard = 4096
    T = inp.total_tokens
    ob = torch.full((T * 2 * 128 + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = ob[guard:guard + T * 2 * 128].view(T, 2, 128)
    st = d["initial_state"].clone()
    o, f = kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, None, st, out=out, final_state=st)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o) and torch.equal(st, ref_f)
    assert bool((ob[:guard] == 7.0).all()) and bool((ob[-guard:] == 7.0).all())


def test_time_split_agrees_with_unsplit(kda):
    inp = kda_inputs.make_inputs([3000], 4, seed=32, random_initial_state=True)
    kda.set_path(16)
    res = {}
    for mode in (1, 2):
        kda.set_time_split(mode)
        res[mode] = H.run_gpu(inp)
    kda.set_time_split(0)
    kda.set_path(0)
    o1, f1 = (x.float().cpu().numpy().astype(np.float64) for x in res[1])
    o2, f2 = (x.float().cpu().numpy().astype(np.float64) for x in res[2])
    mo, ms = H.metrics(o2, o1), H.metrics(f2, f1)
    assert mo["max_abs"] <= H.O_MAX_ABS and mo["rel_rms"] <= 2 * H.O_REL_RMS, mo
    assert ms["rel_rms"] <= 2 * H.S_REL_RMS, ms


def test_time_split_automatic_from_4096_tokens(kda, oracle_mod):
    """One sequence of 4096 tokens with few heads takes the split by default:
    the automatic result equals the forced split bitwise, differs from the
    unsplit run, and meets the oracle."""
    import torch

    inp = kda_inputs.make_inputs([4096], 2, seed=34, random_initial_state=True)
    kda.set_path(16)
    try:
        res = {}
        for mode in (0, 1, 2):
            kda.set_time_split(mode)
            res[mode] = H.run_gpu(inp)
    finally:
        kda.set_time_split(0)
        kda.set_path(0)
    assert torch.equal(res[0][0], res[2][0]) and torch.equal(res[0][1], res[2][1])
    assert not torch.equal(res[0][0], res[1][0])
    o_ref, f_ref = oracle_mod.scan_inputs(inp)
    H.assert_parity(res[0][0], res[0][1], o_ref, f_ref, label="automatic split T=4096")

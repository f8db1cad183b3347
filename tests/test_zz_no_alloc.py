"""kda_fwd_noalloc: the allocation-free entry point of the C ABI.

It is meant for callers that cannot allocate device memory while they run:
kda_fwd takes its scratch ring from a stream-ordered memory pool, which a
serving engine that has reserved the whole device for its own arena (or a
deployment without CUDA memory pools) cannot allow. kda_fwd_noalloc uses a
fixed-size ring declared in device memory by the library instead.

The GPU test calls it through the C ABI twice in a row, on different batches
(so the second call runs on the first call's leftover scratch contents), on
each kernel path and with a few persistent clusters running all the pairs,
and checks that each result is bitwise identical to
kda_fwd's on the same inputs: both run the same deterministic kernel, only
the scratch memory differs. It loads the library itself, so it passes in a
fresh process as well as after the other tests.
"""
import ctypes
import os

import pytest

import kda_inputs
from tests import helpers as H

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MAX_PAIRS = 32  # KDA_NOALLOC_MAX_PAIRS in include/kda.h


@pytest.mark.gpu
@pytest.mark.parametrize("path,clusters", [(16, 0), (64, 0), (16, 3)])
def test_noalloc_matches_kda_fwd_on_two_calls(path, clusters):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kimi_delta_attention_26_b200 as kda

    lib = ctypes.CDLL(kda.library_path())
    P = ctypes.POINTER(kda.TensorDesc)
    fn = lib.kda_fwd_noalloc
    fn.argtypes = [P, P, P, P, P, ctypes.c_float, ctypes.c_void_p, ctypes.c_int32, P, P, P, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    kda.set_path(path)
    # clusters > 0: a few persistent clusters run all the pairs, so each cluster's
    # ring slots carry several pairs' chunks within one call
    kda.set_schedule(2 if clusters else 0, clusters)
    try:
        batches = [
            kda_inputs.make_inputs([300, 17, 0, 129], 4, seed=71, random_initial_state=True),   # 16 pairs
            kda_inputs.make_inputs([1000, 33], 16, seed=72, random_initial_state=True),         # 32 pairs (the cap)
        ]
        for i, inp in enumerate(batches):
            d = H.to_device(inp)
            ref_o, ref_f = kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, d["cu_seqlens"],
                                       d["initial_state"])
            out = torch.empty_like(ref_o)
            fin = torch.empty_like(ref_f)
            descs = [kda.describe(t) for t in (d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"], out, fin)]
            r = [x[0] for x in descs]
            rc = fn(r[0], r[1], r[2], r[3], r[4], inp.scale, d["cu_seqlens"].data_ptr(), inp.num_seqs, r[5], r[6],
                    r[7], torch.cuda.current_stream().cuda_stream)
            assert rc == 0, f"call {i}: status {rc}"
            torch.cuda.synchronize()
            assert torch.equal(out, ref_o), f"call {i}: output bits differ from kda_fwd"
            assert torch.equal(fin, ref_f), f"call {i}: state bits differ from kda_fwd"
    finally:
        kda.set_path(0)
        kda.set_schedule(0)
    assert kda.wait_timeouts(reset=True) == 0

"""kda_fwd_noalloc: the allocation-free entry point of the C ABI.

It is meant for callers that cannot allocate device memory while they run:
kda_fwd takes its scratch ring from a stream-ordered memory pool, which a
serving engine that has reserved the whole device for its own arena (or a
deployment without CUDA memory pools) cannot allow. kda_fwd_noalloc uses a
fixed-size ring declared in device memory by the library instead.

The GPU test calls it through the C ABI twice in a row, on different batches
(so the second call runs on the first call's leftover scratch contents), and
checks each result against kda_fwd on the same inputs within the parity
tolerances of the test suite. It loads the library itself, so it passes in a
fresh process as well as after the other tests.
"""
import ctypes
import os

import numpy as np
import pytest

import kda_inputs
from tests import helpers as H

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MAX_PAIRS = 32  # KDA_NOALLOC_MAX_PAIRS in include/kda.h
KDA_ERR_CAPACITY = 6


def _bind(lib):
    P = ctypes.c_void_p
    fn = lib.kda_fwd_noalloc
    fn.argtypes = [P, P, P, P, P, ctypes.c_float, P, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, P, P, P, P]
    fn.restype = ctypes.c_int
    return fn


def _lib_path():
    return os.path.join(ROOT, "kimi_delta_attention_26_b200", "libkda.so")


def test_capacity_is_rejected_before_any_gpu_work():
    # fails argument validation on the host (fake addresses are never used)
    fn = _bind(ctypes.CDLL(_lib_path()))
    rc = fn(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 1.0, 0x6000, 2, 16, MAX_PAIRS // 2 + 1, None, 0x7000,
            None, None)
    assert rc == KDA_ERR_CAPACITY


@pytest.mark.gpu
def test_noalloc_matches_kda_fwd_on_two_calls():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kimi_delta_attention_26_b200 as kda

    fn = _bind(ctypes.CDLL(kda.library_path()))
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
        stream = torch.cuda.current_stream()
        rc = fn(d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), d["g"].data_ptr(), d["beta"].data_ptr(),
                inp.scale, d["cu_seqlens"].data_ptr(), inp.num_seqs, inp.total_tokens, inp.num_heads,
                d["initial_state"].data_ptr(), out.data_ptr(), fin.data_ptr(), stream.cuda_stream)
        assert rc == 0, f"call {i}: status {rc}"
        torch.cuda.synchronize()
        ref = ref_o.float().cpu().numpy().astype(np.float64)
        got = out.float().cpu().numpy().astype(np.float64)
        m_o = H.metrics(got, ref)
        assert m_o["max_abs"] <= H.O_MAX_ABS and m_o["rel_rms"] <= H.O_REL_RMS, (i, m_o)
        m_s = H.metrics(fin.cpu().numpy().astype(np.float64), ref_f.cpu().numpy().astype(np.float64))
        assert m_s["rel_rms"] <= H.S_REL_RMS, (i, m_s)
    assert kda.wait_timeouts(reset=True) == 0

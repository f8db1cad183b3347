"""Shared helpers for the GPU parity tests (marshalling and error metrics only)."""
import json
import os

import numpy as np

# Tolerances of the KDA prefill parity bar: o (bf16) max-abs <= 3e-2 and
# relative RMS <= 5e-3; final state (fp32) relative RMS <= 5e-3.
O_MAX_ABS = 3e-2
O_REL_RMS = 5e-3
S_REL_RMS = 5e-3

# Parity results of this process, written to $KDA_PARITY_REPORT (JSON) at
# the end of the session when that variable is set.
REPORT = []


def to_device(inp, device="cuda"):
    import torch

    d = {
        "q": torch.from_numpy(inp.q).view(torch.bfloat16).to(device),
        "k": torch.from_numpy(inp.k).view(torch.bfloat16).to(device),
        "v": torch.from_numpy(inp.v).view(torch.bfloat16).to(device),
        "g": torch.from_numpy(inp.g).to(device),
        "beta": torch.from_numpy(inp.beta).to(device),
        "cu_seqlens": torch.from_numpy(inp.cu_seqlens).to(device),
        "initial_state": None if inp.initial_state is None else torch.from_numpy(inp.initial_state).to(device),
    }
    return d


def run_gpu(inp, device="cuda", **kw):
    import torch
    import kimi_delta_attention_26_b200 as kda

    d = to_device(inp, device)
    out, fin = kda.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale=inp.scale,
                           cu_seqlens=d["cu_seqlens"], initial_state=d["initial_state"], **kw)
    torch.cuda.synchronize()
    return out, fin


def o_to_f64(out):
    return out.float().cpu().numpy().astype(np.float64)


def metrics(x, ref):
    err = x - ref
    nref = float(np.linalg.norm(ref))
    return {
        "max_abs": float(np.max(np.abs(err))) if err.size else 0.0,
        "rel_rms": float(np.linalg.norm(err) / nref) if nref > 0 else float(np.linalg.norm(err)),
    }


def record(label, mo, ms):
    REPORT.append({"case": label, "o_max_abs": mo["max_abs"], "o_rel_rms": mo["rel_rms"],
                   "state_rel_rms": None if ms is None else ms["rel_rms"]})


def write_report():
    path = os.environ.get("KDA_PARITY_REPORT")
    if path and REPORT:
        with open(path, "w") as f:
            json.dump(REPORT, f, indent=1)


def assert_parity(out, fin, o_ref, f_ref, cols=slice(None), label=""):
    o = o_to_f64(out)[:, :, cols]
    mo = metrics(o, o_ref[:, :, cols])
    ms = None
    if f_ref is not None:
        f = fin.cpu().numpy().astype(np.float64)[..., cols]
        ms = metrics(f, f_ref[..., cols])
    record(label, mo, ms)
    assert np.isfinite(o).all(), f"{label}: non-finite output"
    assert mo["max_abs"] <= O_MAX_ABS, f"{label}: o max-abs {mo}"
    assert mo["rel_rms"] <= O_REL_RMS, f"{label}: o rel-RMS {mo}"
    if ms is not None:
        assert np.isfinite(fin.cpu().numpy()).all(), f"{label}: non-finite state"
        assert ms["rel_rms"] <= S_REL_RMS, f"{label}: state rel-RMS {ms}"
    return mo, ms

"""fp64 CPU oracle for the KDA forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg may
import this package. The product (the CUDA library and its Python binding)
never imports it, and it imports nothing from the product.

Python side: ctypes marshalling around ``kda_oracle.cpp`` (the arithmetic lives
there, in plain fp64 C++). ``build()`` compiles it with g++ into
``liboracle.so`` next to the source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle (portable x86-64/aarch64 code, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
               "-ffp-contract=off", "-o", tmp, _SRC]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            try:
                lib = ctypes.CDLL(build())
            except OSError:
                lib = ctypes.CDLL(build(force=True))
            P = ctypes.c_void_p
            i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
            scan_args = [P, P, P, P, P, i64, i32, i32, i32, P, i32, f64, P, P, P, i32, i32, i32, i32, i32]
            lib.kda_oracle_scan_bf16.argtypes = scan_args
            lib.kda_oracle_scan_bf16.restype = ctypes.c_int
            lib.kda_oracle_scan_f64.argtypes = scan_args
            lib.kda_oracle_scan_f64.restype = ctypes.c_int
            lib.kda_oracle_chunked_f64.argtypes = [P, P, P, P, P, i64, i32, i32, i32, P, i32, f64, P, P, P, i32, i32]
            lib.kda_oracle_chunked_f64.restype = ctypes.c_int
            lib.kda_oracle_unit_lower_inverse.argtypes = [P, i32, P, i32]
            lib.kda_oracle_unit_lower_inverse.restype = ctypes.c_int
            lib.kda_oracle_preprocess.argtypes = [P, P, P, P, i64, i32, i32, f64, f64, P, P, P, P]
            lib.kda_oracle_preprocess.restype = ctypes.c_int
            bw_args = [P, P, P, P, P, i64, i32, i32, i32, P, i32, f64, P, P, P, P, P, P, P, P, P, i32]
            lib.kda_oracle_backward_bf16.argtypes = bw_args
            lib.kda_oracle_backward_bf16.restype = ctypes.c_int
            lib.kda_oracle_backward_f64.argtypes = bw_args
            lib.kda_oracle_backward_f64.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def scan(q, k, v, g, beta, cu_seqlens, scale, initial_state=None, *, erase=True,
         want_out=True, want_final=True, col_begin=0, col_end=None, col_block=16, nthreads=0):
    """Token-by-token fp64 recurrence.

    ``q``/``k``/``v`` are either uint16 bf16 bit patterns (library format, with
    float32 ``g``/``beta``/``initial_state``) or float64 arrays (all inputs
    float64). Returns ``(out, final_state)`` as float64 arrays (or ``None``
    where not requested); only value columns ``[col_begin, col_end)`` are
    filled, the rest is NaN.
    """
    lib = _load()
    bf16 = np.asarray(q).dtype == np.uint16
    vt = np.uint16 if bf16 else np.float64
    gt = np.float32 if bf16 else np.float64
    q, k, v = _c(q, vt), _c(k, vt), _c(v, vt)
    g, beta = _c(g, gt), _c(beta, gt)
    init = _c(initial_state, gt)
    cu = _c(cu_seqlens, np.int32)
    T, H, dk = q.shape
    dv = v.shape[2]
    nseq = cu.shape[0] - 1
    if col_end is None:
        col_end = dv
    out = np.full((T, H, dv), np.nan) if want_out else None
    fin = np.full((nseq, H, dk, dv), np.nan) if want_final else None
    fn = lib.kda_oracle_scan_bf16 if bf16 else lib.kda_oracle_scan_f64
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), T, H, dk, dv, _ptr(cu), nseq, float(scale),
            _ptr(init), _ptr(out), _ptr(fin), 1 if erase else 0, int(col_begin), int(col_end),
            int(col_block), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle scan rejected its arguments (code {rc})")
    return out, fin


def chunked(q, k, v, g, beta, cu_seqlens, scale, initial_state=None, *, chunk=16, nthreads=0):
    """Naive fp64 chunked (WY-form) rewrite; all inputs converted to float64."""
    lib = _load()
    from kda_inputs import bf16_bits_to_f32  # input-format widening only

    def f64(a):
        a = np.asarray(a)
        if a.dtype == np.uint16:
            a = bf16_bits_to_f32(a)
        return np.ascontiguousarray(a, dtype=np.float64)

    q, k, v, g, beta = map(f64, (q, k, v, g, beta))
    init = None if initial_state is None else f64(initial_state)
    cu = _c(cu_seqlens, np.int32)
    T, H, dk = q.shape
    dv = v.shape[2]
    nseq = cu.shape[0] - 1
    out = np.full((T, H, dv), np.nan)
    fin = np.full((nseq, H, dk, dv), np.nan)
    rc = lib.kda_oracle_chunked_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), T, H, dk, dv, _ptr(cu),
                                    nseq, float(scale), _ptr(init), _ptr(out), _ptr(fin), int(chunk), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle chunked rejected its arguments (code {rc})")
    return out, fin


def unit_lower_inverse(L: np.ndarray, method: str = "substitution") -> np.ndarray:
    """(I + L)^{-1} for strictly lower-triangular L (upper part ignored)."""
    lib = _load()
    L = np.ascontiguousarray(L, dtype=np.float64)
    n = L.shape[0]
    X = np.empty((n, n), dtype=np.float64)
    m = {"substitution": 0, "doubling": 1}[method]
    rc = lib.kda_oracle_unit_lower_inverse(_ptr(L), n, _ptr(X), m)
    if rc != 0:
        raise ValueError(f"oracle inverse rejected its arguments (code {rc})")
    return X


def scan_inputs(inp, **kw):
    """Run the scan on a ``kda_inputs.KDAInputs`` batch."""
    return scan(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.scale, inp.initial_state, **kw)


def preprocess(q_raw, k_raw, g_logit, beta_logit, lower_bound=-5.0, eps=1e-6):
    """fp64 gate preprocessing (see ``kda_oracle_preprocess``): returns
    ``(q_hat, k_hat, g, beta)`` as float64 arrays from bf16-bit q/k and fp32
    logits."""
    lib = _load()
    q_raw, k_raw = _c(q_raw, np.uint16), _c(k_raw, np.uint16)
    g_logit, beta_logit = _c(g_logit, np.float32), _c(beta_logit, np.float32)
    T, H, dk = q_raw.shape
    qo, ko, go = (np.empty((T, H, dk), np.float64) for _ in range(3))
    bo = np.empty((T, H), np.float64)
    rc = lib.kda_oracle_preprocess(_ptr(q_raw), _ptr(k_raw), _ptr(g_logit), _ptr(beta_logit), T, H, dk,
                                   float(lower_bound), float(eps), _ptr(qo), _ptr(ko), _ptr(go), _ptr(bo))
    if rc != 0:
        raise ValueError(f"oracle preprocess rejected its arguments (code {rc})")
    return qo, ko, go, bo


def scan_raw_inputs(inp, lower_bound=-5.0, **kw):
    """Preprocess a batch's raw tensors (``kda_inputs.make_inputs(..., raw=True)``)
    and run the fp64 scan on the result."""
    from kda_inputs import bf16_bits_to_f32  # input-format widening only

    qh, kh, g, beta = preprocess(inp.q_raw, inp.k_raw, inp.g_logit, inp.beta_logit, lower_bound)
    v = bf16_bits_to_f32(inp.v).astype(np.float64)
    init = None if inp.initial_state is None else inp.initial_state.astype(np.float64)
    return scan(qh, kh, v, g, beta, inp.cu_seqlens, inp.scale, init, **kw)


def backward(q, k, v, g, beta, cu_seqlens, scale, dout, initial_state=None, dfinal=None, *, nthreads=0):
    """Gradients of sum(dout * o) + sum(dfinal * S_final) with respect to q, k,
    v, g, beta and the initial state (reverse mode of the token recurrence).

    Inputs as for ``scan`` (bf16 bit patterns with float32 g/beta/states and
    bf16-bit ``dout``, or all float64). Returns a dict of float64 arrays
    ``dq, dk, dv, dg, dbeta, dinit`` (``dinit`` None without an initial state).
    """
    lib = _load()
    bf16 = np.asarray(q).dtype == np.uint16
    vt = np.uint16 if bf16 else np.float64
    gt = np.float32 if bf16 else np.float64
    q, k, v, dout = _c(q, vt), _c(k, vt), _c(v, vt), _c(dout, vt)
    g, beta = _c(g, gt), _c(beta, gt)
    init, dfin = _c(initial_state, gt), _c(dfinal, gt)
    cu = _c(cu_seqlens, np.int32)
    T, H, dk = q.shape
    dv = v.shape[2]
    nseq = cu.shape[0] - 1
    res = {"dq": np.zeros((T, H, dk)), "dk": np.zeros((T, H, dk)), "dv": np.zeros((T, H, dv)),
           "dg": np.zeros((T, H, dk)), "dbeta": np.zeros((T, H)),
           "dinit": np.zeros((nseq, H, dk, dv)) if initial_state is not None else None}
    fn = lib.kda_oracle_backward_bf16 if bf16 else lib.kda_oracle_backward_f64
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), T, H, dk, dv, _ptr(cu), nseq, float(scale), _ptr(init),
            _ptr(dout), _ptr(dfin), _ptr(res["dq"]), _ptr(res["dk"]), _ptr(res["dv"]), _ptr(res["dg"]),
            _ptr(res["dbeta"]), _ptr(res["dinit"]), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle backward rejected its arguments (code {rc})")
    return res


def chunked_backward(q, k, v, g, beta, cu_seqlens, scale, dout, initial_state=None, dfinal=None, *, chunk=16):
    """The gradients ``backward`` computes, by the chunked (WY) form instead of
    the token recurrence: the derivative of the chunked rewrite step by step.

    Per chunk of C tokens, with Gamma the inclusive cumulative sum of g inside
    the chunk, E = exp(Gamma), F = exp(Gamma_last - Gamma), gamma = E_last and
    S the chunk-start state, the forward products are
        A    = strictly lower part of (k E)(k / E)^T,  L = diag(beta) A,
        M    = (I + L)^{-1},  W = M diag(beta),
        X    = V - (k E) S,   Vnew = W X,
        Aqk  = lower part (with the diagonal) of (q E)(k / E)^T,
        O    = scale ((q E) S + Aqk Vnew),
        S'   = diag(gamma) S + (k F)^T Vnew.
    The backward walks the chunks in reverse with the adjoint state dS (the
    gradient at S'): dVnew = (k F) dS + scale Aqk^T dO, dX = W^T dVnew, and
    dS <- diag(gamma) dS + scale (q E)^T dO - (k E)^T dX. Inside a chunk the
    gradients go through M (d(I + L)^{-1} = -M dL M), L = diag(beta) A and the
    two masked products, then through the decay factors into Gamma, and a
    reverse cumulative sum within the chunk turns dGamma into dg.

    Float64 numpy (all inputs float64); returns the same dict as ``backward``.
    Test infrastructure: the plan of a chunked backward, checked against the
    token-level reverse recurrence.
    """
    q, k, v, g = (np.asarray(x, np.float64) for x in (q, k, v, g))
    beta, dout = np.asarray(beta, np.float64), np.asarray(dout, np.float64)
    cu = np.asarray(cu_seqlens, np.int64)
    T, H, dk = q.shape
    dv = v.shape[2]
    nseq = cu.shape[0] - 1
    res = {"dq": np.zeros((T, H, dk)), "dk": np.zeros((T, H, dk)), "dv": np.zeros((T, H, dv)),
           "dg": np.zeros((T, H, dk)), "dbeta": np.zeros((T, H)),
           "dinit": np.zeros((nseq, H, dk, dv)) if initial_state is not None else None}
    for s in range(nseq):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        starts = list(range(t0, t1, chunk))
        for h in range(H):
            S = np.zeros((dk, dv)) if initial_state is None else np.array(initial_state[s, h], np.float64)

            def parts(a, S):
                b = min(a + chunk, t1)
                kk, qq, vv, bb = k[a:b, h], q[a:b, h], v[a:b, h], beta[a:b, h]
                Gam = np.cumsum(g[a:b, h], axis=0)
                E = np.exp(Gam)
                F = np.exp(Gam[-1] - Gam)
                gam = E[-1]
                Kd, Qd, KR, Ke = kk * E, qq * E, kk / E, kk * F
                n = b - a
                strict = np.tril(np.ones((n, n)), -1)
                lower = np.tril(np.ones((n, n)))
                A = (Kd @ KR.T) * strict
                L = bb[:, None] * A
                M = np.linalg.solve(np.eye(n) + L, np.eye(n))
                W = M * bb[None, :]
                X = vv - Kd @ S
                Vn = W @ X
                Aqk = (Qd @ KR.T) * lower
                return dict(a=a, b=b, k=kk, q=qq, beta=bb, E=E, F=F, gam=gam, Kd=Kd, Qd=Qd, KR=KR, Ke=Ke,
                            strict=strict, lower=lower, A=A, M=M, W=W, X=X, Vn=Vn, Aqk=Aqk)

            # forward: the chunk-start states
            states = []
            for a in starts:
                states.append(S)
                c = parts(a, S)
                S = c["gam"][:, None] * S + c["Ke"].T @ c["Vn"]
            # backward over the chunks in reverse
            dS = np.zeros((dk, dv)) if dfinal is None else np.array(dfinal[s, h], np.float64)
            for a, S in zip(reversed(starts), reversed(states)):
                c = parts(a, S)
                a_, b_ = c["a"], c["b"]
                dO = dout[a_:b_, h]
                dVn = c["Ke"] @ dS + scale * c["Aqk"].T @ dO
                dX = c["W"].T @ dVn
                dW = dVn @ c["X"].T
                dKd = -dX @ S.T
                dQd = scale * dO @ S.T
                dAqk = scale * (dO @ c["Vn"].T) * c["lower"]
                dKe = c["Vn"] @ dS.T
                dgam = np.sum(S * dS, axis=1)
                dS_prev = c["gam"][:, None] * dS + scale * c["Qd"].T @ dO - c["Kd"].T @ dX
                # W = M diag(beta); M = (I + L)^{-1}; L = diag(beta) A
                dM = dW * c["beta"][None, :]
                dbeta = np.sum(c["M"] * dW, axis=0)
                dL = -(c["M"].T @ dM @ c["M"].T) * c["strict"]
                dA = c["beta"][:, None] * dL
                dbeta += np.sum(c["A"] * dL, axis=1)
                # A = strict((k E)(k / E)^T), Aqk = lower((q E)(k / E)^T)
                dKd += dA @ c["KR"]
                dKR = dA.T @ c["Kd"] + dAqk.T @ c["Qd"]
                dQd += dAqk @ c["KR"]
                # back to k, q and Gamma (E = exp Gamma, KR = k exp(-Gamma), F = exp(Gamma_last - Gamma))
                E, F = c["E"], c["F"]
                res["dk"][a_:b_, h] = dKd * E + dKR / E + dKe * F
                res["dq"][a_:b_, h] = dQd * E
                dGam = (dKd * c["k"] + dQd * c["q"]) * E - dKR * c["KR"] - dKe * c["Ke"]
                dGam[-1] += np.sum(dKe * c["Ke"], axis=0) + dgam * c["gam"]
                res["dg"][a_:b_, h] = np.cumsum(dGam[::-1], axis=0)[::-1]
                res["dv"][a_:b_, h] = dX
                res["dbeta"][a_:b_, h] = dbeta
                dS = dS_prev
            if res["dinit"] is not None:
                res["dinit"][s, h] = dS
    return res

"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before touching the GPU (CPU only).

Every call here fails validation before any CUDA call, so the fake device
addresses are never dereferenced or handed to the driver. The one test that
lets a call pass validation runs only where no GPU is present (the call then
stops at the CUDA device query).
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KDA_OK, KDA_ERR_NULL, KDA_ERR_SHAPE, KDA_ERR_ALIGN = 0, 1, 2, 3
KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_CAPACITY = 4, 5, 6
KDA_ERR_DTYPE, KDA_ERR_STRIDE, KDA_ERR_DEVICE, KDA_ERR_VALUE = 7, 8, 9, 10
BF16, F32, I32 = 1, 2, 3


class Desc(ctypes.Structure):
    """Mirror of kda_tensor_t (include/kda.h)."""
    _fields_ = [("data", ctypes.c_void_p), ("ndim", ctypes.c_int32), ("dtype", ctypes.c_int),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


def desc(addr, dtype, shape, stride=None):
    d = Desc()
    d.data = addr
    d.ndim = len(shape)
    d.dtype = dtype
    if stride is None:  # contiguous
        stride, acc = [], 1
        for n in reversed(shape):
            stride.insert(0, acc)
            acc *= n
    for i, (n, s) in enumerate(zip(shape, stride)):
        d.shape[i] = n
        d.stride[i] = s
    return d


@pytest.fixture(scope="module")
def lib():
    # load the build script by path so a stale library is rebuilt before use
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "kda_build", os.path.join(ROOT, "kimi_delta_attention_26_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    build.build()
    lib = ctypes.CDLL(build.LIB)
    P = ctypes.POINTER(Desc)
    for name in ("kda_fwd", "kda_fwd_noalloc"):
        fn = getattr(lib, name)
        fn.argtypes = [P, P, P, P, P, ctypes.c_float, ctypes.c_void_p, ctypes.c_int32, P, P, P, ctypes.c_void_p]
        fn.restype = ctypes.c_int
    return lib


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert "kda_fwd" in names and "kda_fwd_noalloc" in names and len(names) >= 8
    for n in names:
        assert hasattr(lib, n), f"libkda.so does not export {n}"


def test_abi_version_and_status_strings(lib):
    lib.kda_abi_version.restype = ctypes.c_int32
    assert lib.kda_abi_version() == 5
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_status_string.argtypes = [ctypes.c_int]
    texts = {lib.kda_status_string(code) for code in range(11)}
    assert len(texts) == 11 and b"unknown status" not in texts
    assert lib.kda_status_string(99) == b"unknown status"


class Call:
    """A valid-looking problem (T tokens, H heads, N sequences) on fake
    16-byte-aligned addresses; tests override one tensor at a time."""

    def __init__(self, T=64, H=2, N=1):
        self.T, self.H, self.N = T, H, N
        self.t = {
            "q": desc(0x10000, BF16, [T, H, 128]),
            "k": desc(0x20000, BF16, [T, H, 128]),
            "v": desc(0x30000, BF16, [T, H, 128]),
            "g": desc(0x40000, F32, [T, H, 128]),
            "beta": desc(0x50000, F32, [T, H]),
            "init": None,
            "out": desc(0x60000, BF16, [T, H, 128]),
            "fin": None,
        }
        self.cu = 0x70000
        self.scale = 1.0

    def run(self, lib, fn="kda_fwd", num_seqs=None, **over):
        t = dict(self.t)
        t.update({k: v for k, v in over.items() if k in t})
        cu = over.get("cu", self.cu)
        ref = {k: (None if d is None else ctypes.byref(d)) for k, d in t.items()}
        return getattr(lib, fn)(ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"], self.scale, cu,
                                self.N if num_seqs is None else num_seqs, ref["init"], ref["out"], ref["fin"], None)


def test_path_and_slice_settings_validated(lib):
    lib.kda_set_slice_columns.argtypes = [ctypes.c_int32]
    lib.kda_set_slice_columns.restype = ctypes.c_int
    lib.kda_set_path.argtypes = [ctypes.c_int32]
    lib.kda_set_path.restype = ctypes.c_int
    for bad in (-1, 1, 8, 24, 64, 128):
        assert lib.kda_set_slice_columns(bad) == KDA_ERR_SHAPE
    for good in (16, 32, 0):
        assert lib.kda_set_slice_columns(good) == KDA_OK
    for bad in (-1, 1, 32, 128):
        assert lib.kda_set_path(bad) == KDA_ERR_SHAPE
    for good in (16, 64, 0):
        assert lib.kda_set_path(good) == KDA_OK
    lib.kda_set_time_split.argtypes = [ctypes.c_int32]
    lib.kda_set_time_split.restype = ctypes.c_int
    for bad in (-1, 3, 16):
        assert lib.kda_set_time_split(bad) == KDA_ERR_SHAPE
    for good in (1, 2, 0):
        assert lib.kda_set_time_split(good) == KDA_OK
    lib.kda_set_schedule.argtypes = [ctypes.c_int32, ctypes.c_int32]
    lib.kda_set_schedule.restype = ctypes.c_int
    for bad in ((-1, 0), (3, 0), (16, 0), (2, -1)):
        assert lib.kda_set_schedule(*bad) == KDA_ERR_SHAPE
    for good in ((1, 0), (2, 3), (0, 0)):
        assert lib.kda_set_schedule(*good) == KDA_OK


@pytest.mark.parametrize("fn", ["kda_fwd", "kda_fwd_noalloc"])
def test_rejects_missing_tensors(lib, fn):
    c = Call()
    for name in ("q", "k", "v", "g", "beta", "out"):
        assert c.run(lib, fn, **{name: None}) == KDA_ERR_NULL, name
    # a descriptor whose data pointer is NULL while T > 0
    assert c.run(lib, fn, q=desc(None, BF16, [64, 2, 128])) == KDA_ERR_NULL
    assert c.run(lib, fn, init=desc(None, F32, [1, 2, 128, 128])) == KDA_ERR_NULL


@pytest.mark.parametrize("fn", ["kda_fwd", "kda_fwd_noalloc"])
def test_rejects_wrong_dtypes(lib, fn):
    c = Call()
    assert c.run(lib, fn, q=desc(0x10000, F32, [64, 2, 128])) == KDA_ERR_DTYPE
    assert c.run(lib, fn, v=desc(0x30000, I32, [64, 2, 128])) == KDA_ERR_DTYPE
    assert c.run(lib, fn, g=desc(0x40000, BF16, [64, 2, 128])) == KDA_ERR_DTYPE
    assert c.run(lib, fn, beta=desc(0x50000, BF16, [64, 2])) == KDA_ERR_DTYPE
    assert c.run(lib, fn, out=desc(0x60000, F32, [64, 2, 128])) == KDA_ERR_DTYPE
    assert c.run(lib, fn, init=desc(0x80000, BF16, [1, 2, 128, 128])) == KDA_ERR_DTYPE
    assert c.run(lib, fn, fin=desc(0x90000, I32, [1, 2, 128, 128])) == KDA_ERR_DTYPE


@pytest.mark.parametrize("fn", ["kda_fwd", "kda_fwd_noalloc"])
def test_rejects_bad_shapes(lib, fn):
    c = Call()
    assert c.run(lib, fn, k=desc(0x20000, BF16, [63, 2, 128])) == KDA_ERR_SHAPE      # T mismatch
    assert c.run(lib, fn, v=desc(0x30000, BF16, [64, 3, 128])) == KDA_ERR_SHAPE      # H mismatch
    assert c.run(lib, fn, g=desc(0x40000, F32, [64, 2, 64])) == KDA_ERR_SHAPE        # head dim
    assert c.run(lib, fn, beta=desc(0x50000, F32, [64, 2, 1])) == KDA_ERR_SHAPE      # ndim
    assert c.run(lib, fn, q=desc(0x10000, BF16, [64, 0, 128]), k=desc(0x20000, BF16, [64, 0, 128])) == KDA_ERR_SHAPE
    assert c.run(lib, fn, init=desc(0x80000, F32, [2, 2, 128, 128])) == KDA_ERR_SHAPE  # N mismatch
    assert c.run(lib, fn, cu=None, num_seqs=2) == KDA_ERR_SHAPE
    assert c.run(lib, fn, num_seqs=0) == KDA_ERR_SHAPE
    big = Call(T=1 << 31, H=1)
    assert big.run(lib, fn) == KDA_ERR_SHAPE


@pytest.mark.parametrize("fn", ["kda_fwd", "kda_fwd_noalloc"])
def test_rejects_bad_strides(lib, fn):
    c = Call()
    T, H = 64, 2
    # innermost dimension not contiguous
    assert c.run(lib, fn, q=desc(0x10000, BF16, [T, H, 128], [H * 256, 256, 2])) == KDA_ERR_STRIDE
    # token stride not a multiple of 16 bytes
    assert c.run(lib, fn, k=desc(0x20000, BF16, [T, H, 128], [H * 128 + 4, 128, 1])) == KDA_ERR_STRIDE
    assert c.run(lib, fn, g=desc(0x40000, F32, [T, H, 128], [H * 128 + 2, 128, 1])) == KDA_ERR_STRIDE
    # zero or negative outer strides
    assert c.run(lib, fn, v=desc(0x30000, BF16, [T, H, 128], [0, 128, 1])) == KDA_ERR_STRIDE
    assert c.run(lib, fn, beta=desc(0x50000, F32, [T, H], [-H, 1])) == KDA_ERR_STRIDE
    # out rows overlapping each other
    assert c.run(lib, fn, out=desc(0x60000, BF16, [T, H, 128], [128, 64, 1])) == KDA_ERR_STRIDE
    # non-contiguous states
    assert c.run(lib, fn, init=desc(0x80000, F32, [1, H, 128, 128], [H * 128 * 128, 128 * 128, 1, 128])) == KDA_ERR_STRIDE
    assert c.run(lib, fn, fin=desc(0x90000, F32, [1, H, 128, 128], [H * 128 * 256, 128 * 256, 256, 1])) == KDA_ERR_STRIDE


@pytest.mark.parametrize("fn", ["kda_fwd", "kda_fwd_noalloc"])
def test_rejects_misaligned_pointers(lib, fn):
    c = Call()
    for name, dt, shape in (("q", BF16, [64, 2, 128]), ("k", BF16, [64, 2, 128]), ("v", BF16, [64, 2, 128]),
                            ("g", F32, [64, 2, 128]), ("out", BF16, [64, 2, 128]),
                            ("init", F32, [1, 2, 128, 128]), ("fin", F32, [1, 2, 128, 128])):
        assert c.run(lib, fn, **{name: desc(0xA0008, dt, shape)}) == KDA_ERR_ALIGN, name
    # beta is read 4 bytes at a time: 4-byte alignment suffices
    assert c.run(lib, fn, beta=desc(0xA0002, F32, [64, 2])) == KDA_ERR_ALIGN
    assert c.run(lib, fn, cu=0xB0008) == KDA_ERR_ALIGN


def test_empty_batch_may_have_null_token_pointers(lib):
    # T = 0: the token tensors are never read or written, so NULL data is fine;
    # the call then stops at the misaligned initial state
    c = Call(T=0)
    z = {n: desc(None, c.t[n].dtype, [0] + list(c.t[n].shape[1:c.t[n].ndim])) for n in ("q", "k", "v", "g", "beta", "out")}
    assert c.run(lib, init=desc(0xA0008, F32, [1, 2, 128, 128]), **z) == KDA_ERR_ALIGN


def test_noalloc_capacity_rejected_before_any_gpu_work(lib):
    H = 32 // 2 + 1  # two sequences: 34 (sequence, head) pairs > 32
    c = Call(T=64, H=H, N=2)
    assert c.run(lib, "kda_fwd_noalloc") == KDA_ERR_CAPACITY


def test_strided_views_pass_validation():
    """q, k, v as slices of one fused [T, H, 3 * 128] projection and beta as a
    column of a wider matrix are accepted (checked on a host without a GPU,
    where the call stops at the device query after validation)."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("validation-only check; needs a host without a GPU")
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "kda_build", os.path.join(ROOT, "kimi_delta_attention_26_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    lib = ctypes.CDLL(build.build())
    P = ctypes.POINTER(Desc)
    lib.kda_fwd.argtypes = [P, P, P, P, P, ctypes.c_float, ctypes.c_void_p, ctypes.c_int32, P, P, P, ctypes.c_void_p]
    lib.kda_fwd.restype = ctypes.c_int
    T, H = 64, 2
    c = Call(T, H)
    fused = [H * 384, 384, 1]
    rc = c.run(lib, q=desc(0x100000, BF16, [T, H, 128], fused), k=desc(0x100100, BF16, [T, H, 128], fused),
               v=desc(0x100200, BF16, [T, H, 128], fused), beta=desc(0x50000, F32, [T, H], [4 * H, 4]),
               out=desc(0x60000, BF16, [T, H, 128], [128, T * 128, 1]))   # head-major output
    assert rc == KDA_ERR_CUDA  # validation passed; no device to run on


def test_device_status_and_wait_counter_reject_null(lib):
    lib.kda_wait_timeouts.argtypes = [ctypes.c_void_p, ctypes.c_int32]
    lib.kda_wait_timeouts.restype = ctypes.c_int
    lib.kda_device_status.argtypes = [ctypes.c_void_p, ctypes.c_int32]
    lib.kda_device_status.restype = ctypes.c_int
    assert lib.kda_wait_timeouts(None, 0) == KDA_ERR_NULL
    assert lib.kda_device_status(None, 0) == KDA_ERR_NULL


# ------------------------------------------------------------------ decode
class DecodeCall:
    """A valid-looking decode step (B requests, H heads, P state slots) on fake
    16-byte-aligned addresses; tests override one argument at a time."""

    def __init__(self, B=4, H=2, P=4):
        self.B, self.H, self.P = B, H, P
        self.t = {
            "q": desc(0x10000, BF16, [B, H, 128]),
            "k": desc(0x20000, BF16, [B, H, 128]),
            "v": desc(0x30000, BF16, [B, H, 128]),
            "g": desc(0x40000, F32, [B, H, 128]),
            "beta": desc(0x50000, F32, [B, H]),
            "state": desc(0x100000, F32, [P, H, 128, 128]),
            "out": desc(0x60000, BF16, [B, H, 128]),
        }
        self.idx = None

    def run(self, lib, **over):
        P = ctypes.POINTER(Desc)
        lib.kda_decode.argtypes = [P, P, P, P, P, ctypes.c_float, P, ctypes.c_void_p, P, ctypes.c_void_p]
        lib.kda_decode.restype = ctypes.c_int
        t = dict(self.t)
        t.update({k: v for k, v in over.items() if k in t})
        idx = over.get("idx", self.idx)
        ref = {k: (None if d is None else ctypes.byref(d)) for k, d in t.items()}
        return lib.kda_decode(ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"], 1.0, ref["state"], idx,
                              ref["out"], None)


def test_decode_rejects_bad_arguments(lib):
    c = DecodeCall()
    for name in c.t:
        assert c.run(lib, **{name: None}) == KDA_ERR_NULL, name
    # dtypes
    assert c.run(lib, q=desc(0x10000, F32, [4, 2, 128])) == KDA_ERR_DTYPE
    assert c.run(lib, g=desc(0x40000, BF16, [4, 2, 128])) == KDA_ERR_DTYPE
    assert c.run(lib, state=desc(0x100000, BF16, [4, 2, 128, 128])) == KDA_ERR_DTYPE
    assert c.run(lib, out=desc(0x60000, F32, [4, 2, 128])) == KDA_ERR_DTYPE
    # shapes: batch or heads disagree, head dim, state dims, too few slots without indices
    assert c.run(lib, k=desc(0x20000, BF16, [3, 2, 128])) == KDA_ERR_SHAPE
    assert c.run(lib, beta=desc(0x50000, F32, [4, 3])) == KDA_ERR_SHAPE
    assert c.run(lib, v=desc(0x30000, BF16, [4, 2, 64])) == KDA_ERR_SHAPE
    assert c.run(lib, state=desc(0x100000, F32, [4, 2, 128, 64])) == KDA_ERR_SHAPE
    assert c.run(lib, state=desc(0x100000, F32, [4, 3, 128, 128])) == KDA_ERR_SHAPE
    assert c.run(lib, state=desc(0x100000, F32, [3, 2, 128, 128])) == KDA_ERR_SHAPE
    # strides: non-unit inner stride, a non-contiguous state
    assert c.run(lib, q=desc(0x10000, BF16, [4, 2, 128], [512, 256, 2])) == KDA_ERR_STRIDE
    assert c.run(lib, state=desc(0x100000, F32, [4, 2, 128, 128], [2 * 128 * 256, 128 * 256, 256, 1])) \
        == KDA_ERR_STRIDE
    # alignment: token tensors, state, indices
    assert c.run(lib, k=desc(0x20008, BF16, [4, 2, 128])) == KDA_ERR_ALIGN
    assert c.run(lib, state=desc(0x100004, F32, [4, 2, 128, 128])) == KDA_ERR_ALIGN
    assert c.run(lib, idx=0x70002) == KDA_ERR_ALIGN


def test_decode_accepts_a_small_pool_with_indices(lib):
    """With state_indices, the pool may hold fewer slots than requests; the
    call then passes validation (and stops at the device query without a GPU)."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("would launch on the fake addresses")
    c = DecodeCall(B=4, H=2, P=2)
    assert c.run(lib, idx=0x70000) in (KDA_ERR_CUDA, KDA_ERR_UNSUPPORTED)
    assert c.run(lib) == KDA_ERR_SHAPE


# ------------------------------------------------------------ fused gate
def test_fused_rejects_lower_bound_and_bad_tensors(lib):
    P = ctypes.POINTER(Desc)
    lib.kda_fwd_fused.argtypes = [P, P, P, P, P, ctypes.c_float, ctypes.c_float, ctypes.c_void_p, ctypes.c_int32,
                                  P, P, P, ctypes.c_void_p]
    lib.kda_fwd_fused.restype = ctypes.c_int
    c = Call()

    def run(lb, **over):
        t = dict(c.t)
        t.update(over)
        ref = {k: (None if d is None else ctypes.byref(d)) for k, d in t.items()}
        return lib.kda_fwd_fused(ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"], 1.0, lb, c.cu, 1, ref["init"],
                                 ref["out"], ref["fin"], None)

    for lb in (-5.5, 0.0, 0.5, float("nan"), float("-inf")):
        assert run(lb) == KDA_ERR_VALUE, lb
    assert run(-5.0, q=None) == KDA_ERR_NULL
    assert run(-5.0, g=desc(0x40000, BF16, [64, 2, 128])) == KDA_ERR_DTYPE
    assert run(-2.0, beta=desc(0x50000, F32, [64, 3])) == KDA_ERR_SHAPE
    assert run(-1.0, k=desc(0x20000, BF16, [64, 2, 128], [256, 128, 2])) == KDA_ERR_STRIDE


# -------------------------------------------------------------- backward
def test_bwd_rejects_bad_arguments(lib):
    P = ctypes.POINTER(Desc)
    lib.kda_bwd.argtypes = [P, P, P, P, P, ctypes.c_float, ctypes.c_void_p, ctypes.c_int32, P, P, P, P, P, P, P, P, P,
                            ctypes.c_void_p]
    lib.kda_bwd.restype = ctypes.c_int
    T, H = 64, 2
    base = {
        "q": desc(0x10000, BF16, [T, H, 128]), "k": desc(0x20000, BF16, [T, H, 128]),
        "v": desc(0x30000, BF16, [T, H, 128]), "g": desc(0x40000, F32, [T, H, 128]),
        "beta": desc(0x50000, F32, [T, H]), "init": None, "dout": desc(0x60000, BF16, [T, H, 128]), "dfin": None,
        "dq": desc(0x100000, F32, [T, H, 128]), "dk": desc(0x200000, F32, [T, H, 128]),
        "dv": desc(0x300000, F32, [T, H, 128]), "dg": desc(0x400000, F32, [T, H, 128]),
        "dbeta": desc(0x500000, F32, [T, H]), "dinit": None,
    }

    def run(**over):
        t = dict(base)
        t.update(over)
        r = {n: (None if d is None else ctypes.byref(d)) for n, d in t.items()}
        return lib.kda_bwd(r["q"], r["k"], r["v"], r["g"], r["beta"], 1.0, 0x70000, 1, r["init"], r["dout"], r["dfin"],
                           r["dq"], r["dk"], r["dv"], r["dg"], r["dbeta"], r["dinit"], None)

    for name in ("q", "dout", "dq", "dk", "dv", "dg", "dbeta"):
        assert run(**{name: None}) == KDA_ERR_NULL, name
    assert run(dout=desc(0x60000, F32, [T, H, 128])) == KDA_ERR_DTYPE
    assert run(dq=desc(0x100000, BF16, [T, H, 128])) == KDA_ERR_DTYPE
    assert run(dbeta=desc(0x500000, BF16, [T, H])) == KDA_ERR_DTYPE
    assert run(dk=desc(0x200000, F32, [T, H, 64])) == KDA_ERR_SHAPE
    assert run(dbeta=desc(0x500000, F32, [T, H + 1])) == KDA_ERR_SHAPE
    assert run(dout=desc(0x60000, BF16, [T + 1, H, 128])) == KDA_ERR_SHAPE
    # gradients must be contiguous; dout may be strided like the inputs
    assert run(dg=desc(0x400000, F32, [T, H, 128], [H * 256, 256, 1])) == KDA_ERR_STRIDE
    assert run(dbeta=desc(0x500000, F32, [T, H], [2 * H, 2])) == KDA_ERR_STRIDE
    assert run(dq=desc(0x100004, F32, [T, H, 128])) == KDA_ERR_ALIGN
    assert run(dinit=desc(0x600000, F32, [1, H, 128, 64])) == KDA_ERR_SHAPE
    assert run(dfin=desc(0x600000, BF16, [1, H, 128, 128])) == KDA_ERR_DTYPE

"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments with the documented codes before
touching the device."""
import ctypes
import os
import re

import pytest

from exact_io_aware_78_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "exactattn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|const char\*|void)\s+(attn_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib(lib_path):
    return B.load_library(lib_path)


def test_header_declares_the_boundary():
    assert declared_functions() == sorted(
        ["attn_fwd", "attn_get_last_error", "attn_status_string", "attn_set_option", "attn_shutdown",
         "attn_version", "attn_fwd_fp32_noalloc", "attn_fwd_decode", "attn_fwd_masked", "attn_bwd", "attn_bwd_masked"])


def declared_constants():
    """Every EA_* enumerator of the header with its value."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for body in re.findall(r"enum\s*\{(.*?)\}", text, flags=re.S):
        for name, value in re.findall(r"(EA_\w+)\s*=\s*(-?\d+)", body):
            out[name] = int(value)
    return out


def test_binding_constants_match_the_header():
    """Element types, status codes and options: the Python binding carries
    exactly the header's values, so the two cannot drift apart."""
    consts = declared_constants()
    assert len(consts) >= 16, consts  # 3 element types, 8 status codes, 5 options
    for name, value in consts.items():
        assert getattr(B, name) == value, (name, getattr(B, name, None), value)
    m = re.search(r"#define\s+EA_NOALLOC_SCRATCH_BYTES\s+\((\d+)u \* (\d+)u \* (\d+)u\)", open(HEADER).read())
    assert m and int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == 16 * 1024 * 1024


def test_library_exports_every_declared_symbol(lib_path):
    raw = ctypes.CDLL(lib_path)
    for name in declared_functions():
        assert hasattr(raw, name), name
    # and the binding wraps exactly those names
    assert sorted(B._SIGNATURES) == declared_functions()


def test_version_and_status_strings(lib):
    assert lib.attn_version() == 10000
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        s = B.status_string(code)
        assert s.startswith("EA_")
    assert B.status_string(123) == "unknown status"


def test_options_validation(lib):
    assert lib.attn_set_option(B.EA_OPT_WAIT_TIMEOUT_NS, 10) == B.EA_EINVAL
    assert lib.attn_set_option(B.EA_OPT_SCHEDULE_ORDER, 3) == B.EA_EINVAL
    assert lib.attn_set_option(B.EA_OPT_SCHEDULE_ORDER, -1) == B.EA_EINVAL
    assert lib.attn_set_option(B.EA_OPT_MAX_CTAS, -1) == B.EA_EINVAL
    assert lib.attn_set_option(99, 0) == B.EA_EINVAL
    assert lib.attn_set_option(B.EA_OPT_SCHEDULE_ORDER, 0) == B.EA_OK
    assert lib.attn_set_option(B.EA_OPT_WAIT_TIMEOUT_NS, 2_000_000_000) == B.EA_OK
    assert lib.attn_set_option(B.EA_OPT_MAX_CTAS, 0) == B.EA_OK
    assert lib.attn_set_option(B.EA_OPT_ITEM_DEAL, 2) == B.EA_EINVAL
    assert lib.attn_set_option(B.EA_OPT_ITEM_DEAL, -1) == B.EA_EINVAL
    assert lib.attn_set_option(B.EA_OPT_ITEM_DEAL, 1) == B.EA_OK
    assert lib.attn_set_option(B.EA_OPT_ITEM_DEAL, 0) == B.EA_OK
    assert lib.attn_set_option(6, 0) == B.EA_EINVAL


# Fake but 16-byte-aligned addresses: every check below fails before any
# device access, so no GPU is needed and nothing is dereferenced.
P = 1 << 20


def call(lib, q=P, k=P, v=P, o=P, lse=P, B_=1, Hq=2, Hkv=1, N=128, d=128, causal=1, window=0, scale=0.125,
         dtype=B.EA_BF16, qs=None, ks=None, vs=None):
    return lib.attn_fwd(q, k, v, o, lse, B_, Hq, Hkv, N, d, causal, window, scale, dtype, qs, ks, vs, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), B.EA_EINVAL),
    (dict(lse=None), B.EA_EINVAL),
    (dict(B_=0), B.EA_EINVAL),
    (dict(N=0), B.EA_EINVAL),
    (dict(N=-5), B.EA_EINVAL),
    (dict(Hq=3, Hkv=2), B.EA_EINVAL),
    (dict(Hkv=0), B.EA_EINVAL),
    (dict(causal=2), B.EA_EINVAL),
    (dict(scale=0.0), B.EA_EINVAL),
    (dict(scale=-1.0), B.EA_EINVAL),
    (dict(scale=float("inf")), B.EA_EINVAL),
    (dict(scale=float("nan")), B.EA_EINVAL),
    (dict(dtype=7), B.EA_EINVAL),
    (dict(dtype=B.EA_FP8_E4M3), B.EA_EINVAL),                    # fp8 needs scales
    (dict(qs=P, ks=P, vs=P), B.EA_EINVAL),                       # scales only with fp8
    (dict(dtype=B.EA_FP8_E4M3, qs=P, ks=None, vs=P), B.EA_EINVAL),
    (dict(d=96), B.EA_EUNSUPPORTED),
    (dict(d=256), B.EA_EUNSUPPORTED),
    (dict(dtype=B.EA_FP32, d=128), B.EA_EUNSUPPORTED),
    (dict(dtype=B.EA_FP8_E4M3, d=64, qs=P, ks=P, vs=P), None),   # valid sizes: reaches the device step
    (dict(q=P + 8), B.EA_EALIGN),
    (dict(o=P + 2), B.EA_EALIGN),
    (dict(lse=P + 2), B.EA_EALIGN),
    (dict(Hq=1 << 16, Hkv=1 << 16, N=1 << 15), B.EA_EINVAL),     # Hq * N >= 2^31
])
def test_argument_errors(lib, kw, code):
    rc = call(lib, **kw)
    if code is None:
        # argument checks passed; without a GPU the device step reports a CUDA error
        assert rc in (B.EA_ECUDA, B.EA_EUNSUPPORTED)
    else:
        assert rc == code


def call_masked(lib, lo=P, hi=P, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B_=1, Hq=2, Hkv=1, N=128, d=128, causal=1, window=0, scale=0.125,
             dtype=B.EA_BF16, qs=None, ks=None, vs=None)
    a.update(kw)
    return lib.attn_fwd_masked(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B_"], a["Hq"], a["Hkv"], a["N"], a["d"],
                               a["causal"], a["window"], lo, hi, a["scale"], a["dtype"], a["qs"], a["ks"], a["vs"],
                               None)


@pytest.mark.parametrize("kw,code", [
    (dict(lo=None), B.EA_EINVAL),
    (dict(hi=None), B.EA_EINVAL),
    (dict(lo=P + 2), B.EA_EALIGN),
    (dict(hi=P + 1), B.EA_EALIGN),
    (dict(q=None), B.EA_EINVAL),                  # the checks of attn_fwd apply too
    (dict(causal=2), B.EA_EINVAL),
    (dict(d=96), B.EA_EUNSUPPORTED),
    (dict(), None),                                # valid: reaches the device step
])
def test_masked_argument_errors(lib, kw, code):
    rc = call_masked(lib, **kw)
    if code is None:
        assert rc in (B.EA_ECUDA, B.EA_EUNSUPPORTED)
    else:
        assert rc == code


def call_bwd(lib, ptrs=None, B_=1, Hq=2, Hkv=1, N=128, d=128, causal=1, window=0, scale=0.125, dtype=B.EA_BF16):
    ptrs = ptrs or {}
    names = ["q", "k", "v", "o", "lse", "do", "dq", "dk", "dv"]
    args = [ptrs.get(n, P) for n in names]
    return lib.attn_bwd(*args, B_, Hq, Hkv, N, d, causal, window, scale, dtype, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ptrs={"do": None}), B.EA_EINVAL),
    (dict(ptrs={"dk": None}), B.EA_EINVAL),
    (dict(N=0), B.EA_EINVAL),
    (dict(Hq=3, Hkv=2), B.EA_EINVAL),
    (dict(causal=5), B.EA_EINVAL),
    (dict(scale=float("nan")), B.EA_EINVAL),
    (dict(dtype=11), B.EA_EINVAL),
    (dict(dtype=B.EA_FP8_E4M3), B.EA_EUNSUPPORTED),
    (dict(dtype=B.EA_FP32, d=64), B.EA_EUNSUPPORTED),
    (dict(d=96), B.EA_EUNSUPPORTED),
    (dict(ptrs={"dq": P + 8}), B.EA_EALIGN),
    (dict(ptrs={"lse": P + 2}), B.EA_EALIGN),
    (dict(Hq=1 << 16, Hkv=1 << 16, N=1 << 15), B.EA_EINVAL),
    (dict(), None),
])
def test_backward_argument_errors(lib, kw, code):
    rc = call_bwd(lib, **kw)
    if code is None:
        assert rc in (B.EA_ECUDA, B.EA_EUNSUPPORTED)
    else:
        assert rc == code


@pytest.mark.parametrize("lo,hi,code", [(None, P, B.EA_EINVAL), (P, None, B.EA_EINVAL), (P + 2, P, B.EA_EALIGN),
                                         (P, P, None)])
def test_backward_masked_argument_errors(lib, lo, hi, code):
    args = [P] * 9
    rc = lib.attn_bwd_masked(*args, 1, 2, 1, 128, 128, 1, 0, lo, hi, 0.125, B.EA_BF16, None)
    if code is None:
        assert rc in (B.EA_ECUDA, B.EA_EUNSUPPORTED)
    else:
        assert rc == code


def test_valid_call_without_gpu_reports_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert call(lib) == B.EA_ECUDA


def test_python_binding_rejects_bad_layouts():
    import torch
    q = torch.zeros(1, 8, 2, 64)
    with pytest.raises(ValueError):
        B.attn_fwd(q, q, q, q, torch.zeros(1, 2, 8))          # CPU tensors
    r = torch.zeros(1, 8, dtype=torch.int32)
    with pytest.raises(ValueError):
        B.attn_fwd_masked(q, q, q, q, torch.zeros(1, 2, 8), r, r)


def call_decode(lib, q=P, k=P, v=P, o=P, lse=P, B_=1, Hq=8, Hkv=2, Nq=1, Nk=4096, d=128, causal=1, window=0,
                scale=0.125, dtype=B.EA_BF16, splits=0):
    return lib.attn_fwd_decode(q, k, v, o, lse, B_, Hq, Hkv, Nq, Nk, d, causal, window, scale, dtype, splits, None)


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), B.EA_EINVAL),
    (dict(Nq=0), B.EA_EINVAL),
    (dict(Nk=0), B.EA_EINVAL),
    (dict(Nq=5, Nk=4), B.EA_EINVAL),                     # more new queries than cached keys
    (dict(Hq=6, Hkv=4), B.EA_EINVAL),
    (dict(causal=3), B.EA_EINVAL),
    (dict(scale=0.0), B.EA_EINVAL),
    (dict(splits=-1), B.EA_EINVAL),
    (dict(dtype=9), B.EA_EINVAL),
    (dict(dtype=B.EA_FP8_E4M3), B.EA_EUNSUPPORTED),
    (dict(dtype=B.EA_FP32), B.EA_EUNSUPPORTED),
    (dict(d=96), B.EA_EUNSUPPORTED),
    (dict(Hq=16, Hkv=2, Nq=2, splits=3), B.EA_EUNSUPPORTED),   # 16 rows per KV head > 8 (CUDA-core kernel)
    (dict(Hq=16, Hkv=1, Nq=3), B.EA_EUNSUPPORTED),             # 48 rows per KV head > 32 (tensor-core kernel)
    (dict(Hq=16, Hkv=2, Nq=2), None),                          # 16 rows: the tensor-core kernel takes them
    (dict(o=P + 8), B.EA_EALIGN),
    (dict(lse=P + 2), B.EA_EALIGN),
    (dict(), None),                                       # valid: reaches the device step
])
def test_decode_argument_errors(lib, kw, code):
    rc = call_decode(lib, **kw)
    if code is None:
        assert rc in (B.EA_ECUDA, B.EA_EUNSUPPORTED)
    else:
        assert rc == code


def test_python_decode_binding_rejects_bad_layouts():
    import torch
    q = torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        B.attn_fwd_decode(q, q, q, q, torch.zeros(1, 8, 1))     # CPU tensors

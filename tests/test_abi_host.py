"""Host-side checks of the C ABI: the library builds for sm_100a, loads
without a GPU, exports every symbol ``include/fa.h`` declares, and rejects
bad arguments before touching the device.  No call here reaches a kernel
launch."""
import ctypes
import os
import re

import pytest

from exact_io_aware_86_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")
FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails validation first


@pytest.fixture(scope="module")
def lib():
    build.ensure_built()
    return api.load_library()


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("fa_prefill", "fa_prefill_ex", "fa_decode_paged", "fa_decode_paged_append",
              "fa_decode_append_workspace_size", "fa_decode_workspace_size",
              "fa_decode_auto_splits", "fa_get_error_string", "fa_get_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"declared but not exported: {missing}"


def test_library_is_built_for_sm100a():
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.NVCC_FLAGS)


def test_error_strings(lib):
    for code in range(6):
        assert api.error_string(code)
    assert api.error_string(99) == "unknown status"


def _prefill(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, cu=FAKE, B=1, Hq=4, Hkv=2, d=128,
             causal=1, scale=0.0, stream=None, T=16, maxlen=16)
    a.update(kw)
    return lib.fa_prefill(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu"], a["B"], a["Hq"],
                          a["Hkv"], a["d"], a["causal"], a["scale"], a["stream"], a["T"],
                          a["maxlen"])


def test_prefill_argument_checks(lib):
    assert _prefill(lib, q=None) == api.FA_ERR_INVALID_ARG
    assert _prefill(lib, cu=None) == api.FA_ERR_INVALID_ARG
    assert _prefill(lib, Hq=6, Hkv=4) == api.FA_ERR_INVALID_ARG      # Hq % Hkv
    assert _prefill(lib, B=-1) == api.FA_ERR_INVALID_ARG
    assert _prefill(lib, T=-5) == api.FA_ERR_INVALID_ARG
    assert _prefill(lib, q=ctypes.c_void_p(0x1008)) == api.FA_ERR_INVALID_ARG  # misaligned
    assert _prefill(lib, d=96) == api.FA_ERR_UNSUPPORTED
    assert _prefill(lib, d=256) == api.FA_ERR_UNSUPPORTED
    assert _prefill(lib, maxlen=4096 * 256 + 1) == api.FA_ERR_UNSUPPORTED
    assert _prefill(lib, Hq=65536, Hkv=1) == api.FA_ERR_UNSUPPORTED   # head index is 16-bit
    # empty problems are a no-op (no launch)
    assert _prefill(lib, B=0) == api.FA_OK
    assert _prefill(lib, T=0) == api.FA_OK


def _prefill_ex(lib, wl=-1, wr=-1, cap=0.0, alibi=None, stride=0, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, cu=FAKE, B=1, Hq=4, Hkv=2, d=128,
             causal=1, scale=0.0, stream=None, T=16, maxlen=16)
    a.update(kw)
    return lib.fa_prefill_ex(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu"], a["B"], a["Hq"],
                             a["Hkv"], a["d"], a["causal"], a["scale"], a["stream"], a["T"],
                             a["maxlen"], wl, wr, cap, alibi, stride)


def test_prefill_ex_argument_checks(lib):
    assert _prefill_ex(lib, cap=-0.5) == api.FA_ERR_INVALID_ARG
    assert _prefill_ex(lib, cap=float("nan")) == api.FA_ERR_INVALID_ARG
    assert _prefill_ex(lib, cap=float("inf")) == api.FA_ERR_INVALID_ARG
    assert _prefill_ex(lib, alibi=FAKE, stride=-1) == api.FA_ERR_INVALID_ARG
    assert _prefill_ex(lib, alibi=ctypes.c_void_p(0x1002)) == api.FA_ERR_INVALID_ARG  # misaligned
    assert _prefill_ex(lib, q=None, wl=4) == api.FA_ERR_INVALID_ARG
    assert _prefill_ex(lib, d=96, wl=4) == api.FA_ERR_UNSUPPORTED
    # empty problems are a no-op whatever the variant
    assert _prefill_ex(lib, B=0, wl=3, wr=2, cap=30.0, alibi=FAKE, stride=4) == api.FA_OK


def _prefill_fp8(lib, qd=1.0, kd=1.0, vd=1.0, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, cu=FAKE, B=1, Hq=4, Hkv=2, d=128,
             causal=1, scale=0.0, stream=None, T=16, maxlen=16)
    a.update(kw)
    return lib.fa_prefill_fp8(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu"], a["B"],
                              a["Hq"], a["Hkv"], a["d"], a["causal"], a["scale"], qd, kd, vd,
                              a["stream"], a["T"], a["maxlen"])


def test_prefill_fp8_argument_checks(lib):
    assert _prefill_fp8(lib, v=None) == api.FA_ERR_INVALID_ARG
    assert _prefill_fp8(lib, Hq=6, Hkv=4) == api.FA_ERR_INVALID_ARG
    assert _prefill_fp8(lib, o=ctypes.c_void_p(0x1004)) == api.FA_ERR_INVALID_ARG  # misaligned
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        assert _prefill_fp8(lib, qd=bad) == api.FA_ERR_INVALID_ARG
        assert _prefill_fp8(lib, kd=bad) == api.FA_ERR_INVALID_ARG
        assert _prefill_fp8(lib, vd=bad) == api.FA_ERR_INVALID_ARG
    assert _prefill_fp8(lib, d=64) == api.FA_ERR_UNSUPPORTED           # e4m3 path is d = 128
    assert _prefill_fp8(lib, Hq=65536, Hkv=1) == api.FA_ERR_UNSUPPORTED
    assert _prefill_fp8(lib, maxlen=4096 * 256 + 1) == api.FA_ERR_UNSUPPORTED
    assert _prefill_fp8(lib, B=0) == api.FA_OK
    assert _prefill_fp8(lib, T=0) == api.FA_OK


def _decode(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, bt=FAKE, sl=FAKE, ps=16, S=0, o=FAKE, stream=None, B=2,
             Hq=32, Hkv=8, d=128, maxb=4, npages=8, scale=0.0, lse=None, ws=None, wsb=0)
    a.update(kw)
    return lib.fa_decode_paged(a["q"], a["k"], a["v"], a["bt"], a["sl"], a["ps"], a["S"], a["o"],
                               a["stream"], a["B"], a["Hq"], a["Hkv"], a["d"], a["maxb"],
                               a["npages"], a["scale"], a["lse"], a["ws"], a["wsb"])


def test_decode_argument_checks(lib):
    assert _decode(lib, bt=None) == api.FA_ERR_INVALID_ARG
    assert _decode(lib, ps=0) == api.FA_ERR_INVALID_ARG
    assert _decode(lib, S=-1) == api.FA_ERR_INVALID_ARG
    assert _decode(lib, Hq=12, Hkv=8) == api.FA_ERR_INVALID_ARG
    assert _decode(lib, ws=ctypes.c_void_p(0x1010)) == api.FA_ERR_INVALID_ARG  # not 256-aligned
    assert _decode(lib, d=80) == api.FA_ERR_UNSUPPORTED
    # explicit workspace that is too small
    need = lib.fa_decode_workspace_size(2, 32, 128, 4)
    assert _decode(lib, S=4, ws=ctypes.c_void_p(0x10000), wsb=need - 1) == api.FA_ERR_INVALID_ARG
    assert _decode(lib, B=0) == api.FA_OK


def _append(lib, **kw):
    a = dict(q=FAKE, kn=FAKE, vn=FAKE, k=FAKE, v=FAKE, bt=FAKE, cs=FAKE, ps=16, S=0, o=FAKE,
             stream=None, B=2, Hq=32, Hkv=8, d=128, maxb=4, npages=8, scale=0.0, lse=None,
             cos=None, sin=None, maxpos=0, rd=0, inter=0, ws=None, wsb=0)
    a.update(kw)
    return lib.fa_decode_paged_append(a["q"], a["kn"], a["vn"], a["k"], a["v"], a["bt"], a["cs"],
                                      a["ps"], a["S"], a["o"], a["stream"], a["B"], a["Hq"],
                                      a["Hkv"], a["d"], a["maxb"], a["npages"], a["scale"],
                                      a["lse"], a["cos"], a["sin"], a["maxpos"], a["rd"],
                                      a["inter"], a["ws"], a["wsb"])


def test_decode_append_argument_checks(lib):
    assert _append(lib, kn=None) == api.FA_ERR_INVALID_ARG
    assert _append(lib, cos=FAKE) == api.FA_ERR_INVALID_ARG                    # cos without sin
    assert _append(lib, cos=FAKE, sin=FAKE, maxpos=10, rd=3) == api.FA_ERR_INVALID_ARG   # odd
    assert _append(lib, cos=FAKE, sin=FAKE, maxpos=10, rd=130) == api.FA_ERR_INVALID_ARG  # > d
    assert _append(lib, cos=FAKE, sin=FAKE, maxpos=0, rd=64) == api.FA_ERR_INVALID_ARG
    assert _append(lib, d=96) == api.FA_ERR_UNSUPPORTED
    need = lib.fa_decode_append_workspace_size(2, 32, 128, 4)
    assert need == (lib.fa_decode_workspace_size(2, 32, 128, 4) + 2 * 32 * 128 * 2 + 256)
    assert _append(lib, S=4, ws=ctypes.c_void_p(0x10000), wsb=need - 1) == api.FA_ERR_INVALID_ARG
    assert _append(lib, B=0) == api.FA_OK


def test_decode_workspace_is_linear_in_splits_not_context(lib):
    """The split workspace holds fp32 partial outputs and LSEs,
    B*Hq*S*(d+1) floats, plus B+1 range counts (each part rounded to
    256-byte blocks), independent of the context length -- nothing of size
    N^2 (or even N) is ever allocated."""
    for B, Hq, d, S in ((64, 32, 128, 19), (2, 32, 128, 256), (1, 1, 64, 2)):
        n = lib.fa_decode_workspace_size(B, Hq, d, S)
        assert n >= B * Hq * S * (d + 1) * 4 + (B + 1) * 4
        assert n <= B * Hq * S * (d + 1) * 4 + (B + 1) * 4 + 768
    assert lib.fa_decode_workspace_size(64, 32, 128, 1) == 0


def test_auto_splits_rule(lib):
    """Automatic ranges span c pages, chosen for whole rounds of ranges per
    SM with little partial-output traffic (at least 256 tokens, at most
    max_blocks); the call returns ceil(max_blocks / c)."""
    # 64 requests x 2048 pages of 16 tokens: c = 69 pages, 30 ranges at most,
    # 64 * 30 = 1920 ranges = 12.97 rounds of 148
    assert lib.fa_decode_auto_splits(64, 32, 8, 2048, 16, 148) == 30
    # 2 requests x 2048 pages of 64 tokens: c = 28, 2 * 74 = 148 ranges, one round
    assert lib.fa_decode_auto_splits(2, 32, 8, 2048, 64, 148) == 74
    # short contexts or many requests: one range per request
    assert lib.fa_decode_auto_splits(2, 32, 8, 3, 16, 148) == 1
    assert lib.fa_decode_auto_splits(10000, 32, 8, 64, 16, 148) == 1
    # invalid shapes fall back to one range
    assert lib.fa_decode_auto_splits(2, 12, 8, 64, 16, 148) == 1


def test_python_binding_rejects_host_tensors():
    import torch
    q = torch.zeros(4, 2, 64, dtype=torch.bfloat16)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    with pytest.raises(ValueError):
        api.fa_prefill(q, q[:, :1], q[:, :1], q, None, cu, True)


@pytest.mark.parametrize("which", ["fa_decode_paged", "fa_decode_paged_noalloc",
                                   "fa_decode_paged_append"])
def test_decode_wrappers_check_the_output_shapes(which):
    """The decode kernels write B*Hq*d elements of o and B*Hq of lse, so each
    decode wrapper refuses an o or lse of another shape before any call
    (a smaller buffer would be written past its end)."""
    import torch
    B, Hq, Hkv, d, ps = 3, 8, 2, 64, 16
    bf = torch.bfloat16
    q = torch.zeros(B, Hq, d, dtype=bf)
    kp = torch.zeros(4, ps, Hkv, d, dtype=bf)
    bt = torch.zeros(B, 2, dtype=torch.int32)
    sl = torch.zeros(B, dtype=torch.int32)
    kn = torch.zeros(B, Hkv, d, dtype=bf)
    fn = getattr(api, which)

    def call(o, lse):
        if which == "fa_decode_paged_append":
            fn(q, kn, kn, kp, kp, bt, sl, 0, o, lse)
        else:
            fn(q, kp, kp, bt, sl, 0, o, lse)

    good_o = torch.zeros(B, Hq, d, dtype=bf)
    good_lse = torch.zeros(B, Hq, dtype=torch.float32)
    for bad_o in (torch.zeros(B, Hq, d // 2, dtype=bf), torch.zeros(B - 1, Hq, d, dtype=bf),
                  torch.zeros(B, Hq - 1, d, dtype=bf)):
        with pytest.raises(ValueError, match="o must have shape"):
            call(bad_o, good_lse)
    for bad_lse in (torch.zeros(B, Hq - 1, dtype=torch.float32),
                    torch.zeros(Hq, B, dtype=torch.float32)):
        with pytest.raises(ValueError, match="lse must have shape"):
            call(good_o, bad_lse)
    # right shapes: refused only because these are host tensors
    with pytest.raises(ValueError, match="CUDA device"):
        call(good_o, good_lse)

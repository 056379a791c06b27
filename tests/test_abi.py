"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

The library must load, export every function include/gdn.h declares, and
reject invalid calls with the documented status before touching the device.
"""
import ctypes
import os
import re

import pytest
import torch

from gated_deltanet_recurrence_rule_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from gated_deltanet_recurrence_rule_b200 import build

    build.build()
    return api.load()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "gdn_prefill" in names and "gdn_decode_step" in names
    for name in names:
        assert hasattr(lib, name), f"libgdn.so does not export {name}"


def test_status_strings(lib):
    for code in range(0, 7):
        assert api.status_string(code).startswith("GDN_")
    assert api.status_string(999) == "GDN_ERR_UNKNOWN"
    assert lib.gdn_version() >= 100


def test_workspace_size_rounds(lib):
    """Tensor-core sizes: the full workspace holds two rounds of records (one
    per chunk and value head, 6 rounds of ceil(129 / 6) = 22 chunks at T=8192);
    smaller rounds bound it; CUDA-core sizes need only the header."""
    full = api.prefill_workspace_size(1, 8192, 16, 48, 128, 128)
    assert 2 * 22 * 48 * 65536 < full < 2 * 23 * 48 * 66560 + (8 << 20)
    r1 = api.prefill_workspace_size(1, 8192, 16, 48, 128, 128, chunks_per_round=1)
    r4 = api.prefill_workspace_size(1, 8192, 16, 48, 128, 128, chunks_per_round=4)
    assert 256 < r1 < r4 < full
    assert r4 - r1 == 3 * (r4 - r1) // 3 and (r4 - r1) // 3 >= 48 * 65536
    assert api.prefill_workspace_size(1, 8192, 16, 48, 128, 128, chunks_per_round=10 ** 6) == full
    assert lib.gdn_prefill_workspace_size_rounds(1, 8192, 16, 48, 128, 128, 0, -1) == 0
    assert api.prefill_workspace_size(1, 256, 2, 6, 64, 64, torch.float32) == 256
    assert api.prefill_workspace_size(1, 256, 2, 6, 64, 64, torch.float32, chunks_per_round=2) == 256


def test_launch_count(lib):
    """One launch for the single-pass and CUDA-core kernels; plan + two per
    round for the two-phase kernels (6 pipelined rounds of 22 chunks at 8k)."""
    full = api.prefill_workspace_size(1, 8192, 16, 48, 128, 128)
    assert api.prefill_launch_count(1, 8192, 16, 48, 128, 128, full) == 1 + 2 * 6
    assert api.prefill_launch_count(1, 8192, 16, 48, 128, 128, 256) == 1
    one_row = api.prefill_workspace_size(1, 8192, 16, 48, 128, 128, chunks_per_round=1)
    assert api.prefill_launch_count(1, 8192, 16, 48, 128, 128, one_row) == 1 + 2 * 129
    assert api.prefill_launch_count(1, 256, 2, 6, 64, 64, 256, torch.float32) == 1
    assert api.prefill_launch_count(0, 0, 16, 48, 128, 128, full) == 0
    assert api.prefill_launch_count(1, 8192, 16, 48, 128, 128, 100) == -1


def test_decode_tokens_validation(lib):
    """Host-side rejections of gdn_decode_tokens (nothing is launched)."""
    vp = ctypes.c_void_p(256)
    args = dict(batch=2, tokens=4, Hqk=16, Hv=48, Dk=128, Dv=128, dtype=0, o_dtype=1, s_dtype=1,
                form=0)

    def call(**kw):
        a = {**args, **kw}
        return lib.gdn_decode_tokens(vp, vp, vp, vp, vp, vp, vp, None, None, 4, vp, a["batch"],
                                     a["tokens"], a["Hqk"], a["Hv"], a["Dk"], a["Dv"], a["dtype"],
                                     a["o_dtype"], a["s_dtype"], a["form"], 1.0, None, None)

    assert call(tokens=17) == api.GDN_ERR_UNSUPPORTED      # more than 16 tokens
    assert call(Dk=96) == api.GDN_ERR_UNSUPPORTED
    assert call(Hv=40) == api.GDN_ERR_INVALID_ARG            # 40 % 16 != 0
    assert call(tokens=-1) == api.GDN_ERR_INVALID_ARG
    assert call(batch=0) == api.GDN_OK and call(tokens=0) == api.GDN_OK
    assert call(batch=5) == api.GDN_ERR_INVALID_ARG          # no slot map: needs batch <= slots
    assert call(s_dtype=2) == api.GDN_ERR_INVALID_ARG        # state dtype neither bf16 nor fp32
    assert call(s_dtype=0, batch=0) == api.GDN_OK            # bf16 states accepted
    assert call(form=5) == api.GDN_ERR_INVALID_ARG           # input form neither prepared nor raw
    assert call(form=1, batch=0) == api.GDN_OK


def test_workspace_size(lib):
    assert api.prefill_workspace_size(1, 8192, 16, 48, 128, 128) >= 256
    assert lib.gdn_prefill_workspace_size(-1, 10, 16, 48, 128, 128, 0) == 0
    assert lib.gdn_prefill_workspace_size(1, 10, 16, 40, 128, 128, 0) == 0  # 40 % 16 != 0
    assert lib.gdn_prefill_workspace_size(1, 10, 16, 48, 128, 128, 7) == 0  # bad dtype


def _prefill(lib, **kw):
    a = dict(q=1 << 12, k=1 << 12, v=1 << 12, g=1 << 12, beta=1 << 12, cu=1 << 12, N=1, T=16,
             Hqk=2, Hv=6, Dk=64, Dv=64, dtype=0, odt=1, sdt=1, form=0, scale=1.0, s0=None,
             sf=None, o=1 << 12, ws=1 << 12, wsb=256)
    a.update(kw)
    return lib.gdn_prefill(a["q"], a["k"], a["v"], a["g"], a["beta"], a["cu"], a["N"], a["T"],
                           a["Hqk"], a["Hv"], a["Dk"], a["Dv"], a["dtype"], a["odt"], a["sdt"],
                           a["form"], a["scale"], a["s0"], a["sf"], a["o"], a["ws"], a["wsb"], None)


def test_prefill_validation(lib):
    # every case is rejected on the host; the fake addresses are never dereferenced
    assert _prefill(lib, q=None) == api.GDN_ERR_INVALID_ARG
    assert _prefill(lib, cu=None) == api.GDN_ERR_INVALID_ARG
    assert _prefill(lib, o=None) == api.GDN_ERR_INVALID_ARG
    assert _prefill(lib, v=(1 << 12) + 8) == api.GDN_ERR_INVALID_ARG  # misaligned
    assert _prefill(lib, Hv=5) == api.GDN_ERR_INVALID_ARG            # Hv % Hqk
    assert _prefill(lib, Hqk=0) == api.GDN_ERR_INVALID_ARG
    assert _prefill(lib, dtype=3) == api.GDN_ERR_INVALID_ARG
    assert _prefill(lib, odt=2) == api.GDN_ERR_INVALID_ARG
    assert _prefill(lib, sdt=2) == api.GDN_ERR_INVALID_ARG             # state dtype
    assert _prefill(lib, form=2) == api.GDN_ERR_INVALID_ARG            # input form
    assert _prefill(lib, T=-1) == api.GDN_ERR_INVALID_ARG
    assert _prefill(lib, N=-1) == api.GDN_ERR_INVALID_ARG
    assert _prefill(lib, Dk=96) == api.GDN_ERR_UNSUPPORTED
    assert _prefill(lib, Dv=256) == api.GDN_ERR_UNSUPPORTED
    assert _prefill(lib, ws=None) == api.GDN_ERR_WORKSPACE
    assert _prefill(lib, ws=(1 << 12) + 16) == api.GDN_ERR_WORKSPACE
    assert _prefill(lib, wsb=8) == api.GDN_ERR_WORKSPACE
    assert _prefill(lib, N=0, T=5) == api.GDN_ERR_INVALID_ARG
    assert _prefill(lib, N=0, T=0) == api.GDN_OK                    # nothing to do


def _decode(lib, **kw):
    a = dict(q=1 << 12, k=1 << 12, v=1 << 12, g=1 << 12, beta=1 << 12, S=1 << 12, o=1 << 12, B=2,
             Hqk=16, Hv=48, Dk=128, Dv=128, dtype=0, odt=1, scale=1.0)
    a.update(kw)
    return lib.gdn_decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], a["S"], a["o"], a["B"],
                               a["Hqk"], a["Hv"], a["Dk"], a["Dv"], a["dtype"], a["odt"], a["scale"],
                               None)


def test_decode_validation(lib):
    assert _decode(lib, S=None) == api.GDN_ERR_INVALID_ARG
    assert _decode(lib, k=None) == api.GDN_ERR_INVALID_ARG
    assert _decode(lib, o=(1 << 12) + 4) == api.GDN_ERR_INVALID_ARG
    assert _decode(lib, Hv=47) == api.GDN_ERR_INVALID_ARG
    assert _decode(lib, B=-3) == api.GDN_ERR_INVALID_ARG
    assert _decode(lib, Dk=32) == api.GDN_ERR_UNSUPPORTED
    assert _decode(lib, odt=-1) == api.GDN_ERR_INVALID_ARG
    assert _decode(lib, B=0) == api.GDN_OK


def test_device_status_validation(lib):
    out = ctypes.c_int32(7)
    assert lib.gdn_get_device_status(None, None, ctypes.byref(out)) == api.GDN_ERR_INVALID_ARG
    assert lib.gdn_get_device_status(1 << 12, None, None) == api.GDN_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(lib):
    import torch

    x = torch.zeros(4, 1, 64)
    with pytest.raises(ValueError):
        api.prefill(x, x, x, torch.zeros(4, 1), torch.zeros(4, 1))


def test_backward_workspace_and_validation(lib):
    """gdn_prefill_backward: workspace arithmetic and host-side rejections
    (nothing is launched; the fake addresses are never dereferenced)."""
    ck = 64 * 1024  # one 128 x 128 fp32 state
    # sequential form.  48 heads fill few SMs: 4 row slices per head, dq/dk/dg/dbeta per slice
    ws = api.prefill_backward_workspace_size(1, 8192, 16, 48, 128, 128, sequential=True)
    need = (512 + 1) * 48 * ck + 48 * 16 * ck + 2 * 8192 * 48 * 4 * (128 * 4 + 4)
    assert need <= ws <= need + 6 * 256
    # 8 sequences x 48 heads fill the GPU: one slice, dq/dk per value head only
    ws8 = api.prefill_backward_workspace_size(8, 8192, 16, 48, 128, 128, sequential=True)
    need8 = (512 + 8) * 48 * ck + 8 * 48 * 16 * ck + 2 * 8192 * 48 * 128 * 4
    assert need8 <= ws8 <= need8 + 4 * 256
    assert (api.prefill_backward_workspace_size(8, 8192, 48, 48, 128, 128, sequential=True)
            == ws8 - 2 * 8192 * 48 * 128 * 4)
    # chunk form: per (chunk, value head) 3 tiles of 64 x 64, 7 of 64 x 128, the state and its
    # gradient (128 x 128 each), 3 x 64 fp32 scalars and 64 fp64 log-decay sums; chunks bounded
    # by ceil(T / 64) + N
    # (the reported size is the larger of the two forms, so it always runs the chunk form)
    per_unit = 4 * (3 * 64 * 64 + 7 * 64 * 128 + 2 * 128 * 128 + 3 * 64) + 8 * 64  # G in fp64
    # (no per-value-head dq, dk: the group's value heads add them in registers)
    wsc1 = api.prefill_backward_workspace_size(1, 8192, 16, 48, 128, 128)
    needc1 = (128 + 1) * 48 * per_unit
    assert wsc1 == max(ws, wsc1) and (wsc1 == ws or needc1 <= wsc1 <= needc1 + 20 * 256)
    wsc8 = api.prefill_backward_workspace_size(8, 8192, 16, 48, 128, 128)
    needc8 = (128 + 8) * 48 * per_unit
    assert wsc8 > ws8 and needc8 <= wsc8 <= needc8 + 20 * 256
    assert api.prefill_backward_workspace_size(8, 8192, 48, 48, 128, 128) == wsc8
    assert lib.gdn_prefill_backward_workspace_size(1, 10, 16, 40, 128, 128) == 0  # 40 % 16
    assert lib.gdn_prefill_backward_workspace_size(1, 10, 16, 48, 96, 128) == 0
    vp = 1 << 12
    a = dict(q=vp, k=vp, v=vp, g=vp, beta=vp, cu=vp, N=1, T=16, Hqk=2, Hv=6, Dk=64, Dv=64, dtype=0,
             scale=1.0, s0=None, do=vp, dsf=None, dq=vp, dk=vp, dv=vp, dg=vp, db=vp, ds0=None,
             ws=vp, wsb=1 << 30)

    for fn in (lib.gdn_prefill_backward, lib.gdn_prefill_backward_sequential):
        def call(**kw):
            x = {**a, **kw}
            return fn(x["q"], x["k"], x["v"], x["g"], x["beta"], x["cu"], x["N"], x["T"], x["Hqk"],
                      x["Hv"], x["Dk"], x["Dv"], x["dtype"], x["scale"], x["s0"], x["do"], x["dsf"],
                      x["dq"], x["dk"], x["dv"], x["dg"], x["db"], x["ds0"], x["ws"], x["wsb"], None)

        assert call(do=None) == api.GDN_ERR_INVALID_ARG
        assert call(dq=vp + 4) == api.GDN_ERR_INVALID_ARG          # misaligned
        assert call(dv=vp + 8) == api.GDN_ERR_INVALID_ARG          # bases are 16-byte aligned
        assert call(Hv=5) == api.GDN_ERR_INVALID_ARG
        assert call(Dk=96) == api.GDN_ERR_UNSUPPORTED
        assert call(wsb=1024) == api.GDN_ERR_WORKSPACE
        assert call(ws=vp + 16) == api.GDN_ERR_WORKSPACE            # not 256-byte aligned
        assert call(N=0, T=0) == api.GDN_OK
        assert call(N=0, T=5) == api.GDN_ERR_INVALID_ARG

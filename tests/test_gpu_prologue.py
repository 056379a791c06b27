"""Raw inputs (GDN_INPUT_RAW) on the GPU against the fp64 oracle: the kernels
normalise q, k and map g = -softplus(a), beta = sigmoid(b) themselves; the
oracle runs its prologue, then the recurrence, on the same raw values."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrence_rule_b200 import api, inputs
from parity import assert_parity, to_np

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _raw_case(lengths, Hqk, Hv, D, dtype, seed, zero_rows=True):
    """Prefill inputs with raw q, k (row norms spread over e^N(0,1), a few rows
    all zero) and raw gate inputs a, b ~ N(0, 1.5^2)."""
    inp = inputs.prefill_inputs(lengths, Hqk, Hv, D, dtype=dtype, seed=seed, init_std=0.1)
    T = sum(lengths)
    gen = torch.Generator().manual_seed(seed + 500)
    qk = []
    for _ in range(2):
        x = torch.randn(T, Hqk, D, generator=gen) * torch.exp(torch.randn(T, Hqk, 1, generator=gen))
        if zero_rows and T > 3:
            x[T // 3, 0] = 0.0
        qk.append(x.to(inputs.DTYPES[dtype]))
    inp["q"], inp["k"] = qk
    inp["g"] = torch.randn(T, Hv, generator=gen) * 1.5   # a
    inp["beta"] = torch.randn(T, Hv, generator=gen) * 1.5  # b
    return inp


def _oracle_raw(inp, **kw):
    q, k, g, beta = oracle.prologue(inp["q"], inp["k"], inp["g"], inp["beta"])
    return oracle.prefill(q, k, inp["v"], g, beta, cu_seqlens=inp["cu_seqlens"],
                          initial_state=inp.get("initial_state"), **kw)


def _gpu_raw(inp, ws_bytes=None):
    dev = {n: (t.to(DEV) if t is not None else None) for n, t in inp.items()}
    ws = None if ws_bytes is None else torch.zeros(ws_bytes, dtype=torch.uint8, device=DEV)
    o, f = api.prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"],
                       cu_seqlens=dev["cu_seqlens"], initial_state=dev["initial_state"],
                       workspace=ws, raw_inputs=True)
    torch.cuda.synchronize()
    if ws is not None:
        assert api.get_device_status(ws) == api.GDN_OK
    return o, f


LENGTHS = [300, 0, 130, 64, 65]


@pytest.mark.parametrize("mode", ["two_phase", "rounds", "single_pass"])
def test_raw_prefill_tensor_cores(mode):
    inp = _raw_case(LENGTHS, 2, 6, 128, "bf16", seed=81)
    N, T = len(LENGTHS), sum(LENGTHS)
    ws = {"two_phase": None, "single_pass": 256,
          "rounds": api.prefill_workspace_size(N, T, 2, 6, 128, 128, chunks_per_round=3)}[mode]
    o, f = _gpu_raw(inp, ws)
    o_ref, f_ref = _oracle_raw(inp)
    assert_parity(torch.bfloat16, to_np(o), o_ref, to_np(f), f_ref, f"raw {mode}")


@pytest.mark.parametrize("D", [64, 128])
def test_raw_prefill_cuda_cores(D):
    inp = _raw_case([200, 0, 77], 2, 6, D, "fp32", seed=82 + D)
    o, f = _gpu_raw(inp)
    o_ref, f_ref = _oracle_raw(inp)
    assert_parity(torch.float32, to_np(o), o_ref, to_np(f), f_ref, f"raw CUDA cores D={D}")


def test_raw_mode_on_normalised_inputs():
    """Raw mode fed normalised q, k (rounded to bf16, so their norms are 1 to
    within 2^-8 and get renormalised) and a, b chosen so that -softplus(a) = g,
    sigmoid(b) = beta: parity with the oracle's prologue on the same values,
    and the prepared run's parity with the prepared oracle alongside."""
    inp = inputs.prefill_inputs([300, 65], 2, 6, 128, dtype="bf16", seed=83, init_std=0.1)
    dev = {n: (t.to(DEV) if t is not None else None) for n, t in inp.items()}
    o1, f1 = api.prefill(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"],
                         cu_seqlens=dev["cu_seqlens"], initial_state=dev["initial_state"])
    g64, b64 = inp["g"].double(), inp["beta"].double()
    raw = dict(inp, g=torch.log(torch.expm1(-g64)).float(),   # -softplus(a) = g
               beta=torch.log(b64 / (1 - b64)).float())       # sigmoid(b) = beta
    o2, f2 = _gpu_raw(raw)
    o_ref, f_ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                  cu_seqlens=inp["cu_seqlens"], initial_state=inp["initial_state"])
    assert_parity(torch.bfloat16, to_np(o1), o_ref, to_np(f1), f_ref, "prepared")
    o_ref2, f_ref2 = _oracle_raw(raw)
    assert_parity(torch.bfloat16, to_np(o2), o_ref2, to_np(f2), f_ref2, "raw on normalised inputs")


@pytest.mark.parametrize("sdt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("Tn", [1, 4])
def test_raw_decode_tokens(sdt, Tn):
    B, Hqk, Hv, D = 3, 2, 6, 128
    inp = _raw_case([Tn] * B, Hqk, Hv, D, "bf16", seed=84 + Tn)
    gen = torch.Generator().manual_seed(90 + Tn)
    pool = (torch.randn(B, Hv, D, D, generator=gen) * 0.3).to(sdt)
    x = {"q": inp["q"].view(B, Tn, Hqk, D), "k": inp["k"].view(B, Tn, Hqk, D),
         "v": inp["v"].view(B, Tn, Hv, D), "g": inp["g"].view(B, Tn, Hv),
         "beta": inp["beta"].view(B, Tn, Hv)}
    S = pool.to(DEV)
    o = api.decode_tokens(*(x[n].to(DEV) for n in ("q", "k", "v", "g", "beta")), S,
                          raw_inputs=True)
    torch.cuda.synchronize()
    inp["initial_state"] = pool
    rest = "bf16" if sdt == torch.bfloat16 else None
    o_ref, f_ref = _oracle_raw(inp, state_at_rest=rest)
    assert_parity(torch.bfloat16, to_np(o).reshape(B * Tn, Hv, D), o_ref, to_np(S), f_ref,
                  f"raw decode Tn={Tn} {sdt}")

"""The entry points inside a CUDA graph: the pipelined prefill (its internal
streams join the capture through events), the pool decode (launched with
programmatic dependent launch) and the backward pass, captured once and
replayed, give the same bits as the eager calls."""
import pytest
import torch

from gated_deltanet_recurrence_rule_b200 import api, inputs

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def test_capture_and_replay_match_eager():
    inp = inputs.prefill_inputs([300, 0, 130], 2, 6, 128, dtype="bf16", seed=91, init_std=0.1)
    x = {n: t.to(DEV) for n, t in inp.items()}
    T, N = x["q"].shape[0], 3
    ws = torch.zeros(api.prefill_workspace_size(N, T, 2, 6, 128, 128), dtype=torch.uint8, device=DEV)
    gen = torch.Generator().manual_seed(92)
    pool0 = (torch.randn(4, 6, 128, 128, generator=gen) * 0.3).to(torch.bfloat16).to(DEV)
    dx = inputs.prefill_inputs([4] * 4, 2, 6, 128, dtype="bf16", seed=93)
    d = {n: dx[n].to(DEV).view(4, 4, *dx[n].shape[1:]) for n in ("q", "k", "v", "g", "beta")}
    d_o = torch.randn(T, 6, 128, generator=gen).to(DEV)

    def calls(o, f, pool, od, grads):
        api.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=x["cu_seqlens"],
                    initial_state=x["initial_state"], final_state=f, o=o, workspace=ws)
        api.decode_tokens(d["q"], d["k"], d["v"], d["g"], d["beta"], pool, o=od)
        out = api.prefill_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], d_o,
                                   cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"],
                                   workspace=grads["ws"])
        for name, t in zip(("dq", "dk", "dv", "dg", "db", "ds0"), out):
            grads[name].copy_(t)

    def buffers():
        o = torch.empty(T, 6, 128, device=DEV)
        f = torch.empty(N, 6, 128, 128, device=DEV)
        od = torch.empty(4, 4, 6, 128, device=DEV)
        grads = {"ws": torch.zeros(api.prefill_backward_workspace_size(N, T, 2, 6, 128, 128),
                                   dtype=torch.uint8, device=DEV),
                 "dq": torch.empty(T, 2, 128, device=DEV), "dk": torch.empty(T, 2, 128, device=DEV),
                 "dv": torch.empty(T, 6, 128, device=DEV), "dg": torch.empty(T, 6, device=DEV),
                 "db": torch.empty(T, 6, device=DEV), "ds0": torch.empty(N, 6, 128, 128, device=DEV)}
        return o, f, od, grads

    eager = buffers()
    pool_e = pool0.clone()
    calls(eager[0], eager[1], pool_e, eager[2], eager[3])
    torch.cuda.synchronize()

    graphed = buffers()
    pool_g = pool0.clone()
    side = torch.cuda.Stream(DEV)
    side.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(side):  # warm-up off the capture: internal streams, kernel attributes
        calls(graphed[0], graphed[1], pool0.clone(), graphed[2], graphed[3])
    torch.cuda.current_stream(DEV).wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        calls(graphed[0], graphed[1], pool_g, graphed[2], graphed[3])
    for t in (graphed[0], graphed[1], graphed[2]):
        t.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == api.GDN_OK
    assert torch.equal(graphed[0], eager[0]) and torch.equal(graphed[1], eager[1])
    assert torch.equal(graphed[2], eager[2]) and torch.equal(pool_g, pool_e)
    for name in ("dq", "dk", "dv", "dg", "db", "ds0"):
        assert torch.equal(graphed[3][name], eager[3][name]), name

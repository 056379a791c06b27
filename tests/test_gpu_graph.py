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


def test_serving_loop_replays():
    """A serving loop's graph: raw-input prefill into bf16 states, then decode
    steps on fp32 states and one-token calls on a bf16 pool, both in place.
    Replayed three times, the graph gives the same bits as three rounds of the
    eager calls (the in-place states advance on every replay)."""
    B, Hqk, Hv, D = 4, 2, 6, 128
    pin = inputs.prefill_inputs([200, 64], Hqk, Hv, D, dtype="bf16", seed=94, init_std=0.1)
    x = {n: t.to(DEV) for n, t in pin.items()}
    T, N = x["q"].shape[0], 2
    s0 = x["initial_state"].to(torch.bfloat16)
    ws = torch.zeros(api.prefill_workspace_size(N, T, Hqk, Hv, D, D), dtype=torch.uint8, device=DEV)
    dx = inputs.prefill_inputs([1] * B, Hqk, Hv, D, dtype="bf16", seed=95)
    d = {n: dx[n].to(DEV) for n in ("q", "k", "v", "g", "beta")}
    gen = torch.Generator().manual_seed(96)
    st0 = (torch.randn(B, Hv, D, D, generator=gen) * 0.3).to(DEV)
    pool0 = st0.to(torch.bfloat16)
    dt = {n: t.view(B, 1, *t.shape[1:]) for n, t in d.items()}

    def buffers():
        return {"o": torch.empty(T, Hv, D, device=DEV),
                "f": torch.empty(N, Hv, D, D, dtype=torch.bfloat16, device=DEV),
                "S": st0.clone(), "pool": pool0.clone(),
                "od": torch.empty(B, Hv, D, device=DEV), "ot": torch.empty(B, 1, Hv, D, device=DEV)}

    def calls(b):
        api.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], cu_seqlens=x["cu_seqlens"],
                    initial_state=s0, final_state=b["f"], o=b["o"], workspace=ws, raw_inputs=True)
        api.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], b["S"], o=b["od"])
        api.decode_tokens(dt["q"], dt["k"], dt["v"], dt["g"], dt["beta"], b["pool"], o=b["ot"])

    eager = buffers()
    for _ in range(3):
        calls(eager)
    torch.cuda.synchronize()

    graphed = buffers()
    side = torch.cuda.Stream(DEV)
    side.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.stream(side):  # warm-up off the capture, on copies of the states
        warm = buffers()
        calls(warm)
    torch.cuda.current_stream(DEV).wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        calls(graphed)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert api.get_device_status(ws) == api.GDN_OK
    for name in ("o", "f", "S", "pool", "od", "ot"):
        assert torch.equal(graphed[name], eager[name]), name

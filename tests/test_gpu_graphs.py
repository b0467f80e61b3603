"""The C-ABI calls inside CUDA graphs.

A serving loop that runs the same shapes over and over can capture one step
(scoring, selection, attention) in a CUDA graph and replay it with new inputs
copied into the captured buffers, paying the launch cost once. Each call only
launches kernels on the caller's stream (the host-buffer call adds two
streams joined by events), so capture must work as is. Replays with fresh
inputs must reproduce the eager results bit for bit.
"""
import pytest
import torch

from block_sparse_long_score_b200 import (xattn_get_device_status, xattn_prefill_host,
                                          xattn_prefill_varlen, xattn_score,
                                          xattn_score_select, xattn_select, xattn_sparse_attn)
from block_sparse_long_score_b200.synth import make_problem

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _step(Q, K, V, prob, out):
    P = xattn_score(Q, K, prob.B, prob.S, prob.causal, probs=out["P"], workspace=out["ws_s"])
    xattn_select(P, out["tau"], prob.causal, out=(out["mask"], out["counts"], out["idx"]))
    xattn_sparse_attn(Q, K, V, out["counts"], out["idx"], prob.B, prob.causal, out=out["O"],
                      lse=out["lse"], workspace=out["ws_a"])


def _buffers(prob, Q):
    from block_sparse_long_score_b200 import (make_shape, xattn_attn_workspace_bytes,
                                              xattn_score_workspace_bytes)
    NB = prob.NB
    shape = make_shape(prob.batch, prob.hq, prob.hkv, prob.L, prob.d, prob.B, prob.S,
                       prob.causal, Q.dtype)
    z = dict(device=DEV, dtype=torch.int32)
    return {
        "P": torch.empty(prob.batch, prob.hq, NB, NB, device=DEV),
        "mask": torch.empty(prob.batch, prob.hq, NB, (NB + 31) // 32, **z),
        "counts": torch.empty(prob.batch, prob.hq, NB, **z),
        "idx": torch.empty(prob.batch, prob.hq, NB, NB, **z),
        "O": torch.empty_like(Q),
        "lse": torch.empty(Q.shape[:3], device=DEV),
        "ws_s": torch.empty(xattn_score_workspace_bytes(shape), device=DEV, dtype=torch.uint8),
        "ws_a": torch.empty(xattn_attn_workspace_bytes(shape), device=DEV, dtype=torch.uint8),
        "tau": torch.tensor(prob.tau.tolist(), dtype=torch.float32, device=DEV),
    }


@pytest.mark.parametrize("name,kw", [("c1", dict(L=4096, hq=4, hkv=2)),        # pair scoring
                                     ("c4", dict(frames=3, frame_tokens=640, hq=2, S=4))])
def test_three_calls_replay_in_a_graph(name, kw):
    a = make_problem(name, seed=11, **kw)
    b = make_problem(name, seed=12, **kw)
    Q, K, V = a.Q.to(DEV), a.K.to(DEV), a.V.to(DEV)
    buf = _buffers(a, Q)
    _step(Q, K, V, a, buf)          # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _step(Q, K, V, a, buf)
    # replay on the second problem's data, copied into the captured inputs
    Q.copy_(b.Q.to(DEV))
    K.copy_(b.K.to(DEV))
    V.copy_(b.V.to(DEV))
    g.replay()
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    got = {k: buf[k].clone() for k in ("P", "counts", "O", "lse")}
    ref = _buffers(b, Q)
    _step(Q, K, V, b, ref)
    torch.cuda.synchronize()
    for k in got:
        assert torch.equal(got[k], ref[k]), k
    # the second problem really differs from the captured one
    buf2 = _buffers(a, Q)
    _step(a.Q.to(DEV), a.K.to(DEV), a.V.to(DEV), a, buf2)
    torch.cuda.synchronize()
    assert not torch.equal(buf2["O"], got["O"])


def test_fused_call_and_varlen_replay_in_a_graph():
    lens = [1024, 520, 2048]
    probs = [make_problem("c1", L=L, hq=2, hkv=1, seed=30 + i) for i, L in enumerate(lens)]
    pack = lambda attr: torch.cat([getattr(p, attr)[0].reshape(-1, 128)
                                   for p in probs]).contiguous().to(DEV)
    Q, K, V = pack("Q"), pack("K"), pack("V")
    tau = probs[0].tau.tolist()
    out = torch.empty_like(Q)
    xattn_prefill_varlen(Q, K, V, lens, 2, 1, 128, 8, True, tau, out=out)
    torch.cuda.synchronize()
    eager = out.clone()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    # the call forks its lanes' streams while the capture runs
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        xattn_prefill_varlen(Q, K, V, lens, 2, 1, 128, 8, True, tau, out=out)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)

    p = probs[2]
    Qd, Kd = p.Q.to(DEV), p.K.to(DEV)
    tau_d = torch.tensor(tau, dtype=torch.float32, device=DEV)
    m1, c1, i1 = xattn_score_select(Qd, Kd, p.B, p.S, p.causal, tau_d)
    torch.cuda.synchronize()
    outs = (torch.zeros_like(m1), torch.zeros_like(c1), torch.zeros_like(i1))
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2):
        xattn_score_select(Qd, Kd, p.B, p.S, p.causal, tau_d, out=outs)
    g2.replay()
    torch.cuda.synchronize()
    assert torch.equal(outs[0], m1) and torch.equal(outs[1], c1)


def test_host_buffer_call_replays_in_a_graph():
    """xattn_prefill_host forks two copy streams off the caller's stream and
    joins them back with events, which a capture records as graph edges."""
    p = make_problem("c1", L=2048, hq=4, hkv=2, seed=40)
    Qh, Kh, Vh = p.Q.pin_memory(), p.K.pin_memory(), p.V.pin_memory()
    eager = xattn_prefill_host(Qh, Kh, Vh, p.B, p.S, p.causal, p.tau.tolist())
    torch.cuda.synchronize()
    eager = eager.clone()
    Oh = torch.zeros_like(eager).pin_memory()
    from block_sparse_long_score_b200 import make_shape, xattn_prefill_host_workspace_bytes
    shape = make_shape(1, 4, 2, p.L, 128, p.B, p.S, p.causal, "bf16")
    ws = torch.empty(xattn_prefill_host_workspace_bytes(shape, 0), device=DEV,
                     dtype=torch.uint8)
    g = torch.cuda.CUDAGraph()
    # the call creates its copy streams and events while the capture runs
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        xattn_prefill_host(Qh, Kh, Vh, p.B, p.S, p.causal, p.tau.tolist(), out=Oh,
                           workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(Oh, eager)


def test_replayed_step_reads_new_tau_from_the_device():
    """Per-head tau lives in a device array the kernels read at run time, so a
    captured step takes new thresholds written into that array, without
    capturing again. Every head's tau changes between the replays."""
    p = make_problem("c1", L=4096, hq=4, hkv=2, seed=50)
    Q, K, V = p.Q.to(DEV), p.K.to(DEV), p.V.to(DEV)
    buf = _buffers(p, Q)
    _step(Q, K, V, p, buf)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _step(Q, K, V, p, buf)
    for taus in ([0.5, 0.6, 0.7, 0.8], [0.99, 0.95, 0.9, 1.0]):
        buf["tau"].copy_(torch.tensor(taus, dtype=torch.float32))
        g.replay()
        torch.cuda.synchronize()
        assert xattn_get_device_status() == 0
        ref = _buffers(p, Q)
        ref["tau"].copy_(torch.tensor(taus, dtype=torch.float32))
        _step(Q, K, V, p, ref)
        torch.cuda.synchronize()
        for k in ("mask", "counts", "O"):
            assert torch.equal(buf[k], ref[k]), (taus, k)
    # tau = 1 on the last head selects every causally allowed block
    NB = p.NB
    assert torch.equal(buf["counts"][0, 3].cpu(), torch.arange(1, NB + 1, dtype=torch.int32))


@pytest.mark.parametrize("bad", [0.0, -0.5, 1.5, float("nan")])
def test_invalid_device_tau_is_reported(bad):
    """A device-resident tau outside (0, 1] cannot be checked on the host: the
    kernels check it, select nothing for that head and report INVALID_ARG
    through the device status, for both selection calls; the other heads are
    unaffected and the context stays usable."""
    p = make_problem("c1", L=2048, hq=2, hkv=1, seed=51)
    Q, K = p.Q.to(DEV), p.K.to(DEV)
    assert xattn_get_device_status() == 0
    tau_ok = torch.tensor([0.9, 0.9], dtype=torch.float32, device=DEV)
    tau_bad = torch.tensor([0.9, bad], dtype=torch.float32, device=DEV)
    P = xattn_score(Q, K, p.B, p.S, p.causal)
    m_ok, c_ok, i_ok = xattn_select(P, tau_ok, p.causal)
    torch.cuda.synchronize()
    assert xattn_get_device_status() == 0
    for call in (lambda: xattn_select(P, tau_bad, p.causal),
                 lambda: xattn_score_select(Q, K, p.B, p.S, p.causal, tau_bad)):
        m, c, _ = call()
        torch.cuda.synchronize()
        assert xattn_get_device_status() == -1          # XATTN_ERR_INVALID_ARG
        assert xattn_get_device_status() == 0           # read and cleared
        assert torch.equal(c[0, 0], c_ok[0, 0]) and torch.equal(m[0, 0], m_ok[0, 0])
        assert int(c[0, 1].abs().sum()) == 0 and int(m[0, 1].abs().sum()) == 0

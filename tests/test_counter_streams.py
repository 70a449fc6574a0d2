"""Counter-scheduled calls on several streams at once.

Packed, block-sparse and long causal backward calls take their work items
from a counter pair in the library.  Each stream owns one pair; a stream
beyond the 64 that own pairs takes over the least recently used pair after
an event wait.  If two calls that run at the same time shared a pair, each
would skip the items the other took, leaving rows of O (or dK/dV) unwritten
with no error raised.  These tests run such calls on several streams with no
ordering between them and compare every result bit for bit with the same
call made alone (the forward and the deterministic backward are bitwise
repeatable, whichever CTA takes which item).
"""

import pytest
import torch
from cuda.bindings import runtime as rt

from exact_attention_147_b200 import fa2 as F
from exact_attention_147_b200 import workloads as W

pytestmark = pytest.mark.gpu

SHORT = W.packed("short", (300, 129, 1, 77), H=2, d=128, causal=True, seed=91)
LONG = W.packed("long", (2048,) * 8, H=16, d=128, seed=92)


def _new_streams(n):
    """n new non-blocking CUDA streams (raw handles, as ints)."""
    out = []
    for _ in range(n):
        err, st = rt.cudaStreamCreateWithFlags(rt.cudaStreamNonBlocking)
        assert err == rt.cudaError_t.cudaSuccess, err
        out.append(int(st))
    return out


def _fwd_inputs(w):
    q, k, v, _ = W.make_inputs(w, "cuda")
    return q, k, v, w.cu_seqlens("cuda")


def test_one_long_call_beside_many_short_calls():
    # stream A: one long packed forward; stream B: 70 short ones queued behind
    # nothing on A.  With pairs handed out per call in turn, B's 64th call
    # would have shared A's pair while A still ran.
    ql, kl, vl, cul = _fwd_inputs(LONG)
    qs, ks, vs, cus = _fwd_inputs(SHORT)
    ref_long = F.fwd_varlen(ql, kl, vl, cul, LONG.N, causal=LONG.causal)
    ref_short = F.fwd_varlen(qs, ks, vs, cus, SHORT.N, causal=SHORT.causal)
    torch.cuda.synchronize()
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    with torch.cuda.stream(sa):
        got_long = F.fwd_varlen(ql, kl, vl, cul, LONG.N, causal=LONG.causal)
    with torch.cuda.stream(sb):
        for _ in range(70):
            outs.append(F.fwd_varlen(qs, ks, vs, cus, SHORT.N, causal=SHORT.causal))
    torch.cuda.synchronize()
    assert F.device_status() == 0
    assert torch.equal(got_long[0], ref_long[0]) and torch.equal(got_long[1], ref_long[1])
    for o, l in outs:
        assert torch.equal(o, ref_short[0]) and torch.equal(l, ref_short[1])


def test_more_streams_than_counter_pairs():
    # 72 streams, each with one forward and one deterministic backward of a
    # small packed batch, then a block-sparse forward: streams 65.. take
    # over pairs from earlier streams and must wait for their calls.
    q, k, v, do = W.make_inputs(SHORT, "cuda")
    cu = SHORT.cu_seqlens("cuda")
    ref_o, ref_l = F.fwd_varlen(q, k, v, cu, SHORT.N, causal=True)
    ref_D = F.bwd_preprocess(ref_o, do)
    ref_g = F.bwd_varlen(do, q, k, v, ref_l, ref_D, cu, SHORT.N, causal=True, deterministic=True)
    bs = W.Workload("bs", B=1, N=512, H=2, d=64, seed=93)
    bq, bk, bv, _ = W.make_inputs(bs, "cuda")
    nb = 4
    mask = (torch.arange(nb)[:, None] >= torch.arange(nb)[None, :]).to(torch.uint8).cuda()
    mask = mask[None, None].expand(1, 2, nb, nb)
    ref_b = F.fwd_blocksparse(bq, bk, bv, mask)
    torch.cuda.synchronize()
    handles = _new_streams(72)  # distinct handles (torch's own pool has fewer)
    try:
        res = []
        for hnd in handles:
            with torch.cuda.stream(torch.cuda.ExternalStream(hnd)):
                o, l = F.fwd_varlen(q, k, v, cu, SHORT.N, causal=True)
                g = F.bwd_varlen(do, q, k, v, l, ref_D, cu, SHORT.N, causal=True,
                                 deterministic=True)
                b = F.fwd_blocksparse(bq, bk, bv, mask)
                res.append((o, l, g, b))
        torch.cuda.synchronize()
        assert F.device_status() == 0
        for o, l, g, b in res:
            assert torch.equal(o, ref_o) and torch.equal(l, ref_l)
            assert all(torch.equal(x, y) for x, y in zip(g, ref_g))
            assert torch.equal(b[0], ref_b[0]) and torch.equal(b[1], ref_b[1])
        del res, o, l, g, b
    finally:
        torch.cuda.synchronize()
        for hnd in handles:
            rt.cudaStreamDestroy(hnd)


def test_counter_calls_inside_a_cuda_graph():
    # A counter-scheduled call captured into a CUDA graph keeps the pair of
    # its capturing stream; the pair is cleared by a captured memset before
    # the kernel, so the graph replays correctly any number of times.  The
    # first call on the stream is made before the capture (it may take the
    # pair over from another stream, which needs an event wait that a capture
    # cannot record).
    q, k, v, do = W.make_inputs(SHORT, "cuda")
    cu = SHORT.cu_seqlens("cuda")
    ref_o, ref_l = F.fwd_varlen(q, k, v, cu, SHORT.N, causal=True)
    ref_D = F.bwd_preprocess(ref_o, do)
    ref_g = F.bwd_varlen(do, q, k, v, ref_l, ref_D, cu, SHORT.N, causal=True, deterministic=True)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    out, lse = torch.empty_like(ref_o), torch.empty_like(ref_l)
    D = torch.empty_like(ref_D)
    g = [torch.empty_like(t) for t in ref_g]
    ws = torch.empty(max(1, F.workspace_size(1, SHORT.total, SHORT.H, SHORT.d, torch.bfloat16, True)),
                     dtype=torch.uint8, device="cuda")

    def step():
        F.fwd_varlen(q, k, v, cu, SHORT.N, causal=True, out=out, lse=lse, stream=s)
        F.bwd_preprocess(out, do, D, stream=s)
        F.bwd_varlen(do, q, k, v, lse, D, cu, SHORT.N, causal=True, deterministic=True, dq=g[0],
                     dk=g[1], dv=g[2], workspace=ws, stream=s)

    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                       # outside the capture: the stream takes its pair
    s.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step()
    for _ in range(2):
        for t in (out, lse, *g):
            t.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert F.device_status() == 0
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
        assert all(torch.equal(a, b) for a, b in zip(g, ref_g))
    del graph


def test_stream_destroyed_while_its_call_runs():
    # The long call's stream is destroyed right after the launch; a new
    # stream (which may be handed the same handle) makes a short call at
    # once.  Each launch waits for the event of its pair's previous launch, so
    # the two cannot split one counter whether or not the handle is reused.
    ql, kl, vl, cul = _fwd_inputs(LONG)
    qs, ks, vs, cus = _fwd_inputs(SHORT)
    ref_long = F.fwd_varlen(ql, kl, vl, cul, LONG.N, causal=LONG.causal)
    ref_short = F.fwd_varlen(qs, ks, vs, cus, SHORT.N, causal=SHORT.causal)
    out_l, lse_l = torch.empty_like(ref_long[0]), torch.empty_like(ref_long[1])
    out_s, lse_s = torch.empty_like(ref_short[0]), torch.empty_like(ref_short[1])
    torch.cuda.synchronize()
    (h1,) = _new_streams(1)
    F.fwd_varlen(ql, kl, vl, cul, LONG.N, causal=LONG.causal, out=out_l, lse=lse_l,
                 stream=torch.cuda.ExternalStream(h1))
    rt.cudaStreamDestroy(h1)
    (h2,) = _new_streams(1)
    try:
        F.fwd_varlen(qs, ks, vs, cus, SHORT.N, causal=SHORT.causal, out=out_s, lse=lse_s,
                     stream=torch.cuda.ExternalStream(h2))
        torch.cuda.synchronize()
        assert F.device_status() == 0
        assert torch.equal(out_l, ref_long[0]) and torch.equal(lse_l, ref_long[1])
        assert torch.equal(out_s, ref_short[0]) and torch.equal(lse_s, ref_short[1])
    finally:
        torch.cuda.synchronize()
        rt.cudaStreamDestroy(h2)

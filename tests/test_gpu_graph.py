"""The library's calls captured into a CUDA graph and replayed.

A serving loop captures its step once and replays it with new inputs written into
the same buffers.  Each test captures a call on a side stream, changes the inputs in
place, replays, and compares with an eager call on the same inputs: the results
must be identical bit for bit (same kernels, same schedule, same split).
"""
import numpy as np
import pytest
import torch

import mla_latent_kv_22_b200 as M
import mla_synth as S
from gpu_helpers import bf16_dev, upload

pytestmark = pytest.mark.gpu


def _replay_matches_eager(run, inputs_a, inputs_b, outs):
    """run() reads the input buffers and writes outs; inputs_* are (buffer, value) pairs."""
    for buf, val in inputs_a:
        buf.copy_(val)
    run()  # warm: library state, workspace, kernel attributes
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    torch.cuda.synchronize()
    for buf, val in inputs_b:
        buf.copy_(val)
    for o in outs:
        o.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert M.mla_get_device_error() == 0
    replayed = [o.clone() for o in outs]
    for o in outs:
        o.fill_(float("nan"))
    run()
    torch.cuda.synchronize()
    for r, o in zip(replayed, outs):
        assert torch.isfinite(r).any()
        assert torch.equal(r, o)
    del g


def test_decode_replayed_from_a_graph():
    a = S.make_decode_case(4, 128, [100, 700, 64, 1], seed=91, poison=True)
    b = S.make_decode_case(4, 128, [100, 700, 64, 1], seed=92, poison=True)
    q, kv, bt, sl = upload(a)
    q_b = bf16_dev(b.q)
    out = torch.empty(4, 128, 512, device="cuda")
    lse = torch.empty(4, 128, device="cuda")
    _replay_matches_eager(lambda: M.mla_decode(q, kv, bt, sl, out, lse, a.softmax_scale),
                          [(q, bf16_dev(a.q))], [(q, q_b)], [out, lse])


def test_layer_and_several_queries_replayed_from_a_graph():
    B, H = 8, 64
    li_a, li_b = S.make_layer_inputs(B, H, seed=93), S.make_layer_inputs(B, H, seed=94)
    case = S.make_decode_case(B, 2 * H, [300, 1, 65, 128, 999, 7, 64, 200], seed=93, poison=True)
    _, kv, bt, sl = upload(case)
    qn, qr = bf16_dev(li_a.q_nope), bf16_dev(li_a.q_rope)
    wk, wv = bf16_dev(li_a.w_uk), bf16_dev(li_a.w_uv)
    qp = torch.empty(B, H, 576, dtype=torch.bfloat16, device="cuda")
    o_lat = torch.empty(B, H, 512, device="cuda")
    lse = torch.empty(B, H, device="cuda")
    out = torch.empty(B, H, 128, device="cuda")
    qm = bf16_dev(case.q).view(B, 2, H, 576)
    out_m = torch.empty(B, 2, H, 512, device="cuda")
    lse_m = torch.empty(B, 2, H, device="cuda")

    def step():
        M.mla_absorb_q(qn, qr, wk, qp)
        M.mla_decode(qp, kv, bt, sl, o_lat, lse, case.softmax_scale)
        M.mla_absorb_o(o_lat, wv, out)
        M.mla_decode_multi(qm, kv, bt, sl, out_m, lse_m, case.softmax_scale)

    qm_b = bf16_dev(S.make_decode_case(B, 2 * H, 1, seed=95).q).view(B, 2, H, 576)
    _replay_matches_eager(step,
                          [(qn, bf16_dev(li_a.q_nope)), (qr, bf16_dev(li_a.q_rope))],
                          [(qn, bf16_dev(li_b.q_nope)), (qr, bf16_dev(li_b.q_rope)), (qm, qm_b)],
                          [out, lse, out_m, lse_m])

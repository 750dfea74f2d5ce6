"""GPU parity of the absorption GEMMs and of the end-to-end absorbed layer
(absorb_q -> decode -> absorb_o) against the fp64 oracle, including the expanded
per-head K/V form on a batch subset."""
import numpy as np
import pytest
import torch

import mla_latent_kv_22_b200 as M
import mla_synth as S
import oracle as O
from gpu_helpers import OUT_ATOL, OUT_RTOL, LSE_ATOL, bf16_dev, upload

pytestmark = pytest.mark.gpu


def _f64(t):
    return t.double().cpu().numpy()


@pytest.mark.parametrize("B,H", [(64, 128), (5, 3), (70, 16), (1, 1), (130, 32), (300, 8)])
def test_absorb_q(B, H):
    li = S.make_layer_inputs(B, H, seed=50 + B)
    qn, qr, wk = bf16_dev(li.q_nope), bf16_dev(li.q_rope), bf16_dev(li.w_uk)
    qo = torch.empty(B, H, 576, dtype=torch.bfloat16, device="cuda")
    M.mla_absorb_q(qn, qr, wk, qo)
    torch.cuda.synchronize()
    ref = O.mla_absorb_q_ref(li.q_nope, li.q_rope, li.w_uk)
    got = _f64(qo)
    # fp32 accumulation rounded once to bf16 (relative 2^-9), plus fp32 sum noise.
    assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5).all()
    assert np.array_equal(got[..., 512:], ref[..., 512:])


@pytest.mark.parametrize("B,H", [(64, 128), (5, 3), (70, 16), (130, 32), (300, 8)])
def test_absorb_o(B, H):
    li = S.make_layer_inputs(B, H, seed=60 + B)
    ol = torch.randn(B, H, 512, generator=torch.Generator().manual_seed(B)).mul_(0.05)
    wv = bf16_dev(li.w_uv)
    out = torch.empty(B, H, 128, device="cuda")
    M.mla_absorb_o(ol.cuda(), wv, out)
    torch.cuda.synchronize()
    # The library rounds out_latent to bf16 on load; feed the oracle those values.
    ol_bf16 = ol.to(torch.bfloat16).double().numpy()
    ref = O.mla_absorb_o_ref(ol_bf16, li.w_uv)
    assert np.abs(_f64(out) - ref).max() <= 1e-5 + 1e-5 * np.abs(ref).max()


def test_layer_end_to_end_config5():
    B, H = 64, 128
    li = S.config_layer_inputs(B)
    case = S.config_case(5)
    _, kv, bt, sl = upload(case)
    qn, qr, wk, wv = (bf16_dev(x) for x in (li.q_nope, li.q_rope, li.w_uk, li.w_uv))
    qp = torch.empty(B, H, 576, dtype=torch.bfloat16, device="cuda")
    o_lat = torch.empty(B, H, 512, device="cuda")
    lse = torch.empty(B, H, device="cuda")
    out = torch.empty(B, H, 128, device="cuda")
    M.mla_absorb_q(qn, qr, wk, qp)
    M.mla_decode(qp, kv, bt, sl, o_lat, lse, case.softmax_scale)
    M.mla_absorb_o(o_lat, wv, out)
    assert M.mla_get_device_error() == 0
    got, got_lse = _f64(out), _f64(lse)

    bs = [0, 31, 63]
    ref_o, ref_l = O.mla_layer_absorbed_ref(li.q_nope, li.q_rope, li.w_uk, li.w_uv, case.kv_cache, case.block_table,
                                            case.cache_seqlens, case.softmax_scale, batch=bs)
    assert (np.abs(got[bs] - ref_o) <= OUT_ATOL + OUT_RTOL * np.abs(ref_o)).all()
    assert np.abs(got_lse[bs] - ref_l).max() <= LSE_ATOL

    hs = [0, 9, 77, 127]
    exp_o, exp_l = O.mla_decode_expanded_ref(li.q_nope, li.q_rope, li.w_uk, li.w_uv, case.kv_cache, case.block_table,
                                             case.cache_seqlens, case.softmax_scale, batch=bs, heads=hs)
    sub = got[bs][:, hs]
    assert (np.abs(sub - exp_o) <= OUT_ATOL + OUT_RTOL * np.abs(exp_o)).all()
    assert np.abs(got_lse[bs][:, hs] - exp_l).max() <= LSE_ATOL

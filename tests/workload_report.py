"""Per-workload report (GPU): times every workload's call (CUDA events per call, a 256 MB
write between calls, median of 20 after 5 warm-ups) on inputs with finite tails, and gives
the largest deviation from the fp64 oracle on the correctness inputs (NaN-poisoned tails
and unused pages), as one markdown table.

    python tests/workload_report.py

Workloads 1-4 call mla_decode; workload 5 calls mla_absorb_q, mla_decode and mla_absorb_o.
Roofline: algorithmic bytes over the measured HBM copy rate (MEASURED_PEAKS.json).  Not a
test (pytest does not collect it); it lives beside the tests because it reads the oracle.
"""
import json
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, ROOT)
sys.path.insert(0, HERE)
import mla_latent_kv_22_b200 as M  # noqa: E402
import mla_synth as S  # noqa: E402
import oracle as O  # noqa: E402
from gpu_helpers import upload, run_decode, bf16_dev  # noqa: E402

HBM = json.load(open(os.path.join(ROOT, 'MEASURED_PEAKS.json')))['hbm_gbs'] * 1e9
flush = torch.empty(256 * 1024 * 1024 // 4, device='cuda')

def alg(case):
    H = case.H; mb = case.block_table.shape[1] if case.block_table is not None else case.kv_cache.shape[1] // 64
    T = case.cache_seqlens.astype(np.int64)
    by = int((T * 1152 + H * (1152 + 2048 + 4) + 4 * mb + 4).sum()); fl = float((2 * H * T * 1088).sum())
    return by, fl

def time_fn(fn, n=20):
    for _ in range(5): fn()
    ts = []
    for _ in range(n):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(); fn(); e1.record(); torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1000)
    return float(np.median(ts))

def errs(out, lse, ro, rl):
    o = out.double().cpu().numpy(); l = lse.double().cpu().numpy()
    return float(np.nanmax(np.abs(o - ro))), float(np.nanmax(np.abs(l - rl)))

rows = []
def decode_row(name, timed, check, sel):
    q, kv, bt, sl = upload(timed)
    out = torch.empty(timed.B, timed.H, 512, device='cuda'); lse = torch.empty(timed.B, timed.H, device='cuda')
    us = time_fn(lambda: M.mla_decode(q, kv, bt, sl, out, lse, timed.softmax_scale))
    by, fl = alg(timed)
    o, l, e = run_decode(check)
    assert e == 0
    ro, rl = O.mla_decode_ref(check.q, check.kv_cache, check.block_table, check.cache_seqlens, check.softmax_scale, **sel)
    if 'batch' in sel: o, l = o[sel['batch']], l[sel['batch']]
    if 'heads' in sel: o, l = o[:, sel['heads']], l[:, sel['heads']]
    eo, el = errs(o, l, ro, rl)
    kv_bytes = int(timed.cache_seqlens.astype(np.int64).sum() * 1152)
    rows.append((name, us, kv_bytes / us / 1e6, fl / us / 1e6, by / HBM * 1e6 / us, by / HBM * 1e6, eo, el, str(sel) if sel else 'all'))

decode_row('1 tiny B1 H16 T256 contiguous', S.config_case(1, poison=False), S.config_case(1), {})
decode_row('2 paged B16 H128 T4096', S.config_case(2, poison=False), S.config_case(2), {})
decode_row('3 var-len B64 H128 T~U[1024,8192]', S.config_case(3, poison=False), S.config_case(3), {})
decode_row('3 headline B64 H128 T8192', S.config_case(3, poison=False, headline=True), S.config_case(3, headline=True), {'batch': [0, 17, 38, 63]})
decode_row('4 long B4 H128 T131072', S.config_case(4, poison=False), S.config_case(4), {'heads': [0, 5, 64, 127]})

# workload 5: absorb_q -> decode -> absorb_o
li = S.config_layer_inputs(); timed = S.config_case(5, poison=False); check = S.config_case(5)
qn, qr, wk, wv = bf16_dev(li.q_nope), bf16_dev(li.q_rope), bf16_dev(li.w_uk), bf16_dev(li.w_uv)
def layer(case, dev):
    _, kv, bt, sl = dev
    qp = torch.empty(64, 128, 576, dtype=torch.bfloat16, device='cuda')
    ol = torch.empty(64, 128, 512, device='cuda'); lse = torch.empty(64, 128, device='cuda')
    out = torch.empty(64, 128, 128, device='cuda')
    def f():
        M.mla_absorb_q(qn, qr, wk, qp)
        M.mla_decode(qp, kv, bt, sl, ol, lse, case.softmax_scale)
        M.mla_absorb_o(ol, wv, out)
    return f, out, lse
dev_t = upload(timed); f, _, _ = layer(timed, dev_t)
us = time_fn(f)
by, fl = alg(timed)
by += 64 * 128 * 192 * 2 + 128 * 128 * 512 * 2 + 64 * 128 * 576 * 2 + 64 * 128 * 512 * 4 + 128 * 512 * 128 * 2 + 64 * 128 * 128 * 4
fl += 2 * 2 * 64 * 128 * 128 * 512
dev_c = upload(check); f, out, lse = layer(check, dev_c); f(); torch.cuda.synchronize()
bs = [0, 31, 63]
ro, rl = O.mla_layer_absorbed_ref(li.q_nope, li.q_rope, li.w_uk, li.w_uv, check.kv_cache, check.block_table, check.cache_seqlens, check.softmax_scale, batch=bs)
eo, el = errs(out[bs], lse[bs], ro, rl)
kv_bytes = int(timed.cache_seqlens.astype(np.int64).sum() * 1152)
rows.append(('5 layer B64 H128 T4096 (absorb_q + decode + absorb_o)', us, kv_bytes / us / 1e6, fl / us / 1e6, by / HBM * 1e6 / us, by / HBM * 1e6, eo, el, "{'batch': [0, 31, 63]}"))
print('| workload | µs/call | cache TB/s | TFLOPS | % of roofline (measured copy rate) | roofline µs | max abs out err | max abs lse err | checked |')
print('|---|---|---|---|---|---|---|---|---|')
for r in rows:
    print(f'| {r[0]} | {r[1]:.1f} | {r[2]:.2f} | {r[3]:.0f} | {100*r[4]:.1f} % | {r[5]:.2f} | {r[6]:.2e} | {r[7]:.2e} | {r[8]} |')

"""The C-ABI library: it loads, exports every symbol include/mla.h declares, and
rejects bad arguments on the host before launching anything.  CPU only (no call
here reaches a kernel launch)."""
import ctypes
import os
import re

import pytest

import mla_latent_kv_22_b200 as M

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "mla.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert "mla_decode" in names and "mla_absorb_q" in names and "mla_absorb_o" in names
    lib = ctypes.CDLL(M.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_knobs():
    for code, name in M.STATUS.items():
        assert M.mla_status_string(code) == name
    old = M.mla_get_knob("min_pages")
    M.mla_set_knob("min_pages", 9)
    assert M.mla_get_knob("min_pages") == 9
    M.mla_set_knob("min_pages", old)
    assert M.lib.mla_set_knob(99, 1) == 1
    assert M.lib.mla_set_knob(0, -1) == 1


def _decode(**kw):
    args = dict(q=16, kv=16, bt=None, sl=16, out=16, lse=16, B=2, H=128, num_pages=10, max_blocks=4, scale=0.1)
    args.update(kw)
    return M.lib.mla_decode(args["q"], args["kv"], args["bt"], args["sl"], args["out"], args["lse"], args["B"],
                            args["H"], args["num_pages"], args["max_blocks"], args["scale"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(kv=None), 1), (dict(sl=None), 1), (dict(out=None), 1), (dict(lse=None), 1),
    (dict(H=0), 2), (dict(H=129), 2), (dict(B=-1), 1), (dict(max_blocks=0), 1),
    (dict(q=24), 1), (dict(kv=8), 1), (dict(out=4), 1), (dict(lse=2), 1),
    (dict(bt=16, num_pages=0), 1), (dict(scale=float("nan")), 1), (dict(scale=float("inf")), 1),
    (dict(max_blocks=1 << 25), 2),
    # batch x (table width + the largest piece cost) must fit the device's 32-bit split arithmetic
    (dict(B=8_000_000, max_blocks=16), 2),
])
def test_decode_host_validation(kw, status):
    assert _decode(**kw) == status
    assert M.lib.mla_last_error_message()


@pytest.mark.parametrize("s_q,H,q,status", [
    (0, 64, 16, 1), (-1, 64, 16, 1), (2, -1, 16, 1), (2, 129, 16, 2), (17, 128, 16, 2), (2049, 1, 16, 2),
    (2, 64, None, 1), (2, 64, 24, 1), (1, 129, 16, 2),
])
def test_decode_multi_host_validation(s_q, H, q, status):
    assert M.lib.mla_decode_multi(q, 16, None, 16, 16, 16, 2, s_q, H, 10, 4, 0.1, None) == status
    assert M.lib.mla_last_error_message()


def test_split_schedule_size_limit_message():
    assert _decode(B=8_000_000, max_blocks=16) == 2
    assert b"32-bit split schedule" in M.lib.mla_last_error_message()
    assert _decode(B=8_000_000, max_blocks=1, q=24) == 1  # 8M x 257 units fit: the next check runs


def test_empty_batch_is_a_no_op():
    assert _decode(B=0, q=None) == 0


@pytest.mark.parametrize("fn,args,status", [
    ("mla_absorb_q", (None, 16, 16, 16, 2, 8, None), 1),
    ("mla_absorb_q", (16, 16, 16, 16, 2, 200, None), 2),
    ("mla_absorb_q", (16, 16, 8, 16, 2, 8, None), 1),
    ("mla_absorb_o", (16, None, 16, 2, 8, None), 1),
    ("mla_absorb_o", (16, 16, 16, 2, 0, None), 2),
    ("mla_absorb_o", (20, 16, 16, 2, 8, None), 1),
])
def test_absorb_host_validation(fn, args, status):
    assert getattr(M.lib, fn)(*args) == status


def test_workspace_alignment_rejected():
    assert M.lib.mla_set_workspace(ctypes.c_void_p(0x1010), 4096) == 1

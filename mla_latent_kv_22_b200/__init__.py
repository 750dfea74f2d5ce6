"""Python binding of libmla.so: absorbed Multi-head Latent Attention decode on B200.

Argument marshalling only.  Every function takes torch tensors, checks dtype,
shape, device and contiguity, and passes raw pointers, sizes and the current CUDA
stream to the C ABI of the same name (include/mla.h); every step of the
computation runs in the library's CUDA kernels.  Importing fails loudly when the
library has not been built (``python mla_latent_kv_22_b200/build.py``); there is
no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MlaError", "mla_decode", "mla_decode_multi", "mla_decode_noalloc", "mla_absorb_q", "mla_absorb_o", "mla_workspace_size", "mla_set_workspace",
    "mla_get_device_error", "mla_status_string", "mla_set_knob", "mla_get_knob", "mla_selected_decode_kernel",
    "mla_timing_enable",
    "mla_timing_read", "lib", "LIB_PATH", "KNOB", "STATUS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla.so")

STATUS = {
    0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_WORKSPACE", 4: "MLA_ERR_CUDA",
    5: "MLA_ERR_DEVICE_BAD_PAGE", 6: "MLA_ERR_DEVICE_TIMEOUT",
}
KNOB = {"num_workers": 0, "min_pages": 1, "decode_kernel": 2, "wait_limit": 3, "withhold_arrive": 4, "split_policy": 5,
        "piece_cost": 6}

D_LATENT, D_ROPE, D_QK, PAGE, D_NOPE, D_V, MAX_HEADS = 512, 64, 576, 64, 128, 128, 128


class MlaError(RuntimeError):
    def __init__(self, status: int, message: str = ""):
        self.status = status
        self.name = STATUS.get(status, f"status {status}")
        super().__init__(f"{self.name}: {message}" if message else self.name)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python mla_latent_kv_22_b200/build.py` "
                          "(nvcc, sm_100a); there is no fallback implementation")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "mla_decode": ([vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, vp], i32),
        "mla_decode_multi": ([vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp], i32),
        "mla_decode_noalloc": ([vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, vp], i32),
        "mla_absorb_q": ([vp, vp, vp, vp, i32, i32, vp], i32),
        "mla_absorb_o": ([vp, vp, vp, i32, i32, vp], i32),
        "mla_workspace_size": ([i32, i32, i32], sz),
        "mla_set_workspace": ([vp, sz], i32),
        "mla_get_device_error": ([vp], i32),
        "mla_status_string": ([i32], ctypes.c_char_p),
        "mla_last_error_message": ([], ctypes.c_char_p),
        "mla_set_knob": ([i32, i32], i32),
        "mla_get_knob": ([i32], i32),
        "mla_selected_decode_kernel": ([i32], i32),
        "mla_timing_enable": ([i32], i32),
        "mla_timing_read": ([ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


lib = _load()


def _check(status: int) -> None:
    if status != 0:
        raise MlaError(status, lib.mla_last_error_message().decode(errors="replace"))


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: tuple | None = None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _cache_args(kv_cache, block_table, B):
    if block_table is None:
        _need(kv_cache, "kv_cache", torch.bfloat16)
        if kv_cache.dim() != 3 or kv_cache.shape[0] != B or kv_cache.shape[2] != D_QK or kv_cache.shape[1] % PAGE:
            raise ValueError("contiguous kv_cache must be [B, Tcap, 576] with Tcap % 64 == 0")
        return int(kv_cache.shape[1]) // PAGE, 0, None
    _need(block_table, "block_table", torch.int32)
    _need(kv_cache, "kv_cache", torch.bfloat16)
    if kv_cache.dim() != 3 or tuple(kv_cache.shape[1:]) != (PAGE, D_QK):
        raise ValueError("paged kv_cache must be [num_pages, 64, 576]")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B, max_blocks]")
    return int(block_table.shape[1]), int(kv_cache.shape[0]), block_table.data_ptr()


def mla_decode(q, kv_cache, block_table, cache_seqlens, out, lse, softmax_scale: float, stream=None) -> None:
    """Absorbed decode (see include/mla.h).  q [B,H,576] bf16; kv_cache paged
    [num_pages,64,576] with block_table [B,max_blocks] int32, or contiguous
    [B,Tcap,576] with block_table None; cache_seqlens [B] int32; out [B,H,512] fp32;
    lse [B,H] fp32."""
    if q.dim() == 4 and q.shape[1] == 1:  # [B, 1, H, 576] (s_q = 1)
        q = q.view(q.shape[0], q.shape[2], q.shape[3])
    B, H = int(q.shape[0]), int(q.shape[1])
    _need(q, "q", torch.bfloat16, (B, H, D_QK))
    _need(cache_seqlens, "cache_seqlens", torch.int32, (B,))
    _need(out, "out", torch.float32, (B, H, D_LATENT))
    _need(lse, "lse", torch.float32, (B, H))
    max_blocks, num_pages, bt = _cache_args(kv_cache, block_table, B)
    _check(lib.mla_decode(q.data_ptr(), kv_cache.data_ptr(), bt, cache_seqlens.data_ptr(), out.data_ptr(),
                          lse.data_ptr(), B, H, num_pages, max_blocks, float(softmax_scale), _stream(stream)))


def mla_decode_multi(q, kv_cache, block_table, cache_seqlens, out, lse, softmax_scale: float, stream=None) -> None:
    """Decode of s_q causal query tokens per sequence (see include/mla.h).
    q [B,s_q,H,576] bf16; out [B,s_q,H,512] fp32; lse [B,s_q,H] fp32; the cache
    arguments are those of mla_decode."""
    if q.dim() != 4:
        raise ValueError("q must be [B, s_q, H, 576]")
    B, SQ, H = int(q.shape[0]), int(q.shape[1]), int(q.shape[2])
    _need(q, "q", torch.bfloat16, (B, SQ, H, D_QK))
    _need(cache_seqlens, "cache_seqlens", torch.int32, (B,))
    _need(out, "out", torch.float32, (B, SQ, H, D_LATENT))
    _need(lse, "lse", torch.float32, (B, SQ, H))
    max_blocks, num_pages, bt = _cache_args(kv_cache, block_table, B)
    _check(lib.mla_decode_multi(q.data_ptr(), kv_cache.data_ptr(), bt, cache_seqlens.data_ptr(), out.data_ptr(),
                                lse.data_ptr(), B, SQ, H, num_pages, max_blocks, float(softmax_scale),
                                _stream(stream)))


def _noalloc_args(q, kv_cache, block_table, cache_seqlens, out, lse):
    if q.dim() == 4 and q.shape[1] == 1:  # [B, 1, H, 576] (s_q = 1)
        q = q.view(q.shape[0], q.shape[2], q.shape[3])
    B, H = int(q.shape[0]), int(q.shape[1])
    _need(q, "q", torch.bfloat16, (B, H, D_QK))
    _need(cache_seqlens, "cache_seqlens", torch.int32, (B,))
    _need(out, "out", torch.float32, (B, H, D_LATENT))
    _need(lse, "lse", torch.float32, (B, H))
    if block_table is None:
        _need(kv_cache, "kv_cache", torch.bfloat16)
        if kv_cache.dim() != 3 or kv_cache.shape[0] != B or kv_cache.shape[2] != D_QK or kv_cache.shape[1] % PAGE:
            raise ValueError("contiguous kv_cache must be [B, Tcap, 576] with Tcap % 64 == 0")
        max_blocks, num_pages, bt = int(kv_cache.shape[1]) // PAGE, 0, None
    else:
        _need(block_table, "block_table", torch.int32)
        _need(kv_cache, "kv_cache", torch.bfloat16)
        if kv_cache.dim() != 3 or tuple(kv_cache.shape[1:]) != (PAGE, D_QK):
            raise ValueError("paged kv_cache must be [num_pages, 64, 576]")
        if block_table.dim() != 2 or block_table.shape[0] != B:
            raise ValueError("block_table must be [B, max_blocks]")
        max_blocks, num_pages, bt = int(block_table.shape[1]), int(kv_cache.shape[0]), block_table.data_ptr()
    return (q.data_ptr(), kv_cache.data_ptr(), bt, cache_seqlens.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H,
            num_pages, max_blocks)


def mla_decode_noalloc(q, kv_cache, block_table, cache_seqlens, out, lse, softmax_scale: float,
                       stream=None) -> None:
    """mla_decode for callers that cannot allocate device memory: same arguments and
    results, scratch from the library's static 32 MiB device array (see include/mla.h)."""
    args = _noalloc_args(q, kv_cache, block_table, cache_seqlens, out, lse)
    _check(lib.mla_decode_noalloc(*args, float(softmax_scale), _stream(stream)))


def mla_absorb_q(q_nope, q_rope, w_uk, q_out, stream=None) -> None:
    """q_out[b,h] = [q_nope[b,h] W_UK[h] | q_rope[b,h]] (bf16, fp32 accumulate)."""
    B, H = int(q_nope.shape[0]), int(q_nope.shape[1])
    _need(q_nope, "q_nope", torch.bfloat16, (B, H, D_NOPE))
    _need(q_rope, "q_rope", torch.bfloat16, (B, H, D_ROPE))
    _need(w_uk, "w_uk", torch.bfloat16, (H, D_NOPE, D_LATENT))
    _need(q_out, "q_out", torch.bfloat16, (B, H, D_QK))
    _check(lib.mla_absorb_q(q_nope.data_ptr(), q_rope.data_ptr(), w_uk.data_ptr(), q_out.data_ptr(), B, H,
                            _stream(stream)))


def mla_absorb_o(out_latent, w_uv, out, stream=None) -> None:
    """out[b,h] = bf16(out_latent[b,h]) W_UV[h] (fp32 accumulate, fp32 out)."""
    B, H = int(out_latent.shape[0]), int(out_latent.shape[1])
    _need(out_latent, "out_latent", torch.float32, (B, H, D_LATENT))
    _need(w_uv, "w_uv", torch.bfloat16, (H, D_LATENT, D_V))
    _need(out, "out", torch.float32, (B, H, D_V))
    _check(lib.mla_absorb_o(out_latent.data_ptr(), w_uv.data_ptr(), out.data_ptr(), B, H, _stream(stream)))


def mla_workspace_size(batch: int, heads: int, max_blocks: int) -> int:
    return int(lib.mla_workspace_size(batch, heads, max_blocks))


def mla_set_workspace(buf: torch.Tensor | None) -> None:
    """Use ``buf`` (a CUDA uint8 tensor the caller keeps alive) as the workspace, or None."""
    if buf is None:
        _check(lib.mla_set_workspace(None, 0))
    else:
        _need(buf, "workspace", torch.uint8)
        _check(lib.mla_set_workspace(buf.data_ptr(), buf.numel()))


def mla_get_device_error(stream=None) -> int:
    """Synchronise and return (and clear) the device error status code (0 = none)."""
    return int(lib.mla_get_device_error(_stream(stream)))


def mla_status_string(status: int) -> str:
    return lib.mla_status_string(status).decode()


def mla_set_knob(name: str, value: int) -> None:
    _check(lib.mla_set_knob(KNOB[name], int(value)))


def mla_get_knob(name: str) -> int:
    return int(lib.mla_get_knob(KNOB[name]))


def mla_selected_decode_kernel(heads: int) -> int:
    """2 = dim-split pair kernel, 3 = head-split pair kernel (what mla_decode runs for ``heads`` now)."""
    return int(lib.mla_selected_decode_kernel(int(heads)))


def mla_timing_enable(enable: bool = True) -> None:
    _check(lib.mla_timing_enable(1 if enable else 0))


def mla_timing_read() -> tuple[list[float], int]:
    """Summed milliseconds of (schedule, decode, combine) since enabling, and the call count."""
    ms = (ctypes.c_float * 3)()
    calls = ctypes.c_int()
    _check(lib.mla_timing_read(ms, ctypes.byref(calls)))
    return [ms[0], ms[1], ms[2]], calls.value

"""ctypes binding of libflashblock.so (include/flashblock.h).

Argument marshalling only: every function here has the name of the C entry
point it calls, takes torch tensors where the C call takes device pointers,
and raises :class:`FlashBlockError` when the call returns a non-zero status.
No arithmetic of the method happens in Python; there is no fallback path --
if the library is missing, loading it raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libflashblock.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "flashblock.h")

FB_BF16, FB_FP32 = 0, 1
STATUS = {0: "FB_OK", 1: "FB_ERR_INVALID_ARG", 2: "FB_ERR_UNSUPPORTED", 3: "FB_ERR_ALIGNMENT",
          4: "FB_ERR_WORKSPACE", 5: "FB_ERR_LAUNCH", 6: "FB_ERR_DEVICE_TIMEOUT", 7: "FB_ERR_BOUNDS"}


class FlashBlockError(RuntimeError):
    def __init__(self, where: str, status: int):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class fb_desc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_len", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("kv_capacity", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("block_table", ctypes.c_void_p),
        ("prefix_lens", ctypes.c_void_p),
        ("chunk_size", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("num_splits", ctypes.c_int32),
    ]


_lib = None


# FB_ABI_VERSION of include/flashblock.h that the signatures below follow.
ABI_VERSION = 2


def load() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FileNotFoundError(
                f"{LIB_PATH} is missing: build it with `python -m block_diffusion_attention_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        D = ctypes.POINTER(fb_desc)
        sig = {
            "fb_cache_rows": (ctypes.c_int64, [D]),
            "fb_workspace_bytes": (SZ, [D]),
            "fb_prefix_partial": (I32, [D, P, P, P, P, P, P, P, SZ, P, P]),
            "fb_prefix_partial_noalloc": (I32, [D, P, P, P, P, P, P, P, P]),
            "fb_block_step": (I32, [D, P, P, P, P, P, P, P, P, SZ, P, P]),
            "fb_block_step_append": (I32, [D, P, P, P, P, P, P, P, P, P, P, P, SZ, P, P]),
            "fb_full_reference_gpu": (I32, [D, P, P, P, P, P, P, P, P, SZ, P, P]),
            "fb_chunk_means": (I32, [D, P, I32, I32, P, P, P]),
            "fb_chunk_means_tail": (I32, [D, P, I32, P, P, P]),
            "fb_select_chunks": (I32, [D, P, P, P, P, P]),
            "fb_kv_append": (I32, [D, P, P, P, P, P, P, P]),
            "fb_complement_chunks": (I32, [D, P, P, I32, P, P]),
            "fb_merge_partials": (I32, [D, P, P, P, P, P, P, P]),
            "fb_headwise_refresh_mask": (I32, [D, P, P, ctypes.c_float, P, P, P]),
            "fb_threshold_refresh_mask": (I32, [D, P, P, P, P, ctypes.c_float, I32, P, P, P, SZ, P]),
            "fb_prefix_partial_masked": (I32, [D, P, P, P, P, P, P, P, P, SZ, P, P]),
            "fb_status_string": (ctypes.c_char_p, [I32]),
            "fb_launch_count": (ctypes.c_uint64, []),
            "fb_abi_version": (I32, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        if lib.fb_abi_version() != ABI_VERSION:
            raise RuntimeError(f"{LIB_PATH} has ABI version {lib.fb_abi_version()}, this binding needs "
                               f"{ABI_VERSION}: rebuild it")
        _lib = lib
    return _lib


def header_functions():
    """Names of the functions declared in include/flashblock.h."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fb_[a-z0-9_]+)\s*\(", src)))


def make_desc(batch, num_q_heads, num_kv_heads, head_dim, block_len, dtype=FB_BF16, softmax_scale=1.0,
              kv_capacity=0, page_size=0, max_pages=0, num_pages=0, block_table=None, prefix_lens=None,
              chunk_size=0, topk=0, num_splits=0) -> fb_desc:
    d = fb_desc()
    d.batch, d.num_q_heads, d.num_kv_heads = batch, num_q_heads, num_kv_heads
    d.head_dim, d.block_len, d.dtype = head_dim, block_len, dtype
    d.softmax_scale = softmax_scale
    d.kv_capacity, d.page_size, d.max_pages, d.num_pages = kv_capacity, page_size, max_pages, num_pages
    d.block_table = None if block_table is None else block_table.data_ptr()
    d.prefix_lens = None if prefix_lens is None else prefix_lens.data_ptr()
    d.chunk_size, d.topk, d.num_splits = chunk_size, topk, num_splits
    return d


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _ok(where: str, st: int):
    if st != 0:
        raise FlashBlockError(where, st)


def fb_cache_rows(d: fb_desc) -> int:
    return load().fb_cache_rows(ctypes.byref(d))


def fb_workspace_bytes(d: fb_desc) -> int:
    return load().fb_workspace_bytes(ctypes.byref(d))


def fb_prefix_partial(d, Q, Kcache, Vcache, chunk_idx, O_pre, LSE_pre, workspace, dev_status, stream=None):
    _ok("fb_prefix_partial", load().fb_prefix_partial(
        ctypes.byref(d), _p(Q), _p(Kcache), _p(Vcache), _p(chunk_idx), _p(O_pre), _p(LSE_pre),
        _p(workspace), _nbytes(workspace), _p(dev_status), _s(stream)))


def fb_prefix_partial_noalloc(d, Q, Kcache, Vcache, chunk_idx, O_pre, LSE_pre, dev_status, stream=None):
    """fb_prefix_partial with the library's static scratch in place of a workspace."""
    _ok("fb_prefix_partial_noalloc", load().fb_prefix_partial_noalloc(
        ctypes.byref(d), _p(Q), _p(Kcache), _p(Vcache), _p(chunk_idx), _p(O_pre), _p(LSE_pre),
        _p(dev_status), _s(stream)))


def fb_block_step(d, Q, Kblk, Vblk, O_pre, LSE_pre, O, LSE_out, dev_status, stream=None, workspace=None):
    _ok("fb_block_step", load().fb_block_step(
        ctypes.byref(d), _p(Q), _p(Kblk), _p(Vblk), _p(O_pre), _p(LSE_pre), _p(O), _p(LSE_out),
        _p(workspace), _nbytes(workspace), _p(dev_status), _s(stream)))


def fb_block_step_append(d, Q, Kblk, Vblk, O_pre, LSE_pre, O, LSE_out, Kcache, Vcache, lens_inout, dev_status,
                         stream=None, workspace=None):
    _ok("fb_block_step_append", load().fb_block_step_append(
        ctypes.byref(d), _p(Q), _p(Kblk), _p(Vblk), _p(O_pre), _p(LSE_pre), _p(O), _p(LSE_out), _p(Kcache),
        _p(Vcache), _p(lens_inout), _p(workspace), _nbytes(workspace), _p(dev_status), _s(stream)))


def fb_full_reference_gpu(d, Q, Kcache, Vcache, Kblk, Vblk, O, LSE_out, workspace, dev_status, stream=None):
    _ok("fb_full_reference_gpu", load().fb_full_reference_gpu(
        ctypes.byref(d), _p(Q), _p(Kcache), _p(Vcache), _p(Kblk), _p(Vblk), _p(O), _p(LSE_out),
        _p(workspace), _nbytes(workspace), _p(dev_status), _s(stream)))


def fb_chunk_means(d, Kcache, chunk_begin, chunk_end, Kmean, dev_status, stream=None):
    _ok("fb_chunk_means", load().fb_chunk_means(
        ctypes.byref(d), _p(Kcache), int(chunk_begin), int(chunk_end), _p(Kmean), _p(dev_status), _s(stream)))


def fb_chunk_means_tail(d, Kcache, rows, Kmean, dev_status, stream=None):
    _ok("fb_chunk_means_tail", load().fb_chunk_means_tail(
        ctypes.byref(d), _p(Kcache), int(rows), _p(Kmean), _p(dev_status), _s(stream)))


def fb_select_chunks(d, Q, Kmean, chunk_idx, dev_status, stream=None):
    _ok("fb_select_chunks", load().fb_select_chunks(
        ctypes.byref(d), _p(Q), _p(Kmean), _p(chunk_idx), _p(dev_status), _s(stream)))


def fb_kv_append(d, Kblk, Vblk, Kcache, Vcache, lens_inout, dev_status, stream=None):
    _ok("fb_kv_append", load().fb_kv_append(
        ctypes.byref(d), _p(Kblk), _p(Vblk), _p(Kcache), _p(Vcache), _p(lens_inout), _p(dev_status),
        _s(stream)))


def fb_complement_chunks(d, chunk_idx, comp_idx, comp_cap, dev_status, stream=None):
    _ok("fb_complement_chunks", load().fb_complement_chunks(
        ctypes.byref(d), _p(chunk_idx), _p(comp_idx), int(comp_cap), _p(dev_status), _s(stream)))


def fb_merge_partials(d, O_a, LSE_a, O_b, LSE_b, O_out, LSE_out, stream=None):
    _ok("fb_merge_partials", load().fb_merge_partials(
        ctypes.byref(d), _p(O_a), _p(LSE_a), _p(O_b), _p(LSE_b), _p(O_out), _p(LSE_out), _s(stream)))


def fb_headwise_refresh_mask(d, Q_now, Q_ref, gamma, unit_mask, sim_out=None, stream=None):
    _ok("fb_headwise_refresh_mask", load().fb_headwise_refresh_mask(
        ctypes.byref(d), _p(Q_now), _p(Q_ref), float(gamma), _p(unit_mask), _p(sim_out), _s(stream)))


def fb_threshold_refresh_mask(d, K_prev, V_prev, K_now, V_now, eps, tau, unit_mask, count_out, workspace,
                              stream=None):
    _ok("fb_threshold_refresh_mask", load().fb_threshold_refresh_mask(
        ctypes.byref(d), _p(K_prev), _p(V_prev), _p(K_now), _p(V_now), float(eps), int(tau), _p(unit_mask),
        _p(count_out), _p(workspace), _nbytes(workspace), _s(stream)))


def fb_prefix_partial_masked(d, Q, Kcache, Vcache, chunk_idx, unit_mask, O_pre, LSE_pre, workspace, dev_status,
                             stream=None):
    """fb_prefix_partial for the units whose unit_mask entry is non-zero."""
    _ok("fb_prefix_partial_masked", load().fb_prefix_partial_masked(
        ctypes.byref(d), _p(Q), _p(Kcache), _p(Vcache), _p(chunk_idx), _p(unit_mask), _p(O_pre), _p(LSE_pre),
        _p(workspace), _nbytes(workspace), _p(dev_status), _s(stream)))


def fb_status_string(status: int) -> str:
    return load().fb_status_string(int(status)).decode()


def fb_launch_count() -> int:
    return int(load().fb_launch_count())


def fb_abi_version() -> int:
    return int(load().fb_abi_version())

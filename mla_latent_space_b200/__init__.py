"""Python binding of libmla_b200.so: MLA decode in absorbed latent space on
B200 (sm_100a).

Argument marshalling only.  Every function takes torch tensors, checks their
dtype / shape / device on the host, and passes raw device pointers and the
current CUDA stream to the C ABI of ``include/mla.h`` under the same name.
All computation happens in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and loading fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_b200.so")

MLA_OK = 0
MLA_CACHE_BF16 = 0
MLA_CACHE_FP8_E4M3 = 1
D_QK, D_V, PAGE, TILE_ROWS = 576, 512, 64, 128
D_HEAD, D_ROPE = 128, 64   # per-head dims before absorption, RoPE dims
FP8_PAGE_BYTES = PAGE * D_V + PAGE * (D_QK - D_V) * 2

EXPORTED = ("mla_schedule_bytes", "mla_workspace_bytes", "mla_get_schedule", "mla_decode_fwd",
            "mla_combine", "mla_get_device_status", "mla_plan_schedule_host",
            "mla_error_string", "mla_version", "mla_decode_fwd_noalloc")


class MLAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {error_string(code)} ({code})")


class mla_shape_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("batch", "s_q", "num_heads", "d_qk", "d_v", "page_size",
                                              "max_pages_per_seq", "num_pages", "cache_dtype", "causal")]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it was never built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m mla_latent_space_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
        sp = ctypes.POINTER(mla_shape_t)
        L.mla_schedule_bytes.argtypes = [sp, i32]
        L.mla_schedule_bytes.restype = sz
        L.mla_workspace_bytes.argtypes = [sp, i32]
        L.mla_workspace_bytes.restype = sz
        L.mla_get_schedule.argtypes = [sp, vp, i32, vp, sz, vp]
        L.mla_get_schedule.restype = i32
        dec = [sp, vp, vp, vp, vp, vp, f32, vp, vp, sz, vp, vp, vp]
        L.mla_decode_fwd.argtypes = dec
        L.mla_decode_fwd.restype = i32
        L.mla_combine.argtypes = [sp, vp, vp, sz, vp, vp, vp]
        L.mla_combine.restype = i32
        L.mla_get_device_status.argtypes = [vp, vp, vp, ctypes.POINTER(i32)]
        L.mla_get_device_status.restype = i32
        L.mla_plan_schedule_host.argtypes = [sp, vp, i32, vp, sz]
        L.mla_plan_schedule_host.restype = i32
        L.mla_decode_fwd_noalloc.argtypes = [sp, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp]
        L.mla_decode_fwd_noalloc.restype = i32
        L.mla_sparse_workspace_bytes.argtypes = [sp, i32, i32]
        L.mla_sparse_workspace_bytes.restype = sz
        L.mla_sparse_decode_fwd.argtypes = [sp, i32, vp, vp, vp, vp, vp, vp, f32, vp, sz, vp, vp, vp]
        L.mla_sparse_decode_fwd.restype = i32
        L.mla_sparse_get_device_status.argtypes = [sp, i32, i32, vp, vp, ctypes.POINTER(i32)]
        L.mla_sparse_get_device_status.restype = i32
        L.mla_var6_workspace_bytes.argtypes = [sp, i32, i32]
        L.mla_var6_workspace_bytes.restype = sz
        L.mla_var6_decode_fwd.argtypes = [sp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, f32, vp, sz, vp, vp, vp]
        L.mla_var6_decode_fwd.restype = i32
        L.mla_var6_get_device_status.argtypes = [sp, i32, i32, vp, vp, ctypes.POINTER(i32)]
        L.mla_var6_get_device_status.restype = i32
        L.mla_absorb_q.argtypes = [i32, i32, vp, vp, vp, vp, vp]
        L.mla_absorb_q.restype = i32
        L.mla_decompress_o.argtypes = [i32, i32, vp, vp, vp, vp, vp]
        L.mla_decompress_o.restype = i32
        L.mla_error_string.argtypes = [i32]
        L.mla_error_string.restype = ctypes.c_char_p
        L.mla_version.argtypes = []
        L.mla_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def error_string(code: int) -> str:
    return lib().mla_error_string(int(code)).decode()


def make_shape(batch, s_q, num_heads, max_pages_per_seq, num_pages, cache_dtype="bf16", causal=False) -> mla_shape_t:
    cd = {"bf16": MLA_CACHE_BF16, "fp8": MLA_CACHE_FP8_E4M3}[cache_dtype] if isinstance(cache_dtype, str) \
        else int(cache_dtype)
    return mla_shape_t(int(batch), int(s_q), int(num_heads), D_QK, D_V, PAGE, int(max_pages_per_seq),
                       int(num_pages), cd, int(bool(causal)))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, where: str):
    if rc != MLA_OK:
        raise MLAError(rc, where)


def _need(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def num_sms(device=None) -> int:
    return torch.cuda.get_device_properties(device if device is not None else torch.cuda.current_device()).multi_processor_count


def mla_schedule_bytes(shape: mla_shape_t, n_sms: int) -> int:
    return int(lib().mla_schedule_bytes(ctypes.byref(shape), int(n_sms)))


def mla_workspace_bytes(shape: mla_shape_t, n_sms: int) -> int:
    return int(lib().mla_workspace_bytes(ctypes.byref(shape), int(n_sms)))


def mla_get_schedule(shape: mla_shape_t, seqlens: torch.Tensor, n_sms: int, sched: torch.Tensor, stream=None):
    _need(seqlens, "seqlens", torch.int32, (shape.batch,))
    _need(sched, "sched", None)
    _check(lib().mla_get_schedule(ctypes.byref(shape), _ptr(seqlens), int(n_sms), _ptr(sched),
                                  sched.numel() * sched.element_size(), _stream(stream)), "mla_get_schedule")


def mla_plan_schedule_host(shape: mla_shape_t, seqlens: torch.Tensor, n_sms: int) -> torch.Tensor:
    """Host planner (same code as the device scheduler); CPU tensors in and out."""
    sl = seqlens.to(torch.int32).contiguous().cpu()
    nbytes = mla_schedule_bytes(shape, n_sms)
    out = torch.zeros(nbytes // 4, dtype=torch.int32)
    _check(lib().mla_plan_schedule_host(ctypes.byref(shape), _ptr(sl), int(n_sms), _ptr(out), nbytes),
           "mla_plan_schedule_host")
    return out


def _check_decode_tensors(shape, q, kv_cache, kv_scale, block_table, seqlens, out, lse):
    b, s, h = shape.batch, shape.s_q, shape.num_heads
    _need(q, "q", torch.bfloat16, (b, s, h, D_QK))
    if shape.cache_dtype == MLA_CACHE_BF16:
        _need(kv_cache, "kv_cache", torch.bfloat16, (shape.num_pages, PAGE, D_QK))
        if kv_scale is not None:
            raise ValueError("kv_scale is only used with the fp8 cache")
    else:
        _need(kv_cache, "kv_cache", torch.uint8, (shape.num_pages, FP8_PAGE_BYTES))
        _need(kv_scale, "kv_scale", torch.float32, (shape.num_pages, PAGE))
    _need(block_table, "block_table", torch.int32, (b, shape.max_pages_per_seq))
    _need(seqlens, "seqlens", torch.int32, (b,))
    if out is not None:
        _need(out, "out", torch.bfloat16, (b, s, h, D_V))
    if lse is not None:
        _need(lse, "lse", torch.float32, (b, s, h))


def _decode_common(fn, where, shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, sched,
                   workspace, out, lse, stream):
    b, s, h = shape.batch, shape.s_q, shape.num_heads
    _need(q, "q", torch.bfloat16, (b, s, h, D_QK))
    if shape.cache_dtype == MLA_CACHE_BF16:
        _need(kv_cache, "kv_cache", torch.bfloat16, (shape.num_pages, PAGE, D_QK))
        if kv_scale is not None:
            raise ValueError("kv_scale is only used with the fp8 cache")
    else:
        _need(kv_cache, "kv_cache", torch.uint8, (shape.num_pages, FP8_PAGE_BYTES))
        _need(kv_scale, "kv_scale", torch.float32, (shape.num_pages, PAGE))
    _need(block_table, "block_table", torch.int32, (b, shape.max_pages_per_seq))
    _need(seqlens, "seqlens", torch.int32, (b,))
    _need(sched, "sched", None)
    _need(workspace, "workspace", None)
    _need(out, "out", torch.bfloat16, (b, s, h, D_V))
    _need(lse, "lse", torch.float32, (b, s, h))
    rc = fn(ctypes.byref(shape), _ptr(q), _ptr(kv_cache), _ptr(kv_scale), _ptr(block_table), _ptr(seqlens),
            float(softmax_scale), _ptr(sched), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _ptr(out), _ptr(lse), _stream(stream))
    _check(rc, where)


def mla_decode_fwd(shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, sched, workspace, out, lse,
                   stream=None):
    _decode_common(lib().mla_decode_fwd, "mla_decode_fwd", shape, q, kv_cache, kv_scale, block_table, seqlens,
                   softmax_scale, sched, workspace, out, lse, stream)


def mla_decode_fwd_noalloc(shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, out, lse,
                           device_status: Optional[torch.Tensor] = None, stream=None):
    """The whole decode step (schedule, decode, combine) with the library's
    static scratch instead of caller buffers; see mla.h for its limits."""
    _check_decode_tensors(shape, q, kv_cache, kv_scale, block_table, seqlens, out, lse)
    if device_status is not None:
        _need(device_status, "device_status", torch.int32)
    rc = lib().mla_decode_fwd_noalloc(ctypes.byref(shape), _ptr(q), _ptr(kv_cache), _ptr(kv_scale),
                                      _ptr(block_table), _ptr(seqlens), float(softmax_scale), _ptr(out), _ptr(lse),
                                      _ptr(device_status), _stream(stream))
    _check(rc, "mla_decode_fwd_noalloc")


def mla_combine(shape, sched, workspace, out, lse, stream=None):
    _need(out, "out", torch.bfloat16, (shape.batch, shape.s_q, shape.num_heads, D_V))
    _need(lse, "lse", torch.float32, (shape.batch, shape.s_q, shape.num_heads))
    _check(lib().mla_combine(ctypes.byref(shape), _ptr(sched), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _ptr(out), _ptr(lse), _stream(stream)),
           "mla_combine")


def mla_get_device_status(sched, workspace, stream=None) -> int:
    st = ctypes.c_int(0)
    _check(lib().mla_get_device_status(_ptr(sched), _ptr(workspace), _stream(stream), ctypes.byref(st)),
           "mla_get_device_status")
    return int(st.value)


def mla_sparse_workspace_bytes(shape: mla_shape_t, topk: int, n_sms: int) -> int:
    return int(lib().mla_sparse_workspace_bytes(ctypes.byref(shape), int(topk), int(n_sms)))


class SparseDecoder:
    """Token-level sparse decode through the C ABI: holds the zero-filled
    workspace (torch allocation) for one shape, list length and device."""

    def __init__(self, shape: mla_shape_t, topk: int, device=None):
        self.shape, self.topk = shape, int(topk)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.n_sms = num_sms(self.device)
        nb = mla_sparse_workspace_bytes(shape, self.topk, self.n_sms)
        if nb == 0:
            raise MLAError(-2, "SparseDecoder: shape not supported (causal=0, topk >= 1)")
        self.workspace = torch.zeros(nb, dtype=torch.uint8, device=self.device)

    def decode(self, q, kv_cache, block_table, seqlens, indices, softmax_scale, out, lse, stream=None,
               kv_scale=None):
        sh = self.shape
        _check_decode_tensors(sh, q, kv_cache, kv_scale, block_table, seqlens, out, lse)
        _need(indices, "indices", torch.int32, (sh.batch, sh.s_q, self.topk))
        rc = lib().mla_sparse_decode_fwd(ctypes.byref(sh), self.topk, _ptr(q), _ptr(kv_cache), _ptr(kv_scale),
                                         _ptr(block_table),
                                         _ptr(seqlens), _ptr(indices), float(softmax_scale), _ptr(self.workspace),
                                         self.workspace.numel(), _ptr(out), _ptr(lse), _stream(stream))
        _check(rc, "mla_sparse_decode_fwd")

    def status(self, stream=None) -> int:
        st = ctypes.c_int(0)
        _check(lib().mla_sparse_get_device_status(ctypes.byref(self.shape), self.topk, self.n_sms,
                                                  _ptr(self.workspace), _stream(stream), ctypes.byref(st)),
               "mla_sparse_get_device_status")
        return int(st.value)


class Var6Decoder:
    """MLAvar6+ split decode through the C ABI: the older tokens in latent
    form, the n newest as decompressed per-head keys and values.  Holds the
    zero-filled workspace for one shape, n and device."""

    def __init__(self, shape: mla_shape_t, n_new: int, device=None):
        self.shape, self.n_new = shape, int(n_new)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.n_sms = num_sms(self.device)
        nb = int(lib().mla_var6_workspace_bytes(ctypes.byref(shape), self.n_new, self.n_sms))
        if nb == 0:
            raise MLAError(-2, "Var6Decoder: shape not supported (s_q <= 32; causal steps need n >= s_q)")
        self.workspace = torch.zeros(nb, dtype=torch.uint8, device=self.device)

    def decode(self, qz, q, kv_cache, block_table, seqlens, k_new, v_new, w_kvb2, softmax_scale, out, lse,
               stream=None, kv_scale=None):
        sh, n = self.shape, self.n_new
        _check_decode_tensors(sh, qz, kv_cache, kv_scale, block_table, seqlens, None, None)
        _need(q, "q", torch.bfloat16, (sh.batch, sh.s_q, sh.num_heads, D_HEAD + D_ROPE))
        _need(k_new, "k_new", torch.bfloat16, (sh.batch, n, sh.num_heads, D_HEAD))
        _need(v_new, "v_new", torch.bfloat16, (sh.batch, n, sh.num_heads, D_HEAD))
        _need(w_kvb2, "w_kvb2", torch.bfloat16, (sh.num_heads, D_HEAD, D_V))
        _need(out, "out", torch.bfloat16, (sh.batch, sh.s_q, sh.num_heads, D_HEAD))
        _need(lse, "lse", torch.float32, (sh.batch, sh.s_q, sh.num_heads))
        rc = lib().mla_var6_decode_fwd(ctypes.byref(sh), n, _ptr(qz), _ptr(q), _ptr(kv_cache), _ptr(kv_scale),
                                       _ptr(block_table), _ptr(seqlens), _ptr(k_new), _ptr(v_new), _ptr(w_kvb2),
                                       float(softmax_scale), _ptr(self.workspace), self.workspace.numel(), _ptr(out),
                                       _ptr(lse), _stream(stream))
        _check(rc, "mla_var6_decode_fwd")

    def status(self, stream=None) -> int:
        st = ctypes.c_int(0)
        _check(lib().mla_var6_get_device_status(ctypes.byref(self.shape), self.n_new, self.n_sms,
                                                _ptr(self.workspace), _stream(stream), ctypes.byref(st)),
               "mla_var6_get_device_status")
        return int(st.value)


def _rows_heads(t: torch.Tensor, name: str, last: int):
    if t.dim() < 2 or t.shape[-1] != last:
        raise ValueError(f"{name} must have shape [..., heads, {last}], got {tuple(t.shape)}")
    return t.numel() // (t.shape[-2] * last), t.shape[-2]


def mla_absorb_q(q, w_k, qz, device_status: Optional[torch.Tensor] = None, stream=None):
    """qz[..., j, :512] = q[..., j, :128] . w_k[j]^T and qz[..., j, 512:] =
    q[..., j, 128:] on the tensor core.  q bf16 [..., h, 192], w_k bf16
    [h, 512, 128], qz bf16 [..., h, 576] (the decode's query rows)."""
    _need(q, "q", torch.bfloat16)
    rows, h = _rows_heads(q, "q", D_HEAD + D_ROPE)
    _need(w_k, "w_k", torch.bfloat16, (h, D_V, D_HEAD))
    _need(qz, "qz", torch.bfloat16, tuple(q.shape[:-1]) + (D_QK,))
    if device_status is not None:
        _need(device_status, "device_status", torch.int32)
    _check(lib().mla_absorb_q(int(rows), int(h), _ptr(q), _ptr(w_k), _ptr(qz), _ptr(device_status),
                              _stream(stream)), "mla_absorb_q")


def mla_decompress_o(o_lat, w_kvb2, out, device_status: Optional[torch.Tensor] = None, stream=None):
    """out[..., j, v] = sum_c o_lat[..., j, c] w_kvb2[j, v, c] on the tensor
    core.  o_lat bf16 [..., h, 512], w_kvb2 bf16 [h, 128, 512], out bf16
    [..., h, 128]."""
    _need(o_lat, "o_lat", torch.bfloat16)
    rows, h = _rows_heads(o_lat, "o_lat", D_V)
    _need(w_kvb2, "w_kvb2", torch.bfloat16, (h, D_HEAD, D_V))
    _need(out, "out", torch.bfloat16, tuple(o_lat.shape[:-1]) + (D_HEAD,))
    if device_status is not None:
        _need(device_status, "device_status", torch.int32)
    _check(lib().mla_decompress_o(int(rows), int(h), _ptr(o_lat), _ptr(w_kvb2), _ptr(out), _ptr(device_status),
                                  _stream(stream)), "mla_decompress_o")


class Decoder:
    """Holds the schedule and workspace buffers (torch allocations) for one
    shape and runs schedule -> decode -> combine through the C ABI."""

    def __init__(self, shape: mla_shape_t, device=None, n_sms: Optional[int] = None):
        self.shape = shape
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.n_sms = num_sms(self.device) if n_sms is None else int(n_sms)
        sb = mla_schedule_bytes(shape, self.n_sms)
        wb = mla_workspace_bytes(shape, self.n_sms)
        if sb == 0 or wb == 0:
            raise MLAError(-1, "Decoder: invalid shape")
        self.sched = torch.empty(sb, dtype=torch.uint8, device=self.device)
        self.workspace = torch.zeros(wb, dtype=torch.uint8, device=self.device)

    def schedule(self, seqlens, stream=None):
        mla_get_schedule(self.shape, seqlens, self.n_sms, self.sched, stream)

    def decode(self, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, out, lse, stream=None,
               decode_fn=None):
        """Decode + combine.  ``decode_fn`` replaces mla_decode_fwd (same
        signature); the tests pass the SIMT kernel of the test library."""
        fn = mla_decode_fwd if decode_fn is None else decode_fn
        fn(self.shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, self.sched, self.workspace,
           out, lse, stream)
        mla_combine(self.shape, self.sched, self.workspace, out, lse, stream)

    def status(self, stream=None) -> int:
        return mla_get_device_status(self.sched, self.workspace, stream)

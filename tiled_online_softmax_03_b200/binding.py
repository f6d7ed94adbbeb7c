"""ctypes binding of libfa.so (include/fa.h): argument marshalling only.

Every step of the attention forward runs in the library's CUDA kernel; this
module checks tensor metadata, allocates the outputs with torch when the
caller does not pass them, and calls ``fa_fwd`` (or ``fa_fwd_splitkv``) on the
current torch stream.
Importing it loads the library and raises if it is missing: there is no
fallback path.
"""

import ctypes
import os

import torch

__all__ = ["FaError", "fa_fwd", "fa_fwd_from_host", "host_chunk_plan", "fa_bwd", "fa_fwd_fp8", "fa_fwd_bias", "fa_fwd_splitkv", "splitkv_workspace_bytes", "load_library", "lib", "FA_OK", "FA_ERR_INVALID_ARG",
           "FA_ERR_UNSUPPORTED", "FA_ERR_CUDA", "FA_ERR_DEVICE_TIMEOUT"]

FA_OK = 0
FA_ERR_INVALID_ARG = -1
FA_ERR_UNSUPPORTED = -2
FA_ERR_CUDA = -3
FA_ERR_DEVICE_TIMEOUT = -4
FA_FP16 = 0
FA_BF16 = 1

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa.so")


class FaError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"fa error {code}: {msg}")
        self.code = code


def load_library(path=LIB_PATH):
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m tiled_online_softmax_03_b200.build` "
            "(there is no non-CUDA fallback)")
    L = ctypes.CDLL(path)
    c_int, c_void_p, c_float = ctypes.c_int, ctypes.c_void_p, ctypes.c_float
    L.fa_fwd.argtypes = [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                         c_int, c_int, c_float, c_int, c_void_p, c_void_p, c_int]
    L.fa_fwd.restype = c_int
    L.fa_bwd.argtypes = [c_void_p] * 9 + [c_int] * 5 + [c_float, c_int, c_void_p, c_void_p,
                                                       ctypes.c_size_t, c_void_p, c_int]
    L.fa_bwd.restype = c_int
    L.fa_bwd_workspace_bytes.argtypes = [c_int] * 4
    L.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
    L.fa_fwd_fp8.argtypes = [c_void_p] * 3 + [c_float] * 3 + [c_void_p, c_void_p] + [c_int] * 5 + \
        [c_float, c_int, c_void_p, c_void_p, ctypes.c_size_t, c_void_p]
    L.fa_fwd_fp8.restype = c_int
    L.fa_fwd_fp8_workspace_bytes.argtypes = [c_int] * 4
    L.fa_fwd_fp8_workspace_bytes.restype = ctypes.c_size_t
    L.fa_fwd_bias.argtypes = [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p,
                              c_void_p, c_int, c_int, c_int, c_int, c_int, c_float, c_int,
                              c_void_p, c_void_p, c_int]
    L.fa_fwd_bias.restype = c_int
    L.fa_fwd_splitkv.argtypes = [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int,
                                 c_int, c_int, c_int, c_float, c_int, c_void_p, c_int, c_void_p,
                                 ctypes.c_size_t, c_void_p, c_int]
    L.fa_fwd_splitkv.restype = c_int
    L.fa_fwd_splitkv_static.argtypes = [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                        c_int, c_int, c_int, c_int, c_float, c_int, c_void_p,
                                        c_int, c_void_p, c_int]
    L.fa_fwd_splitkv_static.restype = c_int
    L.fa_fwd_host.argtypes = [c_void_p] * 5 + [c_int] * 5 + [c_float, c_int, c_void_p] + \
        [c_void_p] * 6 + [c_int, c_void_p, c_int]
    L.fa_fwd_host.restype = c_int
    L.fa_host_chunk_plan.argtypes = [c_int] * 6 + [ctypes.POINTER(ctypes.c_int32), c_int]
    L.fa_host_chunk_plan.restype = c_int
    L.fa_splitkv_workspace_bytes.argtypes = [c_int] * 5
    L.fa_splitkv_workspace_bytes.restype = ctypes.c_size_t
    L.fa_unit_kv_range.argtypes = [c_int] * 8 + [ctypes.POINTER(ctypes.c_int32)]
    L.fa_unit_kv_range.restype = c_int
    L.fa_unit_kv_range_grouped.argtypes = [c_int] * 9 + [ctypes.POINTER(ctypes.c_int32)]
    L.fa_unit_kv_range_grouped.restype = c_int
    L.fa_unit_for_grouped.argtypes = [c_int] * 10
    L.fa_unit_for_grouped.restype = c_int
    L.fa_unit_groups.argtypes = [c_int] * 7 + [ctypes.c_longlong]
    L.fa_unit_groups.restype = c_int
    L.fa_last_error_string.argtypes = []
    L.fa_last_error_string.restype = ctypes.c_char_p
    L.fa_get_device_status.argtypes = []
    L.fa_get_device_status.restype = c_int
    L.fa_set_wait_timeout_ms.argtypes = [c_int]
    L.fa_set_wait_timeout_ms.restype = c_int
    L.fa_num_units.argtypes = [c_int] * 5
    L.fa_num_units.restype = c_int
    L.fa_unit_info.argtypes = [c_int] * 6 + [ctypes.POINTER(ctypes.c_int32)]
    L.fa_unit_info.restype = c_int
    L.fa_unit_for.argtypes = [c_int] * 3
    L.fa_unit_for.restype = c_int
    L.fa_selftest_wait_timeout.argtypes = [c_int]
    L.fa_selftest_wait_timeout.restype = c_int
    L.fa_version.argtypes = []
    L.fa_version.restype = c_int
    return L


lib = load_library()


def last_error():
    return lib.fa_last_error_string().decode(errors="replace")


def check(code):
    if code != FA_OK:
        raise FaError(code, last_error())
    return code


_DTYPES = {torch.float16: FA_FP16, torch.bfloat16: FA_BF16}


def _prepare(q, k, v, key_pad_lens, out, lse, return_lse, scale, stream):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise FaError(FA_ERR_INVALID_ARG, f"{name} must be a contiguous 4-D CUDA tensor")
    if q.dtype not in _DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise FaError(FA_ERR_UNSUPPORTED, "q, k, v must share one dtype: float16 or bfloat16")
    B, Hq, N, d = q.shape
    Hk = k.shape[1]
    if tuple(k.shape) != (B, Hk, N, d) or tuple(v.shape) != (B, Hk, N, d):
        raise FaError(FA_ERR_INVALID_ARG, "k and v must be [B, Hk, N, d] matching q")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    if key_pad_lens is not None:
        if key_pad_lens.dtype != torch.int32 or not key_pad_lens.is_cuda or \
                key_pad_lens.numel() != B:
            raise FaError(FA_ERR_INVALID_ARG, "key_pad_lens must be an int32 CUDA tensor [B]")
    if scale is None:
        scale = float(d) ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    return (B, Hq, Hk, N, d), out, lse, float(scale), stream


def fa_fwd(q, k, v, causal=False, scale=None, key_pad_lens=None, out=None, lse=None,
           return_lse=True, stream=None):
    """O (and LSE) = attention forward of q [B,Hq,N,d] against k, v [B,Hk,N,d].

    Tensors must be CUDA, contiguous, fp16 or bf16 (all the same). ``scale``
    defaults to 1/sqrt(d). ``key_pad_lens`` is an int32 CUDA tensor [B] or
    None. ``out``/``lse`` may be given preallocated. Returns (o, lse) or o.
    """
    (B, Hq, Hk, N, d), out, lse, scale, stream = _prepare(q, k, v, key_pad_lens, out, lse,
                                                          return_lse, scale, stream)
    with torch.cuda.device(q.device):
        check(lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                         lse.data_ptr() if lse is not None else None, B, Hq, Hk, N, d,
                         scale, 1 if causal else 0,
                         key_pad_lens.data_ptr() if key_pad_lens is not None else None,
                         stream, _DTYPES[q.dtype]))
    return (out, lse) if return_lse else out


def _stream_handle(stream, device):
    """(raw cudaStream_t handle, torch stream object or None) for ``stream``: a
    torch.cuda.Stream, a raw handle (int), or None for the device's current
    stream. A torch stream on another device is refused."""
    if stream is None:
        st = torch.cuda.current_stream(device)
        return st.cuda_stream, st
    if isinstance(stream, torch.cuda.Stream):
        if stream.device != device:
            raise FaError(FA_ERR_INVALID_ARG, f"stream is on {stream.device}, not {device}")
        return stream.cuda_stream, stream
    if isinstance(stream, int):
        return stream, torch.cuda.ExternalStream(stream, device=device)
    raise FaError(FA_ERR_INVALID_ARG, "stream must be a torch.cuda.Stream, a raw handle or None")


def fa_fwd_from_host(q, k, v, causal=False, scale=None, key_pad_lens=None, out=None, lse=None,
                     device_buffers=None, device=None, stream=None, chunks=None):
    """``fa_fwd_host`` of the C ABI: the forward on page-locked HOST tensors.

    q [B,Hq,N,d], k and v [B,Hk,N,d] (and key_pad_lens, int32 [B], if given)
    are contiguous pinned CPU tensors; ``out`` [B,Hq,N,d] and ``lse``
    [B,Hq,N] float32, pinned CPU tensors, receive the result (allocated pinned
    when None). The staged device copies live in ``device_buffers``, a dict of
    CUDA tensors 'q', 'k', 'v', 'o', 'lse' of the same shapes and, with
    padding, 'lens' [B] int32; they are allocated on ``device`` (default: the
    current CUDA device) when None. The library cuts the work into ``chunks``
    (None: its default, about 16 MB of inputs each) and overlaps, chunk by
    chunk, the copy in, the attention and the copy out.

    ``stream`` is a torch.cuda.Stream or a raw cudaStream_t handle on
    ``device`` (default: its current stream). The call returns once the work
    is enqueued. Only after ``stream`` has been synchronised (or waited on)
    do ``out`` and ``lse`` hold the result, and only then may q, k, v and
    key_pad_lens be written again: asynchronous copies read them until then.
    Caller-given device buffers must also stay alive until then. Returns
    (out, lse).
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda or not t.is_contiguous() or t.dim() != 4 or not t.is_pinned():
            raise FaError(FA_ERR_INVALID_ARG, f"{name} must be a contiguous 4-D pinned CPU tensor")
    if q.dtype not in _DTYPES or k.dtype != q.dtype or v.dtype != q.dtype:
        raise FaError(FA_ERR_UNSUPPORTED, "q, k, v must share one dtype: float16 or bfloat16")
    B, Hq, N, d = q.shape
    Hk = k.shape[1]
    if tuple(k.shape) != (B, Hk, N, d) or tuple(v.shape) != (B, Hk, N, d):
        raise FaError(FA_ERR_INVALID_ARG, "k and v must be [B, Hk, N, d] matching q")
    if key_pad_lens is not None and (key_pad_lens.is_cuda or key_pad_lens.dtype != torch.int32 or
                                     key_pad_lens.numel() != B or not key_pad_lens.is_pinned()):
        raise FaError(FA_ERR_INVALID_ARG, "key_pad_lens must be a pinned int32 CPU tensor [B]")
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32).pin_memory()
    if out.is_cuda or tuple(out.shape) != tuple(q.shape) or out.dtype != q.dtype or \
            not out.is_contiguous() or not out.is_pinned():
        raise FaError(FA_ERR_INVALID_ARG, "out must be a pinned CPU tensor shaped and typed like q")
    if lse.is_cuda or tuple(lse.shape) != (B, Hq, N) or lse.dtype != torch.float32 or \
            not lse.is_contiguous() or not lse.is_pinned():
        raise FaError(FA_ERR_INVALID_ARG, "lse must be a pinned float32 CPU tensor [B, Hq, N]")
    if device is None:
        device = device_buffers["q"].device if device_buffers is not None and "q" in device_buffers \
            else torch.device("cuda", torch.cuda.current_device())
    device = torch.device(device)
    if device.type != "cuda":
        raise FaError(FA_ERR_INVALID_ARG, "device must be a CUDA device")
    if device.index is None:
        device = torch.device("cuda", torch.cuda.current_device())
    owned = device_buffers is None
    if owned:
        with torch.cuda.device(device):
            device_buffers = {"q": torch.empty(q.shape, dtype=q.dtype, device=device),
                              "k": torch.empty(k.shape, dtype=q.dtype, device=device),
                              "v": torch.empty(v.shape, dtype=q.dtype, device=device),
                              "o": torch.empty(q.shape, dtype=q.dtype, device=device),
                              "lse": torch.empty((B, Hq, N), dtype=torch.float32, device=device),
                              "lens": (torch.empty(B, dtype=torch.int32, device=device)
                                       if key_pad_lens is not None else None)}
    want = {"q": (tuple(q.shape), q.dtype), "k": (tuple(k.shape), q.dtype), "v": (tuple(v.shape), q.dtype),
            "o": (tuple(q.shape), q.dtype), "lse": ((B, Hq, N), torch.float32)}
    if key_pad_lens is not None:
        want["lens"] = ((B,), torch.int32)
    for n, (shape, dt) in want.items():
        t = device_buffers.get(n)
        if t is None or not t.is_cuda or t.device != device or tuple(t.shape) != shape or \
                t.dtype != dt or not t.is_contiguous():
            raise FaError(FA_ERR_INVALID_ARG,
                          f"device_buffers['{n}'] must be a contiguous {dt} tensor {list(shape)} on {device}")
    qd, kd, vd, od, ld = (device_buffers[n] for n in ("q", "k", "v", "o", "lse"))
    lens_d = device_buffers["lens"] if key_pad_lens is not None else None
    handle, st = _stream_handle(stream, device)
    if owned:
        # the library's copy streams finish before `stream` does: tying the
        # buffers to `stream` keeps them alive until every copy has run
        for t in (qd, kd, vd, od, ld) + ((lens_d,) if lens_d is not None else ()):
            t.record_stream(st)
    if scale is None:
        scale = float(d) ** -0.5
    with torch.cuda.device(device):
        check(lib.fa_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                              lse.data_ptr(), B, Hq, Hk, N, d, float(scale), 1 if causal else 0,
                              key_pad_lens.data_ptr() if key_pad_lens is not None else None,
                              qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(),
                              ld.data_ptr(), lens_d.data_ptr() if lens_d is not None else None,
                              0 if chunks is None else int(chunks), handle, _DTYPES[q.dtype]))
    return out, lse


def host_chunk_plan(B, Hq, Hk, N, d, chunks=None):
    """[(b0, b1, hk0, hk1)] chunks fa_fwd_host uses (chunks None: its default)."""
    out = (ctypes.c_int32 * (4 * 64))()
    n = lib.fa_host_chunk_plan(B, Hq, Hk, N, d, 0 if chunks is None else int(chunks), out, 64)
    if n < 0:
        check(n)
    return [tuple(out[4 * i:4 * i + 4]) for i in range(n)]


def fa_fwd_bias(q, k, v, bias, causal=False, scale=None, key_pad_lens=None, out=None, lse=None,
                return_lse=True, stream=None):
    """``fa_fwd`` with an additive bias on the scaled scores.

    ``bias`` is a contiguous CUDA tensor [Bb, Hb, N, N] of q's dtype with Bb in
    {1, B} and Hb in {1, Hq}; it is added to scale·QKᵀ before the mask.
    """
    (B, Hq, Hk, N, d), out, lse, scale, stream = _prepare(q, k, v, key_pad_lens, out, lse,
                                                          return_lse, scale, stream)
    if not bias.is_cuda or not bias.is_contiguous() or bias.dim() != 4 or \
            bias.dtype != q.dtype or tuple(bias.shape[2:]) != (N, N):
        raise FaError(FA_ERR_INVALID_ARG,
                      "bias must be a contiguous [Bb, Hb, N, N] CUDA tensor of q's dtype")
    with torch.cuda.device(q.device):
        check(lib.fa_fwd_bias(q.data_ptr(), k.data_ptr(), v.data_ptr(), bias.data_ptr(),
                              bias.shape[0], bias.shape[1], out.data_ptr(),
                              lse.data_ptr() if lse is not None else None, B, Hq, Hk, N, d,
                              scale, 1 if causal else 0,
                              key_pad_lens.data_ptr() if key_pad_lens is not None else None,
                              stream, _DTYPES[q.dtype]))
    return (out, lse) if return_lse else out


def fa_bwd(q, k, v, o, lse, dout, causal=False, scale=None, key_pad_lens=None, dq=None, dk=None,
           dv=None, workspace=None, stream=None):
    """(dq, dk, dv) of the attention forward for upstream gradient ``dout``.

    ``o`` and ``lse`` are the forward's outputs for the same q, k, v, causal,
    scale and key_pad_lens. The fp32 workspace is allocated here when None.
    """
    (B, Hq, Hk, N, d), _, _, scale, stream = _prepare(q, k, v, key_pad_lens, o, lse, True,
                                                      scale, stream)
    for name, t in (("o", o), ("dout", dout)):
        if not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, Hq, N, d) or \
                t.dtype != q.dtype:
            raise FaError(FA_ERR_INVALID_ARG, f"{name} must be a contiguous CUDA tensor like q")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, N) or not lse.is_contiguous():
        raise FaError(FA_ERR_INVALID_ARG, "lse must be a contiguous float32 [B, Hq, N] tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = lib.fa_bwd_workspace_bytes(B, Hq, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        check(lib.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                         dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hk,
                         N, d, scale, 1 if causal else 0,
                         key_pad_lens.data_ptr() if key_pad_lens is not None else None,
                         workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                         stream, _DTYPES[q.dtype]))
    return dq, dk, dv


def fa_fwd_fp8(q, k, v, q_descale, k_descale, v_descale, causal=False, scale=None,
               key_pad_lens=None, out=None, lse=None, return_lse=True, workspace=None, stream=None):
    """Attention forward on E4M3 inputs (torch.float8_e4m3fn, values = stored × descale).

    O is bfloat16. ``scale`` defaults to 1/sqrt(d) and multiplies the decoded
    scores. The workspace (a transposed copy of V) is allocated when None.
    """
    fp8 = getattr(torch, "float8_e4m3fn", None)
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.dim() != 4 or t.dtype != fp8:
            raise FaError(FA_ERR_INVALID_ARG,
                          f"{name} must be a contiguous 4-D CUDA tensor of torch.float8_e4m3fn")
    B, Hq, N, d = q.shape
    Hk = k.shape[1]
    if tuple(k.shape) != (B, Hk, N, d) or tuple(v.shape) != (B, Hk, N, d):
        raise FaError(FA_ERR_INVALID_ARG, "k and v must be [B, Hk, N, d] matching q")
    if out is None:
        out = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    if key_pad_lens is not None and (key_pad_lens.dtype != torch.int32 or not key_pad_lens.is_cuda
                                     or key_pad_lens.numel() != B):
        raise FaError(FA_ERR_INVALID_ARG, "key_pad_lens must be an int32 CUDA tensor [B]")
    if scale is None:
        scale = float(d) ** -0.5
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    need = lib.fa_fwd_fp8_workspace_bytes(B, Hk, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        check(lib.fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), float(q_descale),
                             float(k_descale), float(v_descale), out.data_ptr(),
                             lse.data_ptr() if lse is not None else None, B, Hq, Hk, N, d,
                             float(scale), 1 if causal else 0,
                             key_pad_lens.data_ptr() if key_pad_lens is not None else None,
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             stream))
    return (out, lse) if return_lse else out


def splitkv_workspace_bytes(B, Hq, N, d, num_splits):
    """Bytes of scratch ``fa_fwd_splitkv`` needs (0 for one split)."""
    return lib.fa_splitkv_workspace_bytes(B, Hq, N, d, num_splits)


def fa_fwd_splitkv(q, k, v, num_splits, causal=False, scale=None, key_pad_lens=None, out=None,
                   lse=None, return_lse=True, workspace=None, stream=None):
    """As ``fa_fwd``, with each Q tile pair's K/V range cut into ``num_splits``
    chunks (1..16) whose partial results a second kernel merges by LSE.

    ``workspace`` is a CUDA tensor of at least ``splitkv_workspace_bytes``
    bytes (allocated here when None); a call in flight owns it until the
    stream reaches the end of the merge.
    """
    (B, Hq, Hk, N, d), out, lse, scale, stream = _prepare(q, k, v, key_pad_lens, out, lse,
                                                          return_lse, scale, stream)
    need = splitkv_workspace_bytes(B, Hq, N, d, num_splits)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace is not None and (not workspace.is_cuda or not workspace.is_contiguous()):
        raise FaError(FA_ERR_INVALID_ARG, "workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(q.device):
        check(lib.fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr() if lse is not None else None, B, Hq, Hk, N, d,
                                 scale, 1 if causal else 0,
                                 key_pad_lens.data_ptr() if key_pad_lens is not None else None,
                                 int(num_splits),
                                 workspace.data_ptr() if workspace is not None else None,
                                 ws_bytes, stream, _DTYPES[q.dtype]))
    return (out, lse) if return_lse else out


STATIC_SCRATCH_BYTES = 32 << 20  # FA_STATIC_SCRATCH_BYTES in include/fa.h


def fa_fwd_splitkv_static(q, k, v, num_splits, causal=False, scale=None, key_pad_lens=None,
                          out=None, lse=None, return_lse=True, stream=None):
    """``fa_fwd_splitkv`` on the library's static scratch: the C call allocates
    nothing (pass ``out`` and ``lse`` to allocate nothing here either).

    Calls on one device share the scratch: calls whose kernels may overlap
    (other streams) race on it. Problems whose split workspace exceeds
    ``STATIC_SCRATCH_BYTES`` raise ``FaError``.
    """
    (B, Hq, Hk, N, d), out, lse, scale, stream = _prepare(q, k, v, key_pad_lens, out, lse,
                                                          return_lse, scale, stream)
    with torch.cuda.device(q.device):
        check(lib.fa_fwd_splitkv_static(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                        lse.data_ptr() if lse is not None else None, B, Hq, Hk,
                                        N, d, scale, 1 if causal else 0,
                                        key_pad_lens.data_ptr() if key_pad_lens is not None
                                        else None, int(num_splits), stream, _DTYPES[q.dtype]))
    return (out, lse) if return_lse else out


def device_status():
    """Synchronise and read (then clear) the kernel's device status word."""
    return lib.fa_get_device_status()


def num_units(B, Hq, Hk, N, causal):
    return lib.fa_num_units(B, Hq, Hk, N, 1 if causal else 0)


def unit_info(B, Hq, Hk, N, causal, u):
    out = (ctypes.c_int32 * 8)()
    check(lib.fa_unit_info(B, Hq, Hk, N, 1 if causal else 0, u, out))
    return list(out)


def unit_for(cta, it, grid):
    return lib.fa_unit_for(cta, it, grid)


def unit_kv_range(B, Hq, Hk, N, causal, num_splits, u, key_len):
    """{b, hk, hq0, mb0, present0, hq1, mb1, present1, split, j0, n0, n1} of unit u."""
    out = (ctypes.c_int32 * 12)()
    check(lib.fa_unit_kv_range(B, Hq, Hk, N, 1 if causal else 0, num_splits, u, key_len, out))
    return list(out)


def unit_groups(B, Hq, Hk, N, d, causal, grid, l2_bytes):
    """Head groups of the causal unit order fa_fwd uses at d = 128 (0: one group)."""
    n = lib.fa_unit_groups(B, Hq, Hk, N, d, 1 if causal else 0, grid, l2_bytes)
    if n < 0:
        check(n)
    return n


def unit_kv_range_grouped(B, Hq, Hk, N, causal, num_splits, groups, u, key_len):
    """unit_kv_range with the unit order cut into `groups` head groups."""
    out = (ctypes.c_int32 * 12)()
    check(lib.fa_unit_kv_range_grouped(B, Hq, Hk, N, 1 if causal else 0, num_splits, groups, u,
                                       key_len, out))
    return list(out)


def unit_for_grouped(B, Hq, Hk, N, causal, num_splits, groups, cta, it, grid):
    """Unit of CTA `cta` on iteration `it` under the grouped order (num_units·splits: done)."""
    u = lib.fa_unit_for_grouped(B, Hq, Hk, N, 1 if causal else 0, num_splits, groups, cta, it, grid)
    if u < 0:
        check(u)
    return u

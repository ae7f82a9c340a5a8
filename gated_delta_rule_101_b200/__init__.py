"""B200-native Kimi Delta Attention (KDA): a thin binding over libkda.

libkda (``libkda.so`` next to this file, built by ``build.py`` from
``csrc/``) implements the entry points of ``include/kda.h``:

* ``chunk_fwd``   -> ``kda_chunk_fwd`` (``kda_chunk_fwd_io`` with fused steps):
  chunk-parallel prefill, C = 64 (tensor cores for bf16) or C = 32 (CUDA cores);
* ``decode_step`` -> ``kda_decode_step`` (``kda_decode_step_io``): one recurrent
  decode token;
* ``chunk_bwd``   -> ``kda_chunk_bwd``: the gradients of a prefill call.

Both take the forget gate as ``log_alpha`` in any of the library's gate
layouts (``kda_gate``), told apart by shape and dtype: ``[..., H, 128]``
fp32 (KDA, one rate per key channel; ``kda_chunk_fwd``), the same in bf16,
``[..., H]`` fp32 (one rate per head: Gated DeltaNet), or ``None`` (no gate:
DeltaNet); the last three go through ``kda_chunk_fwd_gated`` /
``kda_decode_step_gated``.

This module only marshals arguments: it checks dtypes, shapes and devices,
allocates outputs with PyTorch (device memory is PyTorch's job here), and
passes raw device pointers and the current CUDA stream to the C ABI. Every
step of the computation runs in libkda's CUDA kernels; there is no Python or
CPU fallback, and a missing library is an error.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# KDA_DEBUG=1 in the environment selects the KDA_DEBUG build (device-side checks of
# packed-sequence offsets; see include/kda.h).
DEBUG_BUILD = os.environ.get("KDA_DEBUG", "0") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libkda_debug.so" if DEBUG_BUILD else "libkda.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "kda.h")

KDA_BF16, KDA_F32 = 0, 1
KDA_GATE_CHANNEL, KDA_GATE_CHANNEL_BF16, KDA_GATE_HEAD, KDA_GATE_NONE = 0, 1, 2, 3
KDA_GATE_CHANNEL_LOGIT, KDA_GATE_CHANNEL_LOGIT_BF16 = 4, 5
GATE_NAMES = {KDA_GATE_CHANNEL: "channel", KDA_GATE_CHANNEL_BF16: "channel_bf16",
              KDA_GATE_HEAD: "head", KDA_GATE_NONE: "none",
              KDA_GATE_CHANNEL_LOGIT: "channel_logit", KDA_GATE_CHANNEL_LOGIT_BF16: "channel_logit_bf16"}
KDA_OK = 0
STATUS = {0: "KDA_OK", -1: "KDA_ERR_INVALID_ARG", -2: "KDA_ERR_UNSUPPORTED",
          -3: "KDA_ERR_WORKSPACE", -4: "KDA_ERR_CUDA", -5: "KDA_ERR_TIMEOUT",
          -6: "KDA_ERR_SCRATCH_LIMIT"}
HEAD_DIM = 128
CHUNK = 64

_lib = None


class KdaIo(ctypes.Structure):
    """``kda_io`` of include/kda.h: the fused input and output transformations."""
    _fields_ = [("qk_l2norm", ctypes.c_int), ("qk_l2norm_eps", ctypes.c_float),
                ("beta_logits", ctypes.c_int), ("out_gate", ctypes.c_void_p),
                ("out_norm_weight", ctypes.c_void_p), ("out_norm_eps", ctypes.c_float)]


class KDAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed: {STATUS.get(status, status)}")


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    vp, i32, i64, fp = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
    lib.kda_strerror.restype = ctypes.c_char_p
    lib.kda_strerror.argtypes = [i32]
    lib.kda_version.restype = i32
    lib.kda_version.argtypes = []
    lib.kda_chunk_fwd_workspace_size.restype = i32
    lib.kda_chunk_fwd_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32,
                                                 ctypes.POINTER(ctypes.c_size_t)]
    lib.kda_chunk_fwd_launches.restype = i32
    lib.kda_chunk_fwd_launches.argtypes = [i32, i64, i32, i32, i32, i32, ctypes.POINTER(ctypes.c_int)]
    lib.kda_chunk_fwd.restype = i32
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, i32, i64, i32, i32, vp, i32,
                                  vp, i32, vp, ctypes.c_size_t, vp]
    lib.kda_chunk_fwd_noalloc.restype = i32
    lib.kda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, i32, i64, i32, i32, vp,
                                          i32, vp, i32, vp]
    lib.kda_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.kda_noalloc_scratch_bytes.argtypes = []
    lib.kda_get_device_status.restype = i32
    lib.kda_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_int)]
    lib.kda_decode_step.restype = i32
    lib.kda_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, vp, i32, i32, i32, vp]
    lib.kda_chunk_fwd_gated.restype = i32
    lib.kda_chunk_fwd_gated.argtypes = [vp, vp, vp, vp, i32, fp, fp, vp, fp, i32, i64, i32, i32,
                                        vp, i32, vp, i32, vp, ctypes.c_size_t, vp]
    lib.kda_decode_step_gated.restype = i32
    lib.kda_decode_step_gated.argtypes = [vp, vp, vp, vp, i32, fp, fp, vp, i32, i32, i32, vp]
    io = ctypes.POINTER(KdaIo)
    lib.kda_chunk_fwd_io.restype = i32
    lib.kda_chunk_fwd_io.argtypes = [vp, vp, vp, vp, i32, fp, fp, vp, fp, i32, i64, i32, i32, vp, i32,
                                     vp, i32, vp, ctypes.c_size_t, io, vp]
    lib.kda_chunk_fwd_io_launches.restype = i32
    lib.kda_chunk_fwd_io_launches.argtypes = [i32, i64, i32, i32, i32, i32, io, ctypes.POINTER(ctypes.c_int)]
    lib.kda_decode_step_io.restype = i32
    lib.kda_decode_step_io.argtypes = [vp, vp, vp, vp, i32, fp, fp, vp, i32, i32, i32, io, vp]
    lib.kda_chunk_bwd_workspace_size.restype = i32
    lib.kda_chunk_bwd_workspace_size.argtypes = [i32, i64, i32, i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.kda_chunk_bwd.restype = i32
    lib.kda_chunk_bwd.argtypes = [vp, vp, vp, vp, i32, fp, fp, vp, fp, fp, fp, fp, fp, fp, fp, i32, i64, i32,
                                  vp, i32, vp, i32, io, vp, ctypes.c_size_t, vp]
    lib.kda_set_wait_limit_ns.restype = i32
    lib.kda_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.kda_selftest_wait_timeout.restype = i32
    lib.kda_selftest_wait_timeout.argtypes = [vp, vp, vp]
    return lib


def lib() -> ctypes.CDLL:
    """The loaded libkda handle. Raises if the library has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libkda is not built ({LIB_PATH} missing); "
                               "run `python -m gated_delta_rule_101_b200.build`")
        _lib = _bind(ctypes.CDLL(LIB_PATH))
    return _lib


def declared_symbols(header: str = HEADER) -> list[str]:
    """Names of the entry points declared with KDA_API in include/kda.h."""
    text = open(header, encoding="utf-8").read()
    return re.findall(r"KDA_API\s+[^;(]*?\b(kda_\w+)\s*\(", text)


def strerror(status: int) -> str:
    return lib().kda_strerror(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, device) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def gate_kind(log_alpha: torch.Tensor | None, q: torch.Tensor, logits: bool = False) -> int:
    """The kda_gate layout of ``log_alpha`` for inputs shaped like ``q``. With ``logits``
    the per-channel tensor holds the gate's pre-activation z (alpha = sigmoid(z))."""
    if log_alpha is None:
        if logits:
            raise ValueError("gate_logits needs a per-channel gate tensor")
        return KDA_GATE_NONE
    if log_alpha.shape == q.shape and log_alpha.dtype == torch.float32:
        return KDA_GATE_CHANNEL_LOGIT if logits else KDA_GATE_CHANNEL
    if log_alpha.shape == q.shape and log_alpha.dtype == torch.bfloat16:
        return KDA_GATE_CHANNEL_LOGIT_BF16 if logits else KDA_GATE_CHANNEL_BF16
    if logits:
        raise ValueError("gate_logits needs a per-channel gate tensor shaped like q")
    if log_alpha.shape == q.shape[:-1] and log_alpha.dtype == torch.float32:
        return KDA_GATE_HEAD
    raise ValueError(f"log_alpha must be None, fp32/bf16 {tuple(q.shape)} or fp32 "
                     f"{tuple(q.shape[:-1])}; got {log_alpha.dtype} {tuple(log_alpha.shape)}")


def _need_gate(log_alpha, gate: int, device) -> None:
    if gate != KDA_GATE_NONE:
        _need(log_alpha, "log_alpha", log_alpha.dtype, device)


def _stream_handle(stream: torch.cuda.Stream | None, device) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(B: int, T: int, H: int, n_seqs: int = 0, dtype=torch.bfloat16,
                   C: int = CHUNK) -> int:
    out = ctypes.c_size_t(0)
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    st = lib().kda_chunk_fwd_workspace_size(int(B), int(T), int(H), int(C), int(n_seqs), code,
                                            ctypes.byref(out))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_fwd_workspace_size")
    return int(out.value)


def chunk_fwd_launches(B: int, T: int, H: int, n_seqs: int = 0, dtype=torch.bfloat16,
                       C: int = CHUNK, out_epilogue: bool = False) -> int:
    """Number of libkda kernels one chunk_fwd call with these sizes launches
    (``out_epilogue``: a call with an output gate)."""
    out = ctypes.c_int(0)
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    if out_epilogue:  # the query only tests out_gate for NULL; it is never read
        io = KdaIo(0, 0.0, 0, 16, None, 0.0)
        st = lib().kda_chunk_fwd_io_launches(int(B), int(T), int(H), int(C), int(n_seqs), code,
                                             ctypes.byref(io), ctypes.byref(out))
        if st != KDA_OK:
            raise KDAError(st, "kda_chunk_fwd_io_launches")
        return int(out.value)
    st = lib().kda_chunk_fwd_launches(int(B), int(T), int(H), int(C), int(n_seqs), code,
                                      ctypes.byref(out))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_fwd_launches")
    return int(out.value)


def _prefill_args(q, k, v, log_alpha, beta, S0, cu_seqlens, out, state_out, gate_logits=False):
    """Checks the prefill tensors (dtypes, devices, contiguity, shapes) before any pointer
    reaches the library, which trusts the sizes it is given. Returns
    ``(B, T, H, n_seqs, gate, state_shape)``."""
    dev = q.device
    _dtype_code(q)
    packed = cu_seqlens is not None
    if q.dim() != (3 if packed else 4):
        raise ValueError(f"q must be {'[T, H, 128]' if packed else '[B, T, H, 128]'}, got {tuple(q.shape)}")
    if packed:
        T, H, dk = q.shape
        B = 1
        n_seqs = cu_seqlens.numel() - 1
        _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
        if cu_seqlens.dim() != 1 or n_seqs < 1:
            raise ValueError("cu_seqlens must be 1-D with n_seqs + 1 >= 2 offsets")
    else:
        B, T, H, dk = q.shape
        n_seqs = 0
    if dk != HEAD_DIM:
        raise ValueError(f"head dim must be {HEAD_DIM}, got {dk}")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, dev)
        if t.shape != q.shape:
            raise ValueError(f"{name} shape {tuple(t.shape)} != q shape {tuple(q.shape)}")
    gate = gate_kind(log_alpha, q, gate_logits)
    _need_gate(log_alpha, gate, dev)
    _need(beta, "beta", torch.float32, dev)
    if beta.shape != q.shape[:-1]:
        raise ValueError("beta must be q.shape[:-1]")
    sshape = (n_seqs if packed else B, H, HEAD_DIM, HEAD_DIM)
    for name, t in (("S0", S0), ("state_out", state_out)):
        if t is not None:
            _need(t, name, torch.float32, dev)
            if tuple(t.shape) != sshape:
                raise ValueError(f"{name} must be {sshape}, got {tuple(t.shape)}")
    if out is not None:
        _need(out, "out", q.dtype, dev)
        if out.shape != q.shape:
            raise ValueError(f"out shape {tuple(out.shape)} != q shape {tuple(q.shape)}")
    return B, T, H, n_seqs, gate, sshape


def _io(q, qk_l2norm, qk_eps, beta_logits, out_gate, out_norm_weight, out_eps):
    """The kda_io of the fused transformations, or None when none is asked for."""
    if not (qk_l2norm or beta_logits or out_gate is not None):
        return None
    if out_gate is not None:
        _need(out_gate, "out_gate", q.dtype, q.device)
        if out_gate.shape != q.shape:
            raise ValueError(f"out_gate shape {tuple(out_gate.shape)} != q shape {tuple(q.shape)}")
        if out_norm_weight is not None:
            _need(out_norm_weight, "out_norm_weight", torch.float32, q.device)
            if tuple(out_norm_weight.shape) != (HEAD_DIM,):
                raise ValueError("out_norm_weight must be [128]")
    elif out_norm_weight is not None:
        raise ValueError("out_norm_weight is used only with out_gate")
    return KdaIo(int(bool(qk_l2norm)), float(qk_eps), int(bool(beta_logits)),
                 None if out_gate is None else out_gate.data_ptr(),
                 None if out_norm_weight is None else out_norm_weight.data_ptr(), float(out_eps))


def chunk_fwd(q, k, v, log_alpha, beta, S0=None, *, cu_seqlens=None, cu_seqlens_host=None,
              out=None, final_state=True, state_out=None, workspace=None, stream=None, C=CHUNK,
              gate_logits=False, qk_l2norm=False, qk_eps=1e-6, beta_logits=False, out_gate=None,
              out_norm_weight=None, out_eps=1e-6):
    """KDA prefill through ``kda_chunk_fwd``; returns ``(o, S_T)`` (S_T None if not requested).

    ``q, k, v``: ``[B, T, H, 128]`` (or packed ``[T, H, 128]`` with
    ``cu_seqlens``, an int32 device tensor of ``n_seqs + 1`` offsets).
    ``log_alpha``: like ``q`` (fp32 or bf16), ``[B, T, H]`` fp32, or None (see
    ``gate_kind``). ``beta``: ``[B, T, H]``. ``S0``: fp32 ``[n_seqs, H, 128, 128]`` or None.
    ``state_out`` may be ``S0`` itself for in-place carry.

    Fused transformations (``kda_chunk_fwd_io``): ``gate_logits`` (``log_alpha`` holds
    the gate's pre-activation z, alpha = sigmoid(z)), ``qk_l2norm`` / ``qk_eps`` (q, k
    rows normalised in the kernel), ``beta_logits`` (beta = sigmoid(beta)), and
    ``out_gate`` / ``out_norm_weight`` / ``out_eps`` (o <- RMSNorm(o) * w *
    sigmoid(out_gate) per token-head row).
    """
    dev = q.device
    code = _dtype_code(q)
    B, T, H, n_seqs, gate, sshape = _prefill_args(q, k, v, log_alpha, beta, S0, cu_seqlens, out,
                                                  state_out, gate_logits)
    io = _io(q, qk_l2norm, qk_eps, beta_logits, out_gate, out_norm_weight, out_eps)
    if out is None:
        out = torch.empty_like(v)
    S_T = state_out
    if S_T is None and final_state:
        S_T = torch.empty(sshape, dtype=torch.float32, device=dev)
    host_cu = None
    if cu_seqlens_host is not None:
        host_cu = torch.as_tensor(cu_seqlens_host, dtype=torch.int32).contiguous().cpu()
    need = workspace_size(B, T, H, n_seqs, q.dtype, C)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    tail = (_ptr(beta), _ptr(S0), _ptr(out), _ptr(S_T), B, T, H, C, _ptr(cu_seqlens), n_seqs,
            _ptr(host_cu), code, _ptr(workspace), ws_bytes, _stream_handle(stream, dev))
    if io is not None:
        st = lib().kda_chunk_fwd_io(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), gate, *tail[:-1],
                                    ctypes.byref(io), tail[-1])
        where = "kda_chunk_fwd_io"
    elif gate == KDA_GATE_CHANNEL:
        st, where = lib().kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), *tail), "kda_chunk_fwd"
    else:
        st = lib().kda_chunk_fwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), gate, *tail)
        where = "kda_chunk_fwd_gated"
    if st != KDA_OK:
        raise KDAError(st, where)
    return out, S_T


def decode_step(q, k, v, log_alpha, beta, S, *, out=None, stream=None, gate_logits=False,
                qk_l2norm=False, qk_eps=1e-6, beta_logits=False, out_gate=None, out_norm_weight=None,
                out_eps=1e-6):
    """One decode token through ``kda_decode_step``; updates ``S`` in place, returns ``o``.

    ``q, k, v``: ``[N, H, 128]``; ``log_alpha``: like ``q`` (fp32 or bf16), ``[N, H]``
    fp32, or None (see ``gate_kind``); ``beta``: ``[N, H]``; ``S``: fp32 ``[N, H, 128, 128]``.
    """
    dev = q.device
    code = _dtype_code(q)
    if q.dim() != 3:
        raise ValueError(f"q must be [N, H, 128], got {tuple(q.shape)}")
    N, H, dk = q.shape
    if dk != HEAD_DIM:
        raise ValueError(f"head dim must be {HEAD_DIM}, got {dk}")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, dev)
        if t.shape != q.shape:
            raise ValueError(f"{name} shape {tuple(t.shape)} != q shape {tuple(q.shape)}")
    gate = gate_kind(log_alpha, q, gate_logits)
    _need_gate(log_alpha, gate, dev)
    _need(beta, "beta", torch.float32, dev)
    if beta.shape != q.shape[:-1]:
        raise ValueError("beta must be [N, H]")
    io = _io(q, qk_l2norm, qk_eps, beta_logits, out_gate, out_norm_weight, out_eps)
    _need(S, "S", torch.float32, dev)
    if tuple(S.shape) != (N, H, HEAD_DIM, HEAD_DIM):
        raise ValueError("S must be [N, H, 128, 128]")
    if out is None:
        out = torch.empty_like(v)
    _need(out, "out", q.dtype, dev)
    if out.shape != q.shape:
        raise ValueError(f"out shape {tuple(out.shape)} != q shape {tuple(q.shape)}")
    tail = (_ptr(beta), _ptr(S), _ptr(out), N, H, code, _stream_handle(stream, dev))
    if io is not None:
        st = lib().kda_decode_step_io(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), gate, *tail[:-1],
                                      ctypes.byref(io), tail[-1])
        where = "kda_decode_step_io"
    elif gate == KDA_GATE_CHANNEL:
        st, where = lib().kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), *tail), "kda_decode_step"
    else:
        st = lib().kda_decode_step_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), gate, *tail)
        where = "kda_decode_step_gated"
    if st != KDA_OK:
        raise KDAError(st, where)
    return out


def chunk_fwd_noalloc(q, k, v, log_alpha, beta, S0=None, *, out, state_out=None,
                      cu_seqlens=None, cu_seqlens_host=None, stream=None, C=CHUNK):
    """KDA prefill through ``kda_chunk_fwd_noalloc``: no workspace, no allocation.

    For callers that cannot allocate device memory (a plugin whose host framework
    owns all GPU memory, or a loop that must not call cudaMalloc). The caller
    passes the output tensors; the library uses its fixed scratch buffer (see
    include/kda.h for its size limit and the rule that calls sharing it must not
    overlap on the GPU). Returns ``(out, state_out)``.
    """
    dev = q.device
    code = _dtype_code(q)
    if out is None:
        raise ValueError("chunk_fwd_noalloc writes into the caller's `out`")
    B, T, H, n_seqs, gate, _ = _prefill_args(q, k, v, log_alpha, beta, S0, cu_seqlens, out, state_out)
    if gate != KDA_GATE_CHANNEL:
        raise ValueError("kda_chunk_fwd_noalloc takes the per-channel fp32 gate only")
    host_cu = None
    if cu_seqlens_host is not None:
        host_cu = torch.as_tensor(cu_seqlens_host, dtype=torch.int32).contiguous().cpu()
    st = lib().kda_chunk_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(out),
        _ptr(state_out), B, T, H, C, _ptr(cu_seqlens), n_seqs, _ptr(host_cu), code,
        _stream_handle(stream, dev))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_fwd_noalloc")
    return out, state_out


STATUS_TIMEOUT, STATUS_BAD_INPUT = 1, 2


def device_status() -> int:
    """Reads and clears libkda's device status: 0, or a mask of STATUS_TIMEOUT (a
    bounded wait gave up) and STATUS_BAD_INPUT (a KDA_DEBUG build refused device
    offsets)."""
    st = ctypes.c_int(0)
    rc = lib().kda_get_device_status(ctypes.byref(st))
    if rc != KDA_OK:
        raise KDAError(rc, "kda_get_device_status")
    return st.value


def set_wait_limit_ns(ns: int) -> None:
    """Sets the bounded waits' time limit (0 restores the default of one second)."""
    rc = lib().kda_set_wait_limit_ns(int(ns))
    if rc != KDA_OK:
        raise KDAError(rc, "kda_set_wait_limit_ns")


def selftest_wait_timeout(flag: torch.Tensor, result: torch.Tensor, stream=None) -> None:
    """Launches ``kda_selftest_wait_timeout`` on device int32 tensors ``flag`` (kept at
    0 by the caller) and ``result`` (receives the bitmask of waits that gave up)."""
    for t, name in ((flag, "flag"), (result, "result")):
        _need(t, name, torch.int32, flag.device)
    rc = lib().kda_selftest_wait_timeout(_ptr(flag), _ptr(result), _stream_handle(stream, flag.device))
    if rc != KDA_OK:
        raise KDAError(rc, "kda_selftest_wait_timeout")


def bwd_workspace_size(B: int, T: int, H: int, n_seqs: int = 0) -> int:
    """Bytes of workspace ``kda_chunk_bwd`` needs for these sizes."""
    out = ctypes.c_size_t(0)
    st = lib().kda_chunk_bwd_workspace_size(int(B), int(T), int(H), int(n_seqs), ctypes.byref(out))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_bwd_workspace_size")
    return int(out.value)


def chunk_bwd(q, k, v, log_alpha, beta, S0, dout, dS_T=None, *, cu_seqlens=None, cu_seqlens_host=None,
              workspace=None, stream=None, gate_logits=False, qk_l2norm=False, qk_eps=1e-6,
              beta_logits=False):
    """Gradients of sum(o * dout) + sum(S_T * dS_T) through ``kda_chunk_bwd``.

    Arguments as for ``chunk_fwd`` (no output epilogue), plus ``dout`` shaped like q and
    ``dS_T`` (fp32 state shape, or None). Returns a dict of fp32 tensors: dq, dk, dv,
    dgate (the gate's gradient in its layout's shape; None without a gate), dbeta, dS0.
    """
    dev = q.device
    code = _dtype_code(q)
    B, T, H, n_seqs, gate, sshape = _prefill_args(q, k, v, log_alpha, beta, S0, cu_seqlens, None, None,
                                                  gate_logits)
    _need(dout, "dout", q.dtype, dev)
    if dout.shape != q.shape:
        raise ValueError("dout must be shaped like q")
    if dS_T is not None:
        _need(dS_T, "dS_T", torch.float32, dev)
        if tuple(dS_T.shape) != sshape:
            raise ValueError(f"dS_T must be {sshape}")
    io = _io(q, qk_l2norm, qk_eps, beta_logits, None, None, 0.0)
    f32 = lambda shape: torch.empty(shape, dtype=torch.float32, device=dev)
    res = {"dq": f32(q.shape), "dk": f32(q.shape), "dv": f32(q.shape), "dbeta": f32(beta.shape),
           "dS0": f32(sshape),
           "dgate": None if gate == KDA_GATE_NONE else f32(log_alpha.shape)}
    host_cu = None
    if cu_seqlens_host is not None:
        host_cu = torch.as_tensor(cu_seqlens_host, dtype=torch.int32).contiguous().cpu()
    need = bwd_workspace_size(B, T, H, n_seqs)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = lib().kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), gate, _ptr(beta), _ptr(S0),
                             _ptr(dout), _ptr(dS_T), _ptr(res["dq"]), _ptr(res["dk"]), _ptr(res["dv"]),
                             _ptr(res["dgate"]), _ptr(res["dbeta"]), _ptr(res["dS0"]), B, T, H,
                             _ptr(cu_seqlens), n_seqs, _ptr(host_cu), code,
                             None if io is None else ctypes.byref(io), _ptr(workspace), ws_bytes,
                             _stream_handle(stream, dev))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_bwd")
    return res

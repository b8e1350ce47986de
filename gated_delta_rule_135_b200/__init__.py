"""Python binding of the B200 KDA chunked-prefill library (include/kda.h).

Argument marshalling only: every step of the forward runs in the CUDA kernels
of libkda.so.  Tensors are torch CUDA tensors (torch supplies device memory
and the stream); the library never sees a torch type.  If the shared library
is missing the import fails loudly -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# KDA_LIBRARY may name another build of the same library (e.g. the
# phase-clock instrumented libkda_phase.so); the default is libkda.so.
LIB_PATH = os.environ.get("KDA_LIBRARY", os.path.join(_HERE, "libkda.so"))

HEAD_DIM = 128
CHUNK = 64
FUSED_MIN_LOWER_BOUND = -9.5

KDA_OK = 0
STATUS_NAMES = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
                3: "KDA_ERR_ALIGNMENT", 4: "KDA_ERR_CUDA", 5: "KDA_ERR_DEVICE",
                6: "KDA_ERR_WORKSPACE", 7: "KDA_ERR_SCRATCH_LIMIT"}


class KdaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {kda_strerror(status)}")


class kda_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("seqlen", ctypes.c_int64),
                ("num_heads", ctypes.c_int32), ("num_seqs", ctypes.c_int32),
                ("head_dim_k", ctypes.c_int32), ("head_dim_v", ctypes.c_int32)]


class kda_staged_layout(ctypes.Structure):
    _fields_ = [("chunk_table", ctypes.c_size_t), ("gamma", ctypes.c_size_t),
                ("w", ctypes.c_size_t), ("u_tilde", ctypes.c_size_t), ("p", ctypes.c_size_t),
                ("u", ctypes.c_size_t), ("chunk_states", ctypes.c_size_t),
                ("total", ctypes.c_size_t), ("max_chunks", ctypes.c_int64)]


class kda_grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("dq", "dk", "dv", "dg", "dbeta", "dA_log", "ddt_bias",
                                               "d_initial_state")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkda.so not built ({LIB_PATH}); run gated_delta_rule_135_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    vp, f32 = ctypes.c_void_p, ctypes.c_float
    fwd_args = [vp, vp, vp, vp, vp, vp, vp, f32, f32, vp, vp, vp, vp, kda_dims]
    lib.kda_fwd.restype = ctypes.c_int
    lib.kda_fwd.argtypes = fwd_args + [vp]
    lib.kda_fwd_staged.restype = ctypes.c_int
    lib.kda_fwd_staged.argtypes = fwd_args + [vp, ctypes.c_size_t, vp]
    lib.kda_staged_workspace_size.restype = ctypes.c_size_t
    lib.kda_staged_workspace_size.argtypes = [kda_dims, ctypes.c_int]
    lib.kda_fwd_workspace_size.restype = ctypes.c_size_t
    lib.kda_fwd_workspace_size.argtypes = [kda_dims]
    lib.kda_staged_workspace_layout.restype = ctypes.c_int
    lib.kda_staged_workspace_layout.argtypes = [kda_dims, ctypes.c_int, ctypes.POINTER(kda_staged_layout)]
    lib.kda_strerror.restype = ctypes.c_char_p
    lib.kda_strerror.argtypes = [ctypes.c_int]
    lib.kda_check_device_error.restype = ctypes.c_int
    lib.kda_check_device_error.argtypes = [vp]
    lib.kda_last_device_error_bits.restype = ctypes.c_uint32
    lib.kda_last_device_error_bits.argtypes = []
    lib.kda_version.restype = ctypes.c_char_p
    lib.kda_version.argtypes = []
    lib.kda_fwd_staged_noalloc.restype = ctypes.c_int
    lib.kda_fwd_staged_noalloc.argtypes = fwd_args + [vp]
    lib.kda_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.kda_noalloc_scratch_bytes.argtypes = []
    lib.kda_state_affine.restype = ctypes.c_int
    lib.kda_state_affine.argtypes = [vp, vp, vp, vp, ctypes.c_int32, vp]
    lib.kda_gdn_decode.restype = ctypes.c_int
    lib.kda_gdn_decode.argtypes = [vp] * 7 + [f32, f32, vp, vp, ctypes.c_int32, ctypes.c_int32, vp]
    lib.kda_gdn_fwd.restype = ctypes.c_int
    lib.kda_gdn_fwd.argtypes = fwd_args + [vp]
    lib.kda_bwd_workspace_size.restype = ctypes.c_size_t
    lib.kda_bwd_workspace_size.argtypes = [kda_dims, ctypes.c_int]
    lib.kda_bwd.restype = ctypes.c_int
    lib.kda_bwd.argtypes = [vp] * 7 + [f32, f32, vp, vp, vp, vp, ctypes.POINTER(kda_grads), kda_dims, vp,
                                       ctypes.c_size_t, vp]
    lib.kda_decode.restype = ctypes.c_int
    lib.kda_decode.argtypes = [vp] * 7 + [f32, f32, vp, vp, ctypes.c_int32, ctypes.c_int32, vp]
    lib.kda_selftest_wait_timeout.restype = ctypes.c_int
    lib.kda_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp, vp]
    lib.kda_fwd_segments.restype = ctypes.c_int32
    lib.kda_fwd_segments.argtypes = [kda_dims, ctypes.c_int32]
    return lib


_lib = _load()

# Symbols include/kda.h declares (checked by the ABI test).
EXPORTED = ("kda_fwd", "kda_fwd_staged", "kda_staged_workspace_size",
            "kda_staged_workspace_layout", "kda_strerror", "kda_check_device_error",
            "kda_last_device_error_bits", "kda_version", "kda_fwd_staged_noalloc",
            "kda_noalloc_scratch_bytes", "kda_decode", "kda_gdn_fwd", "kda_gdn_decode",
            "kda_state_affine", "kda_bwd", "kda_bwd_workspace_size", "kda_fwd_workspace_size",
            "kda_selftest_wait_timeout", "kda_fwd_segments")


def lib() -> ctypes.CDLL:
    return _lib


def kda_strerror(status: int) -> str:
    return _lib.kda_strerror(int(status)).decode()


def kda_version() -> str:
    return _lib.kda_version().decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_dims(num_heads: int, *, total_tokens: int, cu_seqlens: Optional[torch.Tensor] = None,
              batch: int = 1, seqlen: Optional[int] = None) -> kda_dims:
    if cu_seqlens is not None:
        return kda_dims(1, int(total_tokens), int(num_heads), int(cu_seqlens.numel() - 1),
                        HEAD_DIM, HEAD_DIM)
    seqlen = total_tokens // max(batch, 1) if seqlen is None else seqlen
    return kda_dims(int(batch), int(seqlen), int(num_heads), int(batch), HEAD_DIM, HEAD_DIM)


def _check_tensor(name, t, dtype, device):
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _marshal(q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens, out, final_state,
             batch):
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda: tensors must live on a CUDA device")
    _check_tensor("q", q, torch.bfloat16, dev)
    _check_tensor("k", k, torch.bfloat16, dev)
    _check_tensor("v", v, torch.bfloat16, dev)
    _check_tensor("g", g, torch.float32, dev)
    _check_tensor("beta", beta, torch.float32, dev)
    _check_tensor("A_log", A_log, torch.float32, dev)
    _check_tensor("dt_bias", dt_bias, torch.float32, dev)
    _check_tensor("initial_state", initial_state, torch.float32, dev)
    _check_tensor("cu_seqlens", cu_seqlens, torch.int32, dev)
    _check_tensor("out", out, torch.bfloat16, dev)
    _check_tensor("final_state", final_state, torch.float32, dev)
    H = q.shape[-2]
    total = q.numel() // (H * HEAD_DIM)
    if cu_seqlens is None and q.dim() == 4:
        batch = q.shape[0]
    dims = make_dims(H, total_tokens=total, cu_seqlens=cu_seqlens, batch=batch)
    return dims


def kda_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
            beta: torch.Tensor, A_log: torch.Tensor, dt_bias: torch.Tensor,
            lower_bound: float, scale: float, initial_state: Optional[torch.Tensor] = None,
            cu_seqlens: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
            final_state: Optional[torch.Tensor] = None, *, batch: int = 1, stream=None):
    """Calls kda_fwd.  q/k/v: [.., H, 128] bf16 (packed [Ttot, H, 128] or [B, T, H, 128]);
    g: fp32 like q; beta: fp32 [.., H]; returns (out, final_state)."""
    dims = _marshal(q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens, out,
                    final_state, batch)
    if out is None:
        out = torch.empty(q.shape[:-1] + (HEAD_DIM,), dtype=torch.bfloat16, device=q.device)
    st = _lib.kda_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log), _ptr(dt_bias),
                      float(lower_bound), float(scale), _ptr(initial_state), _ptr(cu_seqlens),
                      _ptr(out), _ptr(final_state), dims, _stream_ptr(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_fwd")
    return out, final_state


@dataclass
class StagedWorkspace:
    buffer: torch.Tensor
    layout: kda_staged_layout

    def view(self, name: str, dtype, shape):
        off = getattr(self.layout, name)
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return self.buffer[off:off + nbytes].view(dtype).view(*shape)


def staged_workspace(q: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None,
                     batch: int = 1) -> StagedWorkspace:
    H = q.shape[-2]
    total = q.numel() // (H * HEAD_DIM)
    if cu_seqlens is None and q.dim() == 4:
        batch = q.shape[0]
    dims = make_dims(H, total_tokens=total, cu_seqlens=cu_seqlens, batch=batch)
    L = kda_staged_layout()
    st = _lib.kda_staged_workspace_layout(dims, int(cu_seqlens is not None), ctypes.byref(L))
    if st != KDA_OK:
        raise KdaError(st, "kda_staged_workspace_layout")
    buf = torch.empty(max(L.total, 256), dtype=torch.uint8, device=q.device)
    return StagedWorkspace(buf, L)


def kda_fwd_staged(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float,
                   initial_state=None, cu_seqlens=None, out=None, final_state=None, *,
                   workspace: Optional[StagedWorkspace] = None, batch: int = 1, stream=None):
    """Calls kda_fwd_staged (four kernels; intermediates left in the workspace)."""
    dims = _marshal(q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens, out,
                    final_state, batch)
    if out is None:
        out = torch.empty(q.shape[:-1] + (HEAD_DIM,), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        workspace = staged_workspace(q, cu_seqlens, batch)
    st = _lib.kda_fwd_staged(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log),
                             _ptr(dt_bias), float(lower_bound), float(scale), _ptr(initial_state),
                             _ptr(cu_seqlens), _ptr(out), _ptr(final_state), dims,
                             _ptr(workspace.buffer), ctypes.c_size_t(workspace.buffer.numel()),
                             _stream_ptr(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_fwd_staged")
    return out, final_state, workspace


def kda_fwd_staged_noalloc(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float,
                           initial_state=None, cu_seqlens=None, out=None, final_state=None, *,
                           batch: int = 1, stream=None):
    """Calls kda_fwd_staged_noalloc: the staged forward on the library's fixed
    16 MiB device scratch (no device allocation; small problems only)."""
    dims = _marshal(q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens, out,
                    final_state, batch)
    if out is None:
        out = torch.empty(q.shape[:-1] + (HEAD_DIM,), dtype=torch.bfloat16, device=q.device)
    st = _lib.kda_fwd_staged_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log),
                                     _ptr(dt_bias), float(lower_bound), float(scale),
                                     _ptr(initial_state), _ptr(cu_seqlens), _ptr(out),
                                     _ptr(final_state), dims, _stream_ptr(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_fwd_staged_noalloc")
    return out, final_state


def kda_noalloc_scratch_bytes() -> int:
    return int(_lib.kda_noalloc_scratch_bytes())


def kda_gdn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor,
                beta: torch.Tensor, A_log: torch.Tensor, dt_bias: torch.Tensor,
                lower_bound: float, scale: float, initial_state: Optional[torch.Tensor] = None,
                cu_seqlens: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                final_state: Optional[torch.Tensor] = None, *, batch: int = 1, stream=None):
    """Calls kda_gdn_fwd (scalar gate).  q/k/v as for kda_fwd; g and beta: fp32 [.., H];
    A_log and dt_bias: fp32 [H].  Returns (out, final_state)."""
    dims = _marshal(q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens, out,
                    final_state, batch)
    if out is None:
        out = torch.empty(q.shape[:-1] + (HEAD_DIM,), dtype=torch.bfloat16, device=q.device)
    st = _lib.kda_gdn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log), _ptr(dt_bias),
                          float(lower_bound), float(scale), _ptr(initial_state), _ptr(cu_seqlens),
                          _ptr(out), _ptr(final_state), dims, _stream_ptr(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_gdn_fwd")
    return out, final_state


def kda_decode(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float, state,
               out=None, *, stream=None):
    """Calls kda_decode: one recurrent step per sequence.  q/k/v: bf16 [B, H, 128];
    g: fp32 [B, H, 128]; beta: fp32 [B, H]; state: fp32 [B, H, 128, 128], updated in
    place.  Returns out (bf16 [B, H, 128])."""
    dev = q.device
    for name, t, dt in (("q", q, torch.bfloat16), ("k", k, torch.bfloat16), ("v", v, torch.bfloat16),
                        ("g", g, torch.float32), ("beta", beta, torch.float32),
                        ("A_log", A_log, torch.float32), ("dt_bias", dt_bias, torch.float32),
                        ("state", state, torch.float32)):
        _check_tensor(name, t, dt, dev)
    B, H = q.shape[0], q.shape[1]
    if out is None:
        out = torch.empty(B, H, HEAD_DIM, dtype=torch.bfloat16, device=dev)
    st = _lib.kda_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log), _ptr(dt_bias),
                         float(lower_bound), float(scale), _ptr(state), _ptr(out), int(B), int(H),
                         _stream_ptr(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode")
    return out


def kda_gdn_decode(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float, state,
               out=None, *, stream=None):
    """Calls kda_gdn_decode, the scalar-gate decode step.  q/k/v: bf16 [B, H, 128];
    g: fp32 [B, H]; beta: fp32 [B, H]; dt_bias: fp32 [H]; state: fp32 [B, H, 128, 128],
    updated in place.  Returns out (bf16 [B, H, 128])."""
    dev = q.device
    for name, t, dt in (("q", q, torch.bfloat16), ("k", k, torch.bfloat16), ("v", v, torch.bfloat16),
                        ("g", g, torch.float32), ("beta", beta, torch.float32),
                        ("A_log", A_log, torch.float32), ("dt_bias", dt_bias, torch.float32),
                        ("state", state, torch.float32)):
        _check_tensor(name, t, dt, dev)
    B, H = q.shape[0], q.shape[1]
    if out is None:
        out = torch.empty(B, H, HEAD_DIM, dtype=torch.bfloat16, device=dev)
    st = _lib.kda_gdn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log), _ptr(dt_bias),
                         float(lower_bound), float(scale), _ptr(state), _ptr(out), int(B), int(H),
                         _stream_ptr(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_gdn_decode")
    return out


def kda_state_affine(A: torch.Tensor, S: torch.Tensor, B: torch.Tensor, out: Optional[torch.Tensor] = None,
                     *, stream=None) -> torch.Tensor:
    """Calls kda_state_affine: out[h] = A[h] @ S[h] + B[h]; all fp32 [H, 128, 128]."""
    dev = A.device
    for name, t in (("A", A), ("S", S), ("B", B)):
        _check_tensor(name, t, torch.float32, dev)
    if out is None:
        out = torch.empty_like(B)
    H = A.numel() // (HEAD_DIM * HEAD_DIM)
    st = _lib.kda_state_affine(_ptr(A), _ptr(S), _ptr(B), _ptr(out), int(H), _stream_ptr(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_state_affine")
    return out


GRAD_NAMES = ("dq", "dk", "dv", "dg", "dbeta", "dA_log", "ddt_bias", "d_initial_state")


def kda_bwd(q, k, v, g, beta, A_log, dt_bias, lower_bound: float, scale: float, d_out,
            initial_state=None, cu_seqlens=None, d_final_state=None, *, want_d_initial: bool = True,
            grads: Optional[dict] = None, workspace: Optional[torch.Tensor] = None, batch: int = 1,
            stream=None) -> dict:
    """Calls kda_bwd: the gradients of <d_out, out> + <d_final_state, final_state> for the
    forward kda_fwd computes from the same arguments.  d_out: bf16 like q;
    d_final_state: fp32 [N, H, 128, 128] or None.  Returns a dict of fp32 tensors
    (GRAD_NAMES; d_initial_state only with want_d_initial).  `grads` may supply some or all
    output tensors; `workspace` a uint8 device buffer of kda_bwd_workspace_size bytes."""
    dims = _marshal(q, k, v, g, beta, A_log, dt_bias, initial_state, cu_seqlens, d_out, None, batch)
    _check_tensor("d_final_state", d_final_state, torch.float32, q.device)
    H = q.shape[-2]
    shapes = {"dq": q.shape, "dk": q.shape, "dv": v.shape, "dg": g.shape, "dbeta": beta.shape,
              "dA_log": A_log.shape, "ddt_bias": dt_bias.shape}
    if want_d_initial:
        N = dims.num_seqs if cu_seqlens is not None else dims.batch
        shapes["d_initial_state"] = (N, H, HEAD_DIM, HEAD_DIM)
    out = dict(grads or {})
    for name, shape in shapes.items():
        if out.get(name) is None:
            out[name] = torch.empty(shape, dtype=torch.float32, device=q.device)
        _check_tensor(name, out[name], torch.float32, q.device)
    gr = kda_grads(*[None if out.get(n) is None else out[n].data_ptr() for n in GRAD_NAMES])
    if workspace is None:
        nbytes = _lib.kda_bwd_workspace_size(dims, int(cu_seqlens is not None))
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    st = _lib.kda_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log), _ptr(dt_bias),
                      float(lower_bound), float(scale), _ptr(initial_state), _ptr(cu_seqlens), _ptr(d_out),
                      _ptr(d_final_state), ctypes.byref(gr), dims, _ptr(workspace),
                      ctypes.c_size_t(workspace.numel()), _stream_ptr(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_bwd")
    return out


def kda_bwd_workspace_size(q: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None, batch: int = 1) -> int:
    H = q.shape[-2]
    total = q.numel() // (H * HEAD_DIM)
    if cu_seqlens is None and q.dim() == 4:
        batch = q.shape[0]
    dims = make_dims(H, total_tokens=total, cu_seqlens=cu_seqlens, batch=batch)
    return int(_lib.kda_bwd_workspace_size(dims, int(cu_seqlens is not None)))


def kda_fwd_segments(num_heads: int, seqlen: int, batch: int = 1, varlen: bool = False) -> int:
    """How many segments kda_fwd / kda_gdn_fwd split a call with these dims into on the current
    device (1: none; only one sequence in the fixed layout is split)."""
    dims = make_dims(num_heads, total_tokens=seqlen * batch, batch=batch, seqlen=seqlen) if not varlen else \
        make_dims(num_heads, total_tokens=seqlen, cu_seqlens=torch.zeros(2, dtype=torch.int32))
    return int(_lib.kda_fwd_segments(dims, 1 if varlen else 0))


def kda_selftest_wait_timeout(limit_ns: int, observed: Optional[torch.Tensor] = None, stream=None) -> None:
    """Makes one bounded device-side wait run out on purpose (diagnostics; see include/kda.h).
    observed: optional int32 CUDA tensor of 2 elements."""
    if observed is not None:
        _check_tensor("observed", observed, torch.int32, observed.device)
        if observed.numel() < 2:
            raise ValueError("observed needs 2 elements")
    st = _lib.kda_selftest_wait_timeout(int(limit_ns), _ptr(observed), _stream_ptr(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_selftest_wait_timeout")


def kda_check_device_error(stream=None) -> int:
    """Synchronises the stream; returns the device error bits (0 = none)."""
    st = _lib.kda_check_device_error(_stream_ptr(stream))
    if st == KDA_OK:
        return 0
    if st == 5:
        return int(_lib.kda_last_device_error_bits())
    raise KdaError(st, "kda_check_device_error")

"""ctypes binding of the KDA C ABI (include/kda.h, libkda.so).

Argument marshalling only: every step of the operator runs in the library's
CUDA kernels.  torch is used for device memory (outputs, workspace) and for
the current CUDA stream.  There is no CPU path: if ``libkda.so`` is missing
the first call raises, and CPU tensors are rejected.

Low-level functions keep the C names (every symbol in ``EXPORTS``) and take
raw pointers and ints.  Tensor-level helpers allocate outputs and workspaces
with torch, check every tensor's shape and dtype against its role, and pass
the current stream: ``forward``, ``forward_g``, ``forward_scalar_gate``,
``forward_checkpoints``, ``forward_norm_gate``, ``forward_conv``,
``short_conv_swish``, ``decode_step``, ``decode_step_norm_gate``,
``cp_local`` / ``cp_finish`` / ``state_compose`` (context parallelism; the
collective lives in ``cp.py``), ``workspace`` and ``check_device_error``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = 0, -1, -2, -3, -4
KDA_F32, KDA_BF16 = 0, 1

# Every symbol include/kda.h declares.
EXPORTS = ("kda_status_string", "kda_version", "kda_forward_workspace_size",
           "kda_forward_launches", "kda_forward",
           "kda_forward_g", "kda_decode_step", "kda_forward_noalloc", "kda_forward_checkpoints",
           "kda_forward_norm_gate", "kda_decode_step_norm_gate", "kda_forward_scalar_gate",
           "kda_short_conv_swish", "kda_forward_conv_workspace_size", "kda_forward_conv",
           "kda_cp_workspace_size", "kda_cp_local", "kda_cp_finish", "kda_state_compose",
           "kda_check_device_error", "kda_debug_set_wait_limit", "kda_decode_step_conv")

# Bytes of the library's fixed scratch array used by kda_forward_noalloc.
KDA_NOALLOC_SCRATCH_BYTES = 64 << 20

_lib = None


class KdaError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def lib():
    """Load libkda.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m gated_delta_rule_98_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    L.kda_status_string.argtypes = [ctypes.c_int]
    L.kda_status_string.restype = ctypes.c_char_p
    L.kda_version.argtypes = []
    L.kda_version.restype = i32
    L.kda_forward_workspace_size.argtypes = [i32] * 6 + [ctypes.c_int, i32]
    L.kda_forward_workspace_size.restype = sz
    L.kda_forward_launches.argtypes = [i32] * 6 + [ctypes.c_int, i32]
    L.kda_forward_launches.restype = i32
    L.kda_forward.argtypes = [vp] * 8 + [i32] * 6 + [ctypes.c_int, i32, vp, vp, vp, sz, vp]
    L.kda_forward.restype = ctypes.c_int
    L.kda_forward_g.argtypes = [vp] * 7 + [i32] * 6 + [ctypes.c_int, i32, vp, vp, vp, sz, vp]
    L.kda_forward_g.restype = ctypes.c_int
    L.kda_decode_step.argtypes = [vp] * 7 + [i32] * 4 + [ctypes.c_int, vp, vp]
    L.kda_decode_step.restype = ctypes.c_int
    L.kda_forward_noalloc.argtypes = [vp] * 8 + [i32] * 6 + [ctypes.c_int, i32, vp, vp, vp]
    L.kda_forward_noalloc.restype = ctypes.c_int
    L.kda_forward_checkpoints.argtypes = ([vp] * 8 + [i32] * 6 + [ctypes.c_int, i32, vp, vp, vp,
                                          i32, vp, sz, vp])
    L.kda_forward_checkpoints.restype = ctypes.c_int
    L.kda_forward_norm_gate.argtypes = ([vp] * 8 + [i32] * 6 + [ctypes.c_int, i32, vp, vp,
                                        ctypes.c_float, vp, vp, vp, sz, vp])
    L.kda_forward_norm_gate.restype = ctypes.c_int
    L.kda_decode_step_norm_gate.argtypes = ([vp] * 7 + [i32] * 4 + [ctypes.c_int, vp, vp,
                                            ctypes.c_float, vp, vp])
    L.kda_decode_step_norm_gate.restype = ctypes.c_int
    L.kda_forward_scalar_gate.argtypes = [vp] * 7 + [i32] * 6 + [ctypes.c_int, i32, vp, vp, vp,
                                                                sz, vp]
    L.kda_forward_scalar_gate.restype = ctypes.c_int
    L.kda_decode_step_conv.argtypes = ([vp] * 6 + [i32, vp] + [vp] * 4 + [i32] * 4 +
                                       [ctypes.c_int, vp, vp])
    L.kda_decode_step_conv.restype = ctypes.c_int
    L.kda_short_conv_swish.argtypes = [vp, vp, vp] + [i32] * 5 + [ctypes.c_int, vp, vp]
    L.kda_short_conv_swish.restype = ctypes.c_int
    L.kda_forward_conv_workspace_size.argtypes = [i32] * 6 + [ctypes.c_int, i32]
    L.kda_forward_conv_workspace_size.restype = sz
    L.kda_forward_conv.argtypes = ([vp] * 6 + [i32] + [vp] * 5 + [i32] * 6 +
                                   [ctypes.c_int, i32, vp, vp, vp, sz, vp])
    L.kda_forward_conv.restype = ctypes.c_int
    L.kda_cp_workspace_size.argtypes = [i32] * 6 + [ctypes.c_int, i32]
    L.kda_cp_workspace_size.restype = sz
    L.kda_cp_local.argtypes = [vp] * 7 + [i32] * 6 + [ctypes.c_int, i32, vp, vp, vp, sz, vp]
    L.kda_cp_local.restype = ctypes.c_int
    L.kda_cp_finish.argtypes = [vp, vp] + [i32] * 6 + [ctypes.c_int, i32, vp, vp, vp, sz, vp]
    L.kda_cp_finish.restype = ctypes.c_int
    L.kda_state_compose.argtypes = [vp] * 4 + [i32] * 3 + [vp]
    L.kda_state_compose.restype = ctypes.c_int
    L.kda_check_device_error.argtypes = [vp, vp]
    L.kda_check_device_error.restype = ctypes.c_int
    L.kda_debug_set_wait_limit.argtypes = [ctypes.c_int64]
    L.kda_debug_set_wait_limit.restype = ctypes.c_int
    _lib = L
    return L


def status_string(s):
    return lib().kda_status_string(int(s)).decode()


# ------------------------------------------------------------ raw C names ---

def kda_forward_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, dt, chunk):
    return lib().kda_forward_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, dt,
                                            chunk)


def kda_forward_launches(num_seqs, total_tokens, max_seqlen, H, dk, dv, dt, chunk):
    return lib().kda_forward_launches(num_seqs, total_tokens, max_seqlen, H, dk, dv, dt, chunk)


def kda_forward(q, k, v, z, A, beta, S0, cu_seqlens, num_seqs, total_tokens, max_seqlen, H,
                dk, dv, dt, chunk, o, S_final, workspace, workspace_bytes, stream):
    return lib().kda_forward(q, k, v, z, A, beta, S0, cu_seqlens, num_seqs, total_tokens,
                             max_seqlen, H, dk, dv, dt, chunk, o, S_final, workspace,
                             workspace_bytes, stream)


def kda_forward_g(q, k, v, g, beta, S0, cu_seqlens, num_seqs, total_tokens, max_seqlen, H,
                  dk, dv, dt, chunk, o, S_final, workspace, workspace_bytes, stream):
    return lib().kda_forward_g(q, k, v, g, beta, S0, cu_seqlens, num_seqs, total_tokens,
                               max_seqlen, H, dk, dv, dt, chunk, o, S_final, workspace,
                               workspace_bytes, stream)


def kda_decode_step(q, k, v, z, A, beta, S_inout, B, H, dk, dv, dt, o, stream):
    return lib().kda_decode_step(q, k, v, z, A, beta, S_inout, B, H, dk, dv, dt, o, stream)


def kda_forward_noalloc(q, k, v, z, A, beta, S0, cu_seqlens, num_seqs, total_tokens,
                        max_seqlen, H, dk, dv, dt, chunk, o, S_final, stream):
    """kda_forward on the library's fixed scratch array (no workspace argument).
    For callers that cannot allocate device memory; see include/kda.h."""
    return lib().kda_forward_noalloc(q, k, v, z, A, beta, S0, cu_seqlens, num_seqs,
                                     total_tokens, max_seqlen, H, dk, dv, dt, chunk, o, S_final,
                                     stream)


def kda_forward_checkpoints(q, k, v, z, A, beta, S0, cu_seqlens, num_seqs, total_tokens,
                            max_seqlen, H, dk, dv, dt, chunk, o, S_final, S_ckpt, interval,
                            workspace, workspace_bytes, stream):
    return lib().kda_forward_checkpoints(q, k, v, z, A, beta, S0, cu_seqlens, num_seqs,
                                         total_tokens, max_seqlen, H, dk, dv, dt, chunk, o,
                                         S_final, S_ckpt, interval, workspace, workspace_bytes,
                                         stream)


def kda_forward_norm_gate(q, k, v, z, A, beta, S0, cu_seqlens, num_seqs, total_tokens,
                          max_seqlen, H, dk, dv, dt, chunk, out_gate, norm_weight, eps, o,
                          S_final, workspace, workspace_bytes, stream):
    return lib().kda_forward_norm_gate(q, k, v, z, A, beta, S0, cu_seqlens, num_seqs,
                                       total_tokens, max_seqlen, H, dk, dv, dt, chunk, out_gate,
                                       norm_weight, eps, o, S_final, workspace, workspace_bytes,
                                       stream)


def kda_decode_step_norm_gate(q, k, v, z, A, beta, S_inout, B, H, dk, dv, dt, out_gate,
                              norm_weight, eps, o, stream):
    return lib().kda_decode_step_norm_gate(q, k, v, z, A, beta, S_inout, B, H, dk, dv, dt,
                                           out_gate, norm_weight, eps, o, stream)


def kda_forward_scalar_gate(q, k, v, g_head, beta, S0, cu_seqlens, num_seqs, total_tokens,
                            max_seqlen, H, dk, dv, dt, chunk, o, S_final, workspace,
                            workspace_bytes, stream):
    return lib().kda_forward_scalar_gate(q, k, v, g_head, beta, S0, cu_seqlens, num_seqs,
                                         total_tokens, max_seqlen, H, dk, dv, dt, chunk, o,
                                         S_final, workspace, workspace_bytes, stream)


def kda_decode_step_conv(x_q, x_k, x_v, w_q, w_k, w_v, conv_width, conv_state, z, A, beta,
                         S_inout, B, H, dk, dv, dt, o, stream):
    return lib().kda_decode_step_conv(x_q, x_k, x_v, w_q, w_k, w_v, conv_width, conv_state, z,
                                      A, beta, S_inout, B, H, dk, dv, dt, o, stream)


def kda_short_conv_swish(x, w, cu_seqlens, num_seqs, total_tokens, max_seqlen, channels, width,
                         dt, y, stream):
    return lib().kda_short_conv_swish(x, w, cu_seqlens, num_seqs, total_tokens, max_seqlen,
                                      channels, width, dt, y, stream)


def kda_forward_conv_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, dt, chunk):
    return lib().kda_forward_conv_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv,
                                                 dt, chunk)


def kda_forward_conv(x_q, x_k, x_v, w_q, w_k, w_v, conv_width, z, A, beta, S0, cu_seqlens,
                     num_seqs, total_tokens, max_seqlen, H, dk, dv, dt, chunk, o, S_final,
                     workspace, workspace_bytes, stream):
    return lib().kda_forward_conv(x_q, x_k, x_v, w_q, w_k, w_v, conv_width, z, A, beta, S0,
                                  cu_seqlens, num_seqs, total_tokens, max_seqlen, H, dk, dv, dt,
                                  chunk, o, S_final, workspace, workspace_bytes, stream)


def kda_cp_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, dt, chunk):
    return lib().kda_cp_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv, dt, chunk)


def kda_cp_local(q, k, v, z, A, beta, cu_seqlens, num_seqs, total_tokens, max_seqlen, H, dk, dv,
                 dt, chunk, M_out, N_out, workspace, workspace_bytes, stream):
    return lib().kda_cp_local(q, k, v, z, A, beta, cu_seqlens, num_seqs, total_tokens,
                              max_seqlen, H, dk, dv, dt, chunk, M_out, N_out, workspace,
                              workspace_bytes, stream)


def kda_cp_finish(S_in, cu_seqlens, num_seqs, total_tokens, max_seqlen, H, dk, dv, dt, chunk, o,
                  S_final, workspace, workspace_bytes, stream):
    return lib().kda_cp_finish(S_in, cu_seqlens, num_seqs, total_tokens, max_seqlen, H, dk, dv,
                               dt, chunk, o, S_final, workspace, workspace_bytes, stream)


def kda_state_compose(M, N, S_in, S_out, count, dk, dv, stream):
    return lib().kda_state_compose(M, N, S_in, S_out, count, dk, dv, stream)


def kda_check_device_error(workspace, stream):
    return lib().kda_check_device_error(workspace, stream)


def kda_debug_set_wait_limit(cycles):
    return lib().kda_debug_set_wait_limit(cycles)


# ------------------------------------------------------- tensor helpers ---

def _dt(t):
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("KDA runs on the GPU only: pass CUDA tensors")
        if t is not None and not t.is_contiguous():
            raise ValueError("KDA tensors must be contiguous")


_F32_ROLES = ("A", "g", "g_head", "S0", "S_final", "S", "norm_weight", "S_ckpt")


def _shapes(T, H, dk, dv, N, dtype, **ts):
    """Raise ValueError unless every tensor given has the shape and dtype of its
    role (the C ABI takes raw pointers and cannot see either)."""
    want = {"q": (T, H, dk), "k": (T, H, dk), "z": (T, H, dk), "g": (T, H, dk),
            "v": (T, H, dv), "o": (T, H, dv), "out_gate": (T, H, dv), "beta": (T, H),
            "g_head": (T, H), "A": (H,), "S0": (N, H, dk, dv), "S_final": (N, H, dk, dv),
            "S": (N, H, dk, dv), "norm_weight": (dv,), "cu_seqlens": (N + 1,)}
    for name, t in ts.items():
        if t is None:
            continue
        if name in want and tuple(t.shape) != want[name]:
            raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {want[name]}")
        if name == "S_ckpt" and (t.dim() != 5 or tuple(t.shape[:2]) != (N, H) or
                                 tuple(t.shape[3:]) != (dk, dv)):
            raise ValueError(f"S_ckpt: shape {tuple(t.shape)}, expected ({N}, {H}, J, {dk}, {dv})")
        need = (torch.float32 if name in _F32_ROLES else
                torch.int32 if name == "cu_seqlens" else dtype)
        if t.dtype != need:
            raise ValueError(f"{name}: dtype {t.dtype}, expected {need}")


def _geometry(q, v, cu_seqlens, num_seqs, max_seqlen):
    T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        N = 1 if num_seqs is None else int(num_seqs)
        L = T // N if N else 0
        max_len = L if max_seqlen is None else int(max_seqlen)
    else:
        N = cu_seqlens.numel() - 1
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        max_len = int(max_seqlen)
    return T, H, dk, dv, N, max_len


def workspace(num_seqs, total_tokens, max_seqlen, H, dk, dv, dtype, chunk, device=None):
    """A uint8 device tensor of kda_forward_workspace_size() bytes."""
    nbytes = kda_forward_workspace_size(num_seqs, total_tokens, max_seqlen, H, dk, dv,
                                        _dt(torch.empty(0, dtype=dtype)), chunk)
    if nbytes == 0:
        raise KdaError(KDA_ERR_UNSUPPORTED, "kda_forward_workspace_size")
    return torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")


# the helpers below take a ``workspace`` argument that shadows the function
_new_workspace = workspace


def _forward(entry, q, k, v, gate_a, gate_b, beta, S0, cu_seqlens, num_seqs, max_seqlen, chunk,
             o, S_final, ws, stream, want_state):
    _check_cuda(q, k, v, gate_a, gate_b, beta, S0, cu_seqlens, o, S_final, ws)
    T, H, dk, dv, N, max_len = _geometry(q, v, cu_seqlens, num_seqs, max_seqlen)
    gate_roles = {"z": dict(z=gate_a, A=gate_b), "g": dict(g=gate_a),
                  "gs": dict(g_head=gate_a)}[entry]
    _shapes(T, H, dk, dv, N, q.dtype, q=q, k=k, v=v, beta=beta, S0=S0, cu_seqlens=cu_seqlens,
            o=o, S_final=S_final, **gate_roles)
    dt = _dt(q)
    if o is None:
        o = torch.empty((T, H, dv), dtype=q.dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(N, T, max_len, H, dk, dv, q.dtype, chunk, device=q.device)
    args = [_p(q), _p(k), _p(v), _p(gate_a)]
    if entry == "z":
        args.append(_p(gate_b))
    args += [_p(beta), _p(S0), _p(cu_seqlens), N, T, max_len, H, dk, dv, dt, chunk, _p(o),
             _p(S_final), _p(ws), ws.numel(), _stream(stream)]
    fn = {"z": kda_forward, "g": kda_forward_g, "gs": kda_forward_scalar_gate}[entry]
    st = fn(*args)
    if st != KDA_OK:
        raise KdaError(st, fn.__name__)
    return o, S_final


def forward(q, k, v, z, A, beta, *, S0=None, cu_seqlens=None, num_seqs=None, max_seqlen=None,
            chunk=64, o=None, S_final=None, workspace=None, stream=None, output_final_state=True):
    """KDA prefill.  q,k,z [T,H,dk], v [T,H,dv], beta [T,H] (all one dtype),
    A [H] fp32, S0 [N,H,dk,dv] fp32 or None, cu_seqlens int32 [N+1] or None
    (then ``num_seqs`` equal sequences).  Returns (o, S_final)."""
    return _forward("z", q, k, v, z, A, beta, S0, cu_seqlens, num_seqs, max_seqlen, chunk, o,
                    S_final, workspace, stream, output_final_state)


def forward_checkpoints(q, k, v, z, A, beta, interval, *, S0=None, cu_seqlens=None,
                        num_seqs=None, max_seqlen=None, chunk=64, o=None, S_final=None,
                        S_ckpt=None, workspace=None, stream=None):
    """KDA prefill that also returns the state after every ``interval`` tokens of
    each sequence: (o, S_final, S_ckpt) with S_ckpt [N, H, max_seqlen // interval,
    dk, dv] fp32 (entries past a sequence's end are left as allocated: zeros
    when the binding allocates them)."""
    _check_cuda(q, k, v, z, A, beta, S0, cu_seqlens, o, S_final, S_ckpt, workspace)
    T, H, dk, dv, N, max_len = _geometry(q, v, cu_seqlens, num_seqs, max_seqlen)
    _shapes(T, H, dk, dv, N, q.dtype, q=q, k=k, v=v, z=z, A=A, beta=beta, S0=S0,
            cu_seqlens=cu_seqlens, o=o, S_final=S_final, S_ckpt=S_ckpt)
    if S_ckpt is not None and S_ckpt.shape[2] != max_len // int(interval):
        raise ValueError(f"S_ckpt: {S_ckpt.shape[2]} checkpoints, expected "
                         f"{max_len // int(interval)}")
    if o is None:
        o = torch.empty((T, H, dv), dtype=q.dtype, device=q.device)
    if S_final is None:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    if S_ckpt is None:
        S_ckpt = torch.zeros((N, H, max_len // interval, dk, dv), dtype=torch.float32,
                             device=q.device)
    ws = workspace if workspace is not None else _new_workspace(N, T, max_len, H, dk, dv,
                                                                q.dtype, chunk, device=q.device)
    st = kda_forward_checkpoints(_p(q), _p(k), _p(v), _p(z), _p(A), _p(beta), _p(S0),
                                 _p(cu_seqlens), N, T, max_len, H, dk, dv, _dt(q), chunk, _p(o),
                                 _p(S_final), _p(S_ckpt), int(interval), _p(ws), ws.numel(),
                                 _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_forward_checkpoints")
    return o, S_final, S_ckpt


def forward_g(q, k, v, g, beta, *, S0=None, cu_seqlens=None, num_seqs=None, max_seqlen=None,
              chunk=64, o=None, S_final=None, workspace=None, stream=None,
              output_final_state=True):
    """KDA prefill with the fp32 log-decay g [T,H,dk] given directly (g in [-5, 0])."""
    return _forward("g", q, k, v, g, None, beta, S0, cu_seqlens, num_seqs, max_seqlen, chunk, o,
                    S_final, workspace, stream, output_final_state)


def forward_scalar_gate(q, k, v, g_head, beta, *, S0=None, cu_seqlens=None, num_seqs=None,
                        max_seqlen=None, chunk=64, o=None, S_final=None, workspace=None,
                        stream=None, output_final_state=True):
    """Gated DeltaNet special case: one fp32 log-decay per token and head,
    g_head [T,H] in [-5, 0], shared by the dk channels."""
    return _forward("gs", q, k, v, g_head, None, beta, S0, cu_seqlens, num_seqs, max_seqlen,
                    chunk, o, S_final, workspace, stream, output_final_state)


def decode_step(q, k, v, z, A, beta, S, *, o=None, stream=None):
    """One recurrent step: q,k,z [B,H,dk], v [B,H,dv], beta [B,H]; S [B,H,dk,dv]
    fp32 is updated in place.  Returns o [B,H,dv]."""
    _check_cuda(q, k, v, z, A, beta, S, o)
    B, H, dk = q.shape
    dv = v.shape[-1]
    _shapes(B, H, dk, dv, B, q.dtype, q=q, k=k, v=v, z=z, A=A, beta=beta, S=S, o=o)
    if o is None:
        o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    st = kda_decode_step(_p(q), _p(k), _p(v), _p(z), _p(A), _p(beta), _p(S), B, H, dk, dv,
                         _dt(q), _p(o), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_step")
    return o


def conv_state_zeros(B, H, dk, dv, width, dtype, device="cuda"):
    """The rolling input window of decode_step_conv before a sequence's first
    token: [B, H*(2*dk+dv), width-1] zeros."""
    return torch.zeros((B, H * (2 * dk + dv), width - 1), dtype=dtype, device=device)


def decode_step_conv(x_q, x_k, x_v, w_q, w_k, w_v, conv_state, z, A, beta, S, *, o=None,
                     stream=None):
    """One recurrent step with the input prologue carried across steps: x_q,
    x_k [B,H,dk], x_v [B,H,dv] are this token's convolution inputs, w_* [H*d,
    width] fp32 the taps, conv_state [B, H*(2dk+dv), width-1] (x's dtype) the
    rolling window, S [B,H,dk,dv] fp32; conv_state and S are updated in place.
    Returns o [B,H,dv]."""
    _check_cuda(x_q, x_k, x_v, w_q, w_k, w_v, conv_state, z, A, beta, S, o)
    B, H, dk = x_q.shape
    dv = x_v.shape[-1]
    _shapes(B, H, dk, dv, B, x_q.dtype, q=x_q, k=x_k, v=x_v, z=z, A=A, beta=beta, S=S, o=o)
    width = w_q.shape[-1]
    for name, w, rows in (("w_q", w_q, H * dk), ("w_k", w_k, H * dk), ("w_v", w_v, H * dv)):
        if tuple(w.shape) != (rows, width) or w.dtype != torch.float32:
            raise ValueError(f"{name}: {tuple(w.shape)} {w.dtype}, expected ({rows}, {width}) "
                             "float32")
    want = (B, H * (2 * dk + dv), width - 1)
    if conv_state is None or tuple(conv_state.shape) != want or conv_state.dtype != x_q.dtype \
            or not conv_state.is_contiguous():
        got = None if conv_state is None else (tuple(conv_state.shape), conv_state.dtype)
        raise ValueError(f"conv_state: {got}, expected contiguous {want} {x_q.dtype}")
    if o is None:
        o = torch.empty((B, H, dv), dtype=x_q.dtype, device=x_q.device)
    st = kda_decode_step_conv(_p(x_q), _p(x_k), _p(x_v), _p(w_q), _p(w_k), _p(w_v), width,
                              _p(conv_state), _p(z), _p(A), _p(beta), _p(S), B, H, dk, dv,
                              _dt(x_q), _p(o), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_step_conv")
    return o


def forward_norm_gate(q, k, v, z, A, beta, out_gate, *, norm_weight=None, eps=1e-6, S0=None,
                      cu_seqlens=None, num_seqs=None, max_seqlen=None, chunk=64, o=None,
                      S_final=None, workspace=None, stream=None):
    """KDA prefill followed by the output epilogue: o = RMSNorm(attention output
    over dv) * norm_weight * sigmoid(out_gate), out_gate [T,H,dv] in q's dtype,
    norm_weight [dv] fp32 or None.  Returns (o, S_final)."""
    _check_cuda(q, k, v, z, A, beta, out_gate, norm_weight, S0, cu_seqlens, o, S_final,
                workspace)
    T, H, dk, dv, N, max_len = _geometry(q, v, cu_seqlens, num_seqs, max_seqlen)
    _shapes(T, H, dk, dv, N, q.dtype, q=q, k=k, v=v, z=z, A=A, beta=beta, out_gate=out_gate,
            norm_weight=norm_weight, S0=S0, cu_seqlens=cu_seqlens, o=o, S_final=S_final)
    if o is None:
        o = torch.empty((T, H, dv), dtype=q.dtype, device=q.device)
    if S_final is None:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    ws = workspace if workspace is not None else _new_workspace(N, T, max_len, H, dk, dv,
                                                                q.dtype, chunk, device=q.device)
    st = kda_forward_norm_gate(_p(q), _p(k), _p(v), _p(z), _p(A), _p(beta), _p(S0),
                               _p(cu_seqlens), N, T, max_len, H, dk, dv, _dt(q), chunk,
                               _p(out_gate), _p(norm_weight), float(eps), _p(o), _p(S_final),
                               _p(ws), ws.numel(), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_forward_norm_gate")
    return o, S_final


def decode_step_norm_gate(q, k, v, z, A, beta, S, out_gate, *, norm_weight=None, eps=1e-6,
                          o=None, stream=None):
    """decode_step followed by the output epilogue (see forward_norm_gate);
    out_gate [B,H,dv].  S is updated in place.  Returns o [B,H,dv]."""
    _check_cuda(q, k, v, z, A, beta, S, out_gate, norm_weight, o)
    B, H, dk = q.shape
    dv = v.shape[-1]
    _shapes(B, H, dk, dv, B, q.dtype, q=q, k=k, v=v, z=z, A=A, beta=beta, S=S, o=o,
            out_gate=out_gate, norm_weight=norm_weight)
    if o is None:
        o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    st = kda_decode_step_norm_gate(_p(q), _p(k), _p(v), _p(z), _p(A), _p(beta), _p(S), B, H, dk,
                                   dv, _dt(q), _p(out_gate), _p(norm_weight), float(eps), _p(o),
                                   _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_decode_step_norm_gate")
    return o


def short_conv_swish(x, w, *, cu_seqlens=None, num_seqs=None, max_seqlen=None, y=None,
                     stream=None):
    """Input prologue on one tensor x [T, ...] (trailing axes = channels):
    y = Swish(causal depthwise convolution with taps w [channels, width])."""
    _check_cuda(x, w, cu_seqlens, y)
    T = x.shape[0]
    C = x.numel() // T if T else int(np.prod(x.shape[1:]))
    if cu_seqlens is None:
        N = 1 if num_seqs is None else int(num_seqs)
        L = T // N if N else 0
    else:
        N = cu_seqlens.numel() - 1
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        L = int(max_seqlen)
    if cu_seqlens is not None and (cu_seqlens.dtype != torch.int32 or
                                   cu_seqlens.numel() != N + 1):
        raise ValueError("cu_seqlens: int32 [N+1] expected")
    if w.dtype != torch.float32 or w.dim() != 2 or w.shape[0] != C:
        raise ValueError(f"w: {tuple(w.shape)} {w.dtype}, expected ({C}, width) float32")
    if y is not None and (y.shape != x.shape or y.dtype != x.dtype):
        raise ValueError("y: must match x in shape and dtype")
    if y is None:
        y = torch.empty_like(x)
    st = kda_short_conv_swish(_p(x), _p(w), _p(cu_seqlens), N, T, L, C, w.shape[-1], _dt(x),
                              _p(y), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_short_conv_swish")
    return y


def forward_conv(x_q, x_k, x_v, w_q, w_k, w_v, z, A, beta, *, S0=None, cu_seqlens=None,
                 num_seqs=None, max_seqlen=None, chunk=64, o=None, S_final=None, workspace=None,
                 stream=None):
    """KDA prefill on the input prologue's outputs: q, k, v = Swish(short causal
    convolution of x_q, x_k, x_v) with taps w_* [H*d, width] fp32.  Returns
    (o, S_final)."""
    _check_cuda(x_q, x_k, x_v, w_q, w_k, w_v, z, A, beta, S0, cu_seqlens, o, S_final, workspace)
    T, H, dk, dv, N, max_len = _geometry(x_q, x_v, cu_seqlens, num_seqs, max_seqlen)
    _shapes(T, H, dk, dv, N, x_q.dtype, q=x_q, k=x_k, v=x_v, z=z, A=A, beta=beta, S0=S0,
            cu_seqlens=cu_seqlens, o=o, S_final=S_final)
    width = w_q.shape[-1]
    for name, w, rows in (("w_q", w_q, H * dk), ("w_k", w_k, H * dk), ("w_v", w_v, H * dv)):
        if tuple(w.shape) != (rows, width) or w.dtype != torch.float32:
            raise ValueError(f"{name}: {tuple(w.shape)} {w.dtype}, expected ({rows}, {width}) "
                             "float32")
    if o is None:
        o = torch.empty((T, H, dv), dtype=x_q.dtype, device=x_q.device)
    if S_final is None:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=x_q.device)
    dt = _dt(x_q)
    if workspace is None:
        nbytes = kda_forward_conv_workspace_size(N, T, max_len, H, dk, dv, dt, chunk)
        if nbytes == 0:
            raise KdaError(KDA_ERR_UNSUPPORTED, "kda_forward_conv_workspace_size")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=x_q.device)
    st = kda_forward_conv(_p(x_q), _p(x_k), _p(x_v), _p(w_q), _p(w_k), _p(w_v), w_q.shape[-1],
                          _p(z), _p(A), _p(beta), _p(S0), _p(cu_seqlens), N, T, max_len, H, dk,
                          dv, dt, chunk, _p(o), _p(S_final), _p(workspace), workspace.numel(),
                          _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_forward_conv")
    return o, S_final


class CpShard:
    """A shard's context-parallel state between cp_local and cp_finish: its
    geometry and the workspace that holds its chunk preparation."""

    def __init__(self, geometry, dtype, cu_seqlens, workspace, chunk):
        self.geometry, self.dtype, self.cu_seqlens = geometry, dtype, cu_seqlens
        self.workspace, self.chunk = workspace, chunk


def cp_local(q, k, v, z, A, beta, *, cu_seqlens=None, num_seqs=None, max_seqlen=None, chunk=64,
             workspace=None, stream=None):
    """Context parallelism, step 1 on this rank's shard: returns (M [N,H,dk,dk],
    N [N,H,dk,dv], shard) with S_after = M S_before + N for each sequence and
    head; ``shard`` carries the workspace to cp_finish."""
    _check_cuda(q, k, v, z, A, beta, cu_seqlens, workspace)
    T, H, dk, dv, N, max_len = _geometry(q, v, cu_seqlens, num_seqs, max_seqlen)
    _shapes(T, H, dk, dv, N, q.dtype, q=q, k=k, v=v, z=z, A=A, beta=beta, cu_seqlens=cu_seqlens)
    dt = _dt(q)
    if workspace is None:
        nbytes = kda_cp_workspace_size(N, T, max_len, H, dk, dv, dt, chunk)
        if nbytes == 0:
            raise KdaError(KDA_ERR_UNSUPPORTED, "kda_cp_workspace_size")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    M = torch.empty((N, H, dk, dk), dtype=torch.float32, device=q.device)
    Nt = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    st = kda_cp_local(_p(q), _p(k), _p(v), _p(z), _p(A), _p(beta), _p(cu_seqlens), N, T, max_len,
                      H, dk, dv, dt, chunk, _p(M), _p(Nt), _p(workspace), workspace.numel(),
                      _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_cp_local")
    return M, Nt, CpShard((T, H, dk, dv, N, max_len), q.dtype, cu_seqlens, workspace, chunk)


def cp_finish(shard, S_in=None, *, o=None, S_final=None, stream=None):
    """Context parallelism, step 4: o of the shard and the state after it, from
    the state entering it (None: zeros) and the workspace cp_local filled."""
    T, H, dk, dv, N, max_len = shard.geometry
    _check_cuda(S_in, o, S_final)
    _shapes(T, H, dk, dv, N, shard.dtype, S0=S_in, o=o, S_final=S_final)
    if o is None:
        o = torch.empty((T, H, dv), dtype=shard.dtype, device=shard.workspace.device)
    if S_final is None:
        S_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=shard.workspace.device)
    st = kda_cp_finish(_p(S_in), _p(shard.cu_seqlens), N, T, max_len, H, dk, dv,
                       _dt(torch.empty(0, dtype=shard.dtype)), shard.chunk, _p(o), _p(S_final),
                       _p(shard.workspace), shard.workspace.numel(), _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_cp_finish")
    return o, S_final


def state_compose(M, N, S_in=None, *, S_out=None, stream=None):
    """S_out = M S_in + N over leading batch axes (fp32; S_in None reads as 0)."""
    _check_cuda(M, N, S_in, S_out)
    dk, dv = N.shape[-2], N.shape[-1]
    count = N.numel() // (dk * dv)
    for name, t, shape in (("M", M, N.shape[:-2] + (dk, dk)), ("S_in", S_in, N.shape),
                           ("S_out", S_out, N.shape)):
        if t is not None and (tuple(t.shape) != tuple(shape) or t.dtype != torch.float32):
            raise ValueError(f"{name}: {tuple(t.shape)} {t.dtype}, expected {tuple(shape)} float32")
    if N.dtype != torch.float32:
        raise ValueError("N: float32 expected")
    if S_out is None:
        S_out = torch.empty_like(N)
    st = kda_state_compose(_p(M), _p(N), _p(S_in), _p(S_out), count, dk, dv, _stream(stream))
    if st != KDA_OK:
        raise KdaError(st, "kda_state_compose")
    return S_out


def check_device_error(ws, stream=None):
    """Status recorded on the device by the last forward call on ``ws``."""
    return kda_check_device_error(_p(ws), _stream(stream))

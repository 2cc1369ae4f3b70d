"""Thin ctypes binding of ``libssd.so`` (argument marshalling only).

Every step of the SSD forward runs in the library's CUDA kernels; this module
checks tensor devices, dtypes and contiguity, allocates outputs and the
workspace with torch (device memory is the only thing torch provides here),
and passes raw device pointers plus the current CUDA stream to the C ABI of
``include/ssd.h``.  There is no fallback: a missing library or a non-zero
status raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libssd.so")
_lib = None

SSD_F32, SSD_BF16 = 0, 1
STATUS = {0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED", 3: "SSD_ERR_CUDA",
          4: "SSD_ERR_TIMEOUT"}

# Every symbol include/ssd.h declares.
EXPORTS = ("ssd_fwd", "ssd_fwd_gated", "ssd_fwd_gated_launch_count", "ssd_fwd_workspace_bytes",
           "ssd_fwd_launch_count", "ssd_fwd_timed",
           "ssd_fwd_stage_name", "ssd_fwd_check", "ssd_fwd_withhold_publish", "ssd_status_string", "ssd_version",
           "ssd_fwd_no_alloc", "ssd_fwd_no_alloc_check", "ssd_step", "ssd_gate_norm", "ssd_split_logdecay",
           "ssd_split_combine", "ssd_split_correct", "ssd_bwd", "ssd_bwd_workspace_bytes", "ssd_bwd_check")


class SSDError(RuntimeError):
    """A non-zero status returned by libssd.so."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status_string(status)})")


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Open libssd.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m structured_state_space_ssd_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, fp, i, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.ssd_fwd.argtypes = [vp, fp, fp, vp, vp, fp, i, fp, vp, fp, i, i, i, i, i, i, i, vp, sz, vp]
    lib.ssd_fwd.restype = i
    lib.ssd_fwd_gated.argtypes = [vp, fp, fp, vp, vp, fp, i, fp, vp, fp, fp, ctypes.c_float, vp, fp, i, i, i, i, i,
                                  i, i, vp, sz, vp]
    lib.ssd_fwd_gated.restype = i
    lib.ssd_fwd_gated_launch_count.argtypes = [i] * 8
    lib.ssd_fwd_gated_launch_count.restype = i
    lib.ssd_fwd_workspace_bytes.argtypes = [i] * 8
    lib.ssd_fwd_workspace_bytes.restype = sz
    lib.ssd_fwd_launch_count.argtypes = [i] * 8
    lib.ssd_fwd_launch_count.restype = i
    lib.ssd_fwd_timed.argtypes = lib.ssd_fwd.argtypes + [fp, i, fp]
    lib.ssd_fwd_timed.restype = i
    lib.ssd_fwd_stage_name.argtypes = [i] * 9
    lib.ssd_fwd_stage_name.restype = ctypes.c_char_p
    lib.ssd_fwd_check.argtypes = [vp, vp]
    lib.ssd_fwd_check.restype = i
    lib.ssd_bwd_check.argtypes = [vp, vp]
    lib.ssd_bwd_check.restype = i
    lib.ssd_fwd_withhold_publish.argtypes = lib.ssd_fwd.argtypes + [i, i, i, ctypes.c_uint]
    lib.ssd_fwd_withhold_publish.restype = i
    lib.ssd_fwd_no_alloc.argtypes = [vp, fp, fp, vp, vp, fp, i, fp, vp, fp, i, i, i, i, i, i, i, vp]
    lib.ssd_fwd_no_alloc.restype = i
    lib.ssd_fwd_no_alloc_check.argtypes = [vp]
    lib.ssd_fwd_no_alloc_check.restype = i
    lib.ssd_status_string.argtypes = [i]
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_version.argtypes = []
    lib.ssd_version.restype = i
    lib.ssd_step.argtypes = [vp, vp, fp, fp, vp, vp, fp, vp, i, i, i, i, i, i, vp]
    lib.ssd_step.restype = i
    lib.ssd_gate_norm.argtypes = [vp, vp, fp, fp, vp, ctypes.c_longlong, i, i, ctypes.c_float, i, vp]
    lib.ssd_gate_norm.restype = i
    lib.ssd_split_logdecay.argtypes = [fp, fp, fp, fp, i, i, i, vp]
    lib.ssd_split_logdecay.restype = i
    lib.ssd_split_combine.argtypes = [fp, fp, fp, i, i, fp, fp, i, i, i, i, vp]
    lib.ssd_split_combine.restype = i
    lib.ssd_split_correct.argtypes = [vp, vp, fp, fp, i, i, i, i, i, i, i, vp]
    lib.ssd_split_correct.restype = i
    lib.ssd_bwd.argtypes = [vp, fp, fp, vp, vp, fp, i, fp, vp, fp, vp, fp, fp, vp, vp, fp, fp] + [i] * 7 + [vp, sz, vp]
    lib.ssd_bwd.restype = i
    lib.ssd_bwd_workspace_bytes.argtypes = [i] * 8
    lib.ssd_bwd_workspace_bytes.restype = sz
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().ssd_status_string(int(status)).decode()


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return SSD_F32
    if t == torch.bfloat16:
        return SSD_BF16
    raise TypeError(f"x/B/C must be float32 or bfloat16, got {t}")


def ssd_fwd_workspace_bytes(batch, T, H, P, G, N, Q, dtype) -> int:
    code = dtype if isinstance(dtype, int) else _dtype_code(dtype)
    return int(load().ssd_fwd_workspace_bytes(batch, T, H, P, G, N, Q, code))


def ssd_fwd_launch_count(batch, T, H, P, G, N, Q, dtype) -> int:
    code = dtype if isinstance(dtype, int) else _dtype_code(dtype)
    return int(load().ssd_fwd_launch_count(batch, T, H, P, G, N, Q, code))


def ssd_fwd_stage_names(batch, T, H, P, G, N, Q, dtype) -> list:
    """Names of the kernels ssd_fwd launches for this problem, in launch order."""
    code = dtype if isinstance(dtype, int) else _dtype_code(dtype)
    lib = load()
    names = []
    while True:
        n = lib.ssd_fwd_stage_name(batch, T, H, P, G, N, Q, code, len(names))
        if n is None:
            return names
        names.append(n.decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def ssd_fwd(x, dt, A, B, C, D, Q: int, init_state=None, *, y=None, final_state=None,
            return_final_state: bool = True, workspace=None, stream=None, stage_ms=None):
    """SSD layer forward on the GPU.

    x [b,T,H,P], B/C [b,T,G,N] (fp32 or bf16, same dtype), dt [b,T,H], A [H],
    D [H], init_state [b,H,P,N] (fp32 or None) -- contiguous CUDA tensors on
    one device.  Returns ``(y, final_state)``; y has x's dtype, final_state is
    fp32 (None when ``return_final_state`` is False and no buffer is given).
    Runs on ``stream`` (default: the current torch stream) without host sync.
    With ``stage_ms`` (a list) the call goes through ``ssd_fwd_timed`` instead:
    it waits for the stream and appends each kernel's milliseconds, then the
    whole call's span, to the list.
    """
    b, T, H, P, G, N, code, workspace, handle = _prepare_fwd(x, dt, A, B, C, D, Q, init_state, workspace, stream,
                                                             "ssd_fwd")
    dev = x.device
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and return_final_state:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
    lib = load()
    args = (_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), int(Q), _ptr(init_state),
            _ptr(y), _ptr(final_state), b, T, H, P, G, N, code, _ptr(workspace),
            ctypes.c_size_t(workspace.numel() * workspace.element_size()), ctypes.c_void_p(handle))
    if stage_ms is None:
        rc = lib.ssd_fwd(*args)
        if rc != 0:
            raise SSDError(rc, "ssd_fwd")
    else:
        ms = (ctypes.c_float * 8)()
        total = ctypes.c_float(0)
        rc = lib.ssd_fwd_timed(*args, ctypes.cast(ms, ctypes.c_void_p), 8,
                               ctypes.cast(ctypes.pointer(total), ctypes.c_void_p))
        if rc != 0:
            raise SSDError(rc, "ssd_fwd_timed")
        k = int(lib.ssd_fwd_launch_count(b, T, H, P, G, N, int(Q), code))
        stage_ms.extend(float(ms[i]) for i in range(min(k, 8)))
        stage_ms.append(float(total.value))
    return y, final_state


def ssd_fwd_gated(x, dt, A, B, C, D, Q: int, z, init_state=None, norm_weight=None, norm_bias=None,
                  eps: float = 1e-5, *, out=None, final_state=None, return_final_state: bool = True,
                  workspace=None, stream=None):
    """The layer forward followed by the gate and a GroupNorm with a group per head, on the GPU.

    Arguments as for ``ssd_fwd``, plus z (x's shape and dtype) and the norm's fp32 [H*P] weight and bias
    (None: 1 and 0).  Returns ``(out, final_state)`` with out = GroupNorm(y * silu(z)) over each head's P
    channels (y itself is not returned).  One fused launch where the tensor-core path takes whole
    64-column heads in one launch; otherwise ``ssd_fwd`` then ``ssd_gate_norm`` in place.
    """
    b, T, H, P, G, N, code, workspace, handle = _prepare_fwd(x, dt, A, B, C, D, Q, init_state, workspace, stream,
                                                             "ssd_fwd_gated")
    dev = x.device
    if z.shape != x.shape or z.dtype != x.dtype or z.device != dev or not z.is_contiguous():
        raise ValueError("z must be a contiguous tensor of x's shape, dtype and device")
    for k, t in (("norm_weight", norm_weight), ("norm_bias", norm_bias)):
        if t is not None and (t.dtype != torch.float32 or t.numel() != H * P or t.device != dev
                              or not t.is_contiguous()):
            raise ValueError(f"{k} must be a contiguous float32 [{H * P}] tensor on {dev}")
    if out is None:
        out = torch.empty_like(x)
    if final_state is None and return_final_state:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
    rc = load().ssd_fwd_gated(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), int(Q), _ptr(init_state),
                              _ptr(z), _ptr(norm_weight), _ptr(norm_bias), float(eps), _ptr(out), _ptr(final_state),
                              b, T, H, P, G, N, code, _ptr(workspace),
                              ctypes.c_size_t(workspace.numel() * workspace.element_size()), ctypes.c_void_p(handle))
    if rc != 0:
        raise SSDError(rc, "ssd_fwd_gated")
    return out, final_state


def _prepare_fwd(x, dt, A, B, C, D, Q, init_state, workspace, stream, what):
    """Argument checks shared by the forward entry points; returns the dims, dtype code, workspace, stream."""
    dev = x.device
    if dev.type != "cuda":
        raise ValueError(f"{what} needs CUDA tensors (there is no CPU path)")
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    code = _dtype_code(x.dtype)
    named = dict(x=x, dt=dt, A=A, B=B, C=C, D=D)
    if init_state is not None:
        named["init_state"] = init_state
    for k, t in named.items():
        if t.device != dev:
            raise ValueError(f"{k} is on {t.device}, x on {dev}")
        if not t.is_contiguous():
            raise ValueError(f"{k} must be contiguous")
    if B.dtype != x.dtype or C.dtype != x.dtype:
        raise TypeError("x, B and C must share one dtype")
    for k in ("dt", "A", "D") + (("init_state",) if init_state is not None else ()):
        if named[k].dtype != torch.float32:
            raise TypeError(f"{k} must be float32")
    if tuple(dt.shape) != (b, T, H) or tuple(A.shape) != (H,) or tuple(D.shape) != (H,):
        raise ValueError("dt must be [b,T,H]; A and D must be [H]")
    if tuple(B.shape) != (b, T, G, N) or tuple(C.shape) != (b, T, G, N):
        raise ValueError("B and C must be [b,T,G,N]")
    if init_state is not None and tuple(init_state.shape) != (b, H, P, N):
        raise ValueError("init_state must be [b,H,P,N]")
    need = int(load().ssd_fwd_workspace_bytes(b, T, H, P, G, N, int(Q), code))
    if need == 0:
        raise SSDError(1, "ssd_fwd_workspace_bytes")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return b, T, H, P, G, N, code, workspace, handle


def ssd_fwd_check(workspace, stream=None) -> int:
    """Wait for the stream and return the device-side status word of the last call."""
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return int(load().ssd_fwd_check(_ptr(workspace), ctypes.c_void_p(handle)))


def ssd_step(state, x, dt, A, B, C, D, *, y=None, stream=None):
    """One decode step on the GPU: updates ``state`` in place and returns y.

    state [b,H,P,N] fp32, x [b,H,P] and B/C [b,G,N] (fp32 or bf16, one dtype),
    dt [b,H], A [H], D [H] fp32 -- contiguous CUDA tensors on one device.
    Runs on ``stream`` (default: the current torch stream) without host sync.
    """
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("ssd_step needs CUDA tensors (there is no CPU path)")
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    code = _dtype_code(x.dtype)
    named = dict(state=state, x=x, dt=dt, A=A, B=B, C=C, D=D)
    for k, t in named.items():
        if t.device != dev:
            raise ValueError(f"{k} is on {t.device}, x on {dev}")
        if not t.is_contiguous():
            raise ValueError(f"{k} must be contiguous")
    if B.dtype != x.dtype or C.dtype != x.dtype:
        raise TypeError("x, B and C must share one dtype")
    for k in ("state", "dt", "A", "D"):
        if named[k].dtype != torch.float32:
            raise TypeError(f"{k} must be float32")
    if tuple(state.shape) != (b, H, P, N) or tuple(dt.shape) != (b, H) or tuple(A.shape) != (H,) \
            or tuple(D.shape) != (H,) or tuple(C.shape) != (b, G, N):
        raise ValueError("expected state [b,H,P,N], dt [b,H], A and D [H], B and C [b,G,N]")
    if y is None:
        y = torch.empty_like(x)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    rc = load().ssd_step(_ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y),
                         b, H, P, G, N, code, ctypes.c_void_p(handle))
    if rc != 0:
        raise SSDError(rc, "ssd_step")
    return y


def ssd_gate_norm(y, z, ngroups: int, eps: float = 1e-5, weight=None, bias=None, *, out=None, stream=None):
    """Swish gate then GroupNorm on the GPU: ``out = GroupNorm(y * silu(z))`` per token.

    y and z have one shape [..., channels] and dtype (fp32 or bf16); the channels of each token split
    into ``ngroups`` contiguous groups.  weight, bias: fp32 [channels] or None.  ``out`` may be y.
    """
    dev = y.device
    if dev.type != "cuda":
        raise ValueError("ssd_gate_norm needs CUDA tensors (there is no CPU path)")
    if z.shape != y.shape or z.dtype != y.dtype or z.device != dev:
        raise ValueError("y and z must have one shape, dtype and device")
    ch = y.shape[-1]
    for k, t in (("y", y), ("z", z), ("weight", weight), ("bias", bias)):
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{k} must be contiguous")
    for k, t in (("weight", weight), ("bias", bias)):
        if t is not None and (t.dtype != torch.float32 or t.numel() != ch or t.device != dev):
            raise ValueError(f"{k} must be a float32 [{ch}] tensor on {dev}")
    if out is None:
        out = torch.empty_like(y)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    rows = y.numel() // ch
    rc = load().ssd_gate_norm(_ptr(y), _ptr(z), _ptr(weight), _ptr(bias), _ptr(out), rows, ch, int(ngroups),
                              float(eps), _dtype_code(y.dtype), ctypes.c_void_p(handle))
    if rc != 0:
        raise SSDError(rc, "ssd_gate_norm")
    return out


# --- sequence split: shards of one sequence run at once and exchange only their states ---------------

def _handle(stream, dev):
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check_cuda_f32(**named):
    for k, t in named.items():
        if t is None:
            continue
        if t.device.type != "cuda":
            raise ValueError(f"{k} must be a CUDA tensor (there is no CPU path)")
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise TypeError(f"{k} must be a contiguous float32 tensor")


def ssd_split_logdecay(dt, A, *, stream=None):
    """Per-token inclusive log-decay prefix of a shard: returns (sig [b,H,T], total [b,H]) fp32."""
    _check_cuda_f32(dt=dt, A=A)
    b, T, H = dt.shape
    sig = torch.empty((b, H, T), dtype=torch.float32, device=dt.device)
    total = torch.empty((b, H), dtype=torch.float32, device=dt.device)
    rc = load().ssd_split_logdecay(_ptr(dt), _ptr(A), _ptr(sig), _ptr(total), b, T, H, _handle(stream, dt.device))
    if rc != 0:
        raise SSDError(rc, "ssd_split_logdecay")
    return sig, total


def ssd_split_combine(fin0_all, total_all, k: int, init_state=None, *, stream=None):
    """State entering shard k and the shard's true final state, from every shard's zero-start final state
    fin0_all [K,b,H,P,N] and total log decay total_all [K,b,H] (shard order)."""
    _check_cuda_f32(fin0_all=fin0_all, total_all=total_all, init_state=init_state)
    K, b, H, P, N = fin0_all.shape
    if tuple(total_all.shape) != (K, b, H) or (init_state is not None and tuple(init_state.shape) != (b, H, P, N)):
        raise ValueError("expected total_all [K,b,H] and init_state [b,H,P,N] matching fin0_all [K,b,H,P,N]")
    s_in = torch.empty((b, H, P, N), dtype=torch.float32, device=fin0_all.device)
    fin = torch.empty_like(s_in)
    rc = load().ssd_split_combine(_ptr(fin0_all), _ptr(total_all), _ptr(init_state), int(k), K, _ptr(s_in),
                                  _ptr(fin), b, H, P, N, _handle(stream, fin0_all.device))
    if rc != 0:
        raise SSDError(rc, "ssd_split_combine")
    return s_in, fin


def ssd_split_correct(y, C, sig, s_in, *, stream=None):
    """y += exp(sig_t) s_in C_t in place (y [b,T,H,P], C [b,T,G,N]); returns y."""
    _check_cuda_f32(sig=sig, s_in=s_in)
    if C.dtype != y.dtype or not (y.is_contiguous() and C.is_contiguous()) or y.device != C.device:
        raise TypeError("y and C must be contiguous tensors of one dtype on one device")
    b, T, H, P = y.shape
    G, N = C.shape[2], C.shape[3]
    if tuple(sig.shape) != (b, H, T) or tuple(s_in.shape) != (b, H, P, N):
        raise ValueError("expected sig [b,H,T] and s_in [b,H,P,N]")
    rc = load().ssd_split_correct(_ptr(y), _ptr(C), _ptr(sig), _ptr(s_in), b, T, H, P, G, N, _dtype_code(y.dtype),
                                  _handle(stream, y.device))
    if rc != 0:
        raise SSDError(rc, "ssd_split_correct")
    return y


def exchange_shard_states(fin0, total, group=None):
    """All-gather every worker's (zero-start final state, total log decay) in rank order: the one exchange
    of the sequence split.  Returns (fin0_all [K,...], total_all [K,...])."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    fin0_all = torch.empty((world,) + tuple(fin0.shape), dtype=fin0.dtype, device=fin0.device)
    total_all = torch.empty((world,) + tuple(total.shape), dtype=total.dtype, device=total.device)
    dist.all_gather(list(fin0_all.unbind(0)), fin0.contiguous(), group=group)
    dist.all_gather(list(total_all.unbind(0)), total.contiguous(), group=group)
    return fin0_all, total_all


def ssd_fwd_sequence_parallel(x, dt, A, B, C, D, Q: int, init_state=None, group=None):
    """This worker's shard of a sequence split across the workers of ``group`` (rank order = shard order).

    Every worker passes its contiguous shard (x [b,T_k,H,P], dt, B, C) and the same A, D and
    init_state (the state before the whole sequence, or None).  Returns (y_k, final_state_k): y of the
    shard and the state after it, as ssd_fwd over the whole sequence would give them; the last worker's
    final_state is the sequence's.
    """
    import torch.distributed as dist
    k = dist.get_rank(group)
    y, fin0 = ssd_fwd(x, dt, A, B, C, D, Q, None)
    sig, total = ssd_split_logdecay(dt, A)
    fin0_all, total_all = exchange_shard_states(fin0, total, group)
    s_in, fin = ssd_split_combine(fin0_all, total_all, k, init_state)
    ssd_split_correct(y, C, sig, s_in)
    return y, fin


# --- backward pass and the autograd wrapper -----------------------------------------------------------

def ssd_bwd_workspace_bytes(batch, T, H, P, G, N, Q, dtype) -> int:
    code = dtype if isinstance(dtype, int) else _dtype_code(dtype)
    return int(load().ssd_bwd_workspace_bytes(batch, T, H, P, G, N, Q, code))


def ssd_bwd(x, dt, A, B, C, D, dy, Q: int = 256, init_state=None, dfinal_state=None, *, need_dinit: bool = True,
            workspace=None, stream=None):
    """Gradients of ``sum(dy * y) + sum(dfinal_state * final_state)`` for ``ssd_fwd``'s inputs, on the GPU.

    Inputs as for :func:`ssd_fwd`, plus dy [b,T,H,P] in x's dtype and dfinal_state [b,H,P,N] fp32
    (None: zero).  Returns a dict with dx [b,T,H,P], dB, dC [b,T,G,N] (x's dtype), ddt [b,T,H],
    dA [H], dD [H] and dinit_state [b,H,P,N] (fp32; None unless ``need_dinit``).
    Runs on ``stream`` (default: the current torch stream) without host sync.
    """
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("ssd_bwd needs CUDA tensors (there is no CPU path)")
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    code = _dtype_code(x.dtype)
    named = dict(x=x, dt=dt, A=A, B=B, C=C, D=D, dy=dy, init_state=init_state, dfinal_state=dfinal_state)
    for k, t in named.items():
        if t is None:
            continue
        if t.device != dev:
            raise ValueError(f"{k} is on {t.device}, x on {dev}")
        if not t.is_contiguous():
            raise ValueError(f"{k} must be contiguous")
    if B.dtype != x.dtype or C.dtype != x.dtype or dy.dtype != x.dtype:
        raise TypeError("x, B, C and dy must share one dtype")
    for k in ("dt", "A", "D", "init_state", "dfinal_state"):
        if named[k] is not None and named[k].dtype != torch.float32:
            raise TypeError(f"{k} must be float32")
    if tuple(dt.shape) != (b, T, H) or tuple(A.shape) != (H,) or tuple(D.shape) != (H,) or dy.shape != x.shape:
        raise ValueError("dt must be [b,T,H]; A and D must be [H]; dy must match x")
    if tuple(B.shape) != (b, T, G, N) or tuple(C.shape) != (b, T, G, N):
        raise ValueError("B and C must be [b,T,G,N]")
    for k in ("init_state", "dfinal_state"):
        if named[k] is not None and tuple(named[k].shape) != (b, H, P, N):
            raise ValueError(f"{k} must be [b,H,P,N]")
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dx": torch.empty_like(x), "ddt": torch.empty((b, T, H), **f32), "dA": torch.empty((H,), **f32),
           "dB": torch.empty_like(B), "dC": torch.empty_like(C), "dD": torch.empty((H,), **f32),
           "dinit_state": torch.empty((b, H, P, N), **f32) if need_dinit else None}
    lib = load()
    need = int(lib.ssd_bwd_workspace_bytes(b, T, H, P, G, N, int(Q), code))
    if need == 0:
        raise SSDError(1, "ssd_bwd_workspace_bytes")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    rc = lib.ssd_bwd(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), int(Q), _ptr(init_state), _ptr(dy),
                     _ptr(dfinal_state), _ptr(out["dx"]), _ptr(out["ddt"]), _ptr(out["dA"]), _ptr(out["dB"]),
                     _ptr(out["dC"]), _ptr(out["dD"]), _ptr(out["dinit_state"]), b, T, H, P, G, N, code,
                     _ptr(workspace), ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                     _handle(stream, dev))
    if rc != 0:
        raise SSDError(rc, "ssd_bwd")
    return out


class _SSDLayer(torch.autograd.Function):
    """ssd_fwd forward, ssd_bwd backward; no arithmetic of its own."""

    @staticmethod
    def forward(ctx, x, dt, A, B, C, D, init_state, Q):
        y, fin = ssd_fwd(x, dt, A, B, C, D, Q, init_state)
        ctx.Q = Q
        ctx.save_for_backward(x, dt, A, B, C, D, init_state)
        return y, fin

    @staticmethod
    def backward(ctx, dy, dfin):
        x, dt, A, B, C, D, init_state = ctx.saved_tensors
        dy = torch.zeros_like(x) if dy is None else dy.to(x.dtype).contiguous()
        dfin = None if dfin is None else dfin.float().contiguous()
        need_dinit = init_state is not None and ctx.needs_input_grad[6]
        g = ssd_bwd(x, dt, A, B, C, D, dy, ctx.Q, init_state, dfin, need_dinit=need_dinit)
        return g["dx"], g["ddt"], g["dA"], g["dB"], g["dC"], g["dD"], g["dinit_state"], None


def ssd_layer(x, dt, A, B, C, D, Q: int = 256, init_state=None):
    """Differentiable SSD layer: returns ``(y, final_state)`` like :func:`ssd_fwd`, with gradients for every
    tensor input through :func:`ssd_bwd` (torch autograd only records the call)."""
    return _SSDLayer.apply(x, dt, A, B, C, D, init_state, int(Q))

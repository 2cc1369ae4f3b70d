"""CPU oracle of the SSD layer forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  It shares
no code with the CUDA path (``structured_state_space_ssd_b200``) and imports
nothing from it; the CUDA path never imports it.

Three independent fp64 evaluations of the same function, each written from
the "Transformers are SSMs" pages:

* :func:`ssd_ref_fwd` -- the token-by-token recurrence (the plain definition,
  analysis page, section "The SSM as a Matrix Transformation", equation (2)
  with the scalar-identity restriction of section "The Scalar-Identity SSM").
  Implemented in C (``ssd_oracle.c``), threaded over (batch, head) pairs.
* :func:`ssd_dual_fwd` -- the quadratic (attention-like) dual: the
  materialised semiseparable matrix ``M = L o (C B^T)`` with
  ``L = 1SS(a)`` built from explicit products of the decays (section
  "The Scalar-Identity SSM", equation (16); English note, section
  "Working Through Four Tokens").  Tiny inputs only.
* :func:`ssd_chunked_fwd` -- the block decomposition, stages 0 to 5 in the
  pages' order (section "The Block-Decomposition SSD Algorithm"), returning
  its intermediates (chunk states, propagated states) for diagnosis.
* :func:`ssd_ref_step` -- one token of the recurrence (the autoregressive
  mode: the same equation advanced by a single step, as the English note's
  section "Working Through Four Tokens" does by hand), in numpy.
* :func:`ref_gate_norm` -- the Mamba-2 block's step after the layer: the
  output gated by Swish of a parallel branch z, then GroupNorm (analysis
  page, section "The Mamba-2 Architecture", paragraphs "Gating" and "Extra
  normalization"), in numpy.

Discretisation (the pages never write it): ``a_t = exp(dt_t * A_h)``, input
term ``B_t x_t^T`` without a dt factor, skip ``D_h * x_t``, initial state
``h_{-1} = init_state`` (so ``a_0`` multiplies it), head ``h`` reads group
``g = h // (H // G)``.

Array layouts (numpy, C-contiguous): x [b,T,H,P], dt [b,T,H], A [H],
B/C [b,T,G,N], D [H], init_state [b,H,P,N] or None.  Outputs y [b,T,H,P] and
final_state [b,H,P,N], fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libssd_oracle.so")
_lib = None
_DP = ctypes.POINTER(ctypes.c_double)
_LP = ctypes.POINTER(ctypes.c_long)


def _declare(lib):
    lib.ssd_ref_fwd_f64.argtypes = [_DP] * 9 + [ctypes.c_long] * 6 + [_LP, ctypes.c_long, ctypes.c_int]
    lib.ssd_ref_fwd_f64.restype = ctypes.c_int
    lib.ssd_ref_default_threads.restype = ctypes.c_int
    return lib


def build_oracle(force: bool = False) -> str:
    """Compile ``ssd_oracle.c`` into ``libssd_oracle.so`` next to it (gcc)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build_oracle()))
    return _lib


def default_threads() -> int:
    """Threads the C oracle uses by default (one per online core)."""
    return int(_load().ssd_ref_default_threads())


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor (any dtype) -> exact fp64 copy
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def ssd_ref_fwd(x, dt, A, B, C, D, init_state=None, pairs=None, nthreads: int = 0, _lib_path=None):
    """Token-by-token fp64 recurrence.

    For every (batch b, head h), with g = h // (H // G) and S = init_state[b, h]
    (or zero), for t = 0 .. T-1::

        a = exp(dt[b, t, h] * A[h])
        S = a * S + outer(x[b, t, h], B[b, t, g])          # S is [P, N]
        y[b, t, h] = S @ C[b, t, g] + D[h] * x[b, t, h]

    and final_state[b, h] = S.  ``pairs`` (a list of (b, h)) restricts the work
    to those sequences; the other slices of the outputs stay zero.
    Returns (y, final_state) as fp64 numpy arrays.  ``_lib_path`` loads another
    build of the same source instead (the tests that plant mistakes use it).
    """
    x, dt, A, B, C, D, init_state = (_f64(v) for v in (x, dt, A, B, C, D, init_state))
    batch, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt.shape == (batch, T, H) and A.shape == (H,) and D.shape == (H,)
    assert B.shape == (batch, T, G, N) and C.shape == B.shape and H % G == 0
    if init_state is not None:
        assert init_state.shape == (batch, H, P, N)
    y = np.zeros((batch, T, H, P))
    fin = np.zeros((batch, H, P, N))
    pa = None
    npairs = 0
    if pairs is not None:
        pa = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
        npairs = pa.shape[0]
        assert ((pa[:, 0] >= 0) & (pa[:, 0] < batch) & (pa[:, 1] >= 0) & (pa[:, 1] < H)).all()
    lib = _load() if _lib_path is None else _declare(ctypes.CDLL(_lib_path))
    rc = lib.ssd_ref_fwd_f64(
        _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state), _ptr(y), _ptr(fin),
        batch, T, H, P, G, N,
        None if pa is None else pa.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), npairs, int(nthreads))
    if rc != 0:
        raise ValueError(f"ssd_ref_fwd_f64 rejected its arguments (status {rc})")
    return y, fin


def segsum_mask(a):
    """1-semiseparable mask ``L = 1SS(a)`` from explicit products.

    ``L[j, i] = a[i+1] * ... * a[j]`` for ``j >= i`` (1 on the diagonal) and 0
    above it -- the mask of section "The Scalar-Identity SSM" and of the
    four-token example of the English note.
    """
    a = np.asarray(a, dtype=np.float64)
    T = a.shape[0]
    L = np.zeros((T, T))
    for j in range(T):
        L[j, j] = 1.0
        for i in range(j - 1, -1, -1):
            L[j, i] = L[j, i + 1] * a[i + 1]
    return L


def ssd_dual_fwd(x, dt, A, B, C, D, init_state=None):
    """Quadratic dual form with the materialised ``M = L o (C B^T)`` (fp64).

    Per (b, h): ``a_t = exp(dt_t A_h)``, ``L = 1SS(a)``, ``M = L * (C_g @ B_g.T)``,
    ``y = M @ x + D_h x``; an initial state adds ``prod(a_0..a_t) C_t^T h_{-1}``
    to row t.  The final state is ``sum_s L[T-1, s] x_s B_s^T`` plus the fully
    decayed initial state.  O(T^2) memory: tiny inputs only.
    Returns (y, final_state, M) where M is [b, H, T, T].
    """
    x, dt, A, B, C, D, init_state = (_f64(v) for v in (x, dt, A, B, C, D, init_state))
    batch, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.zeros((batch, T, H, P))
    fin = np.zeros((batch, H, P, N))
    Ms = np.zeros((batch, H, T, T))
    for b in range(batch):
        for h in range(H):
            g = h // (H // G)
            a = np.exp(dt[b, :, h] * A[h])
            L = segsum_mask(a)
            M = L * (C[b, :, g, :] @ B[b, :, g, :].T)
            Ms[b, h] = M
            xs = x[b, :, h, :]
            y[b, :, h, :] = M @ xs + D[h] * xs
            fin[b, h] = (L[T - 1, :, None] * xs).T @ B[b, :, g, :]
            if init_state is not None:
                decay_to = np.cumprod(a)  # a_0 * ... * a_t
                y[b, :, h, :] += decay_to[:, None] * (C[b, :, g, :] @ init_state[b, h].T)
                fin[b, h] += decay_to[-1] * init_state[b, h]
    return y, fin, Ms


def ssd_chunked_fwd(x, dt, A, B, C, D, Q: int, init_state=None):
    """Block decomposition, stages 0-5 in the pages' order (fp64).

    Stage 0: chunks ``[cQ, min((c+1)Q, T))``, ``nc = ceil(T/Q)``.
    Stage 1: ``Y_diag = (1SS(a_c) o (C_c B_c^T)) X_c``.
    Stage 2: chunk-final states from zero, ``S_c = sum_i a_{end:i} X_i B_i^T``
    (stored [P, N]).
    Stage 3: ``S~_c = a_{chunk c} S~_{c-1} + S_c`` with ``S~_{-1}`` the initial
    state; ``a_{chunk c}`` is the product of every a in chunk c.  (The pages'
    printed centre-factor indices omit ``a_{cQ}``; this takes the reading in
    which ``S~_{c-1}`` is the state at the last row of chunk c-1.)
    Stage 4: ``Y_off[j] = (a_{cQ} ... a_j) C_j^T S~_{c-1}``.
    Stage 5: ``Y = Y_diag + Y_off`` (+ the ``D_h x`` skip).
    Returns (y, final_state, S, S_prev) with S [b,nc,H,P,N] the local chunk
    states and S_prev [b,nc,H,P,N] the state entering each chunk.
    """
    x, dt, A, B, C, D, init_state = (_f64(v) for v in (x, dt, A, B, C, D, init_state))
    batch, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    nc = -(-T // Q)
    y = np.zeros((batch, T, H, P))
    fin = np.zeros((batch, H, P, N))
    S = np.zeros((batch, nc, H, P, N))
    S_prev = np.zeros((batch, nc, H, P, N))
    for b in range(batch):
        for h in range(H):
            g = h // (H // G)
            a = np.exp(dt[b, :, h] * A[h])
            state = np.zeros((P, N)) if init_state is None else init_state[b, h].copy()
            for c in range(nc):
                lo, hi = c * Q, min((c + 1) * Q, T)
                ac, Xc = a[lo:hi], x[b, lo:hi, h, :]
                Bc, Cc = B[b, lo:hi, g, :], C[b, lo:hi, g, :]
                Lc = segsum_mask(ac)
                y_diag = (Lc * (Cc @ Bc.T)) @ Xc                       # stage 1
                right = Lc[-1, :]                                        # a_{end:i}
                S[b, c, h] = (right[:, None] * Xc).T @ Bc                # stage 2
                S_prev[b, c, h] = state
                left = np.cumprod(ac)                                    # a_{cQ} ... a_j
                y_off = left[:, None] * (Cc @ state.T)                   # stage 4
                y[b, lo:hi, h, :] = y_diag + y_off + D[h] * Xc           # stage 5
                state = np.prod(ac) * state + S[b, c, h]                 # stage 3
            fin[b, h] = state
    return y, fin, S, S_prev


def ssd_ref_step(state, x, dt, A, B, C, D):
    """One autoregressive step of the recurrence in fp64 (numpy).

    Layouts: state [b,H,P,N], x [b,H,P], dt [b,H], A [H], B/C [b,G,N], D [H].
    For every (batch b, head h), with g = h // (H // G)::

        a = exp(dt[b, h] * A[h])
        S = a * state[b, h] + outer(x[b, h], B[b, g])      # S is [P, N]
        y[b, h] = S @ C[b, g] + D[h] * x[b, h]

    Returns (new_state, y); the input state is not modified.
    """
    state, x, dt, A, B, C, D = (_f64(v) for v in (state, x, dt, A, B, C, D))
    batch, H, P, N = state.shape
    G = B.shape[1]
    assert x.shape == (batch, H, P) and dt.shape == (batch, H) and A.shape == (H,) and D.shape == (H,)
    assert B.shape == (batch, G, N) and C.shape == B.shape and H % G == 0
    new = np.empty_like(state)
    y = np.empty((batch, H, P))
    for b in range(batch):
        for h in range(H):
            g = h // (H // G)
            a = np.exp(dt[b, h] * A[h])
            new[b, h] = a * state[b, h] + np.outer(x[b, h], B[b, g])
            y[b, h] = new[b, h] @ C[b, g] + D[h] * x[b, h]
    return new, y


def ref_gate_norm(y, z, ngroups, eps=1e-5, weight=None, bias=None):
    """Gate then GroupNorm in fp64 (numpy), per token.

    y, z [..., channels] (channels = H * P, the layer's output flattened per token);
    weight, bias [channels] or None (1 and 0).  With g = y * silu(z) = y * z / (1 + exp(-z)),
    the channels of each token split into ``ngroups`` contiguous groups, and per group::

        out = (g - mean(g)) / sqrt(var(g) + eps) * weight + bias       (var: population variance)
    """
    y, z = _f64(y), _f64(z)
    shape = y.shape
    ch = shape[-1]
    assert z.shape == shape and ch % ngroups == 0
    g = y * z / (1.0 + np.exp(-z))
    gg = g.reshape(-1, ngroups, ch // ngroups)
    mean = gg.mean(axis=2, keepdims=True)
    var = ((gg - mean) ** 2).mean(axis=2, keepdims=True)
    out = ((gg - mean) / np.sqrt(var + eps)).reshape(shape)
    if weight is not None:
        out = out * _f64(weight)
    if bias is not None:
        out = out + _f64(bias)
    return out

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
* :func:`ssd_ref_bwd` -- the gradients of the layer (x, dt, A, B, C, D and
  the initial state) for given output gradients: the adjoint of the
  recurrence stepped in reverse, in numpy.  The pages print no backward; the
  gradient is unique, and its pins are central finite differences of
  :func:`ssd_ref_fwd`, the adjoint identity of the linear map and closed
  forms (``tests/test_oracle_bwd.py``).
* :func:`ssd_ref_bwd_at` -- the same gradients at a few tokens from explicit
  sums (no state history), for checks at full problem sizes.
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


def _bwd_args(x, dt, A, B, C, D, dy, init_state, dfinal_state):
    x, dt, A, B, C, D, dy, init_state, dfinal_state = (
        _f64(v) for v in (x, dt, A, B, C, D, dy, init_state, dfinal_state))
    batch, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt.shape == (batch, T, H) and A.shape == (H,) and D.shape == (H,) and dy.shape == x.shape
    assert B.shape == (batch, T, G, N) and C.shape == B.shape and H % G == 0
    for st in (init_state, dfinal_state):
        assert st is None or st.shape == (batch, H, P, N)
    return x, dt, A, B, C, D, dy, init_state, dfinal_state


def ssd_ref_bwd(x, dt, A, B, C, D, dy, init_state=None, dfinal_state=None):
    """Reverse-mode gradient of the token-by-token recurrence (fp64, numpy).

    The pages give the forward only (analysis page, section "The SSM as a
    Matrix Transformation", equation (2), scalar-identity case); they motivate
    training speed but print no backward algorithm.  The gradient of a
    function is unique, so this oracle is the adjoint of that recurrence,
    taken step by step in reverse order.  With the loss
    ``L = sum(dy * y) + sum(dfinal_state * final_state)`` and, per (b, h), the
    states ``h_t = a_t h_{t-1} + x_t B_t^T`` (``a_t = exp(dt_t A_h)``,
    ``h_{-1}`` the initial state), the adjoint ``g_t = dL/dh_t`` obeys::

        g_{T-1} = dfinal + dy_{T-1} C_{T-1}^T
        g_t     = a_{t+1} g_{t+1} + dy_t C_t^T

    and every input gradient is local to its token::

        dx_t      = g_t B_t + D_h dy_t
        dB_t      = sum over the group's heads of g_t^T x_t
        dC_t      = sum over the group's heads of h_t^T dy_t
        dlog a_t  = <g_t, a_t h_{t-1}>            (a_t = exp(dt_t A_h))
        ddt_t     = A_h dlog a_t,   dA_h = sum_{b,t} dt_t dlog a_t
        dD_h      = sum_{b,t} <dy_t, x_t>,   dinit = a_0 g_0

    Every state of a batch row is kept ([T, H, P, N] fp64): small problems
    only.  Returns a dict with dx [b,T,H,P], ddt [b,T,H], dA [H], dB, dC
    [b,T,G,N], dD [H] and dinit_state [b,H,P,N], all fp64.
    """
    x, dt, A, B, C, D, dy, init_state, dfinal_state = _bwd_args(x, dt, A, B, C, D, dy, init_state, dfinal_state)
    batch, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    hpg = H // G
    grp = np.arange(H) // hpg
    out = {"dx": np.zeros_like(x), "ddt": np.zeros_like(dt), "dA": np.zeros(H), "dB": np.zeros_like(B),
           "dC": np.zeros_like(C), "dD": np.zeros(H), "dinit_state": np.zeros((batch, H, P, N))}
    for b in range(batch):
        Bh, Ch = B[b][:, grp, :], C[b][:, grp, :]          # [T, H, N]: each head's group row
        a = np.exp(dt[b] * A[None, :])                      # [T, H]
        h0 = np.zeros((H, P, N)) if init_state is None else init_state[b]
        states = np.empty((T, H, P, N))
        S = h0
        for t in range(T):
            S = a[t][:, None, None] * S + x[b, t][:, :, None] * Bh[t][:, None, :]
            states[t] = S
        g = np.zeros((H, P, N)) if dfinal_state is None else dfinal_state[b].copy()
        for t in range(T - 1, -1, -1):
            g = g + dy[b, t][:, :, None] * Ch[t][:, None, :]          # g_t
            out["dx"][b, t] = np.einsum("hpn,hn->hp", g, Bh[t]) + D[:, None] * dy[b, t]
            out["dB"][b, t] = np.einsum("hpn,hp->hn", g, x[b, t]).reshape(G, hpg, N).sum(axis=1)
            out["dC"][b, t] = np.einsum("hpn,hp->hn", states[t], dy[b, t]).reshape(G, hpg, N).sum(axis=1)
            prev = states[t - 1] if t > 0 else h0
            dlog = a[t] * np.einsum("hpn,hpn->h", g, prev)
            out["ddt"][b, t] = A * dlog
            out["dA"] += dt[b, t] * dlog
            out["dD"] += np.einsum("hp,hp->h", dy[b, t], x[b, t])
            g = a[t][:, None, None] * g                                 # carried to t-1
        out["dinit_state"][b] = g
    return out


def ssd_ref_bwd_at(x, dt, A, B, C, D, dy, b, tokens, init_state=None, dfinal_state=None):
    """The same gradients at chosen tokens of batch row ``b``, from explicit sums (fp64).

    Instead of stepping the recurrence, each needed state is written out as
    the sum it stands for (the unrolled form of equation (2), section "The SSM
    as a Matrix Transformation"), with the decay products
    ``a_{u+1} ... a_t = exp(sigma_t - sigma_u)`` from the running sum
    ``sigma_t = sum_{v<=t} dt_v A_h`` (the log-space products of section "The
    Scalar-Identity SSM")::

        h_t = sum_{u<=t} exp(sigma_t - sigma_u) x_u B_u^T + exp(sigma_t) h_{-1}
        g_t = sum_{k>=t} exp(sigma_k - sigma_t) dy_k C_k^T + exp(sigma_{T-1} - sigma_t) dfinal

    and the per-token gradients follow as in :func:`ssd_ref_bwd`.  Costs
    O(T P N) per head and token, with no state history: usable at full
    problem sizes on a few tokens.  Returns a dict with dx [k,H,P], ddt [k,H],
    dB, dC [k,G,N] for the k listed tokens.
    """
    x, dt, A, B, C, D, dy, init_state, dfinal_state = _bwd_args(x, dt, A, B, C, D, dy, init_state, dfinal_state)
    _, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    hpg = H // G
    tokens = [int(t) for t in tokens]
    k = len(tokens)
    out = {"dx": np.zeros((k, H, P)), "ddt": np.zeros((k, H)), "dB": np.zeros((k, G, N)), "dC": np.zeros((k, G, N))}
    for h in range(H):
        gi = h // hpg
        sig = np.cumsum(dt[b, :, h] * A[h])                 # sigma_t
        xs, dys = x[b, :, h, :], dy[b, :, h, :]
        Bs, Cs = B[b, :, gi, :], C[b, :, gi, :]
        for i, t in enumerate(tokens):
            def state_at(u):
                if u < 0:
                    return np.zeros((P, N)) if init_state is None else init_state[b, h]
                w = np.exp(sig[u] - sig[:u + 1])
                st = (xs[:u + 1] * w[:, None]).T @ Bs[:u + 1]
                if init_state is not None:
                    st = st + np.exp(sig[u]) * init_state[b, h]
                return st
            w = np.exp(sig[t:] - sig[t])
            g = (dys[t:] * w[:, None]).T @ Cs[t:]
            if dfinal_state is not None:
                g = g + np.exp(sig[T - 1] - sig[t]) * dfinal_state[b, h]
            ht = state_at(t)
            a_t = np.exp(dt[b, t, h] * A[h])
            out["dx"][i, h] = g @ Bs[t] + D[h] * dys[t]
            out["dB"][i, gi] += xs[t] @ g
            out["dC"][i, gi] += dys[t] @ ht
            out["ddt"][i, h] = A[h] * a_t * np.sum(g * state_at(t - 1))
    return out

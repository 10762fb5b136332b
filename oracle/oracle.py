"""KDA CPU oracle -- TEST INFRASTRUCTURE ONLY.

Python entry points for the fp64 token-by-token oracle in ``kda_oracle.c``.
Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It never imports the CUDA package and the
CUDA package never imports it.

What it computes ("Kimi K3: Architecture, Training, and Million-Token Agentic
RL", sections 3.1-3.3): per head, the state edit
``Sbar = Diag(alpha) S; vhat = Sbar^T k; S = Sbar + beta k (v - vhat)^T;
o = S^T q`` with the gate ``g = -5 * sigmoid(exp(A) * z)``, ``alpha = exp(g)``
-- or, as the earlier unbounded gate the pages contrast it with, the negative
Softplus ``g = -softplus(exp(A) * z)``.

Every input is converted to float64 before the call, so the oracle consumes the
exact values the GPU receives (bf16 or fp32 tensors upcast without rounding).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libkda_oracle.so")
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` with gcc (-O2 -fopenmp) into ``oracle/_build``."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        # -ffp-contract=off keeps every multiply and add a separate IEEE
        # operation, so the arithmetic is exactly what the source spells out.
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
               _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        d, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        lib.kda_oracle_prefill.argtypes = [d, d, d, d, d, d, d, i32, i32, i32, i32,
                                           d, d, d, i32]
        lib.kda_oracle_prefill.restype = i32
        lib.kda_oracle_prefill_ckpt.argtypes = [d, d, d, d, d, d, d, i32, i32, i32, i32,
                                                d, d, d, i32, d, i32]
        lib.kda_oracle_prefill_ckpt.restype = i32
        lib.kda_oracle_decode.argtypes = [d, d, d, d, d, d, i32, i32, i32, i32, d,
                                          d, d, i32]
        lib.kda_oracle_decode.restype = i32
        lib.kda_oracle_gate.argtypes = [d, d, i64, i32, i32, d]
        lib.kda_oracle_gate.restype = None
        lib.kda_oracle_gate_kind.argtypes = [d, d, i64, i32, i32, d, i32]
        lib.kda_oracle_gate_kind.restype = None
        lib.kda_oracle_prefill_gate.argtypes = [d, d, d, d, d, d, d, i32, i32, i32, i32,
                                                d, d, d, i32, d, i32, i32]
        lib.kda_oracle_prefill_gate.restype = i32
        lib.kda_oracle_decode_gate.argtypes = [d, d, d, d, d, d, i32, i32, i32, i32, d,
                                               d, d, i32, i32]
        lib.kda_oracle_decode_gate.restype = i32
        lib.kda_oracle_max_threads.argtypes = []
        lib.kda_oracle_max_threads.restype = i32
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact upcast of a numpy array or torch tensor (any float dtype) to float64."""
    if hasattr(x, "detach"):  # torch tensor: upcast on the torch side (bf16 has no numpy dtype)
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    """Number of OpenMP threads the oracle uses by default."""
    return int(_load().kda_oracle_max_threads())


# Gate kinds: the K3 lower-bounded gate (section 3.3 of the note) and the
# unbounded negative Softplus of the earlier Kimi Linear design.
GATES = {"bounded": 0, "softplus": 1}


def gate(z, A, kind: str = "bounded") -> np.ndarray:
    """g[t,h,c] = -5 * sigmoid(exp(A[h,c]) * z[t,h,c]) for z [T,H,dk], A [H,dk];
    with kind="softplus", g = -softplus(exp(A[h,c]) * z[t,h,c])."""
    z, A = _f64(z), _f64(A)
    T, H, dk = z.shape
    g = np.empty_like(z)
    _load().kda_oracle_gate_kind(_ptr(z), _ptr(A), T, H, dk, _ptr(g), GATES[kind])
    return g


def prefill(q, k, v, z, A, beta, cu_seqlens, initial_state=None, nthreads: int = 0,
            gate: str = "bounded"):
    """Token-by-token fp64 recurrence over packed sequences.

    Shapes: q, k, z [T,H,dk]; v [T,H,dv]; beta [T,H]; A [H,dk];
    cu_seqlens [N+1]; initial_state [N,H,dk,dv] or None (zeros).
    ``gate`` selects the gate kind (see ``gate``).
    Returns ``(o [T,H,dv], final_state [N,H,dk,dv])`` as float64 arrays.
    """
    q, k, v, z, A, beta = (_f64(t) for t in (q, k, v, z, A, beta))
    cu = _i32(cu_seqlens)
    T, H, dk = q.shape
    dv = v.shape[2]
    n = cu.shape[0] - 1
    s0 = None if initial_state is None else _f64(initial_state)
    o = np.zeros((T, H, dv), dtype=np.float64)
    sf = np.zeros((n, H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_prefill_gate(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A),
                                         _ptr(beta), _ptr(cu), n, H, dk, dv, _ptr(s0),
                                         _ptr(o), _ptr(sf), 0, None, nthreads, GATES[gate])
    if rc != 0:
        raise MemoryError("kda oracle: allocation failed")
    return o, sf


def checkpoint_count(cu_seqlens, every: int) -> int:
    """sum over sequences of L_n // every (0 when every <= 0)."""
    cu = _i32(cu_seqlens)
    if every <= 0:
        return 0
    return int(sum((int(cu[i + 1]) - int(cu[i])) // every for i in range(len(cu) - 1)))


def prefill_checkpoints(q, k, v, z, A, beta, cu_seqlens, every: int, initial_state=None,
                        nthreads: int = 0):
    """As ``prefill``, plus the state after every ``every`` tokens of each sequence.

    Returns ``(o, final_state, checkpoints [count, H, dk, dv])``; checkpoint j of
    sequence n (j = 1 .. L_n // every) is at row sum_{m<n} L_m // every + j - 1.
    """
    q, k, v, z, A, beta = (_f64(t) for t in (q, k, v, z, A, beta))
    cu = _i32(cu_seqlens)
    T, H, dk = q.shape
    dv = v.shape[2]
    n = cu.shape[0] - 1
    s0 = None if initial_state is None else _f64(initial_state)
    o = np.zeros((T, H, dv), dtype=np.float64)
    sf = np.zeros((n, H, dk, dv), dtype=np.float64)
    ck = np.zeros((checkpoint_count(cu, every), H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_prefill_ckpt(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A),
                                         _ptr(beta), _ptr(cu), n, H, dk, dv, _ptr(s0),
                                         _ptr(o), _ptr(sf), int(every),
                                         _ptr(ck) if ck.size else None, nthreads)
    if rc != 0:
        raise MemoryError("kda oracle: allocation failed")
    return o, sf, ck


def decode_step(q, k, v, z, A, beta, state, slots=None, nthreads: int = 0,
                gate: str = "bounded"):
    """One single-token step per batch row; returns ``(o [B,H,dv], new_state)``.

    ``state`` is the pool [P,H,dk,dv]; it is copied, never modified in place.
    ``slots`` [B] selects the pool row of each batch entry (None = identity).
    """
    q, k, v, z, A, beta = (_f64(t) for t in (q, k, v, z, A, beta))
    st = _f64(state).copy()
    B, H, dk = q.shape
    dv = v.shape[2]
    sl = None if slots is None else _i32(slots)
    o = np.zeros((B, H, dv), dtype=np.float64)
    rc = _load().kda_oracle_decode_gate(_ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(A),
                                        _ptr(beta), B, H, dk, dv, _ptr(st), _ptr(sl),
                                        _ptr(o), nthreads, GATES[gate])
    if rc != 0:
        raise MemoryError("kda oracle: allocation failed")
    return o, st

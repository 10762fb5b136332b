"""Thin ctypes binding of libkda_b200.so (argument marshalling only).

Every function here checks tensor placement and dtype, passes raw device
pointers and sizes to the C ABI declared in ``include/kda.h``, and raises
``KdaError`` on a non-zero status.  All arithmetic runs in the CUDA library;
there is no fallback: if the library is missing the import of this module
fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libkda_b200.so")

KDA_DTYPE = {torch.bfloat16: 0, torch.float32: 1}
KDA_ALGO = {"auto": 0, "cuda_core": 1, "tensor_core": 2, "tensor_core_split": 3}
KDA_GATE = {"bounded": 0, "softplus": 1}
STATUS_NAMES = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
                3: "KDA_ERR_WORKSPACE", 4: "KDA_ERR_CUDA", 5: "KDA_ERR_TIMEOUT"}

# Every exported symbol of include/kda.h, with its ctypes signature.
_P, _I32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
SIGNATURES = {
    "kda_abi_version": ([], _I32),
    "kda_status_string": ([_I32], ctypes.c_char_p),
    "kda_prefill_workspace_size": ([_I32, _I32, _I32, _I32, _I32, _I32, _I32], _SZ),
    "kda_prefill_gated_workspace_size": ([_I32] * 8, _SZ),
    "kda_prefill": ([_P] * 8 + [_I32] * 6 + [_P] * 4 + [_SZ, _P], _I32),
    "kda_prefill_ex": ([_P] * 8 + [_I32] * 6 + [_P] * 4 + [_SZ, _I32, _P, _P, _I32], _I32),
    "kda_prefill_kernel_count": ([_I32] * 7, _I32),
    "kda_prefill_segments": ([_I32] * 7, _I32),
    "kda_prefill_checkpointed": ([_P] * 8 + [_I32] * 6 + [_P] * 4 + [_SZ, _I32, _P, _P, _I32, _I32, _P],
                                 _I32),
    "kda_checkpoint_count": ([_P, _I32, _I32], ctypes.c_int64),
    "kda_prefill_noalloc": ([_P] * 8 + [_I32] * 6 + [_P] * 4, _I32),
    "kda_decode_step": ([_P] * 6 + [_I32] * 5 + [_P, _I32, _P, _P, _P], _I32),
    "kda_decode_step_gated": ([_P] * 6 + [_I32] * 5 + [_P, _I32, _P, _P, _I32, _P], _I32),
    "kda_prefill_gated": ([_P] * 8 + [_I32] * 6 + [_P] * 4 + [_SZ, _I32, _I32, _P], _I32),
    "kda_prefill_debug": ([_P] * 8 + [_I32] * 6 + [_P] * 4 + [_SZ] + [_P] * 5, _I32),
    "kda_decode_check_slots": ([_P, _I32, _I32], _I32),
    "kda_device_status": ([_P, _P], _I32),
    "kda_decode_multi": ([_P] * 6 + [_I32] * 6 + [_P, _I32, _P, _P, _I32, _P, _P], _I32),
    "kda_selftest_wait_timeout": ([ctypes.c_int64, _P], _I32),
}


class KdaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} "
                         f"({_lib.kda_status_string(code).decode()})")
        self.code = code


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"KDA CUDA library not built: {_LIB_PATH} is missing "
                          "(run python -m linear_attention_serving_prefill_b200.build)")
    lib = ctypes.CDLL(_LIB_PATH)
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes, fn.restype = args, res
    return lib


_lib = _load()


def library_path() -> str:
    return _LIB_PATH


def kda_status_string(code: int) -> str:
    return _lib.kda_status_string(code).decode()


def _check(code: int, where: str):
    if code != 0:
        raise KdaError(code, where)


def _dev(t: Optional[torch.Tensor], name: str, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def kda_prefill_workspace_size(total_tokens: int, num_seqs: int, H: int, dk: int, dv: int,
                               dtype=torch.bfloat16, algo: str = "auto") -> int:
    return int(_lib.kda_prefill_workspace_size(total_tokens, num_seqs, H, dk, dv,
                                               KDA_DTYPE[dtype], KDA_ALGO[algo]))


def kda_prefill_gated_workspace_size(total_tokens: int, num_seqs: int, H: int, dk: int, dv: int,
                                     dtype=torch.bfloat16, algo: str = "auto",
                                     gate: str = "bounded") -> int:
    return int(_lib.kda_prefill_gated_workspace_size(total_tokens, num_seqs, H, dk, dv,
                                                     KDA_DTYPE[dtype], KDA_ALGO[algo],
                                                     KDA_GATE[gate]))


def kda_prefill(q, k, v, z, A, beta, cu_seqlens, cu_seqlens_host=None, initial_state=None,
                output_final_state: bool = True, final_state=None, o=None, workspace=None,
                algo: str = "auto", stream=None, stage_events=None, gate: str = "bounded"):
    """Chunked KDA prefill over packed sequences; returns ``(o, final_state)``.

    q, k, z [T,H,dk], v [T,H,dv] (bf16 or fp32, one dtype); A [H,dk] fp32;
    beta [T,H] fp32; cu_seqlens [N+1] int32 on the device; cu_seqlens_host an
    optional CPU copy; initial_state [N,H,dk,dv] fp32 or None.  ``final_state``
    may be passed (e.g. ``initial_state`` itself, for in-place resume);
    otherwise it is allocated when ``output_final_state``.  ``stage_events``
    (a list of recorded ``torch.cuda.Event``) receives the kernel boundaries.
    ``gate="softplus"`` selects the unbounded gate (kda_prefill_gated; no events).
    """
    T, H, dk = q.shape
    dv = v.shape[2]
    N = cu_seqlens.shape[0] - 1
    dt = q.dtype
    if dt not in KDA_DTYPE:
        raise ValueError(f"unsupported dtype {dt}")
    if o is None:
        o = torch.empty(T, H, dv, dtype=dt, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
    need = kda_prefill_gated_workspace_size(T, N, H, dk, dv, dt, algo, gate)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    host = None
    if cu_seqlens_host is not None:
        ch = cu_seqlens_host.to(torch.int32).contiguous()
        host = ctypes.c_void_p(ch.data_ptr())
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if gate != "bounded":
        if stage_events:
            raise ValueError("stage events are recorded for the lower-bounded gate only")
        code = _lib.kda_prefill_gated(
            _dev(q, "q", dt), _dev(k, "k", dt), _dev(v, "v", dt), _dev(z, "z", dt),
            _dev(A, "A", torch.float32), _dev(beta, "beta", torch.float32),
            _dev(cu_seqlens, "cu_seqlens", torch.int32), host, N, T, H, dk, dv, KDA_DTYPE[dt],
            _dev(initial_state, "initial_state", torch.float32),
            _dev(final_state, "final_state", torch.float32), _dev(o, "o", dt),
            _dev(workspace, "workspace"), ws_bytes, KDA_ALGO[algo], KDA_GATE[gate],
            _stream_ptr(stream))
        _check(code, "kda_prefill_gated")
        return o, final_state
    ev_arr, n_ev = None, 0
    if stage_events:
        ev_arr = (ctypes.c_void_p * len(stage_events))(*[e.cuda_event for e in stage_events])
        n_ev = len(stage_events)
    code = _lib.kda_prefill_ex(
        _dev(q, "q", dt), _dev(k, "k", dt), _dev(v, "v", dt), _dev(z, "z", dt),
        _dev(A, "A", torch.float32), _dev(beta, "beta", torch.float32),
        _dev(cu_seqlens, "cu_seqlens", torch.int32), host, N, T, H, dk, dv, KDA_DTYPE[dt],
        _dev(initial_state, "initial_state", torch.float32),
        _dev(final_state, "final_state", torch.float32), _dev(o, "o", dt),
        _dev(workspace, "workspace"), ws_bytes, KDA_ALGO[algo], _stream_ptr(stream), ev_arr, n_ev)
    _check(code, "kda_prefill")
    return o, final_state


def kda_checkpoint_count(cu_seqlens_host, checkpoint_every: int) -> int:
    """Rows of the checkpoint tensor: sum over sequences of L_n // checkpoint_every."""
    ch = cu_seqlens_host.to(torch.int32).contiguous()
    n = _lib.kda_checkpoint_count(ctypes.c_void_p(ch.data_ptr()), ch.numel() - 1, checkpoint_every)
    if n < 0:
        raise KdaError(1, "kda_checkpoint_count")
    return int(n)


def kda_prefill_checkpointed(q, k, v, z, A, beta, cu_seqlens, cu_seqlens_host, checkpoint_every,
                             initial_state=None, final_state=None, o=None, checkpoints=None,
                             workspace=None, algo: str = "auto", stream=None):
    """kda_prefill plus the state after every ``checkpoint_every`` tokens of each
    sequence; returns ``(o, final_state, checkpoints [count, H, dk, dv])``."""
    T, H, dk = q.shape
    dv = v.shape[2]
    N = cu_seqlens.shape[0] - 1
    dt = q.dtype
    if o is None:
        o = torch.empty(T, H, dv, dtype=dt, device=q.device)
    if final_state is None:
        final_state = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
    count = kda_checkpoint_count(cu_seqlens_host, checkpoint_every)
    if checkpoints is None:
        checkpoints = torch.empty(max(count, 1), H, dk, dv, dtype=torch.float32, device=q.device)
    need = kda_prefill_workspace_size(T, N, H, dk, dv, dt, algo)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ch = cu_seqlens_host.to(torch.int32).contiguous()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    code = _lib.kda_prefill_checkpointed(
        _dev(q, "q", dt), _dev(k, "k", dt), _dev(v, "v", dt), _dev(z, "z", dt),
        _dev(A, "A", torch.float32), _dev(beta, "beta", torch.float32),
        _dev(cu_seqlens, "cu_seqlens", torch.int32), ctypes.c_void_p(ch.data_ptr()), N, T, H, dk,
        dv, KDA_DTYPE[dt], _dev(initial_state, "initial_state", torch.float32),
        _dev(final_state, "final_state", torch.float32), _dev(o, "o", dt),
        _dev(workspace, "workspace"), ws_bytes, KDA_ALGO[algo], _stream_ptr(stream), None, 0,
        int(checkpoint_every), _dev(checkpoints, "checkpoints", torch.float32))
    _check(code, "kda_prefill_checkpointed")
    return o, final_state, checkpoints[:count]


def kda_prefill_noalloc(q, k, v, z, A, beta, cu_seqlens, cu_seqlens_host=None,
                        initial_state=None, output_final_state: bool = True, final_state=None,
                        o=None, stream=None):
    """kda_prefill with the library's fixed scratch array instead of a workspace.

    For callers that must not allocate device memory during the call: pass
    preallocated ``o`` (and ``final_state``) to keep this function from
    allocating them.  Returns ``(o, final_state)``.
    """
    T, H, dk = q.shape
    dv = v.shape[2]
    N = cu_seqlens.shape[0] - 1
    dt = q.dtype
    if dt not in KDA_DTYPE:
        raise ValueError(f"unsupported dtype {dt}")
    if o is None:
        o = torch.empty(T, H, dv, dtype=dt, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty(N, H, dk, dv, dtype=torch.float32, device=q.device)
    host = None
    if cu_seqlens_host is not None:
        ch = cu_seqlens_host.to(torch.int32).contiguous()
        host = ctypes.c_void_p(ch.data_ptr())
    code = _lib.kda_prefill_noalloc(
        _dev(q, "q", dt), _dev(k, "k", dt), _dev(v, "v", dt), _dev(z, "z", dt),
        _dev(A, "A", torch.float32), _dev(beta, "beta", torch.float32),
        _dev(cu_seqlens, "cu_seqlens", torch.int32), host, N, T, H, dk, dv, KDA_DTYPE[dt],
        _dev(initial_state, "initial_state", torch.float32),
        _dev(final_state, "final_state", torch.float32), _dev(o, "o", dt), _stream_ptr(stream))
    _check(code, "kda_prefill_noalloc")
    return o, final_state


def kda_prefill_kernel_count(T: int, N: int, H: int, dk: int, dv: int, dtype=torch.bfloat16,
                             algo: str = "auto") -> int:
    return int(_lib.kda_prefill_kernel_count(T, N, H, dk, dv, KDA_DTYPE[dtype], KDA_ALGO[algo]))


def kda_prefill_segments(T: int, N: int, H: int, dk: int, dv: int, dtype=torch.bfloat16,
                         algo: str = "auto") -> int:
    """Segments per sequence the call uses (1 = no split, 0 = invalid arguments)."""
    return int(_lib.kda_prefill_segments(T, N, H, dk, dv, KDA_DTYPE[dtype], KDA_ALGO[algo]))


def kda_decode_step(q, k, v, z, A, beta, state, slots=None, o=None, stream=None,
                    gate: str = "bounded"):
    """One decode step; ``state`` [P,H,dk,dv] fp32 is updated in place; returns o."""
    B, H, dk = q.shape
    dv = v.shape[2]
    dt = q.dtype
    if o is None:
        o = torch.empty(B, H, dv, dtype=dt, device=q.device)
    code = _lib.kda_decode_step_gated(
        _dev(q, "q", dt), _dev(k, "k", dt), _dev(v, "v", dt), _dev(z, "z", dt),
        _dev(A, "A", torch.float32), _dev(beta, "beta", torch.float32), B, H, dk, dv,
        KDA_DTYPE[dt], _dev(state, "state", torch.float32), state.shape[0],
        _dev(slots, "slots", torch.int32), _dev(o, "o", dt), KDA_GATE[gate], _stream_ptr(stream))
    _check(code, "kda_decode_step")
    return o


def kda_decode_multi(q, k, v, z, A, beta, state, slots=None, num_tokens=None,
                     update_state: bool = False, o=None, want_outputs: bool = True, stream=None):
    """Speculative-decoding verify (update_state=False: outputs for every draft
    token, state untouched) or replay (update_state=True: advance each sequence's
    state by its first num_tokens[b] tokens in place).

    q, k, z [B,Tq,H,dk], v [B,Tq,H,dv]; beta [B,Tq,H] fp32; state [P,H,dk,dv] fp32.
    Returns o [B,Tq,H,dv] (or None when want_outputs is False in replay mode).
    """
    B, Tq, H, dk = q.shape
    dv = v.shape[3]
    dt = q.dtype
    if o is None and (want_outputs or not update_state):
        o = torch.empty(B, Tq, H, dv, dtype=dt, device=q.device)
    code = _lib.kda_decode_multi(
        _dev(q, "q", dt), _dev(k, "k", dt), _dev(v, "v", dt), _dev(z, "z", dt),
        _dev(A, "A", torch.float32), _dev(beta, "beta", torch.float32), B, Tq, H, dk, dv,
        KDA_DTYPE[dt], _dev(state, "state", torch.float32), state.shape[0],
        _dev(slots, "slots", torch.int32), _dev(num_tokens, "num_tokens", torch.int32),
        1 if update_state else 0, _dev(o, "o", dt), _stream_ptr(stream))
    _check(code, "kda_decode_multi")
    return o


def kda_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Enqueue the bounded-wait self-test; read the result with kda_device_status()."""
    _check(_lib.kda_selftest_wait_timeout(int(limit_ns), _stream_ptr(stream)),
           "kda_selftest_wait_timeout")


def kda_device_status(stream=None) -> int:
    out = ctypes.c_int32(0)
    _check(_lib.kda_device_status(_stream_ptr(stream), ctypes.byref(out)), "kda_device_status")
    return int(out.value)


def kda_prefill_debug(q, k, v, z, A, beta, cu_seqlens, cu_seqlens_host, initial_state=None,
                      stream=None):
    """Tensor-core prefill plus its stage intermediates; returns a dict with o,
    final_state and G, W, U, delta (fp32 [T, H, 128], see include/kda.h)."""
    T, H, dk = q.shape
    dv = v.shape[2]
    N = cu_seqlens.shape[0] - 1
    dt = q.dtype
    dev = q.device
    out = {"o": torch.empty(T, H, dv, dtype=dt, device=dev),
           "final_state": torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)}
    for name, d in (("G", dk), ("W", dk), ("U", dv), ("delta", dv)):
        out[name] = torch.full((T, H, d), float("nan"), dtype=torch.float32, device=dev)
    need = kda_prefill_workspace_size(T, N, H, dk, dv, dt, "tensor_core")
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    ch = cu_seqlens_host.to(torch.int32).contiguous()
    code = _lib.kda_prefill_debug(
        _dev(q, "q", dt), _dev(k, "k", dt), _dev(v, "v", dt), _dev(z, "z", dt),
        _dev(A, "A", torch.float32), _dev(beta, "beta", torch.float32),
        _dev(cu_seqlens, "cu_seqlens", torch.int32), ctypes.c_void_p(ch.data_ptr()), N, T, H, dk,
        dv, KDA_DTYPE[dt], _dev(initial_state, "initial_state", torch.float32),
        _dev(out["final_state"], "final_state", torch.float32), _dev(out["o"], "o", dt),
        _dev(ws, "workspace"), need, _dev(out["G"], "G"), _dev(out["W"], "W"), _dev(out["U"], "U"),
        _dev(out["delta"], "delta"), _stream_ptr(stream))
    _check(code, "kda_prefill_debug")
    return out


def kda_decode_check_slots(slots_host, pool_size: int) -> bool:
    """True when the host slots are in range and distinct (kda_decode_check_slots)."""
    sl = torch.as_tensor(slots_host, dtype=torch.int32).contiguous()
    return _lib.kda_decode_check_slots(ctypes.c_void_p(sl.data_ptr()), sl.numel(), pool_size) == 0

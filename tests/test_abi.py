"""C-ABI checks that need no GPU: symbols, status strings, host-side validation.

Every call here either fails validation on the host (so nothing is launched and
no pointer is dereferenced) or, for a valid call, runs only where no GPU exists
(it must then return KDA_ERR_CUDA rather than crash).
"""
import ctypes
import os
import re

import pytest
import torch

from linear_attention_serving_prefill_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA = 0, 1, 2, 3, 4
BF16, F32 = 0, 1
AUTO, CORE, TC, SPLIT = 0, 1, 2, 3


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert names, "no declarations parsed"
    lib = ctypes.CDLL(B.library_path())
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/kda.h but not exported"
    assert set(names) == set(B.SIGNATURES), "binding signatures out of sync with the header"


def test_abi_version_and_status_strings():
    assert B._lib.kda_abi_version() == 3
    for code in range(6):
        s = B.kda_status_string(code)
        assert s.startswith(B.STATUS_NAMES[code])
    assert B.kda_status_string(99) == "KDA_ERR_UNKNOWN"


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def _prefill(**kw):
    a = dict(q=_fake(), k=_fake(), v=_fake(), z=_fake(), A=_fake(), beta=_fake(),
             cu=_fake(), cu_host=None, N=2, T=10, H=4, dk=128, dv=128, dt=BF16, s0=None,
             sf=None, o=_fake(), ws=None, ws_bytes=0, algo=AUTO, stream=None)
    a.update(kw)
    return B._lib.kda_prefill_ex(a["q"], a["k"], a["v"], a["z"], a["A"], a["beta"], a["cu"],
                                 a["cu_host"], a["N"], a["T"], a["H"], a["dk"], a["dv"], a["dt"],
                                 a["s0"], a["sf"], a["o"], a["ws"], a["ws_bytes"], a["algo"],
                                 a["stream"], None, 0)


def _host_cu(vals):
    arr = (ctypes.c_int32 * len(vals))(*vals)
    return ctypes.cast(arr, ctypes.c_void_p), arr


def test_prefill_rejects_bad_sizes():
    assert _prefill(dk=96) == UNSUPPORTED
    assert _prefill(dv=48) == UNSUPPORTED
    assert _prefill(dk=0) == INVALID
    assert _prefill(H=0) == INVALID
    assert _prefill(N=-1) == INVALID
    assert _prefill(T=-5) == INVALID
    assert _prefill(dt=7) == INVALID
    assert _prefill(algo=9) == INVALID
    assert _prefill(algo=TC, dt=F32) == UNSUPPORTED
    assert _prefill(algo=TC, dk=64, dv=64) == UNSUPPORTED


def test_kernel_count():
    kc = B._lib.kda_prefill_kernel_count
    assert kc(32768, 1, 96, 128, 128, BF16, AUTO) == 3
    assert kc(4096, 1, 32, 128, 128, BF16, AUTO) == 5      # split: + compose + correct
    assert kc(4096, 1, 32, 128, 128, BF16, TC) == 3
    assert kc(4096, 1, 32, 128, 128, BF16, CORE) == 1
    assert kc(4096, 1, 32, 64, 64, BF16, AUTO) == 1
    assert kc(4096, 1, 32, 128, 128, F32, AUTO) == 1
    assert kc(4096, 1, 32, 96, 128, BF16, AUTO) == 0
    assert kc(4096, 1, 32, 128, 128, F32, SPLIT) == 0


def test_split_segment_count():
    """The split plan: N H (2 G - 1) <= 148 concurrent state chains, G <= 16;
    AUTO also keeps >= 16 chunks per segment; SPLIT forces G >= 2; other
    paths never split."""
    seg = B._lib.kda_prefill_segments
    assert seg(32768, 1, 96, 128, 128, BF16, AUTO) == 1     # 96 chains already fill the GPU
    assert seg(4096, 1, 32, 128, 128, BF16, AUTO) == 2      # 3 x 32 = 96 <= 148
    assert seg(1 << 20, 1, 16, 128, 128, BF16, AUTO) == 5   # 9 x 16 = 144 <= 148
    assert seg(1 << 20, 1, 1, 128, 128, BF16, AUTO) == 16   # capped
    assert seg(2048, 1, 1, 128, 128, BF16, AUTO) == 2       # 32 chunks: 2 segments of 16
    assert seg(1024, 1, 32, 128, 128, BF16, AUTO) == 1      # too short to pay
    assert seg(1024, 1, 32, 128, 128, BF16, SPLIT) == 2
    assert seg(32768, 16, 96, 128, 128, BF16, SPLIT) == 2   # forced even when the GPU is full
    assert seg(4096, 1, 32, 128, 128, BF16, TC) == 1
    assert seg(4096, 1, 32, 128, 128, F32, AUTO) == 1
    assert seg(4096, 1, 32, 128, 128, BF16, CORE) == 1
    assert seg(4096, 1, 32, 64, 64, BF16, SPLIT) == 0       # invalid: split is tensor-core only
    for G in range(2, 17):
        assert seg(1 << 24, 1, 148 // (2 * G - 1), 128, 128, BF16, AUTO) >= G


def test_split_workspace_holds_the_segment_buffers():
    ws = B._lib.kda_prefill_workspace_size
    T, N, H = 4096, 1, 32
    whole = ws(T, N, H, 128, 128, BF16, TC)
    split = ws(T, N, H, 128, 128, BF16, SPLIT)
    # Sx, Mx (fp32 64 KiB), S_in images (32 KiB) per (sequence, segment, head),
    # E images (16 KiB) per (chunk, head), the first region 1 KiB aligned.
    extra = N * 2 * H * (2 * 65536 + 32768) + H * (T // 64) * 16384
    assert split - whole >= extra and split - whole < extra + 1024
    assert ws(T, N, H, 128, 128, BF16, AUTO) == split


def test_prefill_rejects_null_and_misaligned_pointers():
    for name in ("q", "k", "v", "z", "A", "beta", "o", "cu"):
        assert _prefill(**{name: None}) == INVALID, name
    for name in ("q", "k", "v", "z", "o"):
        assert _prefill(**{name: _fake(0x10008)}) == INVALID, name
    assert _prefill(s0=_fake(0x10004)) == INVALID
    assert _prefill(sf=_fake(0x10002)) == INVALID
    assert _prefill(A=_fake(0x10002)) == INVALID


def test_prefill_rejects_malformed_cu_seqlens_host():
    for vals in ([1, 5, 10], [0, 5, 9], [0, 6, 5], [0, 11, 10]):
        p, keep = _host_cu(vals)
        assert _prefill(cu_host=p) == INVALID, vals


def test_prefill_workspace_checks():
    need = B._lib.kda_prefill_workspace_size(10, 2, 4, 128, 128, BF16, AUTO)
    if need == 0:
        pytest.skip("this configuration needs no workspace")
    assert _prefill(ws=None, ws_bytes=0) == WORKSPACE
    assert _prefill(ws=_fake(), ws_bytes=need - 1) == WORKSPACE


def test_workspace_size_rejects_invalid_and_is_shape_only():
    assert B._lib.kda_prefill_workspace_size(10, 2, 4, 96, 128, BF16, AUTO) == 0
    assert B._lib.kda_prefill_workspace_size(-1, 2, 4, 128, 128, BF16, AUTO) == 0
    a = B._lib.kda_prefill_workspace_size(1000, 3, 8, 128, 128, BF16, AUTO)
    b = B._lib.kda_prefill_workspace_size(1000, 3, 8, 128, 128, BF16, AUTO)
    assert a == b


def test_empty_batch_is_a_no_op():
    # N = 0, T = 0: nothing to launch, no pointer needed, no CUDA call made.
    assert _prefill(N=0, T=0, q=None, k=None, v=None, z=None, A=None, beta=None, o=None,
                    cu=None) == OK
    assert B._lib.kda_decode_step(None, None, None, None, None, None, 0, 4, 128, 128, BF16,
                                  None, 0, None, None, None) == OK


def _decode(**kw):
    a = dict(q=_fake(), k=_fake(), v=_fake(), z=_fake(), A=_fake(), beta=_fake(), Bn=4, H=2,
             dk=128, dv=128, dt=BF16, state=_fake(), P=4, slots=None, o=_fake(), stream=None)
    a.update(kw)
    return B._lib.kda_decode_step(a["q"], a["k"], a["v"], a["z"], a["A"], a["beta"], a["Bn"],
                                  a["H"], a["dk"], a["dv"], a["dt"], a["state"], a["P"],
                                  a["slots"], a["o"], a["stream"])


def test_decode_rejects_bad_arguments():
    assert _decode(dk=100) == UNSUPPORTED
    assert _decode(H=0) == INVALID
    assert _decode(Bn=-1) == INVALID
    assert _decode(P=3) == INVALID          # pool smaller than the batch without slots
    assert _decode(state=None) == INVALID
    assert _decode(q=_fake(0x10004)) == INVALID
    assert _decode(slots=_fake(0x10002)) == INVALID
    assert _decode(dt=3) == INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_valid_call_without_gpu_reports_cuda_error():
    p, keep = _host_cu([0, 4, 10])
    need = B._lib.kda_prefill_workspace_size(10, 2, 4, 128, 128, BF16, AUTO)
    assert _prefill(cu_host=p, ws=_fake(), ws_bytes=need) == CUDA
    out = ctypes.c_int32(0)
    assert B._lib.kda_device_status(None, ctypes.byref(out)) == CUDA


def test_binding_rejects_cpu_tensors():
    x = torch.zeros(4, 2, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        B.kda_decode_step(x, x, x, x, torch.zeros(2, 32), torch.zeros(4, 2),
                          torch.zeros(4, 2, 32, 32))


def test_noalloc_rejects_calls_beyond_its_scratch_limit():
    # 64 MiB of scratch holds about 900 chunk-head tiles; 96 heads x 16 chunks do not fit.
    args = [_fake()] * 6 + [_fake(), None, 1, 16 * 64, 96, 128, 128, BF16, None, None, _fake(), None]
    assert B._lib.kda_prefill_noalloc(*args) == WORKSPACE
    args = [_fake()] * 6 + [_fake(), None, 1, 64, 1, 64, 64, BF16, None, None, _fake(), None]
    assert B._lib.kda_prefill_noalloc(*args) == UNSUPPORTED


def test_noalloc_limit_edge_is_576_tokens_at_96_heads():
    """The scratch limit (64 MiB) against the tensor-core workspace: one sequence
    of 576 tokens at 96 heads (9 chunks) fits, 577 tokens (10 chunks) does not,
    and neither do two sequences of 288 (their ragged-tail bound is 9 chunks + 1)."""
    limit = 64 << 20
    assert B.kda_prefill_workspace_size(576, 1, 96, 128, 128, torch.bfloat16, "tensor_core") <= limit
    assert B.kda_prefill_workspace_size(577, 1, 96, 128, 128, torch.bfloat16, "tensor_core") > limit
    assert B.kda_prefill_workspace_size(576, 2, 96, 128, 128, torch.bfloat16, "tensor_core") > limit
    args = [_fake()] * 6 + [_fake(), None, 1, 577, 96, 128, 128, BF16, None, None, _fake(), None]
    assert B._lib.kda_prefill_noalloc(*args) == WORKSPACE


def test_selftest_rejects_out_of_range_limits():
    assert B._lib.kda_selftest_wait_timeout(0, None) == INVALID
    assert B._lib.kda_selftest_wait_timeout(20_000_000_000, None) == INVALID


def test_checkpoint_count_and_validation():
    p, keep = _host_cu([0, 130, 130, 700])
    assert B._lib.kda_checkpoint_count(p, 3, 64) == 2 + 0 + 8
    assert B._lib.kda_checkpoint_count(p, 3, 128) == 1 + 0 + 4
    assert B._lib.kda_checkpoint_count(p, 3, 100) == -1      # not a multiple of 64
    assert B._lib.kda_checkpoint_count(None, 3, 64) == -1
    args = dict(q=_fake(), k=_fake(), v=_fake(), z=_fake(), A=_fake(), beta=_fake())
    common = [args[k] for k in ("q", "k", "v", "z", "A", "beta")] + [_fake(), None, 2, 10, 4, 64, 64,
                                                                      BF16, None, None, _fake(), None,
                                                                      0, AUTO, None, None, 0]
    assert B._lib.kda_prefill_checkpointed(*common, 96, _fake()) == INVALID   # not a multiple of 64
    assert B._lib.kda_prefill_checkpointed(*common, 64, None) == INVALID      # no buffer
    assert B._lib.kda_prefill_checkpointed(*common, 64, _fake(0x10008)) == INVALID  # misaligned
    split = list(common)
    split[10:12] = [128, 128]          # dk, dv
    split[-4] = SPLIT
    assert B._lib.kda_prefill_checkpointed(*split, 64, _fake()) == UNSUPPORTED


def test_decode_multi_rejects_bad_arguments():
    def call(**kw):
        a = dict(Bn=2, Tq=4, H=2, dk=128, dv=128, dt=BF16, state=_fake(), P=2, slots=None, nt=None,
                 upd=0, o=_fake())
        a.update(kw)
        return B._lib.kda_decode_multi(_fake(), _fake(), _fake(), _fake(), _fake(), _fake(), a["Bn"],
                                       a["Tq"], a["H"], a["dk"], a["dv"], a["dt"], a["state"], a["P"],
                                       a["slots"], a["nt"], a["upd"], a["o"], None)
    assert call(Tq=0) == INVALID
    assert call(Tq=65) == INVALID
    assert call(upd=2) == INVALID
    assert call(o=None, upd=0) == INVALID      # verify needs outputs
    assert call(dk=48) == UNSUPPORTED
    assert call(nt=_fake(0x10002)) == INVALID
    assert call(Bn=0) == OK


def test_gated_entry_points_validate_the_gate():
    """The unbounded gate on the tensor-core path needs its larger workspace
    (the pair kernel's diagonal tiles); fp32 or d != 128 cannot take that path;
    a gate outside the enum is rejected before anything is launched."""
    def gated(algo, gate, dt=BF16, dk=128, dv=128, ws=None, ws_bytes=0):
        return B._lib.kda_prefill_gated(_fake(), _fake(), _fake(), _fake(), _fake(), _fake(),
                                        _fake(), None, 2, 10, 4, dk, dv, dt, None, None, _fake(),
                                        ws, ws_bytes, algo, gate, None)
    size = B._lib.kda_prefill_gated_workspace_size
    bounded, unbounded = size(10, 2, 4, 128, 128, BF16, TC, 0), size(10, 2, 4, 128, 128, BF16, TC, 1)
    assert bounded == B._lib.kda_prefill_workspace_size(10, 2, 4, 128, 128, BF16, TC)
    # two (chunk, head) tiles per head here: (10 + 63 * 2) // 64 = 2 chunks x 4 heads x 8 KiB
    assert unbounded >= bounded + 2 * 4 * 8192
    assert size(10, 2, 4, 128, 128, BF16, CORE, 1) == 0
    assert size(10, 2, 4, 128, 128, BF16, TC, 5) == 0
    assert gated(TC, 1, ws=_fake(), ws_bytes=bounded) == WORKSPACE
    assert gated(SPLIT, 1, ws=None, ws_bytes=0) == WORKSPACE
    assert gated(AUTO, 7) == INVALID
    assert gated(CORE, -1) == INVALID
    assert gated(TC, 1, dt=F32) == UNSUPPORTED
    dec = B._lib.kda_decode_step_gated(_fake(), _fake(), _fake(), _fake(), _fake(), _fake(), 2, 2,
                                       128, 128, BF16, _fake(), 2, None, _fake(), 3, None)
    assert dec == INVALID


def test_decode_slot_check_and_debug_validation():
    ok = (ctypes.c_int32 * 4)(3, 0, 2, 1)
    dup = (ctypes.c_int32 * 3)(0, 2, 2)
    oor = (ctypes.c_int32 * 2)(0, 4)
    chk = B._lib.kda_decode_check_slots
    assert chk(ctypes.cast(ok, ctypes.c_void_p), 4, 4) == OK
    assert chk(ctypes.cast(dup, ctypes.c_void_p), 3, 4) == INVALID
    assert chk(ctypes.cast(oor, ctypes.c_void_p), 2, 4) == INVALID
    assert chk(None, 2, 4) == INVALID
    assert chk(None, 0, 4) == OK
    assert B.kda_decode_check_slots([1, 0], 2) and not B.kda_decode_check_slots([1, 1], 2)

    def dbg(dt=BF16, dk=128, G=None):
        return B._lib.kda_prefill_debug(_fake(), _fake(), _fake(), _fake(), _fake(), _fake(), _fake(),
                                        None, 2, 10, 4, dk, 128, dt, None, None, _fake(), None, 0,
                                        G, None, None, None, None)
    assert dbg(dt=F32) == UNSUPPORTED
    assert dbg(dk=64) == UNSUPPORTED
    assert dbg(dk=96) == UNSUPPORTED
    assert dbg(G=_fake(0x10004)) == INVALID

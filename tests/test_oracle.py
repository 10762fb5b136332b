"""Pins for the CPU oracle (no GPU).

The oracle (``oracle/kda_oracle.c``) is checked against things other than
itself: the product form of the recurrence and its unrolled brute-force
product, closed forms (beta = 0, read-after-write at T = 1, a scalar channel
solved by ``scipy.signal.lfilter``), special cases (alpha = 1 gives the plain
delta rule; orthonormal keys with beta = 1 store exact associations), the
gate's range and saturation values the pages print, invariants (per-step write
identity, resume at any split, varlen = per-sequence loop, affine segment
composition), and the naive chunkwise form at several chunk sizes.

Sources: "Kimi K3: Architecture, Training, and Million-Token Agentic RL",
sections 3.1 (recurrence, delta rule), 3.2 (edit order), 3.3 (gate, chunk
bound, chunk I/O); "Kimi K3 Under the Hood", sections "Sequence mixing" (gate)
and "Infrastructure for a 3T-class MoE" (segments as affine maps composed by a
prefix scan).
"""
import json
import os

import numpy as np
import pytest
import scipy.signal

from oracle import chunkwise, oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _inputs(lengths, H=2, dk=5, dv=4, seed=0, s0=True, z_mean=0.0, beta=None):
    rs = np.random.RandomState(seed)
    T = sum(lengths)
    q = rs.randn(T, H, dk); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rs.randn(T, H, dk); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rs.randn(T, H, dv)
    z = rs.randn(T, H, dk) + z_mean
    b = 1.0 / (1.0 + np.exp(-rs.randn(T, H))) if beta is None else np.full((T, H), beta)
    A = rs.uniform(-1, 1, size=(H, dk))
    S0 = rs.randn(len(lengths), H, dk, dv) * 0.3 if s0 else None
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return dict(q=q, k=k, v=v, z=z, A=A, beta=b, cu_seqlens=cu, initial_state=S0)


def _relerr(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


# ---------------------------------------------------------------- the gate ----

def test_gate_range_and_saturation_match_pages():
    consts = json.load(open(os.path.join(GOLDEN, "pages_constants.json")))
    gmin = consts["g_min"]["value"]
    lo, hi = consts["gate_range"]["value"]
    rs = np.random.RandomState(1)
    z = rs.randn(50, 3, 7) * 4
    A = rs.uniform(-1, 1, (3, 7))
    g = oracle.gate(z, A)
    assert np.all(g >= lo) and np.all(g <= hi)
    # exp(A) * z -> +inf saturates the sigmoid to 1: g = g_min exactly.
    assert np.all(oracle.gate(np.full((2, 3, 7), 1e4), A) == gmin)
    # -> -inf: sigmoid underflows to 0, g = 0 (alpha = 1 exactly).
    assert np.all(oracle.gate(np.full((2, 3, 7), -1e4), A) == 0.0)
    # sigmoid(0) = 1/2: g = g_min / 2 exactly, whatever A is.
    assert np.all(oracle.gate(np.zeros((1, 3, 7)), A) == gmin / 2)
    # monotone decreasing in z for every A (exp(A) > 0).
    zz = np.linspace(-6, 6, 101)[:, None, None] * np.ones((1, 3, 7))
    assert np.all(np.diff(oracle.gate(zz, A), axis=0) < 0)
    # the value at A = 0 is g_min / (1 + e^{-z}), checked against scipy's expit
    from scipy.special import expit
    zs = rs.randn(9, 1, 4)
    np.testing.assert_allclose(oracle.gate(zs, np.zeros((1, 4))), gmin * expit(zs), rtol=1e-15)


def test_tile_cumulative_bound_matches_pages():
    consts = json.load(open(os.path.join(GOLDEN, "pages_constants.json")))
    tile = consts["secondary_tile"]["value"]
    lo, hi = consts["tile_cumulative_log_decay_range"]["value"]
    bexp = consts["reciprocal_scaling_bound_exponent"]["value"]
    A = np.zeros((1, 4))
    g_sat = oracle.gate(np.full((tile, 1, 4), 1e4), A)
    G = np.cumsum(g_sat[:, 0, :], axis=0)
    assert G[-1, 0] == lo               # the closed endpoint is reached exactly
    rs = np.random.RandomState(2)
    G2 = np.cumsum(oracle.gate(rs.randn(tile, 1, 4) * 10, A)[:, 0, :], axis=0)
    assert np.all(G2 >= lo) and np.all(G2 <= hi)
    # e^{+80} and e^{-80} are finite, normal numbers in fp32 (and bf16 shares fp32's exponent).
    f = np.float32
    assert np.isfinite(f(np.exp(bexp))) and f(np.exp(-bexp)) > np.finfo(np.float32).tiny


# ------------------------------------------------------ the recurrence -------

def test_matches_product_form_and_unrolled_brute_force():
    """Section 3.1 product form S_t = (I - b k k^T) Diag(a) S_{t-1} + b k v^T,
    evaluated step by step and as an unrolled product of explicit matrices."""
    for seed, (T, dk, dv) in enumerate([(1, 1, 1), (3, 2, 3), (8, 8, 8), (7, 5, 2)]):
        x = _inputs([T], H=2, dk=dk, dv=dv, seed=seed)
        o, sf = oracle.prefill(**x)
        g = oracle.gate(x["z"], x["A"])
        for h in range(2):
            S = x["initial_state"][0, h].copy()
            Ms, Bs = [], []
            for t in range(T):
                kk, b = x["k"][t, h], x["beta"][t, h]
                M = (np.eye(dk) - b * np.outer(kk, kk)) @ np.diag(np.exp(g[t, h]))
                S = M @ S + b * np.outer(kk, x["v"][t, h])
                Ms.append(M); Bs.append(b * np.outer(kk, x["v"][t, h]))
                np.testing.assert_allclose(o[t, h], S.T @ x["q"][t, h], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(sf[0, h], S, rtol=1e-12, atol=1e-14)
            # unrolled: S_T = M_T..M_1 S0 + sum_t M_T..M_{t+1} B_t
            prod = np.eye(dk)
            S_unrolled = np.zeros((dk, dv))
            for t in range(T):
                P = np.eye(dk)
                for u in range(t + 1, T):
                    P = Ms[u] @ P
                S_unrolled += P @ Bs[t]
            for u in range(T):
                prod = Ms[u] @ prod
            S_unrolled += prod @ x["initial_state"][0, h]
            np.testing.assert_allclose(sf[0, h], S_unrolled, rtol=1e-12, atol=1e-14)


def test_read_after_write_single_token():
    """T = 1 from a zero state: S_1 = b k v^T, so o_1 = b (k . q) v (the read
    follows the write, section 3.2)."""
    x = _inputs([1], H=3, dk=6, dv=5, seed=3, s0=False)
    o, sf = oracle.prefill(**x)
    for h in range(3):
        kk, qq, vv, b = x["k"][0, h], x["q"][0, h], x["v"][0, h], x["beta"][0, h]
        np.testing.assert_allclose(o[0, h], b * (kk @ qq) * vv, rtol=1e-13)
        np.testing.assert_allclose(sf[0, h], b * np.outer(kk, vv), rtol=1e-13)


def test_alpha_one_reduces_to_delta_rule():
    """z -> -inf gives alpha = 1 exactly; the step is then the section 3.1 delta
    rule vhat = S^T k, S += b k (v - vhat)^T, coded separately here."""
    x = _inputs([9], H=2, dk=4, dv=3, seed=4)
    x["z"][:] = -1e4
    o, sf = oracle.prefill(**x)
    for h in range(2):
        S = x["initial_state"][0, h].copy()
        for t in range(9):
            kk = x["k"][t, h]
            err = x["v"][t, h] - S.T @ kk
            S = S + x["beta"][t, h] * np.outer(kk, err)
            np.testing.assert_allclose(o[t, h], S.T @ x["q"][t, h], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(sf[0, h], S, rtol=1e-12, atol=1e-14)


def test_orthonormal_keys_store_exact_associations():
    """alpha = 1, beta = 1 and orthonormal keys from a zero state: the delta
    rule writes each association exactly, so S = sum_i k_i v_i^T and
    S^T k_i = v_i (linear algebra of the edit)."""
    dk, dv = 6, 4
    rs = np.random.RandomState(5)
    Q, _ = np.linalg.qr(rs.randn(dk, dk))
    keys = Q.T  # rows orthonormal
    x = _inputs([dk], H=1, dk=dk, dv=dv, seed=6, s0=False, beta=1.0)
    x["k"][:, 0] = keys
    x["z"][:] = -1e4
    _, sf = oracle.prefill(**x)
    S = sf[0, 0]
    np.testing.assert_allclose(S, keys.T @ x["v"][:, 0], atol=1e-13)
    np.testing.assert_allclose(keys @ S, x["v"][:, 0], atol=1e-13)


def test_beta_zero_leaves_decayed_state():
    """beta = 0: no edit, S_T = Diag(prod_t alpha_t) S0 and o_t = (Diag(e^{G_t}) S0)^T q_t."""
    x = _inputs([11], H=2, dk=5, dv=3, seed=7, beta=0.0)
    o, sf = oracle.prefill(**x)
    g = oracle.gate(x["z"], x["A"])
    for h in range(2):
        G = np.cumsum(g[:, h], axis=0)
        S0 = x["initial_state"][0, h]
        for t in range(11):
            np.testing.assert_allclose(o[t, h], (np.exp(G[t])[:, None] * S0).T @ x["q"][t, h],
                                       rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(sf[0, h], np.exp(G[-1])[:, None] * S0, rtol=1e-12)


def test_decay_scales_rows_scalar_channel_via_lfilter():
    """Diag(alpha) scales ROWS (key channels), section 3.1.  With every key equal
    to e_0 and constant z, beta, rows c != 0 only decay, and row 0 follows the
    first-order filter s_t = (1 - b) a s_{t-1} + b v_t, solved by scipy.signal.lfilter."""
    T, dk, dv = 25, 4, 3
    x = _inputs([T], H=1, dk=dk, dv=dv, seed=8, beta=0.37)
    x["k"][:] = 0.0
    x["k"][:, 0, 0] = 1.0
    x["z"][:] = x["z"][0:1]
    _, sf = oracle.prefill(**x)
    g = oracle.gate(x["z"][:1], x["A"])[0, 0]
    a = np.exp(g)
    S0 = x["initial_state"][0, 0]
    b = 0.37
    for j in range(dv):
        y, _ = scipy.signal.lfilter([b], [1.0, -(1 - b) * a[0]], x["v"][:, 0, j],
                                    zi=[(1 - b) * a[0] * S0[0, j]])
        np.testing.assert_allclose(sf[0, 0, 0, j], y[-1], rtol=1e-12)
    np.testing.assert_allclose(sf[0, 0, 1:], (a[1:] ** T)[:, None] * S0[1:], rtol=1e-12)


def test_per_step_write_identity():
    """With unit k: S_t^T k_t = (1 - b_t) Sbar_t^T k_t + b_t v_t; at b = 1 the
    association is written exactly (S_t^T k_t = v_t)."""
    for beta in (None, 1.0):
        x = _inputs([6], H=1, dk=7, dv=5, seed=9, beta=beta)
        g = oracle.gate(x["z"], x["A"])
        for t in range(1, 6):
            def run(n):
                sub = {kk: x[kk][:n] for kk in ("q", "k", "v", "z", "beta")}
                return oracle.prefill(**sub, A=x["A"], cu_seqlens=np.array([0, n], np.int32),
                                      initial_state=x["initial_state"])[1]
            S_prev, S_t = run(t - 1), run(t)
            kk, b = x["k"][t - 1, 0], x["beta"][t - 1, 0]
            Sbar = np.exp(g[t - 1, 0])[:, None] * S_prev[0, 0]
            lhs = S_t[0, 0].T @ kk
            rhs = (1 - b) * (Sbar.T @ kk) + b * x["v"][t - 1, 0]
            np.testing.assert_allclose(lhs, rhs, rtol=1e-11, atol=1e-13)
            if beta == 1.0:
                np.testing.assert_allclose(lhs, x["v"][t - 1, 0], rtol=1e-11, atol=1e-13)


# ----------------------------------------------- structure and composition ----

def test_resume_at_any_split_equals_whole():
    """Chunk I/O contract, section 3.3: S_in[c+1] = S_out[c]; resuming from the
    final state of a prefix reproduces the whole sequence (prefix-cache resume)."""
    x = _inputs([40], H=2, dk=6, dv=4, seed=10)
    o, sf = oracle.prefill(**x)
    for t1 in (1, 15, 16, 17, 32, 39):
        a = {kk: x[kk][:t1] for kk in ("q", "k", "v", "z", "beta")}
        b = {kk: x[kk][t1:] for kk in ("q", "k", "v", "z", "beta")}
        oa, sa = oracle.prefill(**a, A=x["A"], cu_seqlens=np.array([0, t1], np.int32),
                                initial_state=x["initial_state"])
        ob, sb = oracle.prefill(**b, A=x["A"], cu_seqlens=np.array([0, 40 - t1], np.int32),
                                initial_state=sa)
        np.testing.assert_allclose(np.concatenate([oa, ob]), o, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(sb, sf, rtol=1e-12, atol=1e-14)


def test_varlen_packing_equals_per_sequence_loop():
    lengths = [5, 0, 1, 17, 16, 3]
    x = _inputs(lengths, H=3, dk=4, dv=3, seed=11)
    o, sf = oracle.prefill(**x)
    cu = x["cu_seqlens"]
    for i, L in enumerate(lengths):
        sl = slice(cu[i], cu[i + 1])
        oi, si = oracle.prefill(**{kk: x[kk][sl] for kk in ("q", "k", "v", "z", "beta")},
                                A=x["A"], cu_seqlens=np.array([0, L], np.int32),
                                initial_state=x["initial_state"][i:i + 1])
        np.testing.assert_array_equal(oi, o[sl])
        np.testing.assert_array_equal(si[0], sf[i])
    # an empty sequence passes its initial state through
    np.testing.assert_array_equal(sf[1], x["initial_state"][1])


def test_segments_compose_as_affine_maps():
    """Each segment maps S_in -> M S_in + B (a dk x dk transition and a state
    built from zero); two segments compose as (M2 M1, M2 B1 + B2) -- the
    associative combine that KDA context parallelism scans ("Kimi K3 Under the
    Hood", section "Infrastructure for a 3T-class MoE").  M also equals the
    explicit product of the per-token matrices (I - b k k^T) Diag(alpha)."""
    dk, dv, L1, L2 = 4, 3, 7, 9
    x = _inputs([L1 + L2], H=1, dk=dk, dv=dv, seed=12)
    g = oracle.gate(x["z"], x["A"])

    def seg(lo, hi):
        sub = {kk: x[kk][lo:hi] for kk in ("q", "k", "v", "z", "beta")}
        cu = np.array([0, hi - lo], np.int32)
        _, B = oracle.prefill(**sub, A=x["A"], cu_seqlens=cu, initial_state=None)
        M = np.zeros((dk, dk))
        for c in range(dk):
            e = np.zeros((1, 1, dk, dv)); e[0, 0, c, 0] = 1.0
            _, Sc = oracle.prefill(**sub, A=x["A"], cu_seqlens=cu, initial_state=e)
            M[:, c] = Sc[0, 0, :, 0] - B[0, 0, :, 0]
        P = np.eye(dk)
        for t in range(lo, hi):
            kk, b = x["k"][t, 0], x["beta"][t, 0]
            P = (np.eye(dk) - b * np.outer(kk, kk)) @ np.diag(np.exp(g[t, 0])) @ P
        np.testing.assert_allclose(M, P, rtol=1e-11, atol=1e-14)
        return M, B[0, 0]

    M1, B1 = seg(0, L1)
    M2, B2 = seg(L1, L1 + L2)
    _, sf = oracle.prefill(**x)
    S0 = x["initial_state"][0, 0]
    np.testing.assert_allclose((M2 @ M1) @ S0 + (M2 @ B1 + B2), sf[0, 0], rtol=1e-11, atol=1e-14)


def test_decode_step_continues_prefill():
    """Decode and prefill are the same recurrence (section 3.3): prefill(T)
    followed by one decode step equals prefill(T + 1)."""
    x = _inputs([12], H=2, dk=5, dv=4, seed=13)
    o, sf = oracle.prefill(**x)
    sub = {kk: x[kk][:11] for kk in ("q", "k", "v", "z", "beta")}
    _, s11 = oracle.prefill(**sub, A=x["A"], cu_seqlens=np.array([0, 11], np.int32),
                            initial_state=x["initial_state"])
    od, sd = oracle.decode_step(*(x[kk][11:12] for kk in ("q", "k", "v", "z")), x["A"],
                                x["beta"][11:12], s11)
    np.testing.assert_allclose(od[0], o[11], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(sd, sf, rtol=1e-12, atol=1e-14)


def test_decode_slots_touch_only_their_rows():
    rs = np.random.RandomState(14)
    B, H, dk, dv, P = 3, 2, 4, 3, 6
    q = rs.randn(B, H, dk); k = rs.randn(B, H, dk); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v, z = rs.randn(B, H, dv), rs.randn(B, H, dk)
    beta, A = rs.uniform(0, 1, (B, H)), rs.uniform(-1, 1, (H, dk))
    pool = rs.randn(P, H, dk, dv)
    slots = np.array([4, 0, 2], np.int32)
    o, new = oracle.decode_step(q, k, v, z, A, beta, pool, slots)
    for untouched in (1, 3, 5):
        np.testing.assert_array_equal(new[untouched], pool[untouched])
    for b, s in enumerate(slots):
        ob, sb = oracle.decode_step(q[b:b + 1], k[b:b + 1], v[b:b + 1], z[b:b + 1], A,
                                    beta[b:b + 1], pool[s:s + 1])
        np.testing.assert_array_equal(ob[0], o[b])
        np.testing.assert_array_equal(sb[0], new[s])


# ----------------------------------------------- the chunkwise second witness ----

@pytest.mark.parametrize("chunk", [1, 2, 4, 16, 32, 64])
def test_chunkwise_form_equals_recurrence(chunk):
    lengths = [0, 1, 15, 16, 17, 33, 70]
    x = _inputs(lengths, H=2, dk=6, dv=5, seed=20 + chunk)
    o, sf = oracle.prefill(**x)
    oc, sc = chunkwise.prefill(**x, chunk=chunk)
    assert _relerr(oc, o) < 1e-12
    assert _relerr(sc, sf) < 1e-12


def test_chunkwise_form_at_saturated_gate():
    """All gates at g_min: e^{-G} reaches e^{80} over 16 tokens -- the pages'
    worst case -- and the chunkwise form still agrees at chunk = 16."""
    x = _inputs([48], H=1, dk=4, dv=3, seed=30)
    x["z"][:] = 1e4
    o, sf = oracle.prefill(**x)
    oc, sc = chunkwise.prefill(**x, chunk=16)
    assert _relerr(oc, o) < 1e-10 and _relerr(sc, sf) < 1e-10


def test_oracle_regression_fixture():
    """tests/golden/tiny_case.json was written by tests/golden/make_golden.py from
    the oracle; it guards against drift of the oracle build itself."""
    d = json.load(open(os.path.join(GOLDEN, "tiny_case.json")))
    arr = {kk: np.array(d[kk]) for kk in ("q", "k", "v", "z", "beta", "A", "initial_state")}
    o, sf = oracle.prefill(**arr, cu_seqlens=np.array(d["cu_seqlens"], np.int32))
    np.testing.assert_allclose(o, np.array(d["o"]), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(sf, np.array(d["final_state"]), rtol=1e-13, atol=1e-15)


def test_checkpoints_are_prefix_final_states():
    """A checkpoint is, by definition, the final state of the sequence's prefix
    of that length; the oracle's checkpoint output is checked against separate
    prefix runs (and the plain prefill is unchanged by asking for checkpoints)."""
    lengths = [130, 0, 64, 200, 63]
    x = _inputs(lengths, H=2, dk=4, dv=3, seed=40)
    for every in (16, 64, 100):
        o, sf, ck = oracle.prefill_checkpoints(**x, every=every)
        o2, sf2 = oracle.prefill(**x)
        np.testing.assert_array_equal(o, o2)
        np.testing.assert_array_equal(sf, sf2)
        assert ck.shape[0] == sum(L // every for L in lengths)
        row = 0
        cu = x["cu_seqlens"]
        for i, L in enumerate(lengths):
            for j in range(1, L // every + 1):
                sl = slice(cu[i], cu[i] + j * every)
                _, s_pref = oracle.prefill(**{kk: x[kk][sl] for kk in ("q", "k", "v", "z", "beta")},
                                          A=x["A"], cu_seqlens=np.array([0, j * every], np.int32),
                                          initial_state=x["initial_state"][i:i + 1])
                np.testing.assert_array_equal(ck[row], s_pref[0])
                row += 1
        assert row == ck.shape[0]


# ------------------------------------------- the unbounded (Softplus) gate ----
# "Kimi K3: Architecture, Training, and Million-Token Agentic RL", section 3.3,
# and "Kimi K3 Under the Hood", section "Sequence mixing": the earlier Kimi
# Linear gate was an unbounded negative Softplus, whose 16-token cumulative decay
# has no lower bound, so reciprocal decay overflows and diagonal tiles need a
# position-pair path.  Read here as g = -softplus(exp(A) * z).

def test_softplus_gate_closed_forms():
    rs = np.random.RandomState(11)
    A = rs.uniform(-1, 1, (3, 7))
    # at z = 0: -log 2 exactly, whatever A is
    np.testing.assert_allclose(oracle.gate(np.zeros((1, 3, 7)), A, "softplus"), -np.log(2.0),
                               rtol=1e-15)
    # A = 0 reduces to -log(1 + e^z), scipy's log-sum-exp of (0, z)
    from scipy.special import logsumexp
    zs = rs.randn(9, 1, 4) * 3
    ref = -logsumexp(np.stack([np.zeros_like(zs), zs]), axis=0)
    np.testing.assert_allclose(oracle.gate(zs, np.zeros((1, 4)), "softplus"), ref, rtol=1e-14)
    # asymptotes: -x + e^{-x} terms for large x, -e^{x} for very negative x
    big = np.full((1, 1, 1), 40.0)
    assert abs(oracle.gate(big, np.zeros((1, 1)), "softplus")[0, 0, 0] + 40.0) < 1e-15
    small = np.full((1, 1, 1), -40.0)
    np.testing.assert_allclose(oracle.gate(small, np.zeros((1, 1)), "softplus"), -np.exp(-40.0),
                               rtol=1e-12)
    # unbounded below: g = -exp(A) z once exp(A) z is large
    z = np.full((1, 3, 7), 1e4)
    np.testing.assert_allclose(oracle.gate(z, A, "softplus"), -np.exp(A)[None] * 1e4, rtol=1e-12)
    # strictly negative and decreasing in z
    zz = np.linspace(-6, 6, 101)[:, None, None] * np.ones((1, 3, 7))
    gg = oracle.gate(zz, A, "softplus")
    assert np.all(gg < 0) and np.all(np.diff(gg, axis=0) < 0)


def test_softplus_tile_decay_leaves_the_bound():
    """With z = 60 the 16-token cumulative decay passes -80 (and -745, where
    e^{-G} overflows even fp64): the separable chunk form breaks down, the
    position-pair form stays finite and equals the token recurrence."""
    x = _inputs([40], H=2, dk=6, dv=5, seed=12, z_mean=60.0)
    g = oracle.gate(x["z"], x["A"], "softplus")
    G16 = np.cumsum(g[:16], axis=0)
    assert G16[-1].min() < -745.0
    o, sf = oracle.prefill(**x, gate="softplus")
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(sf))
    with np.errstate(all="ignore"):
        o_sep, _ = chunkwise.prefill(**x, chunk=16, gate="softplus")
    assert not np.all(np.isfinite(o_sep))
    o_pw, sf_pw = chunkwise.prefill(**x, chunk=16, gate="softplus", pairwise=True)
    assert _relerr(o_pw, o) < 1e-12 and _relerr(sf_pw, sf) < 1e-12


@pytest.mark.parametrize("gate", ["bounded", "softplus"])
@pytest.mark.parametrize("chunk", [1, 3, 16])
def test_pairwise_chunk_form_equals_recurrence(gate, chunk):
    x = _inputs([37, 16, 5], H=2, dk=6, dv=4, seed=13 + chunk, z_mean=1.0)
    o, sf = oracle.prefill(**x, gate=gate)
    o_pw, sf_pw = chunkwise.prefill(**x, chunk=chunk, gate=gate, pairwise=True)
    assert _relerr(o_pw, o) < 1e-11 and _relerr(sf_pw, sf) < 1e-11


def test_softplus_recurrence_matches_brute_force_product():
    x = _inputs([6], H=1, dk=4, dv=3, seed=14, z_mean=2.0)
    o, sf = oracle.prefill(**x, gate="softplus")
    g = oracle.gate(x["z"], x["A"], "softplus")
    S = x["initial_state"][0, 0].copy()
    for t in range(6):
        kk, b = x["k"][t, 0], x["beta"][t, 0]
        S = (np.eye(4) - b * np.outer(kk, kk)) @ np.diag(np.exp(g[t, 0])) @ S + b * np.outer(kk, x["v"][t, 0])
        np.testing.assert_allclose(o[t, 0], S.T @ x["q"][t, 0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(sf[0, 0], S, rtol=1e-12, atol=1e-14)


def test_softplus_decode_continues_prefill():
    x = _inputs([9], H=2, dk=5, dv=4, seed=15, z_mean=3.0)
    o, sf = oracle.prefill(**x, gate="softplus")
    head = {key: x[key][:8] for key in ("q", "k", "v", "z", "beta")}
    _, s8 = oracle.prefill(**head, A=x["A"], cu_seqlens=np.array([0, 8], np.int32),
                           initial_state=x["initial_state"], gate="softplus")
    od, sd = oracle.decode_step(*(x[key][8:9] for key in ("q", "k", "v", "z")), x["A"],
                                x["beta"][8:9], s8, gate="softplus")
    np.testing.assert_allclose(od[0], o[8], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(sd, sf, rtol=1e-12, atol=1e-14)


# ------------------------------------------- stage intermediates (debug dumps) ----

def test_chunk_intermediates_satisfy_their_definitions():
    """W and U solve (I + A) W = Diag(beta) Kt and (I + A) U = Diag(beta) V (checked
    by multiplication, not by another inverse); D = U - W S0; and the stages put
    together give the recurrence's outputs and final state."""
    x = _inputs([70, 64, 9], H=2, dk=6, dv=5, seed=16)
    ref_o, ref_s = oracle.prefill(**x)
    got = chunkwise.prefill_intermediates(**x, chunk=64)
    assert _relerr(got["o"], ref_o) < 1e-11 and _relerr(got["final_state"], ref_s) < 1e-11
    q, k, v, b = x["q"][:64, 0], x["k"][:64, 0], x["v"][:64, 0], x["beta"][:64, 0]
    g = oracle.gate(x["z"][:64], x["A"])[:, 0]
    r = chunkwise.chunk_intermediates(q, k, v, g, b, x["initial_state"][0, 0])
    G = np.cumsum(g, axis=0)
    np.testing.assert_allclose(r["G"], G, rtol=1e-13)
    M = np.eye(64) + r["A"]
    np.testing.assert_allclose(M @ r["W"], b[:, None] * k * np.exp(G), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(M @ r["U"], b[:, None] * v, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(r["D"], r["U"] - r["W"] @ x["initial_state"][0, 0], rtol=1e-12, atol=1e-14)

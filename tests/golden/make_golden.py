"""Writes tests/golden/tiny_case.json from the CPU oracle alone.

The inputs are drawn here with NumPy (seeded) and stored exactly; the expected
outputs are the oracle's.  The file pins the oracle against silent drift (a
changed build flag, a refactor); the independent pins live in tests/test_oracle.py.
Run: python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
from oracle import oracle  # noqa: E402


def main():
    rs = np.random.RandomState(20261202)
    lengths = [4, 0, 3]
    T, H, dk, dv = sum(lengths), 2, 3, 2
    q = rs.randn(T, H, dk); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rs.randn(T, H, dk); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rs.randn(T, H, dv)
    z = rs.randn(T, H, dk)
    beta = 1.0 / (1.0 + np.exp(-rs.randn(T, H)))
    A = rs.uniform(-1, 1, size=(H, dk))
    s0 = rs.randn(len(lengths), H, dk, dv) * 0.5
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    o, sf = oracle.prefill(q, k, v, z, A, beta, cu, s0)
    out = dict(
        _about="Oracle regression fixture written by tests/golden/make_golden.py (oracle only).",
        lengths=lengths, H=H, dk=dk, dv=dv,
        q=q.tolist(), k=k.tolist(), v=v.tolist(), z=z.tolist(), beta=beta.tolist(),
        A=A.tolist(), initial_state=s0.tolist(), cu_seqlens=cu.tolist(),
        o=o.tolist(), final_state=sf.tolist())
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_case.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()

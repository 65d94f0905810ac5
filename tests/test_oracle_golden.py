"""The oracle against small examples worked by hand (tests/golden/*.txt,
each deriving its values from the definitions in its header)."""
import os

import numpy as np

from oracle import ckks as C

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            key, *vals = line.split()
            out[key] = [int(v) for v in vals]
    return out


def test_ntt_and_automorphism_worked_by_hand():
    g = _read("ntt_n4_q17.txt")
    q = g["q"][0]
    P = C.Params(2, 1, 1, 1, q=[q], p=[41])
    assert P.psi[0] == g["psi"][0]
    a = np.array([g["coeffs"]], dtype=np.uint64)
    assert C.ntt_rows(a, [q], P)[0].tolist() == g["ntt"]
    assert C.intt_rows(np.array([g["ntt"]], dtype=np.uint64), [q], P)[0].tolist() == g["coeffs"]
    k, *want = g["automorph"]
    assert C.automorph_coeff_rows(a, k, [q], P)[0].tolist() == want


def test_base_conversion_worked_by_hand():
    g = _read("base_conv_q7_q11.txt")
    x = np.array([[v] for v in g["x"]], dtype=np.uint64)
    assert C.base_conv(x, g["src"], g["dst"])[:, 0].tolist() == g["conv"]
    assert C.base_conv(x, g["src"], g["dst"], centred=True)[:, 0].tolist() == g["conv_centred"]


def test_encoding_worked_by_hand():
    lines = [ln.split() for ln in open(os.path.join(GOLDEN, "encode_n4.txt"))
             if ln.strip() and not ln.startswith("#")]
    scale = float(lines[0][1])
    P = C.Params(2, 1, 1, 1, q=[17], p=[41])
    cases = [(lines[i], lines[i + 1]) for i in range(1, len(lines), 2)]
    assert len(cases) == 2
    for zl, cl in cases:
        v = [float(t) for t in zl[1:]]
        z = np.array([v[0] + 1j * v[1], v[2] + 1j * v[3]])
        want = [int(t) for t in cl[1:]]
        assert C.encode_coeffs(z, scale, P).astype(np.int64).tolist() == want

"""The oracle's pins have teeth: each build below plants one plausible
mistake in one step of the oracle (a swapped nibble order, a double
rounding, a wrong zero-point group, a flipped tie-break, biased weights, a
reversed dispatch order, a dropped bias, a SwiGLU without its gate factor, a
dropped gate/up gradient term, unweighted combine, a missing SwiGLU-VJP
factor, a missing softmax-VJP term, a wrong dweights dot, a COPY VJP that
sums one selection only, an NF4 byte read low nibble first), and the oracle's
own CPU tests must fail on every one of them.  CPU only."""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
from oracle.build import build_mutant  # noqa: E402

PINS = [os.path.join(ROOT, "tests", f) for f in
        ("test_oracle_pins.py", "test_oracle_bruteforce.py", "test_oracle_invariants.py", "test_oracle_nf4.py")]

MUTANTS = {
    1: "unpack ignores the 0,2,4,6,1,3,5,7 order",
    2: "coefficient rounded as RNE(RNE(q s) - RNE(z s))",
    3: "zero points taken from the next group",
    4: "top-k ties go to the higher expert ID",
    5: "weights from the biased (selection) logits",
    6: "rows inside an expert in descending token order",
    7: "projection bias dropped",
    8: "SwiGLU without the gate factor (sigmoid(G) U)",
    9: "gate/up input VJP drops the up-projection term",
    10: "combine ignores the routing weights",
    11: "SwiGLU VJP drops the (1 + G (1 - s)) factor",
    12: "router-logit VJP drops the - <w, dw> term",
    13: "combine VJP dweights dot uses dOut instead of y",
    14: "COPY VJP sums only the first selection of each token",
    15: "NF4 codes read low nibble first",
}


def _run_pins(lib_path):
    env = dict(os.environ)
    if lib_path:
        env["ORACLE_LIB"] = lib_path
    else:
        env.pop("ORACLE_LIB", None)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PINS],
                       capture_output=True, text=True, env=env, cwd=ROOT, timeout=600)
    return r.returncode, r.stdout[-1500:]


def test_unmutated_oracle_passes_the_pins():
    rc, out = _run_pins(None)
    assert rc == 0, out


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=[MUTANTS[m] for m in sorted(MUTANTS)])
def test_pins_catch_planted_mistake(mutant):
    with tempfile.TemporaryDirectory() as d:
        lib = build_mutant(mutant, d)
        rc, out = _run_pins(lib)
    assert rc != 0, "the pins did not catch: %s\n%s" % (MUTANTS[mutant], out)

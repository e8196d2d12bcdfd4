"""The oracle's pins reject planted mistakes.

Each case builds the oracle with one plausible slip compiled in (the
ORC_MUTANT switches of oracle/dsa_oracle.c; the default build has none) and
runs tests/test_oracle_pins.py against it in a child process: at least one pin
must fail.  A mistake that every pin accepted would be a mistake the oracle
could carry unnoticed into every parity test.  CPU only.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

MUTANTS = {
    1: "ReLU dropped from the token score",
    2: "ties broken towards the higher index",
    3: "causal mask excludes the query's own position",
    4: "head weight w dropped from the token score",
    5: "k_len ignored",
    6: "boundary block averaged over the full block size",
    7: "router sums w ReLU(.) without the absolute value",
    8: "router breaks head ties towards the higher head",
    9: "HISA coarse score drops the head weight",
    10: "e4m3 rounding half away from zero instead of to even",
    11: "query operand indexed with heads and dim transposed",
    12: "dot product drops its last term",
    13: "e4m3 subnormal step 2^-10 instead of 2^-9",
    14: "quantisation scale amax / 240 instead of amax / 448",
    15: "padding index 0 instead of -1",
    16: "block representative kept unrounded (not the key type)",
    17: "boundary block reads past the causal position",
    18: "MISA-dagger pool one candidate short",
    19: "HISA keeps one block fewer than r",
    20: "stacked HISA reranks with every head instead of the routed ones",
    21: "default query position 0 instead of n_k - n_q",
    22: "router reports E = S instead of S / M_t",
    23: "MISA scores tokens with every head instead of the routed ones",
    24: "MISA-dagger reranks with the routed heads instead of all heads",
    25: "bf16 words decoded with a 15-bit shift",
    26: "e4m3 encode truncates instead of rounding",
    28: "blocks cover full blocks only (the boundary block dropped)",
    29: "router takes |q . k~| instead of ReLU(q . k~)",
    30: "tolerance scale nu sums signed w instead of |w|",
    31: "tolerance scale nu without the 1/sqrt(d) factor",
    32: "tolerance scale nu with the squared key norm",
    33: "split query drops its low e4m3 part",
    34: "indexer LISA ranks by the full ReLU score instead of the linear term",
    35: "ResMiSA residual takes ReLU(q . k) instead of ReLU(-q . k)",
    36: "residual bound pairs q+ with the block maximum (wrong extreme)",
    37: "residual router weighs the bound by signed w instead of |w|",
    38: "residual bound blocks reach past the causal position",
    39: "LISA-dagger pool one candidate short",
    40: "sparse attention logits without the softmax scale",
    41: "sparse attention value taken from the wrong end of the latent row",
    43: "sparse attention reads an empty (-1) entry as position 0",
    44: "backward mask 1[z >= 0] instead of 1[z > 0]",
    45: "backward drops the head weight from dq and dk",
    46: "backward dw uses z instead of ReLU(z)",
    47: "DoSA block bound takes q . kmin for the largest dot product",
    48: "DoSA lower bound weighs the wrong box extreme by the head sign",
    49: "DoSA seed set counts a partial block as full",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: f"m{m}")
def test_pins_reject_mutant(mutant):
    env = dict(os.environ, DSA_ORACLE_MUTANT=str(mutant))
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(HERE, "test_oracle_pins.py"),
                        "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    # pytest exit status 1: tests ran and at least one failed
    assert r.returncode == 1, (f"mutant {mutant} ({MUTANTS[mutant]}) was not rejected "
                               f"(pytest status {r.returncode}):\n{r.stdout[-2000:]}")

"""The pins are strong enough: each deliberately wrong build of the oracle
(ORACLE_MUTANT = k in ssd_oracle.c) must fail at least one pin.

Mutants: 1 drops the D skip; 2 reads y from the state before the update;
3 swaps the roles of B and C; 4 flips the sign of the decay exponent; 5 drops
dt_bias; 6 maps heads to groups round-robin instead of contiguously; 7 drops dt
from the input term; 8 replaces softplus by exp; 9 ignores the initial state;
10 gates with sigmoid(z) instead of silu(z); 11 reverses the convolution
kernel; 12 shifts the convolution one token ahead; 13 ignores the carried
convolution inputs; in the backward pass, 14 drops the decay when the adjoint
steps back a token; 15 drops the decay's share A*da of ddt; 16 drops the
softplus derivative of ddt_raw; 17 adds dy_t C_t^T to the adjoint only after
using it; in the diagonal-A selective scan, 18 decays every state with the
channel's first A entry; 19 feeds channel 0's x to every channel; in the
gated RMSNorm, 20 normalises before the gate; 21 divides by the root of the
sum of squares instead of their mean.
"""
import pytest

import oracle
import pins

MUTANTS = list(range(1, 22))


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    return str(tmp_path_factory.mktemp("oracle_mutants"))


@pytest.mark.parametrize("k", MUTANTS)
def test_mutant_is_caught(k, mutant_dir):
    orc = oracle.load(mutant=k, out_dir=mutant_dir)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {k} passed every pin"

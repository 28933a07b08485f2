"""The parity bars the GPU tests use are the ones stated for this forward pass:
max|x - x_ref| / max|x_ref| <= 1e-4 for float32 inputs and <= 5e-3 for bfloat16 inputs, for the
outputs o and for the final state.  They live in one place (parity_util.TOL); no test module may
define a bar of its own."""
import os
import re

import torch

from parity_util import TOL

HERE = os.path.dirname(os.path.abspath(__file__))


def test_parity_bars_are_the_stated_ones():
    assert TOL == {torch.float32: 1e-4, torch.bfloat16: 5e-3}


def test_no_test_module_defines_its_own_bar():
    for name in sorted(os.listdir(HERE)):
        if not name.endswith(".py") or name == "parity_util.py":
            continue
        text = open(os.path.join(HERE, name)).read()
        assert not re.search(r"^\s*TOL\s*=", text, flags=re.M), f"{name} defines its own TOL"

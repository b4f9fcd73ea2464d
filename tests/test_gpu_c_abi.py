"""The C ABI driven from plain C (tests/c_abi/flce_c_driver.c): forward and
backward through device pointers from cudaMalloc, no PyTorch in the process,
checked against the float64 oracle."""
import subprocess

import numpy as np
import pytest

import flce_inputs as fi
import oracle
from tests import _c_driver
from tests import _gpu as G

pytestmark = pytest.mark.gpu
IGN = fi.IGNORE_INDEX


@pytest.mark.parametrize("softcap,reduction", [(0.0, "sum"), (2.0, "mean")])
def test_c_caller_matches_oracle(tmp_path, softcap, reduction):
    inp = G.small_inputs(N=300, H=128, V=1000, seed=27, n_ign=40, w_std=0.1)
    exe = _c_driver.build_driver(str(tmp_path))
    fin, fout = str(tmp_path / "in.bin"), str(tmp_path / "out.bin")
    _c_driver.write_input(fin, inp.hidden_bits, inp.weight_bits, inp.labels, IGN, softcap, 0.5,
                          0 if reduction == "sum" else 1)
    res = subprocess.run([exe, fin, fout], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr
    got = _c_driver.read_output(fout, 300, 128, 1000)
    assert got["status"] == 0
    rf = oracle.forward(inp.hidden, inp.weight, inp.labels, IGN, softcap, reduction)
    rb = oracle.backward(inp.hidden, inp.weight, inp.labels, IGN, softcap, reduction,
                         grad_scale=0.5)
    assert got["ntok"] == rf["num_tokens"]
    G.check_loss(got["loss"], rf["loss"])
    G.check_lse(got["lse"], rf["lse"], inp.labels, 1000)
    assert np.all(got["dh"][inp.labels == IGN] == 0.0)
    assert G.rel_l2(got["dh"], rb["d_hidden"]) <= G.GRAD_RL2
    assert G.rel_l2(got["dw"], rb["d_weight"]) <= G.GRAD_RL2

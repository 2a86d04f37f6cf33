"""The C ABI from C: the header compiles as C99 on its own, a plain-C program
builds against it and libsfn.so (CPU), and on a GPU that program's output
matches the oracle (parity rules of tests/parity.py)."""
import os
import subprocess

import numpy as np
import pytest

import c_demo
from predictor_gated_channel_b200 import build as sfn_build

ROOT = c_demo.ROOT


def test_header_compiles_as_c99(tmp_path):
    src = tmp_path / "h.c"
    src.write_text('#include "sfn.h"\nint main(void) { return sfn_abi_version() > 0 ? 0 : 1; }\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-I",
                    os.path.join(ROOT, "include"), str(src)], check=True)


def test_c_demo_builds(tmp_path):
    sfn_build.build()
    exe = c_demo.build_demo(str(tmp_path / "abi_demo"))
    assert os.path.exists(exe)


@pytest.mark.gpu
def test_c_demo_matches_oracle(tmp_path):
    import oracle
    import parity
    from predictor_gated_channel_b200.inputs import WORKLOADS, make_layer, make_tokens

    sfn_build.build()
    exe = c_demo.build_demo(str(tmp_path / "abi_demo"))
    wl = WORKLOADS["tiny"]
    layer = make_layer(wl)
    x = make_tokens(wl)
    inp = tmp_path / "in.bin"
    with open(inp, "wb") as f:
        f.write(np.array([wl.T, wl.d, wl.d_i, wl.r, wl.bank, wl.k], np.int64).tobytes())
        for a in (x, layer["A"], layer["B"], layer["Wg"], layer["Wu"], layer["Wd"]):
            f.write(a.numpy().astype(np.float32).tobytes())
    out = tmp_path / "out.bin"
    subprocess.run([exe, str(inp), str(out)], check=True)
    raw = out.read_bytes()
    ny = wl.T * wl.d * 4
    y = np.frombuffer(raw[:ny], np.float32).reshape(wl.T, wl.d).astype(np.float64)
    mask = np.frombuffer(raw[ny:], np.uint64).reshape(wl.T, wl.n_banks)
    logits = oracle.predict(x, layer["A"], layer["B"])
    parity.check_mask(mask, logits, wl.bank, wl.k)
    ref = oracle.forward_given_mask(x, logits, mask, layer["Wg"], layer["Wu"], layer["Wd"],
                                    wl.bank)
    assert parity.y_error(y, ref) <= parity.Y_TOL["f32"]

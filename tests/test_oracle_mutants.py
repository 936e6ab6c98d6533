"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that
the pins catch every one of them: a dropped term, a wrong sign or index, a
transposed operand, a missing scale, reading before writing."""
import os
import re
import subprocess
import tempfile

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

MUTANTS = {
    "drop_decay": ("S[r * dk + c] *= alpha[c];", "(void)0;"),
    "decay_on_value_index": ("S[r * dk + c] *= alpha[c];", "S[r * dk + c] *= alpha[r % dk];"),
    "error_sign": ("e[r] = bt * (vt[r] - vhat[r]);", "e[r] = bt * (vhat[r] - vt[r]);"),
    "drop_beta": ("e[r] = bt * (vt[r] - vhat[r]);", "e[r] = (vt[r] - vhat[r]);"),
    "write_with_query": ("S[r * dk + c] += e[r] * kt[c];", "S[r * dk + c] += e[r] * qt[c];"),
    "missing_scale": ("acc += S[r * dk + c] * (scale * qt[c]);", "acc += S[r * dk + c] * qt[c];"),
    "read_with_key": ("acc += S[r * dk + c] * (scale * qt[c]);", "acc += S[r * dk + c] * (scale * kt[c]);"),
    "gate_sign": ("alpha[c] = exp(g[(row * H + h) * dk + c]);", "alpha[c] = exp(-g[(row * H + h) * dk + c]);"),
    "gate_previous_token": ("alpha[c] = exp(g[(row * H + h) * dk + c]);",
                            "alpha[c] = exp(g[((row > start ? row - 1 : row) * H + h) * dk + c]);"),
    "ignore_S0": ("if (S0) memcpy(S, S0, sizeof(double) * (size_t)dv * dk);", "if (0) (void)S0;"),
    "value_heads_interleaved": ("const int hk = h / (H / Hk);", "const int hk = h % Hk;"),
    "value_heads_ignored": ("const int hk = h / (H / Hk);", "const int hk = 0;"),
    "predict_before_decay": (None, None),
    "read_before_write": (None, None),
}


def _mutate(src, name):
    old, new = MUTANTS[name]
    if name == "predict_before_decay":
        # move the forget loop after the predict step
        forget = re.search(r"        /\* 1\. forget.*?\n(.*?\n.*?\n)", src, re.S)
        block = forget.group(0)
        src = src.replace(block, "")
        return src.replace("        /* 3. correct", block + "        /* 3. correct")
    if name == "read_before_write":
        read = re.search(r"        /\* 5\. read.*?\n        }\n", src, re.S).group(0)
        src = src.replace(read, "")
        return src.replace("        /* 4. write", read + "        /* 4. write")
    assert old in src, name
    return src.replace(old, new)


@pytest.fixture(scope="module")
def src():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(src, name, tmp_path):
    msrc = _mutate(src, name)
    assert msrc != src
    c = tmp_path / "mut.c"
    so = tmp_path / "libmut.so"
    c.write_text(msrc)
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so),
                           str(c), "-lm"])
    lib = oracle.bind(str(so))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"

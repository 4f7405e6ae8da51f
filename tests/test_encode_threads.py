"""The host encoder splits its passes over threads; its output must not
depend on the thread count.  Each count runs in a fresh process (the count is
read once per process from UW_ENCODE_THREADS) and compares against the
oracle's encoding byte for byte."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys
import numpy as np
sys.path.insert(0, ROOT)
from mlp_huffman_coded_b200 import synth, uw
from oracle import uw_oracle as O

def cases():
    yield synth.weight_matrix(256, 512, 0.02, 5e-4, 200.0, 0)
    yield synth.weight_matrix(203, 192, 0.02, 2e-3, 100.0, 3)       # ragged rows
    yield synth.weight_matrix(128, 640, 0.02, 3e-2, 300.0, 4)       # many verbatim groups
    w = synth.weight_matrix(64, 128, 0.02, 0.0, 1.0, 5)
    for i in range(64):
        w[i, i % 128] = np.uint16((150 + i) << 7)                   # every group verbatim
    yield w
    yield np.full((96, 256), 0x3F80, dtype=np.uint16)               # one symbol only
    yield synth.all_patterns_matrix()

for w in cases():
    e = uw.encode(w, chunk_groups=3)
    o = O.encode(w, chunk_groups=3)
    assert np.array_equal(e.sm.ravel(), o.sm.ravel()), "sm"
    assert np.array_equal(e.stream, o.stream), "stream"
    assert np.array_equal(e.chunk_bit_off, o.chunk_bit_off)
    assert np.array_equal(e.vflags.ravel(), o.vflags.ravel())
    assert np.array_equal(e.vprefix, o.vprefix)
    assert np.array_equal(e.verbatim.reshape(-1), o.verbatim.reshape(-1))
    assert [int(v) for v in e.cb.palette] == [int(v) for v in o.cb.palette]
print("ok")
"""


@pytest.mark.parametrize("threads", [2, 3, 7, 13])
def test_encoder_output_does_not_depend_on_threads(threads):
    env = dict(os.environ, UW_ENCODE_THREADS=str(threads))
    res = subprocess.run([sys.executable, "-c", SCRIPT.replace("ROOT", repr(ROOT))], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-3000:]
    assert res.stdout.strip().endswith("ok")

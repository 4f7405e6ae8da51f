"""Property tests over random matrices (hypothesis, CPU): the oracle's
decode of its encoding gives back W bit for bit, the verbatim rule holds,
the code satisfies Kraft equality, and the library's encoder writes the
oracle's bytes.  Shapes, value spreads, outlier rates and chunk sizes vary."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from mlp_huffman_coded_b200 import uw
from oracle import uw_oracle as O


@st.composite
def matrices(draw):
    rows = draw(st.integers(1, 40))
    cols = 64 * draw(st.integers(1, 6))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    kind = draw(st.sampled_from(["normal", "wide", "bits", "few"]))
    if kind == "bits":  # arbitrary BF16 bit patterns (NaN payloads, Inf, subnormals, zeros)
        return rng.integers(0, 1 << 16, size=(rows, cols), dtype=np.uint16)
    if kind == "few":   # a handful of distinct exponents (degenerate palettes)
        e = rng.integers(100, 100 + draw(st.integers(1, 5)), size=(rows, cols))
        s = rng.integers(0, 2, size=(rows, cols))
        m = rng.integers(0, 128, size=(rows, cols))
        return ((s << 15) | (e << 7) | m).astype(np.uint16)
    sigma = 0.02 if kind == "normal" else 10.0 ** draw(st.integers(-4, 2))
    w = rng.standard_normal((rows, cols)).astype(np.float32) * np.float32(sigma)
    rate = draw(st.sampled_from([0.0, 1e-3, 3e-2]))
    mask = rng.random((rows, cols)) < rate
    w[mask] *= np.float32(draw(st.sampled_from([50.0, 1e4])))
    bits = w.view(np.uint32)
    rounded = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16  # round to nearest even
    return rounded.astype(np.uint16)


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(w=matrices(), chunk_groups=st.integers(1, 16))
def test_round_trip_verbatim_rule_kraft_and_library_bytes(w, chunk_groups):
    enc = O.encode(w, chunk_groups=chunk_groups)
    assert np.array_equal(O.decode_full(enc), w)
    # verbatim rule: flagged <=> some exponent of the group is outside the palette
    pal = set(int(v) for v in enc.cb.palette)
    exps = ((w >> 7) & 0xFF).reshape(w.shape[0], -1, 64)
    want = np.array([[any(int(e) not in pal for e in g) for g in row] for row in exps])
    assert np.array_equal(O.verbatim_groups(w, enc.cb.palette), want)
    used = [int(l) for l in enc.cb.lengths if l > 0]
    if len(used) >= 2:
        assert O.kraft_sum(used) == 1.0
    lib = uw.encode(w, chunk_groups=chunk_groups)
    assert np.array_equal(lib.stream, enc.stream)
    assert np.array_equal(lib.chunk_bit_off, enc.chunk_bit_off)
    assert np.array_equal(lib.sm.ravel(), enc.sm.ravel())
    assert np.array_equal(lib.vflags.ravel(), enc.vflags.ravel())
    assert np.array_equal(lib.verbatim.reshape(-1), enc.verbatim.reshape(-1))

"""Pins for the CPU oracle: values and properties fixed by the Unweight page
and by mathematics, independent of the oracle's own code.

Each check is a function of the oracle module so that the mutation tests at
the bottom can run it against a deliberately broken copy of the oracle and
see it fail.
"""
import math
import os
import types

import numpy as np
import pytest

from mlp_huffman_coded_b200 import synth
from oracle import uw_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = v.split()
    return out


def bits_to_words(bits: str, pad: int = 2):
    n = -(-len(bits) // 32)
    bits = bits.ljust(32 * n, "0")
    return [int(bits[32 * i:32 * i + 32], 2) for i in range(n)] + [0] * pad


# ---------------------------------------------------------------------------
# golden worked examples
# ---------------------------------------------------------------------------

def golden_1x64_matrix(g):
    pattern = [int(v) for v in g["pattern"]]
    k = np.arange(64)
    exp = np.array([pattern[i % 8] for i in k], dtype=np.uint16)
    mant = ((5 * k) % 128).astype(np.uint16)
    sign = (k % 3 == 0).astype(np.uint16)
    return ((sign << 15) | (exp << 7) | mant).astype(np.uint16).reshape(1, 64)


def check_golden_huffman(orc):
    g = read_golden("huffman_1x64.txt")
    w = golden_1x64_matrix(g)
    enc = orc.encode(w, chunk_groups=4)
    assert [int(v) for v in enc.cb.palette] == [int(v) for v in g["palette"]]
    assert [int(v) for v in enc.cb.freqs] == [int(v) for v in g["freqs"]]
    assert [int(v) for v in enc.cb.lengths] == [int(v) for v in g["lengths"]]
    codes = [format(int(enc.cb.codes[i]), "0%db" % int(enc.cb.lengths[i])) for i in range(4)]
    assert codes == g["codes"]
    bits = g["bits8"][0] * 8
    assert enc.total_bits == int(g["total_bits"][0]) == len(bits)
    assert [int(v) for v in enc.stream] == bits_to_words(bits)
    assert [int(v) for v in enc.chunk_bit_off] == [0, len(bits)]
    assert enc.n_verbatim == 0
    assert np.array_equal(orc.decode_full(enc, lockstep=False), w)
    assert np.array_equal(orc.decode_full(enc, lockstep=True), w)
    lengths = [int(v) for v in g["canonical_case_lengths"]]
    codes = orc.canonical_codes(lengths)
    got = [format(int(codes[i]), "0%db" % lengths[i]) for i in range(len(lengths))]
    assert got == g["canonical_case_codes"]


def golden_2x128_matrix():
    r = np.arange(2)[:, None]
    c = np.arange(128)[None, :]
    exp = (100 + (c % 16)) * np.ones_like(r)
    exp = exp.astype(np.uint16)
    exp[1, 5] = 50
    mant = (c % 128).astype(np.uint16) * np.ones_like(r, dtype=np.uint16)
    return ((exp << 7) | mant).astype(np.uint16)


def check_golden_verbatim(orc):
    g = read_golden("verbatim_2x128.txt")
    w = golden_2x128_matrix()
    enc = orc.encode(w, chunk_groups=1)
    assert [int(v) for v in enc.cb.palette] == [int(v) for v in g["palette"]]
    assert enc.n_verbatim == 1
    assert [int(v) for v in enc.vflags.ravel()] == [int(v) for v in g["vflags"]]
    assert [int(v) for v in enc.vprefix] == [int(v) for v in g["vprefix"]]
    assert np.array_equal(enc.verbatim[0], w[1, :64])
    assert [int(v) for v in enc.cb.lengths] == [int(v) for v in g["lengths"]]
    per_group = [int(v, 16) for v in g["stream_words_per_group"]]
    assert [int(v) for v in enc.stream] == per_group * 3 + [0, 0]
    assert [int(v) for v in enc.chunk_bit_off] == [int(v) for v in g["chunk_bit_off"]]
    idx4 = orc.transcode_palette(enc, lockstep=False)
    assert [int(v) for v in idx4[0, :4]] == [int(v, 16) for v in g["idx4_row0_first4"]]
    assert (idx4[1, :32] == 0).all()
    assert np.array_equal(orc.decode_full(enc, lockstep=False), w)


def check_golden_sm(orc):
    g = read_golden("sm_layout.txt")
    w = np.array([[int(v, 16) for v in g["words"]]], dtype=np.uint16)
    assert [int(v) for v in orc.sm_bytes(w)[0]] == [int(v, 16) for v in g["sm"]]


def test_golden_huffman_1x64():
    check_golden_huffman(O)


def test_golden_verbatim_2x128():
    check_golden_verbatim(O)


def test_golden_sm_layout():
    check_golden_sm(O)


# ---------------------------------------------------------------------------
# lossless round trip ("bit-identical outputs": section "Key Points" /
# article introduction of the Unweight page)
# ---------------------------------------------------------------------------

def check_round_trip(orc, w, chunk_groups=4):
    enc = orc.encode(w, chunk_groups=chunk_groups)
    assert np.array_equal(orc.decode_full(enc, lockstep=False), w)
    assert np.array_equal(orc.decode_full(enc, lockstep=True), w)
    exp = ((w >> 7) & 0xFF).astype(np.uint8)
    assert np.array_equal(orc.decode_exponent_only(enc, lockstep=False), exp)
    idx4 = orc.transcode_palette(enc, lockstep=False)
    assert np.array_equal(orc.rebuild_from_idx4(enc, idx4), w)
    return enc


def test_round_trip_small_config():
    p = synth.WORKLOADS["small_256x512"]
    w = synth.weight_matrix(p["rows"], p["cols"], p["sigma"], p["outlier_rate"], p["outlier_scale"], p["seed"])
    enc = check_round_trip(O, w)
    # verbatim groups and longest code of this exact generator (seed 0), worked out
    # independently of the oracle when the workload was specified
    assert enc.n_verbatim == 66 and enc.n_groups == 2048 and enc.cb.max_len == 12


def test_round_trip_every_bf16_pattern():
    w = synth.all_patterns_matrix()
    enc = check_round_trip(O, w, chunk_groups=3)
    # every exponent occurs 256 times: palette = exponents 0..15 (value order)
    assert [int(v) for v in enc.cb.palette] == list(range(16))


def test_round_trip_special_values_only():
    # only exponents 0 and 255: +-0, subnormals, +-Inf, NaN payloads
    rng = np.random.default_rng(3)
    mant = rng.integers(0, 128, size=(8, 128)).astype(np.uint16)
    sign = rng.integers(0, 2, size=(8, 128)).astype(np.uint16)
    exp = np.where(rng.random((8, 128)) < 0.7, 0, 255).astype(np.uint16)
    w = ((sign << 15) | (exp << 7) | mant).astype(np.uint16)
    enc = check_round_trip(O, w)
    assert enc.n_verbatim == 0
    assert enc.cb.n_symbols == 2 and sorted(enc.cb.lengths[enc.cb.lengths > 0]) == [1, 1]


@pytest.mark.parametrize("chunk_groups", [1, 2, 4, 5, 64])
def test_round_trip_chunk_sizes(chunk_groups):
    w = synth.weight_matrix(64, 640, 0.03, 2e-3, 300.0, 11)
    check_round_trip(O, w, chunk_groups=chunk_groups)


def test_ragged_rows_and_partial_last_chunk():
    w = synth.weight_matrix(3, 192, 0.02, 1e-2, 100.0, 5)   # 9 groups, chunks of 4
    enc = check_round_trip(O, w, chunk_groups=4)
    assert enc.n_chunks == 3 and enc.chunk_bit_off.size == 4


# ---------------------------------------------------------------------------
# the verbatim rule (section "How to compress model weights effectively")
# ---------------------------------------------------------------------------

def check_verbatim_invariant(orc, w):
    enc = orc.encode(w)
    pal = set(int(v) for v in enc.cb.palette)
    rows, cols = w.shape
    for r in range(rows):
        for gi in range(cols // 64):
            grp = w[r, gi * 64:(gi + 1) * 64]
            outside = any(((int(v) >> 7) & 0xFF) not in pal for v in grp)
            flag = (int(enc.vflags[r, gi // 32]) >> (gi % 32)) & 1
            assert bool(flag) == outside, (r, gi)
    # flag count, prefix total and store size agree
    assert int(enc.vprefix[-1]) == enc.n_verbatim == int(sum(bin(int(v)).count("1") for v in enc.vflags.ravel()))


def test_verbatim_invariant_brute_force():
    check_verbatim_invariant(O, synth.weight_matrix(16, 256, 0.02, 3e-3, 200.0, 9))


def test_at_most_16_exponents_means_no_verbatim_rows():
    rng = np.random.default_rng(4)
    exp = rng.choice(np.arange(100, 116), size=(32, 256)).astype(np.uint16)
    w = ((exp << 7) | rng.integers(0, 128, size=exp.shape).astype(np.uint16)).astype(np.uint16)
    assert O.encode(w).n_verbatim == 0


def test_one_group_with_a_17th_exponent():
    rng = np.random.default_rng(5)
    exp = rng.choice(np.arange(100, 116), size=(4, 256)).astype(np.uint16)
    exp[2, 130] = 7                                   # row 2, group 2
    w = (exp << 7).astype(np.uint16)
    enc = O.encode(w)
    assert enc.n_verbatim == 1
    assert int(enc.vflags[2, 0]) == 1 << 2 and int(enc.vflags.sum()) == 1 << 2


def test_all_verbatim_matrix_has_empty_stream():
    # 17 rows; row r is exponent 10+r everywhere except one element with
    # exponent 100+r.  Counts: 10..26 -> 63 each, 100..116 -> 1 each.
    # Palette = 10..25; row 16 (exponent 26) and every row's 100+r element
    # fall outside, so every group is verbatim and the stream is empty.
    w = np.zeros((17, 64), dtype=np.uint16)
    for r in range(17):
        w[r, :] = (10 + r) << 7
        w[r, 7] = (100 + r) << 7
    enc = O.encode(w)
    assert enc.n_verbatim == enc.n_groups == 17
    assert enc.total_bits == 0 and [int(v) for v in enc.stream] == [0, 0]
    assert enc.cb.n_symbols == 0
    check_round_trip(O, w)


# ---------------------------------------------------------------------------
# palette (section "How to compress model weights effectively")
# ---------------------------------------------------------------------------

def test_palette_is_top16_by_count_then_value():
    counts = {e: 0 for e in range(256)}
    rng = np.random.default_rng(6)
    vals = []
    for e, c in [(120, 50), (121, 50), (90, 49), (3, 49)] + [(200 + i, 10) for i in range(20)]:
        vals += [e] * c
        counts[e] += c
    vals = np.array(vals, dtype=np.uint16)
    vals = np.concatenate([vals, np.full((-vals.size) % 64, 120, dtype=np.uint16)])
    counts[120] += (-len(vals)) % 64
    rng.shuffle(vals)
    w = (vals << 7).astype(np.uint16).reshape(1, -1)
    brute = sorted(counts, key=lambda e: (-counts[e], e))[:16]
    assert [int(v) for v in O.build_palette(w)] == brute
    # 120 and 121 tie -> 120 first; 90 and 3 tie -> 3 first; then 200..211
    assert [int(v) for v in O.build_palette(w)[:4]] == [120, 121, 3, 90]


def test_palette_with_fewer_than_16_exponents_fills_unused_ascending():
    w = (np.array([5, 5, 9, 2] * 16, dtype=np.uint16) << 7).reshape(1, 64)
    assert [int(v) for v in O.build_palette(w)] == [5, 2, 9, 0, 1, 3, 4, 6, 7, 8, 10, 11, 12, 13, 14, 15]


# ---------------------------------------------------------------------------
# Huffman optimality (textbook properties)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(12))
def test_huffman_matches_brute_force_optimum(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 7 if seed < 10 else 8))
    f = rng.integers(1, 50, size=n)
    lengths = O.huffman_code_lengths(f)
    assert int((f * lengths).sum()) == O.brute_force_optimal_cost(f)


@pytest.mark.parametrize("seed", range(8))
def test_kraft_equality_and_shannon_bounds(seed):
    rng = np.random.default_rng(200 + seed)
    n = int(rng.integers(2, 17))
    f = np.zeros(16, dtype=np.int64)
    f[:n] = rng.geometric(0.3, size=n) * rng.integers(1, 1000, size=n)
    lengths = O.huffman_code_lengths(f)
    assert O.kraft_sum(lengths) == 1.0
    p = f[f > 0] / f.sum()
    H = float(-(p * np.log2(p)).sum())
    mean = float((f * lengths).sum() / f.sum())
    assert H - 1e-12 <= mean < H + 1
    assert lengths.max() <= 15


def test_canonical_codes_are_prefix_free_and_ordered():
    f = np.array([40, 30, 10, 10, 5, 3, 1, 1, 0, 0, 0, 0, 0, 0, 0, 0])
    lengths = O.huffman_code_lengths(f)
    codes = O.canonical_codes(lengths)
    words = [format(int(codes[i]), "0%db" % int(lengths[i])) for i in range(16) if lengths[i] > 0]
    for a in words:
        for b in words:
            if a != b:
                assert not b.startswith(a)
    order = sorted((int(lengths[i]), i) for i in range(16) if lengths[i] > 0)
    vals = [int(codes[i]) << (16 - int(lengths[i])) for _, i in order]
    assert vals == sorted(vals) and len(set(vals)) == len(vals)


def test_single_symbol_gets_length_one():
    w = np.full((2, 64), 120 << 7, dtype=np.uint16)
    enc = O.encode(w)
    assert int(enc.cb.lengths[0]) == 1 and int(enc.cb.codes[0]) == 0
    assert enc.total_bits == 128 and not enc.stream.any()
    check_round_trip(O, w)


# ---------------------------------------------------------------------------
# the page's numbers on a trained-weight-like distribution (section "How to
# compress model weights effectively": top-16 covers >99%, ~2.6 bits;
# article introduction: ~30% smaller MLP weights)
# ---------------------------------------------------------------------------

def test_page_numbers_on_synthetic_gaussian_weights():
    w = synth.weight_matrix(2048, 2048, 0.02, 1e-4, 100.0, 1)
    enc = O.encode(w)
    assert O.palette_coverage(w, enc.cb.palette) > 0.99
    H = O.symbol_entropy_bits(enc.cb)
    mean = O.mean_code_bits(enc.cb)
    assert H <= mean < H + 1
    assert abs(mean - 2.6) < 0.15
    assert abs(O.exponent_entropy_bits(w) - 2.6) < 0.15
    saving = 1 - enc.huffman_form_bytes() / w.nbytes
    assert 0.25 <= saving <= 0.35


# ---------------------------------------------------------------------------
# decoder robustness
# ---------------------------------------------------------------------------

def test_wrong_chunk_offsets_are_detected():
    w = synth.weight_matrix(8, 256, 0.02, 0.0, 1.0, 12)
    enc = O.encode(w)
    enc.chunk_bit_off = enc.chunk_bit_off.copy()
    enc.chunk_bit_off[1] += 1
    with pytest.raises(ValueError):
        O.decode_indices(enc)
    with pytest.raises(ValueError):
        O.decode_indices_lockstep(enc)


# ---------------------------------------------------------------------------
# GEMM and MLP block (plain definitions, brute force on tiny inputs)
# ---------------------------------------------------------------------------

def test_gemm_brute_force_tiny():
    w = synth.weight_matrix(5, 64, 0.5, 0.0, 1.0, 13)
    x = synth.activations(3, 64, 14)
    wf = synth.bf16_bits_to_f32(w).astype(float)
    xf = synth.bf16_bits_to_f32(x).astype(float)
    y = O.gemm(w, x)
    for b in range(3):
        for n in range(5):
            s = math.fsum(float(wf[n, k]) * float(xf[b, k]) for k in range(64))
            assert abs(y[b, n] - s) <= 1e-12 * max(1.0, abs(s))


def test_gemm_one_hot_selects_a_column():
    w = synth.weight_matrix(16, 128, 0.02, 1e-2, 100.0, 15)
    x = np.zeros((1, 128), dtype=np.uint16)
    x[0, 77] = 0x3F80                                 # 1.0
    assert np.array_equal(O.gemm(w, x)[0], synth.bf16_bits_to_f32(w[:, 77]).astype(np.float64))


def test_gemm_small_integers_exact():
    w = synth.small_integer_matrix(8, 256, -8, 8, 16)
    x = synth.small_integer_matrix(2, 256, -8, 8, 17)
    wi = synth.bf16_bits_to_f32(w).astype(np.int64)
    xi = synth.bf16_bits_to_f32(x).astype(np.int64)
    assert np.array_equal(O.gemm(w, x), (xi @ wi.T).astype(np.float64))


def test_mlp_block_brute_force_tiny():
    g = synth.weight_matrix(6, 64, 0.2, 0.0, 1.0, 18)
    u = synth.weight_matrix(6, 64, 0.2, 0.0, 1.0, 19)
    d = synth.weight_matrix(4, 6, 0.2, 0.0, 1.0, 20)
    x = synth.activations(2, 64, 21)
    gf, uf, df, xf = (synth.bf16_bits_to_f32(a).astype(float) for a in (g, u, d, x))
    y = O.mlp_block(g, u, d, x)
    for b in range(2):
        h = []
        for j in range(6):
            gj = math.fsum(gf[j, k] * xf[b, k] for k in range(64))
            uj = math.fsum(uf[j, k] * xf[b, k] for k in range(64))
            h.append(O.silu_scalar(gj) * uj)
        for n in range(4):
            s = math.fsum(df[n, j] * h[j] for j in range(6))
            assert abs(y[b, n] - s) <= 1e-12 * max(1.0, abs(s))


def test_silu_closed_forms():
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert abs(O.silu(np.array([30.0]))[0] - 30.0) < 1e-9
    assert abs(O.silu(np.array([-30.0]))[0]) < 1e-9
    assert abs(O.silu(np.array([1.0]))[0] - 1.0 / (1.0 + math.e ** -1)) < 1e-15


# ---------------------------------------------------------------------------
# mutation tests: plausible oracle mistakes must fail a pin
# ---------------------------------------------------------------------------

def mutated(**overrides):
    m = types.ModuleType("uw_oracle_mutant")
    m.__dict__.update(O.__dict__)
    m.__dict__.update(overrides)
    # functions look globals up in their own module dict: rebind them
    for name, obj in list(m.__dict__.items()):
        if isinstance(obj, types.FunctionType) and obj.__module__ == O.__name__:
            m.__dict__[name] = types.FunctionType(obj.__code__, m.__dict__, obj.__name__,
                                                  obj.__defaults__, obj.__closure__)
    for k, v in overrides.items():
        m.__dict__[k] = v
    return m


def _codes_by_index_only(lengths):
    codes = np.zeros(len(lengths), dtype=np.int64)
    code, prev = 0, None
    for i, l in enumerate(lengths):
        if l > 0:
            if prev is not None:
                code <<= max(int(l) - prev, 0)
            codes[i] = code
            code += 1
            prev = int(l)
    return codes


def _palette_ties_by_value_desc(w):
    counts = O.exponent_histogram(w)
    order = sorted(range(256), key=lambda e: (-int(counts[e]), -e))
    return np.array(order[:16], dtype=np.uint8)


def _sm_own_sign(w2d):
    sign, _, mant = O.fields(w2d)
    return ((mant << 1) | sign).astype(np.uint8)


def _pack_lsb_first(values, lengths, extra_words=2):
    words, total = O.pack_bits_msb_first(values, lengths, extra_words)
    rev = np.array([int(format(int(v), "032b")[::-1], 2) for v in words], dtype=np.uint32)
    return rev, total


@pytest.mark.parametrize("mutation,check", [
    (dict(canonical_codes=_codes_by_index_only), check_golden_huffman),
    (dict(build_palette=_palette_ties_by_value_desc), check_golden_verbatim),
    (dict(sm_bytes=_sm_own_sign), check_golden_sm),
    (dict(pack_bits_msb_first=_pack_lsb_first), check_golden_huffman),
    (dict(GROUP=32), check_golden_verbatim),
])
def test_pins_catch_planted_mistakes(mutation, check):
    m = mutated(**mutation)
    with pytest.raises(Exception):
        check(m)

"""The per-element GEMM tolerance of the GPU tests rests on a BF16 rounding
function written from the definition of the format; pin it to the seeded
input generator's own float32 -> BF16 conversion and to hand-worked ties."""
import numpy as np

from mlp_huffman_coded_b200 import synth
from oracle import uw_oracle as O

from gpu_util import bf16_round, within_tol


def test_bf16_round_matches_float32_conversion():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    got = bf16_round(v.astype(np.float64))
    ref = O.bf16_to_f64(synth.f32_to_bf16_bits(v))
    assert np.array_equal(got, ref)


def test_bf16_round_ties_go_to_even():
    # the BF16 ulp at 1 is 2^-7: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    assert bf16_round(1 + 2.0 ** -8) == 1.0
    assert bf16_round(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    assert bf16_round(-(1 + 3 * 2.0 ** -8)) == -(1 + 2.0 ** -6)
    assert bf16_round(1 + 2.0 ** -8 + 2.0 ** -30) == 1 + 2.0 ** -7
    assert bf16_round(0.0) == 0.0


def test_within_tol_allows_the_rounding_distance_and_no_more():
    y_ref = np.array([[100.0 + 0.4, 1.0, -1.0, 0.5]])
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    # 100.4 -> nearest BF16 is 100.5 (ulp 0.5 in [64, 128))
    y = synth.f32_to_bf16_bits(np.array([[100.5, 1.0, -1.0, 0.5]], dtype=np.float32))
    assert within_tol(y, y_ref, tol=0.0)[0]
    # one ulp further is out unless the accumulation term allows it
    y_bad = synth.f32_to_bf16_bits(np.array([[101.0, 1.0, -1.0, 0.5]], dtype=np.float32))
    assert not within_tol(y_bad, y_ref, tol=0.0)[0]
    assert within_tol(y_bad, y_ref, acc=np.full_like(y_ref, 0.6), tol=0.0)[0]
    assert within_tol(y_bad, y_ref, tol=0.6 / rms)[0]

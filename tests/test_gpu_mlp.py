"""GPU parity of the SwiGLU glue, the MLP block and the autotuner."""
import numpy as np
import pytest

from mlp_huffman_coded_b200 import synth
from mlp_huffman_coded_b200 import uw
from oracle import uw_oracle as O

from gpu_util import device_matrix, empty_bf16, mlp_check, to_dev, to_host_u16

pytestmark = pytest.mark.gpu


def test_swiglu_kernel_against_float64():
    rng = np.random.default_rng(60)
    g = synth.f32_to_bf16_bits(rng.standard_normal(10007, dtype=np.float32) * 4)
    u = synth.f32_to_bf16_bits(rng.standard_normal(10007, dtype=np.float32))
    h = empty_bf16(10007)
    uw.swiglu(to_dev(g), to_dev(u), h)
    ref = O.silu(O.bf16_to_f64(g)) * O.bf16_to_f64(u)
    got = O.bf16_to_f64(to_host_u16(h))
    # one BF16 rounding of an FP32 result: relative 2^-8, plus FP32 slack
    assert np.all(np.abs(got - ref) <= 2 ** -8 * np.abs(ref) + 1e-30)


def _block(d, ffn, seed):
    gate = synth.weight_matrix(ffn, d, 0.02, 1e-3, 100.0, seed)
    up = synth.weight_matrix(ffn, d, 0.02, 1e-3, 100.0, seed + 10)
    down = synth.weight_matrix(d, ffn, 0.02, 1e-3, 100.0, seed + 20)
    return gate, up, down


@pytest.mark.parametrize("B", [1, 8, 33, 100, 200])
def test_mlp_block_small(B):
    gate, up, down = _block(512, 1536, 61)
    dms = [device_matrix(m) for m in (gate, up, down)]
    x = synth.activations(B, 512, 62)
    outs = []
    for pipes in ([3, 3, 3], [0, 1, 2], [2, 3, 0], [1, 1, 1]):
        ws = uw.Workspace(uw.mlp_workspace_bytes(*dms, pipes, B))
        y = empty_bf16(B, 512)
        uw.mlp_block(*dms, pipes, to_dev(x), y, ws)
        ws.check("mlp")
        ok, err, rms = mlp_check(to_host_u16(y), gate, up, down, x)
        assert ok, (pipes, err, rms)
        outs.append(to_host_u16(y))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_fused_swiglu_epilogue_equals_separate_kernels():
    gate, up, down = _block(256, 1024, 63)
    dms = [device_matrix(m) for m in (gate, up, down)]
    B = 6
    x = to_dev(synth.activations(B, 256, 64))
    ws = uw.Workspace(uw.mlp_workspace_bytes(*dms, [3, 3, 3], B))
    y = empty_bf16(B, 256)
    uw.mlp_block(*dms, [3, 3, 3], x, y, ws)
    g, u, h, y2 = empty_bf16(B, 1024), empty_bf16(B, 1024), empty_bf16(B, 1024), empty_bf16(B, 256)
    uw.gemm_direct_palette(dms[0], x, g, ws)
    uw.gemm_direct_palette(dms[1], x, u, ws)
    uw.swiglu(g, u, h)
    uw.gemm_direct_palette(dms[2], h, y2, ws)
    ws.check()
    assert np.array_equal(to_host_u16(y), to_host_u16(y2))


@pytest.mark.parametrize("B", [4, 40])
def test_block_with_heavy_verbatim_and_ragged_rows(B):
    """Direct-palette block whose gate and up tiles carry many verbatim rows
    (some beyond the rows staged on chip) and whose hidden size (1088) leaves
    a partial last row tile.  It must equal the exponent-only pipeline bit
    for bit and meet the MLP bar against the float64 oracle."""
    d, ffn = 512, 1088
    gate = synth.weight_matrix(ffn, d, 0.02, 2e-2, 300.0, 67)
    up = synth.weight_matrix(ffn, d, 0.02, 2e-2, 300.0, 68)
    down = synth.weight_matrix(d, ffn, 0.02, 1e-3, 100.0, 69)
    dms = [device_matrix(m) for m in (gate, up, down)]
    x = synth.activations(B, d, 70)
    outs = []
    for pipes in ([3, 3, 3], [1, 1, 3]):
        ws = uw.Workspace(uw.mlp_workspace_bytes(*dms, pipes, B))
        y = empty_bf16(B, d)
        uw.mlp_block(*dms, pipes, to_dev(x), y, ws)
        ws.check("mlp")
        outs.append(to_host_u16(y))
    assert np.array_equal(outs[0], outs[1])
    ok, err, rms = mlp_check(outs[0], gate, up, down, x)
    assert ok, (err, rms)


def test_full_size_mlp_block_batch8():
    gate, up, down = synth.mlp_block()
    dms = [device_matrix(m) for m in (gate, up, down)]
    x = synth.activations(8, 4096, 3)
    ws = uw.Workspace(uw.mlp_workspace_bytes(*dms, [3, 3, 3], 8))
    y = empty_bf16(8, 4096)
    uw.mlp_block(*dms, [3, 3, 3], to_dev(x), y, ws)
    ws.check()
    ok, err, rms = mlp_check(to_host_u16(y), gate, up, down, x)
    assert ok, (err, rms)


def test_autotune_picks_the_fastest_it_measured():
    import torch
    w = synth.weight_matrix(2048, 2048, 0.02, 1e-4, 100.0, 65)
    dm = device_matrix(w)
    batches = [1, 16, 128]
    x = to_dev(synth.activations(128, 2048, 66))
    y = empty_bf16(128, 2048)
    ws = uw.Workspace(max(uw.workspace_bytes(dm, p, b) for p in range(4) for b in batches))
    flush = torch.empty(64 << 20, dtype=torch.uint8, device="cuda")
    choice, us = uw.autotune(dm, batches, 5, x, y, ws, flush=flush)
    assert us.shape == (3, 4) and np.isfinite(us).all() and (us > 0).all()
    for i in range(3):
        assert choice[i] == int(np.argmin(us[i]))
    # without the load-time pack, DIRECT is unavailable
    dm.mat.pack = None
    choice, us = uw.autotune(dm, [4], 3, x, y, ws)
    assert np.isinf(us[0, 3]) and choice[0] != 3

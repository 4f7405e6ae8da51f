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


def _chained_blocks(layers, dms, pipes, x):
    """Layer outputs of uw_mlp_block calls chained through the host, each
    checked against the float64 oracle given that layer's own input."""
    B = x.shape[0]
    h, outs = x, []
    for (g, u, dn), dl, p in zip(layers, dms, pipes):
        ws = uw.Workspace(uw.mlp_workspace_bytes(*dl, p, B))
        y = empty_bf16(B, g.shape[1])
        uw.mlp_block(*dl, p, to_dev(h), y, ws)
        ws.check("block")
        h_next = to_host_u16(y)
        ok, err, rms = mlp_check(h_next, g, u, dn, h)
        assert ok, (len(outs), p, err, rms)
        outs.append(h_next)
        h = h_next
    return outs


@pytest.mark.parametrize("B", [1, 8, 33])
def test_stack_equals_chained_blocks(B):
    """Three layers (d = 512; ffn 1536, 1024, 1536; a different pipeline mix
    per layer): uw_mlp_stack equals the blocks chained on the host bit for
    bit, and each layer meets the MLP bar against the oracle."""
    d = 512
    layers = [_block(d, ffn, seed) for ffn, seed in ((1536, 71), (1024, 74), (1536, 77))]
    dms = [[device_matrix(m) for m in triple] for triple in layers]
    pipes = [[3, 3, 3], [1, 3, 2], [3, 0, 3]]
    x = synth.activations(B, d, 80)
    outs = _chained_blocks(layers, dms, pipes, x)
    ws = uw.Workspace(uw.mlp_stack_workspace_bytes(dms, pipes, B))
    y = empty_bf16(B, d)
    uw.mlp_stack(dms, pipes, to_dev(x), y, ws)
    ws.check("stack")
    assert np.array_equal(to_host_u16(y), outs[-1])
    # a one-layer stack is the block itself
    ws1 = uw.Workspace(uw.mlp_stack_workspace_bytes(dms[:1], pipes[:1], B))
    y1 = empty_bf16(B, d)
    uw.mlp_stack(dms[:1], pipes[:1], to_dev(x), y1, ws1)
    ws1.check("stack")
    assert np.array_equal(to_host_u16(y1), outs[0])


def test_stack_rejects_bad_arguments():
    d = 256
    a = [device_matrix(m) for m in _block(d, 512, 81)]
    b = [device_matrix(m) for m in _block(2 * d, 512, 84)]  # maps 512 -> 512: does not chain with a
    x = to_dev(synth.activations(2, d, 85))
    y = empty_bf16(2, d)
    assert uw.mlp_stack_workspace_bytes([a, b], [3, 3, 3], 2) == 0
    need = uw.mlp_stack_workspace_bytes([a, a], [3, 3, 3], 2)
    assert need > uw.mlp_workspace_bytes(*a, [3, 3, 3], 2)
    small = uw.Workspace(need - 256)
    with pytest.raises(uw.UwError) as e:
        uw.mlp_stack([a, a], [3, 3, 3], x, y, small)
    assert e.value.status == uw.UW_ERR_WORKSPACE_TOO_SMALL
    ws = uw.Workspace(need)
    with pytest.raises(uw.UwError) as e:
        uw.mlp_stack([a, b], [3, 3, 3], x, y, ws)
    assert e.value.status == uw.UW_ERR_INVALID_ARG


@pytest.fixture(scope="module")
def two_full_layers():
    layers = [synth.stack_layer(layer) for layer in (0, 1)]
    return layers, [[device_matrix(m) for m in triple] for triple in layers]


@pytest.mark.parametrize("B", [1, 64])
def test_full_size_two_layer_stack(two_full_layers, B):
    """The first two layers of the 32-layer stack (gate/up 14336x4096, down
    4096x14336, 1e-3 outliers), direct palette throughout, in the launch
    configuration the stack benchmark times."""
    layers, dms = two_full_layers
    pipes = [[3, 3, 3]] * 2
    x = synth.activations(B, 4096, 86)
    outs = _chained_blocks(layers, dms, pipes, x)
    ws = uw.Workspace(uw.mlp_stack_workspace_bytes(dms, pipes, B))
    y = empty_bf16(B, 4096)
    uw.mlp_stack(dms, pipes, to_dev(x), y, ws)
    ws.check("stack")
    assert np.array_equal(to_host_u16(y), outs[-1])

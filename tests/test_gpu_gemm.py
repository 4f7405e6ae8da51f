"""GPU parity of the reconstructive GEMM (all four pipelines plus the BF16
comparator) against the float64 oracle, called through the C ABI.

Bar: max |y - y_ref| <= 2e-2 * rms(y_ref) against the float64 oracle, and
bit-identical y across the four pipelines (same K split, same reduction
order, same rebuilt tiles)."""
import numpy as np
import pytest

from mlp_huffman_coded_b200 import synth
from mlp_huffman_coded_b200 import uw
from oracle import uw_oracle as O

from gpu_util import device_matrix, empty_bf16, gemm_all, gemm_ref, to_dev, to_host_u16, within_tol

pytestmark = pytest.mark.gpu


def _check_gemm(w, x, dm=None, pipelines=(0, 1, 2, 3)):
    if dm is None:
        dm = device_matrix(w)
    ys = gemm_all(dm, to_dev(x), pipelines)
    y_ref, acc = gemm_ref(w, x)
    first = ys[pipelines[0]]
    ok, err, rms = within_tol(first, y_ref, acc)
    assert ok, (err, rms)
    for p in pipelines[1:]:
        assert np.array_equal(ys[p], first), f"pipeline {p} differs from {pipelines[0]}"
    # uncompressed comparator through the same kernel
    ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_BF16, x.shape[0]))
    y = empty_bf16(x.shape[0], w.shape[0])
    uw.gemm_bf16(to_dev(w), to_dev(x), y, ws)
    ws.check("gemm_bf16")
    assert np.array_equal(to_host_u16(y), first)
    return first


def test_small_config_batch4():
    p = synth.WORKLOADS["small_256x512"]
    w = synth.weight_matrix(p["rows"], p["cols"], p["sigma"], p["outlier_rate"], p["outlier_scale"], p["seed"])
    x = synth.activations(p["batch"], p["cols"], p["seed"] + 1)
    _check_gemm(w, x)


@pytest.mark.parametrize("B", [1, 2, 3, 8, 15, 16, 17, 31, 33, 64, 100, 128, 255, 256, 257, 300, 512])
def test_batch_sweep(B):
    w = synth.weight_matrix(512, 1024, 0.02, 1e-3, 100.0, 30)
    x = synth.activations(B, 1024, 31)
    _check_gemm(w, x)


@pytest.mark.parametrize("rows,cols", [(128, 64), (200, 512), (1000, 640), (384, 64 * 37), (64, 4096)])
def test_ragged_shapes(rows, cols):
    w = synth.weight_matrix(rows, cols, 0.02, 2e-3, 100.0, rows + cols)
    x = synth.activations(5, cols, 7)
    _check_gemm(w, x)


@pytest.mark.parametrize("rows,cols,B", [(203, 512, 1), (203, 512, 40), (1001, 192, 8), (77, 64, 300)])
def test_rows_not_multiple_of_8_use_per_element_stores(rows, cols, B):
    # output rows of N*2 bytes are not 16-byte multiples: the epilogue cannot
    # use TMA tensor stores and writes element by element
    w = synth.weight_matrix(rows, cols, 0.02, 2e-3, 100.0, rows * 7 + cols)
    x = synth.activations(B, cols, 9)
    _check_gemm(w, x)


def test_one_hot_input_selects_a_column_exactly():
    w = synth.weight_matrix(384, 1024, 0.02, 2e-3, 100.0, 40)
    dm = device_matrix(w)
    x = np.zeros((16, 1024), dtype=np.uint16)
    cols = [0, 1, 63, 64, 65, 500, 1022, 1023, 7, 77, 128, 129, 255, 256, 511, 777]
    for b, k in enumerate(cols):
        x[b, k] = 0x3F80  # 1.0
    ys = gemm_all(dm, to_dev(x))
    for p, y in ys.items():
        for b, k in enumerate(cols):
            assert np.array_equal(y[b], w[:, k]), (p, b, k)


def test_small_integers_are_exact():
    w = synth.small_integer_matrix(256, 2048, -8, 8, 41)
    x = synth.small_integer_matrix(24, 2048, -8, 8, 42)
    dm = device_matrix(w)
    ys = gemm_all(dm, to_dev(x))
    exact = synth.f32_to_bf16_bits(O.gemm(w, x).astype(np.float32))
    for p, y in ys.items():
        assert np.array_equal(y, exact), p


def test_verbatim_heavy_matrix_overflows_the_staged_slots():
    # 1e-2 outliers x300: most 64-element rows hold a rare exponent, so tiles
    # carry more verbatim rows than the kernel stages on chip
    w = synth.weight_matrix(256, 1024, 0.02, 2e-2, 300.0, 43)
    enc = uw.encode(w)
    # verbatim rows per (128-row tile, 64-column block): some exceed the 16
    # slots staged on chip
    vg = O.verbatim_groups(w, np.array(list(enc.cb.palette), np.uint8))
    per_tile = vg.reshape(2, 128, 16).sum(axis=1)
    assert per_tile.max() > 16
    x = synth.activations(9, 1024, 44)
    _check_gemm(w, x)


def test_all_verbatim_and_single_symbol_matrices():
    w = np.zeros((128, 64), dtype=np.uint16)
    for r in range(128):
        w[r, :] = ((100 + r % 17) << 7) | (r % 128)
        w[r, 5] = ((20 + r % 50) << 7) | 3
    x = synth.activations(3, 64, 45)
    _check_gemm(w, x)
    w = np.full((128, 128), (120 << 7) | 5, dtype=np.uint16)
    _check_gemm(w, x[:, :64].repeat(2, axis=1))


def test_mixed_top_bit_palette_uses_general_lookup():
    # the small config's palette holds exponents on both sides of 128
    p = synth.WORKLOADS["small_256x512"]
    w = synth.weight_matrix(p["rows"], p["cols"], p["sigma"], p["outlier_rate"], p["outlier_scale"], p["seed"])
    pal = np.array(list(uw.encode(w).cb.palette))
    assert (pal >= 128).any() and (pal < 128).any()
    _check_gemm(w, synth.activations(4, 512, 1))


def test_general_lookup_equals_fast_lookup():
    w = synth.weight_matrix(512, 1024, 0.02, 1e-3, 100.0, 46)
    dm = device_matrix(w)
    x = to_dev(synth.activations(16, 1024, 47))
    ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, 16))
    y1, y2 = empty_bf16(16, 512), empty_bf16(16, 512)
    uw.gemm_direct_palette(dm, x, y1, ws)
    uw.gemm_direct_palette(dm, x, y2, ws, general_lookup=True)
    ws.check()
    assert np.array_equal(to_host_u16(y1), to_host_u16(y2))


@pytest.mark.parametrize("which", ["gate", "down"])
@pytest.mark.parametrize("B", [1, 8, 32])
def test_full_size_mlp_matrices(which, B):
    gate, up, down = synth.mlp_block()
    w = gate if which == "gate" else down
    x = synth.activations(B, w.shape[1], 3)
    dm = device_matrix(w)
    ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, B))
    y = empty_bf16(B, w.shape[0])
    uw.gemm_direct_palette(dm, to_dev(x), y, ws)
    ws.check()
    ok, err, rms = within_tol(to_host_u16(y), *gemm_ref(w, x))
    assert ok, (err, rms)
    if B == 8:
        ys = gemm_all(dm, to_dev(x))
        for p in ys:
            assert np.array_equal(ys[p], to_host_u16(y)), p


def test_repeated_calls_are_deterministic_and_leave_counters_clean():
    w = synth.weight_matrix(1024, 4096, 0.02, 1e-4, 100.0, 48)
    dm = device_matrix(w)
    x = to_dev(synth.activations(8, 4096, 49))
    ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, 8))
    outs = []
    for _ in range(5):
        y = empty_bf16(8, 1024)
        uw.gemm_direct_palette(dm, x, y, ws)
        outs.append(to_host_u16(y))
    ws.check()
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
    # the tile counters are back at zero (header is 256 bytes)
    assert int(ws.t[256:256 + 4 * 8].sum()) == 0


def test_argument_errors():
    w = synth.weight_matrix(128, 256, 0.02, 0.0, 1.0, 50)
    dm = device_matrix(w)
    ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, 4))
    x = to_dev(synth.activations(4, 256, 51))
    y = empty_bf16(4, 128)
    with pytest.raises(uw.UwError) as e:
        uw.gemm(dm, uw.PIPE_DIRECT, to_dev(synth.activations(600, 256, 1)), empty_bf16(600, 128), ws)
    assert e.value.status == uw.UW_ERR_UNSUPPORTED_SHAPE
    small = uw.Workspace(300)
    with pytest.raises(uw.UwError) as e:
        uw.gemm(dm, uw.PIPE_FULL, x, y, small)
    assert e.value.status == uw.UW_ERR_WORKSPACE_TOO_SMALL
    dm.mat.pack = None
    with pytest.raises(uw.UwError) as e:
        uw.gemm_direct_palette(dm, x, y, ws)
    assert e.value.status == uw.UW_ERR_INVALID_ARG


def test_pack_offsets_pointing_outside_the_pack_are_reported_not_faulted():
    """Verbatim-row offsets of the direct-palette pack tampered on the device:
    the GEMM reports UW_ERR_CORRUPT, copies nothing outside the pack, and the
    workspace is usable again after the status is read."""
    w = synth.weight_matrix(512, 2048, 0.02, 3e-3, 100.0, 52)
    dm = device_matrix(w)
    x_host = synth.activations(8, 2048, 53)
    x = to_dev(x_host)
    ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, 8))
    y = empty_bf16(8, 512)
    good = dm.pack_off.clone()
    dm.pack_off[3:40] = 2 ** 31 - 1
    uw.gemm_direct_palette(dm, x, y, ws)
    assert ws.status() == uw.UW_ERR_CORRUPT
    dm.pack_off.copy_(good)
    uw.gemm_direct_palette(dm, x, y, ws)
    ws.check("after restoring the offsets")
    ok, err, rms = within_tol(to_host_u16(y), *gemm_ref(w, x_host))
    assert ok, (err, rms)


def test_workspace_shared_by_matrices_with_different_tile_counts():
    """One workspace serves GEMMs whose plans differ (96 and 8 row tiles,
    every tile split over several CTAs): each call leaves nothing that
    changes the next one, so outputs equal those of fresh workspaces."""
    big = device_matrix(synth.weight_matrix(12288, 4096, 0.02, 1e-4, 100.0, 95))
    small = device_matrix(synth.weight_matrix(1024, 4096, 0.02, 1e-4, 100.0, 96))
    x = to_dev(synth.activations(8, 4096, 97))

    def run(dm, ws):
        y = empty_bf16(8, int(dm.mat.L.rows))
        uw.gemm_direct_palette(dm, x, y, ws)
        ws.check()
        return to_host_u16(y)
    fresh = {id(dm): run(dm, uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, 8))) for dm in (big, small)}
    shared = uw.Workspace(max(uw.workspace_bytes(dm, uw.PIPE_DIRECT, 8) for dm in (big, small)))
    for dm in (big, small, big, small, big):
        assert np.array_equal(run(dm, shared), fresh[id(dm)])


@pytest.mark.parametrize("name,rows,cols,B", [
    ("q_proj / o_proj", 4096, 4096, 1),
    ("q_proj / o_proj", 4096, 4096, 8),
    ("k_proj / v_proj (8 KV heads)", 1024, 4096, 8),
    ("k_proj / v_proj (8 KV heads)", 1024, 4096, 64),
])
def test_attention_projection_shapes(name, rows, cols, B):
    """The same scheme on attention matrices (weights drawn with the MLP
    recipe): every pipeline meets the GEMM bar and all four agree bit for
    bit."""
    w = synth.weight_matrix(rows, cols, 0.02, 1e-4, 100.0, 120 + rows // 1024 + B)
    dm = device_matrix(w)
    x = synth.activations(B, cols, 121)
    ys = gemm_all(dm, to_dev(x))
    y_ref, acc = gemm_ref(w, x)
    for p, y in ys.items():
        ok, err, rms = within_tol(y, y_ref, acc)
        assert ok, (name, p, err, rms)
        assert np.array_equal(y, ys[3]), (name, p)


def test_lm_head_shape_sampled_rows():
    """An output projection with a 32000-token vocabulary (32000 x 4096),
    batch 4, direct palette: 2048 sampled output columns against the
    float64 oracle (computed one row of W at a time)."""
    w = synth.weight_matrix(32000, 4096, 0.02, 1e-4, 100.0, 122)
    dm = device_matrix(w)
    x = synth.activations(4, 4096, 123)
    ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, 4))
    y = empty_bf16(4, 32000)
    uw.gemm_direct_palette(dm, to_dev(x), y, ws)
    ws.check()
    got = to_host_u16(y)
    cols = np.sort(np.random.default_rng(124).choice(32000, 2048, replace=False))
    y_ref, acc = gemm_ref(w[cols], x)
    ok, err, rms = within_tol(got[:, cols], y_ref, acc)
    assert ok, (err, rms)

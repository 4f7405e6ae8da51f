"""GPU parity of the three Huffman decoders (full BF16, exponent bytes,
4-bit palette transcode) against the oracle: bit-exact, called through the
C ABI."""
import numpy as np
import pytest

from mlp_huffman_coded_b200 import synth
from mlp_huffman_coded_b200 import uw
from oracle import uw_oracle as O

from gpu_util import device_matrix, to_dev, to_host_u16, empty_bf16
from pack_reader import unpack_to_w

pytestmark = pytest.mark.gpu


def _decode_all(dm):
    import torch
    n = dm.rows * dm.cols
    ws = uw.Workspace(256)
    full = empty_bf16(n)
    exp8 = torch.empty(n, dtype=torch.uint8, device="cuda")
    idx4 = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    uw.decode_full(dm, full, ws)
    uw.decode_exponent_only(dm, exp8, ws)
    uw.transcode_palette(dm, idx4, ws)
    ws.check("decode")
    return (to_host_u16(full).reshape(dm.rows, dm.cols), exp8.cpu().numpy().reshape(dm.rows, dm.cols),
            idx4.cpu().numpy().reshape(dm.rows, dm.cols // 2))


def _expected_idx4(w, palette):
    """Plain definition: palette index per element, 0 in verbatim groups."""
    vg = np.repeat(O.verbatim_groups(w, palette), 64, axis=1)
    idx = np.where(vg, 0, O.palette_lookup(palette)[(w >> 7) & 0xFF]).astype(np.uint8)
    return (idx[:, 0::2] | (idx[:, 1::2] << 4)).astype(np.uint8)


def _check(w, chunk_groups=4, oracle_stream=False):
    if oracle_stream:
        # decode the oracle's own encoding (no product code on the input side)
        ref = O.encode(w, chunk_groups=chunk_groups)
        enc = uw.encode(w, chunk_groups=chunk_groups)
        enc.sm[:] = ref.sm.ravel()
        enc.stream[:] = ref.stream
        enc.chunk_bit_off[:] = ref.chunk_bit_off
        enc.vflags[:] = ref.vflags.ravel()
        enc.vprefix[:] = ref.vprefix
        enc.verbatim[:] = ref.verbatim.ravel()
        dm = uw.DeviceMatrix(enc)
    else:
        dm = device_matrix(w, chunk_groups, direct=False)
    full, exp8, idx4 = _decode_all(dm)
    assert np.array_equal(full, w)
    assert np.array_equal(exp8, ((w >> 7) & 0xFF).astype(np.uint8))
    assert np.array_equal(idx4, _expected_idx4(w, np.array(list(dm.enc.cb.palette), np.uint8)))


def test_small_config_bit_exact():
    p = synth.WORKLOADS["small_256x512"]
    w = synth.weight_matrix(p["rows"], p["cols"], p["sigma"], p["outlier_rate"], p["outlier_scale"], p["seed"])
    _check(w)
    _check(w, oracle_stream=True)


def test_every_bf16_pattern_bit_exact():
    _check(synth.all_patterns_matrix(), chunk_groups=3)


def test_special_values_and_degenerate_codes():
    rng = np.random.default_rng(3)
    exp = np.where(rng.random((8, 128)) < 0.7, 0, 255).astype(np.uint16)
    w = ((rng.integers(0, 2, (8, 128)).astype(np.uint16) << 15) | (exp << 7)
         | rng.integers(0, 128, (8, 128)).astype(np.uint16)).astype(np.uint16)
    _check(w)
    _check(np.full((3, 128), 120 << 7, dtype=np.uint16))          # one symbol
    w = np.zeros((17, 64), dtype=np.uint16)                          # every group verbatim
    for r in range(17):
        w[r, :] = (10 + r) << 7
        w[r, 7] = (100 + r) << 7
    _check(w)


@pytest.mark.parametrize("chunk_groups", [1, 2, 4, 5, 16])
def test_chunk_sizes_and_ragged_tail(chunk_groups):
    # 37 x 640: 370 groups, last chunk partial for most chunk sizes
    _check(synth.weight_matrix(37, 640, 0.03, 2e-3, 300.0, 11), chunk_groups)


def test_long_codes_use_the_slow_path():
    # a very skewed exponent distribution: codes longer than 11 bits
    rng = np.random.default_rng(9)
    probs = 0.5 ** np.arange(1, 17)
    probs /= probs.sum()
    exp = rng.choice(np.arange(100, 116), size=(64, 1024), p=probs).astype(np.uint16)
    w = ((exp << 7) | rng.integers(0, 128, exp.shape).astype(np.uint16)).astype(np.uint16)
    enc = uw.encode(w)
    assert enc.cb.max_len > 11
    _check(w)


def _flat_exponents(rows, cols, seed):
    """Exponents drawn evenly from 16 values: every code is 4 bits long."""
    rng = np.random.default_rng(seed)
    exp = rng.integers(110, 126, (rows, cols)).astype(np.uint16)
    return ((rng.integers(0, 2, exp.shape).astype(np.uint16) << 15) | (exp << 7)
            | rng.integers(0, 128, exp.shape).astype(np.uint16)).astype(np.uint16)


@pytest.mark.parametrize("chunk_groups", [1, 4, 16])
def test_wide_codes_read_the_stream_from_global_memory(chunk_groups):
    # 4-bit codes: the stream words of a warp's 32 chunks (256 * chunk_groups
    # words) outgrow its shared-memory copy, so the lanes read the stream
    # from global memory instead
    w = _flat_exponents(96, 2048, 12)
    assert set(uw.encode(w, chunk_groups=chunk_groups).cb.code_len) == {4}
    _check(w, chunk_groups)


def test_warps_mixing_staged_and_global_streams():
    # rows alternate between 4-bit codes and the usual ~2.6-bit ones, so
    # neighbouring warps take different stream paths in one launch
    a = _flat_exponents(64, 2048, 13)
    b = synth.weight_matrix(64, 2048, 0.02, 1e-4, 100.0, 14)
    w = np.empty((128, 2048), np.uint16)
    w[0::2], w[1::2] = a, b
    for cg in (1, 4):
        _check(w, cg)


def test_invalid_codes_of_an_incomplete_code_are_reported():
    # a one-symbol code ("0"): every 1 bit in the stream is an invalid code
    w = np.full((64, 1024), 120 << 7, dtype=np.uint16)
    enc = uw.encode(w)
    assert enc.cb.n_symbols == 1
    enc.stream[:-2] = np.uint32(0xFFFFFFFF)
    dm = uw.DeviceMatrix(enc)
    ws = uw.Workspace(256)
    import torch
    out = torch.empty(64 * 1024 // 2, dtype=torch.uint8, device="cuda")
    uw.transcode_palette(dm, out, ws)
    assert ws.status() == uw.UW_ERR_CORRUPT


def test_full_size_gate_matrix_bit_exact():
    p = synth.WORKLOADS["gate_14336x4096"]
    w = synth.weight_matrix(p["rows"], p["cols"], p["sigma"], p["outlier_rate"], p["outlier_scale"], p["seed"])
    _check(w)


def test_corrupt_offsets_are_reported_not_faulted():
    w = synth.weight_matrix(64, 512, 0.02, 1e-3, 100.0, 5)
    enc = uw.encode(w)
    enc.chunk_bit_off[5] += 3           # chunk 4 ends early, chunk 5 starts late
    dm = uw.DeviceMatrix(enc)
    ws = uw.Workspace(256)
    out = empty_bf16(64 * 512)
    uw.decode_full(dm, out, ws)
    assert ws.status() == uw.UW_ERR_CORRUPT
    assert ws.status() == uw.UW_OK      # reading clears the sticky word


def test_garbage_stream_stays_in_bounds():
    w = synth.weight_matrix(64, 512, 0.02, 1e-3, 100.0, 6)
    enc = uw.encode(w)
    rng = np.random.default_rng(0)
    enc.stream[:-2] = rng.integers(0, 2**32, enc.stream.size - 2, dtype=np.uint64).astype(np.uint32)
    dm = uw.DeviceMatrix(enc)
    ws = uw.Workspace(256)
    import torch
    out = torch.empty(64 * 512, dtype=torch.uint8, device="cuda")
    uw.decode_exponent_only(dm, out, ws)
    assert ws.status() == uw.UW_ERR_CORRUPT


@pytest.mark.parametrize("rows,cols,rate", [(256, 512, 5e-4), (200, 640, 2e-2), (384, 4096, 1e-4),
                                           (128, 128, 0.5)])
def test_direct_pack_reads_back_as_w(rows, cols, rate):
    """The load-time pack, read by an independent reader of the documented
    layout, gives back every BF16 word of W (the plain definition)."""
    w = synth.weight_matrix(rows, cols, 0.02, rate, 300.0, rows + 1)
    dm = device_matrix(w)
    off = dm.pack_off.cpu().numpy().view(np.uint32)
    got = unpack_to_w(rows, cols, np.array(list(dm.enc.cb.palette)), dm.pack.cpu().numpy(), off)
    assert np.array_equal(got, w)


def test_prefixes_pointing_outside_the_store_are_reported_not_faulted():
    """Flag prefixes tampered on the host after encoding (uploaded without
    uw_validate) point verbatim groups past the store: the decoders and the
    run-time transcode GEMM report UW_ERR_CORRUPT and read nothing outside
    the store."""
    import torch
    w = synth.weight_matrix(256, 1024, 0.02, 3e-3, 100.0, 12)
    enc = uw.encode(w)
    assert enc.layout.n_verbatim > 0
    enc.vprefix[1:] += np.uint32(1 << 24)
    dm = uw.DeviceMatrix(enc)
    ws = uw.Workspace(256)
    out = empty_bf16(256 * 1024)
    uw.decode_full(dm, out, ws)
    assert ws.status() == uw.UW_ERR_CORRUPT
    e8 = torch.empty(256 * 1024, dtype=torch.uint8, device="cuda")
    uw.decode_exponent_only(dm, e8, ws)
    assert ws.status() == uw.UW_ERR_CORRUPT
    x = to_dev(synth.activations(4, 1024, 13))
    y = empty_bf16(4, 256)
    wsg = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_TRANSCODE, 4))
    uw.gemm(dm, uw.PIPE_TRANSCODE, x, y, wsg)
    assert wsg.status() == uw.UW_ERR_CORRUPT
    assert wsg.status() == uw.UW_OK


def _gather(dm, rows):
    import torch
    ws = uw.Workspace(256)
    out = empty_bf16(len(rows), dm.cols)
    uw.decode_rows(dm, torch.tensor(rows, dtype=torch.int32, device="cuda"), out, ws)
    return ws, to_host_u16(out).reshape(len(rows), dm.cols)


@pytest.mark.parametrize("rows,cols,chunk_groups,rate", [
    (300, 640, 3, 2e-2),    # 10 groups per row: chunks straddle rows
    (257, 4096, 4, 1e-3),   # chunks aligned with rows, ragged last row tile
    (64, 1024, 16, 0.0),    # one chunk per row
])
def test_decode_rows_is_the_rows_of_w(rows, cols, chunk_groups, rate):
    """Embedding lookup: every requested row (repeats, first, last, in any
    order) comes back bit for bit, verbatim groups included."""
    w = synth.weight_matrix(rows, cols, 0.02, rate, 300.0, 101)
    dm = device_matrix(w, chunk_groups=chunk_groups, direct=False)
    ids = [rows - 1, 0, 5, 5, rows // 2, 1, rows - 1] + list(np.random.default_rng(102).integers(0, rows, 40))
    ws, got = _gather(dm, ids)
    ws.check("decode rows")
    assert np.array_equal(got, w[ids])


def test_decode_rows_embedding_table():
    """A vocabulary-sized table (32000 x 4096, the shape of a 32K-token
    embedding): 512 random token ids."""
    w = synth.weight_matrix(32000, 4096, 0.02, 1e-4, 100.0, 103)
    dm = device_matrix(w, direct=False)
    ids = list(np.random.default_rng(104).integers(0, 32000, 512))
    ws, got = _gather(dm, ids)
    ws.check("decode rows")
    assert np.array_equal(got, w[ids])


def test_decode_rows_outside_the_matrix_are_reported():
    w = synth.weight_matrix(100, 512, 0.02, 1e-3, 100.0, 105)
    dm = device_matrix(w, direct=False)
    ws, got = _gather(dm, [3, 100, -1, 99])
    with pytest.raises(uw.UwError) as e:
        ws.check("decode rows")
    assert e.value.status == uw.UW_ERR_INVALID_ARG
    assert np.array_equal(got[0], w[3]) and np.array_equal(got[3], w[99])
    assert not got[1].any() and not got[2].any()


def test_decode_rows_argument_errors():
    """Rejected on the host before anything is launched: a negative count
    and a row-id pointer that is not 4-byte aligned."""
    import ctypes as C
    import torch
    w = synth.weight_matrix(64, 256, 0.02, 0.0, 1.0, 106)
    dm = device_matrix(w, direct=False)
    ws = uw.Workspace(256)
    ids = torch.zeros(8, dtype=torch.int32, device="cuda")
    out = empty_bf16(4, 256)
    f = uw.lib().uw_decode_rows
    assert f(C.byref(dm.mat), ids.data_ptr(), -1, out.data_ptr(), ws.ptr, ws.nbytes, None) == uw.UW_ERR_INVALID_ARG
    assert f(C.byref(dm.mat), ids.data_ptr() + 2, 4, out.data_ptr(), ws.ptr, ws.nbytes, None) == uw.UW_ERR_INVALID_ARG
    ws.check("no launch happened")

"""GPU load-time compression (uw_build_palette_codebook_gpu, uw_encode_gpu):
byte-equal to the host encoder and to the oracle's encoding, and usable by
the GEMM directly."""
import numpy as np
import pytest

from mlp_huffman_coded_b200 import synth
from mlp_huffman_coded_b200 import uw
from oracle import uw_oracle as O

from gpu_util import empty_bf16, gemm_ref, to_dev, to_host_u16, within_tol

pytestmark = pytest.mark.gpu


def _host_u32(t):
    return t.cpu().numpy().view(np.uint32)


def _assert_same(dm, enc):
    """Every field of the GPU encoding equals the host encoding."""
    L, H = dm.mat.L, enc.layout
    for f in ("rows", "cols", "chunk_groups", "words_per_row", "n_groups", "n_chunks", "n_verbatim",
              "stream_words", "total_bits"):
        assert getattr(L, f) == getattr(H, f), f
    assert np.array_equal(dm.sm.cpu().numpy(), enc.sm)
    assert np.array_equal(_host_u32(dm.stream), enc.stream)
    assert np.array_equal(_host_u32(dm.chunk_bit_off), enc.chunk_bit_off)
    assert np.array_equal(_host_u32(dm.vflags), enc.vflags)
    assert np.array_equal(_host_u32(dm.vprefix), enc.vprefix)
    if H.n_verbatim:
        assert np.array_equal(dm.verbatim.cpu().numpy().view(np.uint16), enc.verbatim)


def _assert_same_codebook(a, b):
    assert bytes(a) == bytes(b)


def _matrices():
    rng = np.random.default_rng(3)
    exp = np.where(rng.random((8, 128)) < 0.7, 0, 255).astype(np.uint16)
    specials = ((rng.integers(0, 2, (8, 128)).astype(np.uint16) << 15) | (exp << 7)
                | rng.integers(0, 128, (8, 128)).astype(np.uint16)).astype(np.uint16)
    all_verbatim = np.zeros((17, 64), dtype=np.uint16)
    for r in range(17):
        all_verbatim[r, :] = (10 + r) << 7
        all_verbatim[r, 7] = (100 + r) << 7
    return {
        "small": synth.weight_matrix(256, 512, 0.02, 5e-4, 200.0, 0),
        "ragged_37x640": synth.weight_matrix(37, 640, 0.03, 2e-2, 300.0, 111),      # 10 groups per row
        "two_flag_words": synth.weight_matrix(99, 2560, 0.01, 1e-3, 100.0, 112),    # 40 groups per row
        "every_pattern": synth.all_patterns_matrix(),
        "specials": specials,
        "one_symbol": np.full((3, 128), 120 << 7, dtype=np.uint16),
        "all_verbatim": all_verbatim,
    }


@pytest.mark.parametrize("name", list(_matrices()))
def test_codebook_and_encoding_equal_the_host(name):
    import torch
    w = _matrices()[name]
    cb_host = uw.build_codebook(w)
    for cg in (1, 3, 4, 16):
        enc = uw.encode(w, chunk_groups=cg, cb=cb_host)
        dm = uw.DeviceMatrix.encode_on_device(torch.from_numpy(w.view(np.int16)).cuda(), chunk_groups=cg)
        _assert_same_codebook(dm.mat.cb, cb_host)
        _assert_same(dm, enc)


def test_encoding_equals_the_oracle():
    """The small configuration against the oracle's own encoding (the
    oracle is independent of both encoders)."""
    import torch
    w = synth.weight_matrix(256, 512, 0.02, 5e-4, 200.0, 0)
    ref = O.encode(w, chunk_groups=4)
    dm = uw.DeviceMatrix.encode_on_device(torch.from_numpy(w.view(np.int16)).cuda(), chunk_groups=4)
    assert np.array_equal(np.array(list(dm.mat.cb.palette), np.uint8), ref.cb.palette)
    assert np.array_equal(np.array(list(dm.mat.cb.code_len)), ref.cb.lengths)
    assert np.array_equal(dm.sm.cpu().numpy(), ref.sm.ravel())
    assert np.array_equal(_host_u32(dm.stream), ref.stream)
    assert np.array_equal(_host_u32(dm.chunk_bit_off), ref.chunk_bit_off)
    assert np.array_equal(_host_u32(dm.vflags), ref.vflags.ravel())
    assert np.array_equal(_host_u32(dm.vprefix), ref.vprefix)
    assert np.array_equal(dm.verbatim.cpu().numpy().view(np.uint16), ref.verbatim.ravel())


def test_full_size_matrix_encodes_like_the_host_and_feeds_the_gemm():
    """14336 x 4096 gate-shaped matrix: byte-equal encoding, then the
    direct-palette GEMM on the GPU-encoded matrix meets the GEMM bar."""
    import torch
    w = synth.weight_matrix(14336, 4096, 0.02, 1e-4, 100.0, 1)
    enc = uw.encode(w)
    dm = uw.DeviceMatrix.encode_on_device(torch.from_numpy(w.view(np.int16)).cuda())
    _assert_same_codebook(dm.mat.cb, enc.cb)
    _assert_same(dm, enc)
    ws0 = uw.Workspace(256)
    dm.prepare_direct_palette(ws0, keep_idx4=False)
    ws0.check("prepare")
    x = synth.activations(8, 4096, 113)
    ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, 8))
    y = empty_bf16(8, 14336)
    uw.gemm_direct_palette(dm, to_dev(x), y, ws)
    ws.check()
    ok, err, rms = within_tol(to_host_u16(y), *gemm_ref(w, x))
    assert ok, (err, rms)


def test_codebook_that_leaves_an_index_uncoded_is_rejected():
    """A codebook whose used palette index has no code: both encoders report
    UW_ERR_CORRUPT."""
    import torch
    w = synth.weight_matrix(64, 256, 0.02, 0.0, 1.0, 114)
    cb = uw.build_codebook(w)
    used = [i for i in range(16) if cb.freq[i] > 0]
    cb.code_len[used[-1]] = 0
    with pytest.raises(uw.UwError) as e:
        uw.encode(w, cb=cb)
    assert e.value.status == uw.UW_ERR_CORRUPT
    with pytest.raises(uw.UwError) as e:
        uw.DeviceMatrix.encode_on_device(torch.from_numpy(w.view(np.int16)).cuda(), cb=cb)
    assert e.value.status == uw.UW_ERR_CORRUPT

"""CPU tests of the C-ABI library: it loads, exports every declared symbol,
and its host codec (palette, Huffman code, encoder, validator) produces the
oracle's encoding byte for byte.  No device call is made here."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from mlp_huffman_coded_b200 import synth
from mlp_huffman_coded_b200 import uw
from oracle import uw_oracle as O

from pack_reader import verbatim_rows_per_tile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="session", autouse=True)
def built_library():
    from mlp_huffman_coded_b200 import build
    build.build()
    return uw.lib()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"UW_API\s+[\w\s\*]*?\b(uw_\w+)\s*\(", txt))
    return sorted(names)


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 19
    lib = C.CDLL(uw.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    # the binding knows every declared symbol too
    assert set(names) <= set(uw._SIGS)


def test_struct_sizes_match_the_header():
    assert C.sizeof(uw.Codebook) == 200
    assert C.sizeof(uw.Layout) == 64
    assert C.sizeof(uw.Matrix) == 64 + 200 + 9 * 8


def test_status_strings_and_version():
    lib = uw.lib()
    assert lib.uw_status_string(0) == b"ok"
    assert lib.uw_status_string(3) == b"corrupt compressed data"
    assert uw.version() == 100


def _same_as_oracle(w, chunk_groups=4):
    ref = O.encode(w, chunk_groups=chunk_groups)
    enc = uw.encode(w, chunk_groups=chunk_groups)
    assert list(enc.cb.palette) == [int(v) for v in ref.cb.palette]
    assert list(enc.cb.code_len) == [int(v) for v in ref.cb.lengths]
    assert list(enc.cb.freq) == [int(v) for v in ref.cb.freqs]
    used = ref.cb.lengths > 0
    assert [c for c, u in zip(enc.cb.code, used) if u] == [int(c) for c, u in zip(ref.cb.codes, used) if u]
    assert enc.cb.max_len == ref.cb.max_len and enc.cb.n_symbols == ref.cb.n_symbols
    assert enc.layout.total_bits == ref.total_bits
    assert enc.layout.n_verbatim == ref.n_verbatim
    assert np.array_equal(enc.sm, ref.sm.ravel())
    assert np.array_equal(enc.stream, ref.stream)
    assert np.array_equal(enc.chunk_bit_off, ref.chunk_bit_off)
    assert np.array_equal(enc.vflags, ref.vflags.ravel())
    assert np.array_equal(enc.vprefix, ref.vprefix)
    assert np.array_equal(enc.verbatim, ref.verbatim.ravel())
    assert uw.validate(enc) == 0
    return enc


def test_codec_matches_oracle_small_config():
    p = synth.WORKLOADS["small_256x512"]
    w = synth.weight_matrix(p["rows"], p["cols"], p["sigma"], p["outlier_rate"], p["outlier_scale"], p["seed"])
    enc = _same_as_oracle(w)
    assert enc.layout.n_verbatim == 66


def test_codec_matches_oracle_every_bf16_pattern():
    _same_as_oracle(synth.all_patterns_matrix(), chunk_groups=3)


@pytest.mark.parametrize("chunk_groups", [1, 2, 4, 7, 16])
def test_codec_matches_oracle_chunk_sizes(chunk_groups):
    _same_as_oracle(synth.weight_matrix(96, 640, 0.03, 2e-3, 300.0, 11), chunk_groups)


def test_codec_matches_oracle_degenerate_cases():
    # single symbol
    _same_as_oracle(np.full((3, 128), 120 << 7, dtype=np.uint16))
    # all groups verbatim: empty stream
    w = np.zeros((17, 64), dtype=np.uint16)
    for r in range(17):
        w[r, :] = (10 + r) << 7
        w[r, 7] = (100 + r) << 7
    enc = _same_as_oracle(w)
    assert enc.layout.total_bits == 0 and enc.layout.n_verbatim == 17
    # only special values: +-0, subnormals, Inf/NaN
    rng = np.random.default_rng(3)
    exp = np.where(rng.random((8, 128)) < 0.7, 0, 255).astype(np.uint16)
    w = ((rng.integers(0, 2, (8, 128)).astype(np.uint16) << 15) | (exp << 7)
         | rng.integers(0, 128, (8, 128)).astype(np.uint16)).astype(np.uint16)
    _same_as_oracle(w)
    # K = 64 * 40 (flag words per row = 2 with a partial second word), odd rows
    _same_as_oracle(synth.weight_matrix(5, 64 * 40, 0.02, 5e-3, 100.0, 21))


@pytest.mark.slow
def test_codec_matches_oracle_full_size_gate():
    p = synth.WORKLOADS["gate_14336x4096"]
    w = synth.weight_matrix(p["rows"], p["cols"], p["sigma"], p["outlier_rate"], p["outlier_scale"], p["seed"])
    enc = _same_as_oracle(w)
    # the page's ~30% claim on the Huffman form
    assert 0.28 < 1 - enc.compressed_bytes("huffman") / w.nbytes < 0.35


def test_size_query_and_argument_errors():
    w = synth.weight_matrix(8, 128, 0.02, 0.0, 1.0, 1)
    cb = uw.build_codebook(w)
    L = uw.Layout()
    lib = uw.lib()
    assert lib.uw_encode(w.ctypes.data, 8, 128, C.byref(cb), 4, C.byref(L), None, None, None, None, None, None) == 0
    assert L.rows == 8 and L.cols == 128 and L.n_groups == 16 and L.n_chunks == 4 and L.words_per_row == 1
    assert L.stream_words == (L.total_bits + 31) // 32 + 2
    bad = np.zeros((8, 96), np.uint16)
    assert lib.uw_build_palette_codebook(bad.ctypes.data, 8, 96, C.byref(cb)) == uw.UW_ERR_UNSUPPORTED_SHAPE
    assert lib.uw_build_palette_codebook(None, 8, 128, C.byref(cb)) == uw.UW_ERR_INVALID_ARG
    assert lib.uw_encode(w.ctypes.data, 8, 128, C.byref(cb), 0, C.byref(L), None, None, None, None, None,
                         None) == uw.UW_ERR_UNSUPPORTED_SHAPE
    assert lib.uw_encode(w.ctypes.data, 8, 128, C.byref(cb), 17, C.byref(L), None, None, None, None, None,
                         None) == uw.UW_ERR_UNSUPPORTED_SHAPE
    # a codebook that lacks a code for a used symbol
    cb2 = uw.build_codebook(w)
    cb2.code_len[0] = 0
    assert lib.uw_encode(w.ctypes.data, 8, 128, C.byref(cb2), 4, C.byref(L), None, None, None, None, None,
                         None) == uw.UW_ERR_CORRUPT



def test_decoders_reject_a_code_length_above_max_len_on_the_host():
    """The decoders index per-length tables by each code length: a codebook
    whose code_len exceeds its own max_len is refused before any launch (the
    pointers here are never dereferenced)."""
    w = synth.weight_matrix(64, 256, 0.02, 0.0, 1.0, 5)
    enc = uw.encode(w)
    m = uw.Matrix()
    m.L = enc.layout
    m.cb = enc.cb
    for f in ("sm", "stream", "chunk_bit_off", "vflags", "vprefix"):
        setattr(m, f, 0x10000)
    i = int(np.argmax(np.array(list(m.cb.code_len))))
    m.cb.code_len[i] = m.cb.max_len + 1
    lib = uw.lib()
    for fn in (lib.uw_decode_full, lib.uw_decode_exponent_only, lib.uw_transcode_palette):
        assert fn(C.byref(m), 0x20000, 0x30000, 256, None) == uw.UW_ERR_CORRUPT


def test_workspace_bytes_is_host_only():
    w = synth.weight_matrix(256, 512, 0.02, 5e-4, 200.0, 0)
    enc = uw.encode(w)
    n0 = uw.workspace_bytes(enc.layout, uw.PIPE_DIRECT, 0)
    assert n0 == 256
    n_direct = uw.workspace_bytes(enc.layout, uw.PIPE_DIRECT, 4)
    n_full = uw.workspace_bytes(enc.layout, uw.PIPE_FULL, 4)
    assert n_full - n_direct == 256 * 512 * 2
    assert uw.workspace_bytes(enc.layout, uw.PIPE_DIRECT, 513) == 0
    assert uw.workspace_bytes(enc.layout, 9, 4) == 0


@pytest.mark.parametrize("tamper", ["offset", "offset_end", "prefix", "flag_beyond_row", "noncanonical",
                                    "kraft", "dup_palette", "layout"])
def test_validate_rejects_tampered_encodings(tamper):
    w = synth.weight_matrix(64, 256, 0.02, 5e-3, 200.0, 4)
    enc = uw.encode(w)
    assert uw.validate(enc) == 0
    if tamper == "offset":
        enc.chunk_bit_off[3] = enc.chunk_bit_off[2] - 1
    elif tamper == "offset_end":
        enc.chunk_bit_off[-1] += 1
    elif tamper == "prefix":
        enc.vprefix[5] += 1
    elif tamper == "flag_beyond_row":
        enc.vflags[0] |= 1 << 10          # row has only 4 groups
    elif tamper == "noncanonical":
        i = int(np.argmax(np.array(list(enc.cb.code_len)) > 0))
        enc.cb.code[i] ^= 1
    elif tamper == "kraft":
        i = int(np.argmax(np.array(list(enc.cb.code_len))))
        enc.cb.code_len[i] = 1
    elif tamper == "dup_palette":
        enc.cb.palette[1] = enc.cb.palette[0]
    elif tamper == "layout":
        enc.layout.n_chunks += 1
    assert uw.validate(enc) in (uw.UW_ERR_CORRUPT, uw.UW_ERR_UNSUPPORTED_SHAPE)


def test_oracle_decodes_the_library_stream():
    w = synth.weight_matrix(128, 384, 0.02, 3e-3, 150.0, 8)
    enc = uw.encode(w)
    ref = O.encode(w)
    ref.stream = enc.stream.copy()
    ref.chunk_bit_off = enc.chunk_bit_off.copy()
    assert np.array_equal(O.decode_full(ref, lockstep=False), w)


@pytest.mark.parametrize("rows,cols,rate", [(256, 512, 5e-4), (200, 640, 2e-2), (128, 64, 0.3)])
def test_direct_pack_offsets_count_verbatim_rows_per_tile(rows, cols, rate):
    """pack_off[t] = verbatim groups of all tiles before t; the pack is one
    12304-byte body per tile plus 128 bytes per verbatim group (uw.h)."""
    w = synth.weight_matrix(rows, cols, 0.02, rate, 300.0, rows)
    enc = uw.encode(w)
    off, total = enc.pack_offsets()
    vg = O.verbatim_groups(w, O.build_palette(w))
    ref = verbatim_rows_per_tile(vg)
    assert np.array_equal(off, ref)
    n_tiles = -(-rows // 128) * (cols // 64)
    assert int(ref[-1]) == int(vg.sum()) == int(enc.layout.n_verbatim)
    assert total == n_tiles * 12304 + 128 * int(ref[-1])

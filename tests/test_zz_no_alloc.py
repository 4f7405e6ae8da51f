"""The allocation-free direct-palette GEMM (uw_gemm_direct_palette_noalloc).

Callers such as inference engines that hand a plugin only its inputs and
outputs cannot allocate a workspace; this entry point keeps its scratch in a
fixed array inside the library.  Its output must equal the workspace entry
point's, call after call (the array keeps the previous call's contents).
Kept in a file of its own that pytest collects last."""
import numpy as np
import pytest

from mlp_huffman_coded_b200 import synth
from mlp_huffman_coded_b200 import uw
from oracle import uw_oracle as O

from gpu_util import device_matrix, empty_bf16, gemm_ref, to_dev, to_host_u16, within_tol

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols,B", [(1024, 4096, 8), (14336, 4096, 16), (256, 512, 3)])
def test_noalloc_matches_workspace_entry_point_twice(rows, cols, B):
    w = synth.weight_matrix(rows, cols, 0.02, 1e-4, 100.0, 70 + B)
    dm = device_matrix(w)
    ws = uw.Workspace(uw.workspace_bytes(dm, uw.PIPE_DIRECT, B))
    y_ref = empty_bf16(B, rows)
    ys = []
    for call in range(2):
        x_host = synth.activations(B, cols, 80 + call)
        x = to_dev(x_host)
        uw.gemm_direct_palette(dm, x, y_ref, ws)
        ws.check("workspace entry point")
        y = empty_bf16(B, rows)
        uw.gemm_direct_palette_noalloc(dm, x, y)
        got, ref = to_host_u16(y), to_host_u16(y_ref)
        # against the float64 oracle, with the tolerance the other GPU tests use
        ok, err, rms = within_tol(got, *gemm_ref(w, x_host))
        assert ok, (call, err, rms)
        # and the same bits as the workspace entry point (same kernel, same split)
        assert np.array_equal(got, ref), call
        ys.append(got)
    assert not np.array_equal(ys[0], ys[1])  # different inputs really ran


def test_noalloc_rejects_sizes_beyond_its_array():
    w = synth.weight_matrix(14336, 256, 0.02, 0.0, 1.0, 90)
    dm = device_matrix(w)
    x = to_dev(synth.activations(512, 256, 91))
    y = empty_bf16(512, 14336)
    with pytest.raises(uw.UwError) as e:
        uw.gemm_direct_palette_noalloc(dm, x, y)
    assert e.value.status == uw.UW_ERR_WORKSPACE_TOO_SMALL


def _scratch_need(rows, B, sms):
    """Bytes the call needs in the fixed array (the formula documented in
    uw.h): header + tile counters + split-K partials."""
    n_ntiles = -(-B // 256)
    ntile = -(-(-(-B // n_ntiles)) // 16) * 16
    tiles = -(-rows // 128) * n_ntiles
    counters = 64 * 1024  # fixed region, the same for every plan
    return 256 + counters + (tiles + sms) * ntile * 128 * 4


def test_noalloc_size_limit_on_the_gate_matrix():
    """14336 x 4096: the largest batch whose scratch fits the documented
    16 MiB array runs and matches the oracle; the next batch tile is
    rejected before anything is launched."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    limit = 16 << 20
    fits = [B for B in range(1, 257) if _scratch_need(14336, B, sms) <= limit]
    B_max = max(fits)
    assert B_max + 1 not in fits
    w = synth.weight_matrix(14336, 4096, 0.02, 1e-4, 100.0, 92)
    dm = device_matrix(w)
    x_host = synth.activations(B_max, 4096, 93)
    y = empty_bf16(B_max, 14336)
    uw.gemm_direct_palette_noalloc(dm, to_dev(x_host), y)
    ok, err, rms = within_tol(to_host_u16(y), *gemm_ref(w, x_host))
    assert ok, (B_max, err, rms)
    with pytest.raises(uw.UwError) as e:
        uw.gemm_direct_palette_noalloc(dm, to_dev(synth.activations(B_max + 1, 4096, 94)), empty_bf16(B_max + 1, 14336))
    assert e.value.status == uw.UW_ERR_WORKSPACE_TOO_SMALL

"""Thin ctypes binding of libuw (include/uw.h).

Argument marshalling only: every step of the compressed-weight path runs in
the C++ host codec or the CUDA kernels of libuw.so.  PyTorch is used for
device memory (``tensor.data_ptr()``) and streams
(``torch.cuda.current_stream().cuda_stream``) and nothing else.

``lib()`` raises ``UwError`` when the library has not been built; there is no
fallback.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# UW_LIB_PATH selects another build of the same library (e.g. a tuning build)
LIB_PATH = os.environ.get("UW_LIB_PATH") or os.path.join(_HERE, "libuw.so")

PIPE_FULL, PIPE_EXPONENT, PIPE_TRANSCODE, PIPE_DIRECT, PIPE_BF16 = 0, 1, 2, 3, 4
PIPELINES = {"full": PIPE_FULL, "exponent": PIPE_EXPONENT, "transcode": PIPE_TRANSCODE,
             "direct": PIPE_DIRECT}
PIPE_NAMES = {v: k for k, v in PIPELINES.items()}
PIPE_NAMES[PIPE_BF16] = "bf16"

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "corrupt compressed data",
          4: "on-GPU wait timed out", 5: "CUDA error", 6: "workspace too small", 7: "no sm_100 device"}
UW_OK, UW_ERR_INVALID_ARG, UW_ERR_UNSUPPORTED_SHAPE, UW_ERR_CORRUPT = 0, 1, 2, 3
UW_ERR_TIMEOUT, UW_ERR_CUDA, UW_ERR_WORKSPACE_TOO_SMALL, UW_ERR_NO_DEVICE = 4, 5, 6, 7


class UwError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        super().__init__(f"{what}: {STATUS.get(int(status), 'status %d' % status)} ({int(status)})")


class Codebook(C.Structure):
    _fields_ = [("palette", C.c_uint8 * 16), ("code_len", C.c_uint8 * 16), ("code", C.c_uint16 * 16),
                ("freq", C.c_uint64 * 16), ("n_symbols", C.c_uint8), ("max_len", C.c_uint8),
                ("reserved", C.c_uint8 * 6)]


class Layout(C.Structure):
    _fields_ = [("rows", C.c_int64), ("cols", C.c_int64), ("chunk_groups", C.c_int32),
                ("words_per_row", C.c_int32), ("n_groups", C.c_int64), ("n_chunks", C.c_int64),
                ("n_verbatim", C.c_int64), ("stream_words", C.c_int64), ("total_bits", C.c_int64)]


class Matrix(C.Structure):
    _fields_ = [("L", Layout), ("cb", Codebook), ("sm", C.c_void_p), ("stream", C.c_void_p),
                ("chunk_bit_off", C.c_void_p), ("vflags", C.c_void_p), ("vprefix", C.c_void_p),
                ("verbatim", C.c_void_p), ("idx4", C.c_void_p), ("pack", C.c_void_p),
                ("pack_off", C.c_void_p)]


_P = C.c_void_p
_SIGS = {
    "uw_build_palette_codebook": (C.c_int, [_P, C.c_int64, C.c_int64, C.POINTER(Codebook)]),
    "uw_encode": (C.c_int, [_P, C.c_int64, C.c_int64, C.POINTER(Codebook), C.c_int32, C.POINTER(Layout),
                            _P, _P, _P, _P, _P, _P]),
    "uw_validate": (C.c_int, [C.POINTER(Matrix)]),
    "uw_encode_gpu_workspace_bytes": (C.c_size_t, [C.c_int64, C.c_int64]),
    "uw_build_palette_codebook_gpu": (C.c_int, [_P, C.c_int64, C.c_int64, C.POINTER(Codebook), _P, C.c_size_t, _P]),
    "uw_encode_gpu": (C.c_int, [_P, C.c_int64, C.c_int64, C.POINTER(Codebook), C.c_int32, C.POINTER(Layout),
                                _P, _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "uw_direct_pack_offsets": (C.c_int, [C.POINTER(Layout), _P, _P, C.POINTER(C.c_uint64)]),
    "uw_selftest_bounded_wait": (C.c_int, [_P, C.c_size_t, C.c_uint32, _P]),
    "uw_pack_direct_palette": (C.c_int, [C.POINTER(Matrix), _P, _P, _P]),
    "uw_workspace_bytes": (C.c_size_t, [C.POINTER(Layout), C.c_int32, C.c_int32]),
    "uw_workspace_init": (C.c_int, [_P, C.c_size_t, _P]),
    "uw_workspace_status": (C.c_int, [_P, _P]),
    "uw_decode_full": (C.c_int, [C.POINTER(Matrix), _P, _P, C.c_size_t, _P]),
    "uw_decode_exponent_only": (C.c_int, [C.POINTER(Matrix), _P, _P, C.c_size_t, _P]),
    "uw_transcode_palette": (C.c_int, [C.POINTER(Matrix), _P, _P, C.c_size_t, _P]),
    "uw_decode_rows": (C.c_int, [C.POINTER(Matrix), _P, C.c_int32, _P, _P, C.c_size_t, _P]),
    "uw_gemm_direct_palette": (C.c_int, [C.POINTER(Matrix), _P, C.c_int32, _P, _P, C.c_size_t, _P]),
    "uw_gemm_direct_palette_general_lookup": (C.c_int, [C.POINTER(Matrix), _P, C.c_int32, _P, _P,
                                                        C.c_size_t, _P]),
    "uw_gemm_direct_palette_noalloc": (C.c_int, [C.POINTER(Matrix), _P, C.c_int32, _P, _P]),
    "uw_gemm": (C.c_int, [C.POINTER(Matrix), C.c_int32, _P, C.c_int32, _P, _P, C.c_size_t, _P]),
    "uw_gemm_bf16": (C.c_int, [_P, C.c_int64, C.c_int64, _P, C.c_int32, _P, _P, C.c_size_t, _P]),
    "uw_swiglu": (C.c_int, [_P, _P, _P, C.c_int64, _P]),
    "uw_mlp_workspace_bytes": (C.c_size_t, [C.POINTER(Matrix), C.POINTER(Matrix), C.POINTER(Matrix),
                                            C.POINTER(C.c_int32), C.c_int32]),
    "uw_mlp_block": (C.c_int, [C.POINTER(Matrix), C.POINTER(Matrix), C.POINTER(Matrix), C.POINTER(C.c_int32),
                               _P, C.c_int32, _P, _P, C.c_size_t, _P]),
    "uw_mlp_stack_workspace_bytes": (C.c_size_t, [C.POINTER(C.POINTER(Matrix)), C.POINTER(C.c_int32), C.c_int32,
                                                  C.c_int32]),
    "uw_mlp_stack": (C.c_int, [C.POINTER(C.POINTER(Matrix)), C.POINTER(C.c_int32), C.c_int32, _P, C.c_int32, _P,
                               _P, C.c_size_t, _P]),
    "uw_autotune": (C.c_int, [C.POINTER(Matrix), C.POINTER(C.c_int32), C.c_int32, C.c_int32, _P, _P, _P,
                              C.c_size_t, _P, C.c_size_t, C.POINTER(C.c_int32), C.POINTER(C.c_float), _P]),
    "uw_status_string": (C.c_char_p, [C.c_int]),
    "uw_version": (C.c_int32, []),
    "uw_launch_count": (C.c_uint64, []),
}

_lib = None


def lib() -> C.CDLL:
    """Load libuw.so (built by ``python -m mlp_huffman_coded_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise UwError(UW_ERR_NO_DEVICE, f"libuw.so not built at {LIB_PATH}")
        h = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def _check(status: int, what: str):
    if status != UW_OK:
        raise UwError(status, what)


def _ptr(a) -> int:
    """Address of a numpy array or torch tensor (None -> NULL)."""
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    return a.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---------------------------------------------------------------------------
# host codec
# ---------------------------------------------------------------------------

@dataclass
class HostEncoded:
    layout: Layout
    cb: Codebook
    sm: np.ndarray
    stream: np.ndarray
    chunk_bit_off: np.ndarray
    vflags: np.ndarray
    vprefix: np.ndarray
    verbatim: np.ndarray

    @property
    def rows(self):
        return int(self.layout.rows)

    @property
    def cols(self):
        return int(self.layout.cols)

    def matrix(self) -> Matrix:
        """uw_matrix whose pointers are these host arrays (for uw_validate)."""
        m = Matrix()
        m.L = self.layout
        m.cb = self.cb
        m.sm, m.stream, m.chunk_bit_off = _ptr(self.sm), _ptr(self.stream), _ptr(self.chunk_bit_off)
        m.vflags, m.vprefix = _ptr(self.vflags), _ptr(self.vprefix)
        m.verbatim = _ptr(self.verbatim) if self.verbatim.size else None
        m.idx4 = None
        m.pack = None
        m.pack_off = None
        return m

    def pack_offsets(self):
        """Direct-palette pack offsets (verbatim rows before each tile) and
        total pack bytes."""
        return _pack_offsets(self.layout, self.vflags)

    def compressed_bytes(self, form: str = "huffman") -> int:
        meta = self.vflags.nbytes + self.vprefix.nbytes + self.verbatim.nbytes
        if form == "huffman":
            return self.sm.nbytes + self.stream.nbytes + self.chunk_bit_off.nbytes + meta
        if form == "palette":
            return self.sm.nbytes + self.rows * self.cols // 2 + meta
        raise ValueError(form)


def _pack_offsets(layout: Layout, vflags: np.ndarray):
    n_tiles = -(-int(layout.rows) // 128) * (int(layout.cols) // 64)
    off = np.empty(n_tiles + 1, np.uint32)
    total = C.c_uint64()
    vflags = np.ascontiguousarray(vflags, dtype=np.uint32)
    _check(lib().uw_direct_pack_offsets(C.byref(layout), _ptr(vflags), _ptr(off), C.byref(total)),
           "uw_direct_pack_offsets")
    return off, int(total.value)


def build_codebook(w: np.ndarray) -> Codebook:
    w = np.ascontiguousarray(w, dtype=np.uint16)
    cb = Codebook()
    _check(lib().uw_build_palette_codebook(_ptr(w), w.shape[0], w.shape[1], C.byref(cb)),
           "uw_build_palette_codebook")
    return cb


def encode(w: np.ndarray, chunk_groups: int = 4, cb: Codebook | None = None) -> HostEncoded:
    w = np.ascontiguousarray(w, dtype=np.uint16)
    rows, cols = w.shape
    if cb is None:
        cb = build_codebook(w)
    L = Layout()
    f = lib().uw_encode
    _check(f(_ptr(w), rows, cols, C.byref(cb), chunk_groups, C.byref(L), None, None, None, None, None, None),
           "uw_encode (sizes)")
    sm = np.empty(rows * cols, np.uint8)
    stream = np.empty(L.stream_words, np.uint32)
    off = np.empty(L.n_chunks + 1, np.uint32)
    vflags = np.empty(rows * L.words_per_row, np.uint32)
    vprefix = np.empty(rows * L.words_per_row + 1, np.uint32)
    verbatim = np.empty(L.n_verbatim * 64, np.uint16)
    _check(f(_ptr(w), rows, cols, C.byref(cb), chunk_groups, C.byref(L), _ptr(sm), _ptr(stream), _ptr(off),
             _ptr(vflags), _ptr(vprefix), _ptr(verbatim) if verbatim.size else None), "uw_encode")
    return HostEncoded(L, cb, sm, stream, off, vflags, vprefix, verbatim)


def validate(enc: HostEncoded) -> int:
    """Host-side format check; returns the status code (0 = ok)."""
    m = enc.matrix()
    return int(lib().uw_validate(C.byref(m)))


# ---------------------------------------------------------------------------
# device side
# ---------------------------------------------------------------------------

class Workspace:
    """Caller-owned device workspace (a torch uint8 tensor), zeroed once."""

    def __init__(self, nbytes: int, device="cuda"):
        import torch
        self.nbytes = max(int(nbytes), 256)
        self.t = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        with torch.cuda.device(self.t.device):
            _check(lib().uw_workspace_init(self.ptr, self.nbytes, _stream(None)), "uw_workspace_init")

    @property
    def ptr(self) -> int:
        return self.t.data_ptr()

    def status(self, stream=None) -> int:
        return int(lib().uw_workspace_status(self.ptr, _stream(stream)))

    def check(self, what="device", stream=None):
        _check(self.status(stream), what)


class DeviceMatrix:
    """One compressed matrix uploaded to the GPU (torch tensors own memory)."""

    def __init__(self, enc: HostEncoded, device="cuda"):
        import torch

        def up(a):
            return torch.from_numpy(np.ascontiguousarray(a)).to(device)

        self.enc = enc
        self.device = device
        self.sm = up(enc.sm)
        self.stream = up(enc.stream.view(np.int32))
        self.chunk_bit_off = up(enc.chunk_bit_off.view(np.int32))
        self.vflags = up(enc.vflags.view(np.int32))
        self.vprefix = up(enc.vprefix.view(np.int32))
        self.verbatim = up(enc.verbatim.view(np.int16)) if enc.verbatim.size else None
        self.idx4 = None
        self.mat = Matrix()
        self.mat.L = enc.layout
        self.mat.cb = enc.cb
        self.mat.sm, self.mat.stream = self.sm.data_ptr(), self.stream.data_ptr()
        self.mat.chunk_bit_off = self.chunk_bit_off.data_ptr()
        self.mat.vflags, self.mat.vprefix = self.vflags.data_ptr(), self.vprefix.data_ptr()
        self.mat.verbatim = self.verbatim.data_ptr() if self.verbatim is not None else None
        self.mat.idx4 = None
        self.mat.pack = None
        self.mat.pack_off = None
        self.pack = None
        self.pack_off = None

    @property
    def rows(self):
        return int(self.mat.L.rows)

    @property
    def cols(self):
        return int(self.mat.L.cols)

    @classmethod
    def encode_on_device(cls, w, chunk_groups: int = 4, cb: Codebook | None = None, stream=None):
        """Compress a device-resident BF16 matrix on the GPU (torch int16 /
        bfloat16 tensor [rows, cols]): uw_build_palette_codebook_gpu and
        uw_encode_gpu, whose outputs equal the host encoder's byte for
        byte.  No host copy of W is made."""
        import torch
        w = w.contiguous()
        rows, cols = w.shape
        dev = w.device
        wsn = int(lib().uw_encode_gpu_workspace_bytes(rows, cols))
        if wsn == 0:
            raise UwError(UW_ERR_UNSUPPORTED_SHAPE, "uw_encode_gpu_workspace_bytes")
        ws = torch.empty(wsn, dtype=torch.uint8, device=dev)
        st = _stream(stream)
        if cb is None:
            cb = Codebook()
            _check(lib().uw_build_palette_codebook_gpu(w.data_ptr(), rows, cols, C.byref(cb), ws.data_ptr(), wsn, st),
                   "uw_build_palette_codebook_gpu")
        L = Layout()
        f = lib().uw_encode_gpu
        _check(f(w.data_ptr(), rows, cols, C.byref(cb), chunk_groups, C.byref(L), None, None, None, None, None, None,
                 ws.data_ptr(), wsn, st), "uw_encode_gpu (sizes)")
        self = cls.__new__(cls)
        self.enc = None
        self.device = dev
        self.sm = torch.empty(rows * cols, dtype=torch.uint8, device=dev)
        self.stream = torch.empty(int(L.stream_words), dtype=torch.int32, device=dev)
        self.chunk_bit_off = torch.empty(int(L.n_chunks) + 1, dtype=torch.int32, device=dev)
        self.vflags = torch.empty(rows * int(L.words_per_row), dtype=torch.int32, device=dev)
        self.vprefix = torch.empty(rows * int(L.words_per_row) + 1, dtype=torch.int32, device=dev)
        self.verbatim = torch.empty(int(L.n_verbatim) * 64, dtype=torch.int16, device=dev) if L.n_verbatim else None
        _check(f(w.data_ptr(), rows, cols, C.byref(cb), chunk_groups, C.byref(L), self.sm.data_ptr(),
                 self.stream.data_ptr(), self.chunk_bit_off.data_ptr(), self.vflags.data_ptr(),
                 self.vprefix.data_ptr(), _ptr(self.verbatim), ws.data_ptr(), wsn, st), "uw_encode_gpu")
        self.idx4 = None
        self.mat = Matrix()
        self.mat.L = L
        self.mat.cb = cb
        self.mat.sm, self.mat.stream = self.sm.data_ptr(), self.stream.data_ptr()
        self.mat.chunk_bit_off = self.chunk_bit_off.data_ptr()
        self.mat.vflags, self.mat.vprefix = self.vflags.data_ptr(), self.vprefix.data_ptr()
        self.mat.verbatim = self.verbatim.data_ptr() if self.verbatim is not None else None
        self.mat.idx4 = None
        self.mat.pack = None
        self.mat.pack_off = None
        self.pack = None
        self.pack_off = None
        return self

    def prepare_direct_palette(self, ws: Workspace, stream=None, keep_idx4: bool = True):
        """Load-time preparation of the direct-palette form: transcode to 4-bit
        palette indices, then gather sm + indices + verbatim rows into one
        record per 128x64 tile (uw_pack_direct_palette)."""
        import torch
        self.idx4 = torch.empty(self.rows * self.cols // 2, dtype=torch.uint8, device=self.device)
        transcode_palette(self, self.idx4, ws, stream)
        self.mat.idx4 = self.idx4.data_ptr()
        if self.enc is not None:
            off, nbytes = self.enc.pack_offsets()
        else:
            off, nbytes = _pack_offsets(self.mat.L, self.vflags.cpu().numpy().view(np.uint32))
        self.pack_off = torch.from_numpy(off.view(np.int32)).to(self.device)
        self.pack = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        _check(lib().uw_pack_direct_palette(C.byref(self.mat), self.pack_off.data_ptr(), self.pack.data_ptr(),
                                            _stream(stream)), "uw_pack_direct_palette")
        self.mat.pack = self.pack.data_ptr()
        self.mat.pack_off = self.pack_off.data_ptr()
        if not keep_idx4:
            self.mat.idx4 = None
            self.idx4 = None
        return self

    def direct_palette_bytes(self) -> int:
        """Bytes the direct-palette GEMM reads from HBM for W: the pack
        records (sm + 4-bit indices + masks + inline verbatim rows)."""
        return int(self.pack.numel()) if self.pack is not None else 0


def workspace_bytes(dm_or_layout, pipeline: int, batch: int) -> int:
    L = dm_or_layout.mat.L if isinstance(dm_or_layout, DeviceMatrix) else dm_or_layout
    return int(lib().uw_workspace_bytes(C.byref(L), pipeline, batch))


def decode_full(dm: DeviceMatrix, out, ws: Workspace, stream=None):
    _check(lib().uw_decode_full(C.byref(dm.mat), _ptr(out), ws.ptr, ws.nbytes, _stream(stream)), "uw_decode_full")


def decode_exponent_only(dm: DeviceMatrix, out, ws: Workspace, stream=None):
    _check(lib().uw_decode_exponent_only(C.byref(dm.mat), _ptr(out), ws.ptr, ws.nbytes, _stream(stream)),
           "uw_decode_exponent_only")


def decode_rows(dm: DeviceMatrix, rows, out, ws: Workspace, stream=None):
    """out[i] = row rows[i] of W (rows: device int32 tensor)."""
    _check(lib().uw_decode_rows(C.byref(dm.mat), _ptr(rows), rows.numel(), _ptr(out), ws.ptr, ws.nbytes,
                                _stream(stream)), "uw_decode_rows")


def transcode_palette(dm: DeviceMatrix, out, ws: Workspace, stream=None):
    _check(lib().uw_transcode_palette(C.byref(dm.mat), _ptr(out), ws.ptr, ws.nbytes, _stream(stream)),
           "uw_transcode_palette")


def gemm(dm: DeviceMatrix, pipeline: int, x, y, ws: Workspace, stream=None):
    _check(lib().uw_gemm(C.byref(dm.mat), pipeline, _ptr(x), x.shape[0], _ptr(y), ws.ptr, ws.nbytes,
                         _stream(stream)), "uw_gemm")


def gemm_direct_palette(dm: DeviceMatrix, x, y, ws: Workspace, stream=None, general_lookup=False):
    f = lib().uw_gemm_direct_palette_general_lookup if general_lookup else lib().uw_gemm_direct_palette
    _check(f(C.byref(dm.mat), _ptr(x), x.shape[0], _ptr(y), ws.ptr, ws.nbytes, _stream(stream)),
           "uw_gemm_direct_palette")


def gemm_direct_palette_noalloc(dm: DeviceMatrix, x, y, stream=None):
    """Direct-palette GEMM for callers that cannot allocate: the scratch is
    the library's own fixed device array (see uw.h)."""
    _check(lib().uw_gemm_direct_palette_noalloc(C.byref(dm.mat), _ptr(x), x.shape[0], _ptr(y), _stream(stream)),
           "uw_gemm_direct_palette_noalloc")


def gemm_bf16(w, x, y, ws: Workspace, stream=None):
    _check(lib().uw_gemm_bf16(_ptr(w), w.shape[0], w.shape[1], _ptr(x), x.shape[0], _ptr(y), ws.ptr, ws.nbytes,
                              _stream(stream)), "uw_gemm_bf16")


def swiglu(g, u, h, stream=None):
    _check(lib().uw_swiglu(_ptr(g), _ptr(u), _ptr(h), g.numel(), _stream(stream)), "uw_swiglu")


def _pipes(pipelines):
    arr = (C.c_int32 * 3)(*[int(p) for p in pipelines])
    return arr


def mlp_workspace_bytes(gate: DeviceMatrix, up: DeviceMatrix, down: DeviceMatrix, pipelines, batch: int) -> int:
    return int(lib().uw_mlp_workspace_bytes(C.byref(gate.mat), C.byref(up.mat), C.byref(down.mat),
                                            _pipes(pipelines), batch))


def mlp_block(gate: DeviceMatrix, up: DeviceMatrix, down: DeviceMatrix, pipelines, x, y, ws: Workspace,
              stream=None):
    _check(lib().uw_mlp_block(C.byref(gate.mat), C.byref(up.mat), C.byref(down.mat), _pipes(pipelines),
                              _ptr(x), x.shape[0], _ptr(y), ws.ptr, ws.nbytes, _stream(stream)), "uw_mlp_block")


def _stack_args(layers, pipelines):
    """layers: [(gate, up, down), ...] DeviceMatrix triples; pipelines: one
    triple per layer (or one triple for every layer)."""
    mats = [m for triple in layers for m in triple]
    if len(pipelines) == 3 and not hasattr(pipelines[0], "__len__"):
        pipelines = [pipelines] * len(layers)
    pipes = [int(p) for triple in pipelines for p in triple]
    if len(mats) != 3 * len(layers) or len(pipes) != len(mats):
        raise ValueError("one (gate, up, down) triple and one pipeline triple per layer")
    arr = (C.POINTER(Matrix) * len(mats))(*[C.pointer(m.mat) for m in mats])
    return arr, (C.c_int32 * len(pipes))(*pipes), len(layers)


def mlp_stack_workspace_bytes(layers, pipelines, batch: int) -> int:
    arr, pipes, n = _stack_args(layers, pipelines)
    return int(lib().uw_mlp_stack_workspace_bytes(arr, pipes, n, batch))


def mlp_stack(layers, pipelines, x, y, ws: Workspace, stream=None):
    """One decode step's MLP work through the stack: y = MLP_{L-1}(...
    MLP_0(x)) (uw_mlp_stack)."""
    arr, pipes, n = _stack_args(layers, pipelines)
    _check(lib().uw_mlp_stack(arr, pipes, n, _ptr(x), x.shape[0], _ptr(y), ws.ptr, ws.nbytes, _stream(stream)),
           "uw_mlp_stack")


def autotune(dm: DeviceMatrix, batches, reps: int, x, y, ws: Workspace, flush=None, stream=None):
    """Returns (choice[n_batches], us[n_batches, 4])."""
    n = len(batches)
    b = (C.c_int32 * n)(*batches)
    choice = (C.c_int32 * n)()
    us = (C.c_float * (4 * n))()
    _check(lib().uw_autotune(C.byref(dm.mat), b, n, reps, _ptr(x), _ptr(y), _ptr(flush),
                             0 if flush is None else flush.numel() * flush.element_size(), ws.ptr, ws.nbytes,
                             choice, us, _stream(stream)), "uw_autotune")
    return list(choice), np.array(list(us), dtype=np.float64).reshape(n, 4)


def selftest_bounded_wait(ws: Workspace, limit_us: int, stream=None):
    """Launch the bounded-wait self-test (see uw.h); the status it leaves is
    read with ws.status()."""
    _check(lib().uw_selftest_bounded_wait(ws.ptr, ws.nbytes, int(limit_us), _stream(stream)),
           "uw_selftest_bounded_wait")


def launch_count() -> int:
    return int(lib().uw_launch_count())


def version() -> int:
    return int(lib().uw_version())

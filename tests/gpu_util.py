"""Helpers for the GPU tests: upload seeded inputs, call the library through
its C ABI, bring results back as BF16 bit patterns."""
import numpy as np

from mlp_huffman_coded_b200 import uw
from oracle import uw_oracle as O

TOL = 2e-2  # the GEMM bar: max |y - y_ref| <= TOL * rms(y_ref) against the float64 oracle


def to_dev(a: np.ndarray):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda()
    if a.dtype == np.uint32:
        return torch.from_numpy(a.view(np.int32)).cuda()
    return torch.from_numpy(a).cuda()


def to_host_u16(t) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def empty_bf16(*shape):
    import torch
    return torch.empty(*shape, dtype=torch.int16, device="cuda")


def bf16_f64(a: np.ndarray) -> np.ndarray:
    return O.bf16_to_f64(a)


def bf16_round(v):
    """Nearest BF16 value of each float64, ties to even, from the definition
    of BF16's 8-bit significand: v = m 2^e with 0.5 <= |m| < 1 keeps m to a
    multiple of 2^-8 (np.round rounds halves to even)."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.round(np.ldexp(m, 8)), e - 8)


def accumulation_bound(w: np.ndarray, x: np.ndarray) -> np.ndarray:
    """2 K 2^-24 sum_k |W[n, k] x[b, k]| per output.

    The BF16 x BF16 products are exact in FP32, so the FP32 sum of K of them
    is within K 2^-24 sum_k |W x| of the exact sum when every addition rounds
    to nearest; tensor cores add 16 products per step and may truncate
    (2^-23 per step, K/16 steps), which stays inside the same bound.  The
    factor 2 is the midpoint crossing explained in within_tol."""
    K = w.shape[1]
    return 2.0 * K * 2.0 ** -24 * (np.abs(O.bf16_to_f64(x)) @ np.abs(O.bf16_to_f64(w)).T)


def gemm_ref(w: np.ndarray, x: np.ndarray):
    """float64 oracle y = x W^T and its per-element accumulation bound."""
    return O.gemm(w, x), accumulation_bound(w, x)


def within_tol(y_u16, y_ref, acc=None, tol: float = TOL, extra=None):
    """Per element |y - y_ref| <= tol * rms(y_ref) + |bf16(y_ref) - y_ref| + acc (+ extra).

    tol * rms(y_ref) is the GEMM bar.  The BF16 output of an FP32 sum s with
    |s - y_ref| <= d is the BF16 value nearest s: it equals bf16(y_ref)
    (error |bf16(y_ref) - y_ref|) unless a rounding midpoint lies between s
    and y_ref, in which case y_ref is within d of that midpoint and the error
    is at most half an ulp + d <= |bf16(y_ref) - y_ref| + 2d.  `acc` is that
    2d (accumulation_bound); without it only the rounding term is allowed.
    `extra` (array) adds a bound for rounding of intermediates.
    """
    y = bf16_f64(y_u16)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    diff = np.abs(y - y_ref)
    allowed = tol * rms + np.abs(bf16_round(y_ref) - y_ref)
    if acc is not None:
        allowed = allowed + acc
    if extra is not None:
        allowed = allowed + extra
    i = int(np.argmax(diff - allowed))
    ok = bool(np.all(diff <= allowed))
    return ok, (float(diff.max()), float(diff.flat[i]), float(np.abs(y_ref).flat[i])), rms


def device_matrix(w: np.ndarray, chunk_groups: int = 4, direct: bool = True):
    enc = uw.encode(w, chunk_groups=chunk_groups)
    dm = uw.DeviceMatrix(enc)
    if direct:
        ws = uw.Workspace(256)
        dm.prepare_direct_palette(ws)
        ws.check("transcode")
    return dm


def gemm_all(dm, x_dev, pipelines=(0, 1, 2, 3)):
    """y for every pipeline (dict pipeline -> uint16 [B, rows])."""
    B = x_dev.shape[0]
    out = {}
    nb = max(uw.workspace_bytes(dm, p, B) for p in pipelines)
    ws = uw.Workspace(nb)
    for p in pipelines:
        y = empty_bf16(B, dm.rows)
        uw.gemm(dm, p, x_dev, y, ws)
        ws.check(f"gemm pipeline {p}")
        out[p] = to_host_u16(y)
    return out


def mlp_check(y_u16, gate, up, down, x):
    """MLP block bar: the GEMM bar plus the effect of rounding g, u and
    h = SiLU(g) * u to BF16 (each a relative error <= 2^-9, so at most
    ~2^-7 relative on every h_j), propagated through the down projection:
    2^-7 * sum_j |W_down[n, j] h_j|."""
    g = O.gemm(gate, x)
    u = O.gemm(up, x)
    h = O.silu(g) * u
    wd = O.bf16_to_f64(down)
    y_ref = h @ wd.T
    habs = np.abs(h) @ np.abs(wd).T
    inter = 2.0 ** -7 * habs
    acc = 2.0 * down.shape[1] * 2.0 ** -24 * habs
    return within_tol(y_u16, y_ref, acc=acc, extra=inter)

"""CPU oracle for lossless exponent coding of BF16 MLP weights and the
reconstructive GEMM that consumes them.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow reference that the
CUDA library is checked against.  Only the test suite, the smoke check in
``__graft_entry__`` and the benchmark's CPU-baseline leg may import it; the
product path never does, and it shares no code with the CUDA library (only
the seeded input generators in ``mlp_huffman_coded_b200.synth`` serve both).

The method is the one described in Cloudflare's "Unweight: how we compressed
an LLM 22% without sacrificing quality":

* section "How to compress model weights effectively": a BF16 word is 1 sign
  bit, 8 exponent bits and 7 mantissa bits; sign and mantissa are left raw;
  the exponent is Huffman coded; the 16 most frequent exponents of a matrix
  form its palette; a 64-element row that holds any exponent outside the
  palette is stored verbatim, so the hot loop checks once per row and never
  branches per element;
* section "Four ways to use compressed weights": full decode to BF16,
  exponent-only decode, transcode to 4-bit palette indices at run time, and
  the same transcode done once at load time ("direct palette");
* section "How the reconstructive matmul works": the GEMM rebuilds BF16 from
  sign+mantissa bytes plus exponent data (or palette indices) plus the
  verbatim rows, and feeds the result to the tensor cores.

Where the page is silent the oracle takes the following readings (each is
repeated where it is used):

R1  A "64-element row" is 64 consecutive elements along the input dimension
    (K) of the row-major [out_features, in_features] matrix; K % 64 == 0.
R2  Palette: the 16 exponent values with the highest count over the whole
    matrix, ties broken by smaller exponent value; with fewer than 16
    distinct exponents the free slots take the unused values in ascending
    order (they get no code).
R3  Huffman frequencies are counted over non-verbatim groups only (only
    those are coded).  Lengths come from the textbook two-smallest merge with
    a min-heap keyed by (weight, node id): leaves carry their palette index
    0..15, merged nodes take ids 16, 17, ... in creation order.  A single
    used symbol gets length 1; no used symbol gives an empty stream.
R4  Canonical codes in order of (length, palette index), written MSB first.
R5  Container: the codes of the non-verbatim groups in row-major group order,
    packed MSB-first into 32-bit words (bit p of the stream is bit 31-(p%32)
    of word p//32), followed by two zero words; a chunk is `chunk_groups`
    consecutive groups and chunk_bit_off[c] is the stream bit where chunk c
    starts (one extra entry holds the total bit count).
R6  Verbatim store: the full 64 BF16 words of each verbatim group, in group
    order.  vflags holds one bit per group (bit g%32 of word g//32 of the
    row's ceil(K/64/32) words); vprefix[w] counts the verbatim groups in all
    flag words before w (plus one final total).
R7  Sign+mantissa byte (one per element, dense over the whole matrix,
    verbatim groups included): byte k = (mantissa_k << 1) | sign_{k^1}, i.e.
    each byte carries its own mantissa and the sign of its pair partner
    (elements 2j and 2j+1 of a row swap signs).  This is a storage layout
    choice; the bits stay raw.
R8  exp8 output: the true exponent byte of every element (verbatim groups
    filled from the verbatim store).  idx4 output: palette index per element,
    element 2j in the low nibble and 2j+1 in the high nibble of byte j of the
    row; nibbles of verbatim groups are 0.
R9  GEMM: y[b, n] = sum_k W[n, k] * x[b, k] evaluated in float64 on the exact
    BF16 values.  MLP block: y = W_down (SiLU(W_gate x) * (W_up x)), float64.
"""
from __future__ import annotations

import heapq
import math
from dataclasses import dataclass, field

import numpy as np

GROUP = 64          # elements per verbatim-check row (R1)
PALETTE_SIZE = 16   # top-16 exponents (section "How to compress model weights effectively")
PAD_WORDS = 2       # zero words after the stream (R5)


# ---------------------------------------------------------------------------
# BF16 fields (section "How to compress model weights effectively")
# ---------------------------------------------------------------------------

def fields(w: np.ndarray):
    """Split BF16 words into (sign, exponent, mantissa): 1 + 8 + 7 bits."""
    w = np.asarray(w, dtype=np.uint16)
    sign = (w >> 15) & 1
    exp = (w >> 7) & 0xFF
    mant = w & 0x7F
    return sign.astype(np.uint8), exp.astype(np.uint8), mant.astype(np.uint8)


def bf16_to_f64(w: np.ndarray) -> np.ndarray:
    """Exact value of each BF16 word as float64."""
    w = np.ascontiguousarray(w, dtype=np.uint16)
    return (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sm_bytes(w2d: np.ndarray) -> np.ndarray:
    """Raw sign+mantissa byte per element, laid out per R7."""
    w2d = np.asarray(w2d, dtype=np.uint16)
    assert w2d.ndim == 2 and w2d.shape[1] % 2 == 0
    sign, _, mant = fields(w2d)
    partner_sign = sign.reshape(w2d.shape[0], -1, 2)[:, :, ::-1].reshape(w2d.shape)
    return ((mant << 1) | partner_sign).astype(np.uint8)


def word_from_fields(sign, exp, mant) -> np.ndarray:
    """Reassemble BF16 words from their three fields."""
    return ((np.asarray(sign, np.uint16) << 15) | (np.asarray(exp, np.uint16) << 7)
            | np.asarray(mant, np.uint16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# Palette (R2) and verbatim rule (R1, R6)
# ---------------------------------------------------------------------------

def exponent_histogram(w: np.ndarray) -> np.ndarray:
    _, exp, _ = fields(w)
    return np.bincount(exp.ravel(), minlength=256).astype(np.int64)


def build_palette(w: np.ndarray) -> np.ndarray:
    """The 16 most frequent exponents, ordered by (count desc, value asc).

    Sorting all 256 values by that key also fills missing slots with the
    unused values in ascending order (R2).
    """
    counts = exponent_histogram(w)
    order = sorted(range(256), key=lambda e: (-int(counts[e]), e))
    return np.array(order[:PALETTE_SIZE], dtype=np.uint8)


def palette_lookup(palette: np.ndarray) -> np.ndarray:
    """256-entry map exponent -> palette index, 255 for 'not in palette'."""
    lut = np.full(256, 255, dtype=np.uint8)
    for i, e in enumerate(palette):
        lut[int(e)] = i
    return lut


def verbatim_groups(w2d: np.ndarray, palette: np.ndarray) -> np.ndarray:
    """bool[rows, cols/64]: True where the 64-element row holds an exponent
    outside the palette (section "How to compress model weights effectively")."""
    rows, cols = w2d.shape
    assert cols % GROUP == 0
    _, exp, _ = fields(w2d)
    outside = palette_lookup(palette)[exp] == 255
    return outside.reshape(rows, cols // GROUP, GROUP).any(axis=2)


# ---------------------------------------------------------------------------
# Huffman code (R3, R4)
# ---------------------------------------------------------------------------

def huffman_code_lengths(freqs) -> np.ndarray:
    """Code length per symbol from the textbook Huffman construction.

    Repeatedly merge the two lightest nodes; a leaf's length is its depth in
    the final tree.  Ties: min-heap on (weight, node id) (R3).
    """
    freqs = [int(f) for f in freqs]
    n = len(freqs)
    lengths = np.zeros(n, dtype=np.int64)
    used = [i for i in range(n) if freqs[i] > 0]
    if not used:
        return lengths
    if len(used) == 1:
        lengths[used[0]] = 1
        return lengths
    heap = [(freqs[i], i) for i in used]
    heapq.heapify(heap)
    children = {}
    next_id = n
    while len(heap) > 1:
        wa, a = heapq.heappop(heap)
        wb, b = heapq.heappop(heap)
        children[next_id] = (a, b)
        heapq.heappush(heap, (wa + wb, next_id))
        next_id += 1
    root = heap[0][1]
    stack = [(root, 0)]
    while stack:
        node, depth = stack.pop()
        if node in children:
            a, b = children[node]
            stack.append((a, depth + 1))
            stack.append((b, depth + 1))
        else:
            lengths[node] = depth
    return lengths


def canonical_codes(lengths) -> np.ndarray:
    """Canonical code values: symbols taken in (length, index) order, each
    code one more than the previous, shifted left when the length grows (R4)."""
    lengths = [int(l) for l in lengths]
    codes = np.zeros(len(lengths), dtype=np.int64)
    order = sorted((l, i) for i, l in enumerate(lengths) if l > 0)
    code = 0
    prev = order[0][0] if order else 0
    for l, i in order:
        code <<= (l - prev)
        codes[i] = code
        code += 1
        prev = l
    return codes


@dataclass
class Codebook:
    palette: np.ndarray      # uint8[16] exponent values
    lengths: np.ndarray      # int64[16], 0 = symbol not coded
    codes: np.ndarray        # int64[16] canonical code values
    freqs: np.ndarray        # int64[16] counts over non-verbatim groups

    @property
    def max_len(self) -> int:
        return int(self.lengths.max()) if self.lengths.size else 0

    @property
    def n_symbols(self) -> int:
        return int((self.lengths > 0).sum())


def build_codebook(w2d: np.ndarray) -> Codebook:
    """Palette + Huffman code for one matrix (R2, R3, R4)."""
    w2d = np.asarray(w2d, dtype=np.uint16)
    palette = build_palette(w2d)
    vg = verbatim_groups(w2d, palette)
    _, exp, _ = fields(w2d)
    rows, cols = w2d.shape
    idx = palette_lookup(palette)[exp].reshape(rows, cols // GROUP, GROUP)
    coded = idx[~vg]                     # [n_coded_groups, 64]
    freqs = np.bincount(coded.ravel(), minlength=PALETTE_SIZE)[:PALETTE_SIZE].astype(np.int64)
    lengths = huffman_code_lengths(freqs)
    return Codebook(palette=palette, lengths=lengths, codes=canonical_codes(lengths), freqs=freqs)


# ---------------------------------------------------------------------------
# Encoder (R5-R7)
# ---------------------------------------------------------------------------

@dataclass
class Encoded:
    rows: int
    cols: int
    chunk_groups: int
    cb: Codebook
    sm: np.ndarray            # uint8[rows, cols]
    stream: np.ndarray        # uint32[stream_words]
    chunk_bit_off: np.ndarray # uint32[n_chunks + 1]
    vflags: np.ndarray        # uint32[rows, words_per_row]
    vprefix: np.ndarray       # uint32[rows * words_per_row + 1]
    verbatim: np.ndarray      # uint16[n_verbatim, 64]
    total_bits: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def n_groups(self) -> int:
        return self.rows * self.cols // GROUP

    @property
    def n_chunks(self) -> int:
        return -(-self.n_groups // self.chunk_groups)

    @property
    def words_per_row(self) -> int:
        return -(-(self.cols // GROUP) // 32)

    @property
    def n_verbatim(self) -> int:
        return int(self.verbatim.shape[0])

    def huffman_form_bytes(self) -> int:
        """Bytes of the Huffman storage form (everything a decoder reads)."""
        return (self.sm.nbytes + self.stream.nbytes + self.chunk_bit_off.nbytes
                + self.vflags.nbytes + self.vprefix.nbytes + self.verbatim.nbytes)

    def palette_form_bytes(self) -> int:
        """Bytes of the direct-palette form: sm + 4-bit indices + verbatim data."""
        return (self.sm.nbytes + self.rows * self.cols // 2 + self.vflags.nbytes
                + self.vprefix.nbytes + self.verbatim.nbytes)


def pack_bits_msb_first(values: np.ndarray, lengths: np.ndarray, extra_words: int = PAD_WORDS):
    """Concatenate codes MSB-first into uint32 words (R5).

    Each code (<= 15 bits) starting at bit p lands in word p//32 and, when it
    crosses the word boundary, in word p//32 + 1.
    """
    values = np.asarray(values, dtype=np.uint64)
    lengths = np.asarray(lengths, dtype=np.uint64)
    total = int(lengths.sum())
    words = np.zeros(-(-total // 32) + extra_words, dtype=np.uint64)
    if total == 0:
        return words.astype(np.uint32), 0
    start = np.concatenate([[0], np.cumsum(lengths)[:-1]]).astype(np.uint64)
    off = start & np.uint64(31)
    # place the code in a 64-bit window whose top bit is bit 0 of word start//32
    window = values << (np.uint64(64) - lengths - off)
    widx = (start >> np.uint64(5)).astype(np.int64)
    np.bitwise_or.at(words, widx, window >> np.uint64(32))
    np.bitwise_or.at(words, widx + 1, window & np.uint64(0xFFFFFFFF))
    return words.astype(np.uint32), total


def encode(w2d: np.ndarray, chunk_groups: int = 4, cb: Codebook | None = None) -> Encoded:
    """Compress one BF16 matrix into the storage form (R1-R7)."""
    w2d = np.ascontiguousarray(w2d, dtype=np.uint16)
    rows, cols = w2d.shape
    assert cols % GROUP == 0 and rows >= 1 and chunk_groups >= 1
    if cb is None:
        cb = build_codebook(w2d)
    gpr = cols // GROUP
    vg = verbatim_groups(w2d, cb.palette)                       # [rows, gpr]
    _, exp, _ = fields(w2d)
    idx = palette_lookup(cb.palette)[exp].reshape(rows * gpr, GROUP)
    vg_flat = vg.ravel()

    # codes of the non-verbatim groups, in row-major group order
    sym = idx[~vg_flat].ravel().astype(np.int64)
    if sym.size:
        assert (cb.lengths[sym] > 0).all(), "codebook does not cover a coded symbol"
    lens = cb.lengths[sym] if sym.size else np.zeros(0, np.int64)
    vals = cb.codes[sym] if sym.size else np.zeros(0, np.int64)
    stream, total = pack_bits_msb_first(vals, lens)

    # bits per group, then the bit offset where every chunk starts
    bits_per_group = np.zeros(rows * gpr, dtype=np.int64)
    if sym.size:
        bits_per_group[~vg_flat] = lens.reshape(-1, GROUP).sum(axis=1)
    group_start = np.concatenate([[0], np.cumsum(bits_per_group)])
    n_chunks = -(-(rows * gpr) // chunk_groups)
    chunk_first_group = np.minimum(np.arange(n_chunks + 1) * chunk_groups, rows * gpr)
    chunk_bit_off = group_start[chunk_first_group]
    assert chunk_bit_off[-1] == total and total < 2**32
    chunk_bit_off = chunk_bit_off.astype(np.uint32)

    # verbatim flags, per-word prefix counts and the verbatim store (R6)
    wpr = -(-gpr // 32)
    vflags = np.zeros((rows, wpr), dtype=np.uint32)
    for g in range(gpr):
        vflags[:, g // 32] |= (vg[:, g].astype(np.uint32) << np.uint32(g % 32))
    popc = np.array([bin(int(v)).count("1") for v in vflags.ravel()], dtype=np.int64)
    vprefix = np.concatenate([[0], np.cumsum(popc)]).astype(np.uint32)
    verbatim = w2d.reshape(rows * gpr, GROUP)[vg_flat].copy()

    return Encoded(rows=rows, cols=cols, chunk_groups=chunk_groups, cb=cb,
                   sm=sm_bytes(w2d), stream=stream, chunk_bit_off=chunk_bit_off,
                   vflags=vflags, vprefix=vprefix, verbatim=verbatim, total_bits=total)


# ---------------------------------------------------------------------------
# Decoder (canonical decoding, R4/R5) and the three decode outputs
# ---------------------------------------------------------------------------

class CanonicalDecoder:
    """Textbook canonical Huffman decoding: read bits one at a time and stop
    at the first length whose code range contains the value read."""

    def __init__(self, cb: Codebook):
        self.max_len = cb.max_len
        self.first = [0] * (self.max_len + 2)   # first code value of each length
        self.count = [0] * (self.max_len + 2)   # number of codes of each length
        self.offset = [0] * (self.max_len + 2)  # index of that length's first symbol
        self.symbols = [i for l, i in sorted((int(l), i) for i, l in enumerate(cb.lengths) if l > 0)]
        for l in cb.lengths:
            if l > 0:
                self.count[int(l)] += 1
        code = 0
        pos = 0
        for l in range(1, self.max_len + 1):
            self.first[l] = code
            self.offset[l] = pos
            code = (code + self.count[l]) << 1
            pos += self.count[l]

    def decode(self, stream: np.ndarray, bit: int, n: int):
        """Decode n symbols starting at stream bit `bit`; return (symbols, end bit)."""
        out = []
        for _ in range(n):
            code = 0
            for l in range(1, self.max_len + 1):
                word = int(stream[bit >> 5])
                code = (code << 1) | ((word >> (31 - (bit & 31))) & 1)
                bit += 1
                if code - self.first[l] < self.count[l]:
                    out.append(self.symbols[self.offset[l] + code - self.first[l]])
                    break
            else:
                raise ValueError("invalid code in stream")
        return out, bit


def _group_is_verbatim(enc: Encoded, g: int) -> bool:
    gpr = enc.cols // GROUP
    r, j = divmod(g, gpr)
    return bool((int(enc.vflags[r, j // 32]) >> (j % 32)) & 1)


def _verbatim_slot(enc: Encoded, g: int) -> int:
    gpr = enc.cols // GROUP
    r, j = divmod(g, gpr)
    w = r * enc.words_per_row + j // 32
    below = int(enc.vflags[r, j // 32]) & ((1 << (j % 32)) - 1)
    return int(enc.vprefix[w]) + bin(below).count("1")


def decode_indices(enc: Encoded) -> np.ndarray:
    """Palette index of every element, decoded chunk by chunk from the stream.

    Chunks are decoded independently from their own start offset, which is
    how a parallel decoder uses them; the bits a chunk consumes must end
    exactly where the next chunk starts.  Verbatim groups get index 255.
    Pure Python: for small matrices only.
    """
    dec = CanonicalDecoder(enc.cb)
    idx = np.full(enc.n_groups * GROUP, 255, dtype=np.uint8)
    for c in range(enc.n_chunks):
        bit = int(enc.chunk_bit_off[c])
        for g in range(c * enc.chunk_groups, min((c + 1) * enc.chunk_groups, enc.n_groups)):
            if _group_is_verbatim(enc, g):
                continue
            syms, bit = dec.decode(enc.stream, bit, GROUP)
            idx[g * GROUP:(g + 1) * GROUP] = syms
        if bit != int(enc.chunk_bit_off[c + 1]):
            raise ValueError(f"chunk {c} consumed bits up to {bit}, expected {int(enc.chunk_bit_off[c + 1])}")
    return idx.reshape(enc.rows, enc.cols)


def decode_indices_lockstep(enc: Encoded) -> np.ndarray:
    """Same result as decode_indices, vectorised across chunks with numpy.

    Every chunk advances one symbol per step; the code length is found by the
    canonical rule (first length l whose left-aligned range holds the next
    16 bits).  Used for full-size matrices.
    """
    cb = enc.cb
    n_groups = enc.n_groups
    C = enc.chunk_groups
    idx = np.full(n_groups * GROUP, 255, dtype=np.uint8)
    if cb.n_symbols == 0:
        return idx.reshape(enc.rows, enc.cols)
    gpr = enc.cols // GROUP
    g_all = np.arange(n_groups)
    r, j = np.divmod(g_all, gpr)
    vflag = ((enc.vflags[r, j // 32] >> (j % 32).astype(np.uint32)) & 1).astype(bool)
    # per chunk: element offsets of its coded symbols, in order
    n_chunks = enc.n_chunks
    coded_groups = np.where(~vflag)[0]
    chunk_of = coded_groups // C
    counts = np.bincount(chunk_of, minlength=n_chunks)
    order_in_chunk = np.arange(coded_groups.size) - np.concatenate([[0], np.cumsum(counts)])[chunk_of]
    max_groups = int(counts.max()) if counts.size else 0
    # table[c, t] = first element of the t-th coded group of chunk c
    table = np.full((n_chunks, max(max_groups, 1)), -1, dtype=np.int64)
    table[chunk_of, order_in_chunk] = coded_groups * GROUP

    dec = CanonicalDecoder(cb)
    L = dec.max_len
    # left-aligned 16-bit limits: value v has length l iff (v >> (16-l)) - first[l] < count[l]
    words = enc.stream.astype(np.uint64)
    bit = enc.chunk_bit_off[:-1].astype(np.int64).copy()
    sym_tab = np.array(dec.symbols, dtype=np.uint8)
    for t in range(max_groups * GROUP):
        gi, e = divmod(t, GROUP)
        base = table[:, gi]
        act = base >= 0
        if not act.any():
            break
        b = bit[act]
        w0 = words[b >> 5]
        w1 = words[(b >> 5) + 1]
        win = ((w0 << np.uint64(32)) | w1) << (b & 31).astype(np.uint64)
        peek = ((win >> np.uint64(48)) & np.uint64(0xFFFF)).astype(np.int64)
        length = np.zeros(b.size, dtype=np.int64)
        sym = np.zeros(b.size, dtype=np.int64)
        for l in range(1, L + 1):
            if dec.count[l] == 0:
                continue
            code = peek >> (16 - l)
            hit = (length == 0) & (code - dec.first[l] >= 0) & (code - dec.first[l] < dec.count[l])
            length[hit] = l
            sym[hit] = sym_tab[dec.offset[l] + code[hit] - dec.first[l]]
        if (length == 0).any():
            raise ValueError("invalid code in stream")
        idx[base[act] + e] = sym
        bit[act] = b + length
    if not np.array_equal(bit, enc.chunk_bit_off[1:].astype(np.int64)):
        raise ValueError("chunk bit counts do not match the chunk offsets")
    return idx.reshape(enc.rows, enc.cols)


def _verbatim_words(enc: Encoded) -> np.ndarray:
    """uint16[rows, cols] holding the verbatim store at the verbatim groups'
    positions (found through vflags + vprefix) and 0 elsewhere."""
    out = np.zeros((enc.rows * enc.cols // GROUP, GROUP), dtype=np.uint16)
    flagged = np.flatnonzero(_verbatim_mask(enc)[:, ::GROUP].ravel())
    for g in flagged:
        out[g] = enc.verbatim[_verbatim_slot(enc, int(g))]
    return out.reshape(enc.rows, enc.cols)


def _verbatim_mask(enc: Encoded) -> np.ndarray:
    gpr = enc.cols // GROUP
    g = np.arange(gpr)
    m = ((enc.vflags[:, g // 32] >> (g % 32).astype(np.uint32)) & 1).astype(bool)
    return np.repeat(m, GROUP, axis=1)


def _indices(enc: Encoded, lockstep: bool | None) -> np.ndarray:
    if lockstep is None:
        lockstep = enc.rows * enc.cols > 1 << 16
    return decode_indices_lockstep(enc) if lockstep else decode_indices(enc)


def rebuild_from_sm(sm: np.ndarray, exp: np.ndarray) -> np.ndarray:
    """BF16 words from sign+mantissa bytes (R7) and exponent bytes."""
    sm = np.asarray(sm, dtype=np.uint8)
    mant = sm >> 1
    partner_sign = sm & 1
    rows = sm.shape[0]
    sign = partner_sign.reshape(rows, -1, 2)[:, :, ::-1].reshape(sm.shape)
    return word_from_fields(sign, exp, mant)


def decode_full(enc: Encoded, lockstep: bool | None = None) -> np.ndarray:
    """Full decode to BF16 (section "Four ways to use compressed weights")."""
    idx = _indices(enc, lockstep)
    vmask = _verbatim_mask(enc)
    exp = enc.cb.palette[np.where(vmask, 0, idx)]
    w = rebuild_from_sm(enc.sm, exp)
    return np.where(vmask, _verbatim_words(enc), w).astype(np.uint16)


def decode_exponent_only(enc: Encoded, lockstep: bool | None = None) -> np.ndarray:
    """Exponent byte of every element (R8)."""
    idx = _indices(enc, lockstep)
    vmask = _verbatim_mask(enc)
    exp = enc.cb.palette[np.where(vmask, 0, idx)]
    vexp = ((_verbatim_words(enc) >> 7) & 0xFF).astype(np.uint8)
    return np.where(vmask, vexp, exp).astype(np.uint8)


def transcode_palette(enc: Encoded, lockstep: bool | None = None) -> np.ndarray:
    """4-bit palette index per element, two per byte (R8)."""
    idx = _indices(enc, lockstep)
    vmask = _verbatim_mask(enc)
    nib = np.where(vmask, 0, idx).astype(np.uint8)
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def rebuild_from_idx4(enc: Encoded, idx4: np.ndarray) -> np.ndarray:
    """BF16 matrix from sm + 4-bit indices + verbatim store: what the
    reconstructive GEMM builds in on-chip memory, written out in full."""
    nib = np.empty((enc.rows, enc.cols), dtype=np.uint8)
    nib[:, 0::2] = idx4 & 0xF
    nib[:, 1::2] = idx4 >> 4
    w = rebuild_from_sm(enc.sm, enc.cb.palette[nib])
    return np.where(_verbatim_mask(enc), _verbatim_words(enc), w).astype(np.uint16)


# ---------------------------------------------------------------------------
# GEMM and MLP block (R9)
# ---------------------------------------------------------------------------

def gemm(w2d: np.ndarray, x: np.ndarray) -> np.ndarray:
    """y[b, n] = sum_k W[n, k] x[b, k] in float64 on exact BF16 values."""
    return bf16_to_f64(x) @ bf16_to_f64(w2d).T


def silu(v: np.ndarray) -> np.ndarray:
    return v / (1.0 + np.exp(-v))


def mlp_block(w_gate, w_up, w_down, x) -> np.ndarray:
    """SwiGLU block: y = W_down (SiLU(W_gate x) * (W_up x)), all float64."""
    g = gemm(w_gate, x)
    u = gemm(w_up, x)
    h = silu(g) * u
    return h @ bf16_to_f64(w_down).T


# ---------------------------------------------------------------------------
# Statistics the page quotes (section "How to compress model weights effectively")
# ---------------------------------------------------------------------------

def exponent_entropy_bits(w: np.ndarray) -> float:
    c = exponent_histogram(w).astype(np.float64)
    p = c[c > 0] / c.sum()
    return float(-(p * np.log2(p)).sum())


def palette_coverage(w: np.ndarray, palette: np.ndarray) -> float:
    c = exponent_histogram(w)
    return float(c[palette.astype(np.int64)].sum() / c.sum())


def mean_code_bits(cb: Codebook) -> float:
    f = cb.freqs.astype(np.float64)
    return float((f * cb.lengths).sum() / f.sum()) if f.sum() else 0.0


def symbol_entropy_bits(cb: Codebook) -> float:
    f = cb.freqs[cb.freqs > 0].astype(np.float64)
    p = f / f.sum()
    return float(-(p * np.log2(p)).sum())


def kraft_sum(lengths) -> float:
    return float(sum(2.0 ** -int(l) for l in lengths if l > 0))


def brute_force_optimal_cost(freqs) -> int:
    """Minimum sum f_i * l_i over every prefix-code length vector (Kraft sum
    <= 1, lengths 1..n-1) for a small alphabet; exhaustive search."""
    import itertools
    f = [int(v) for v in freqs if v > 0]
    n = len(f)
    if n <= 1:
        return sum(f)
    best = None
    for ls in itertools.product(range(1, n), repeat=n):
        if sum(2.0 ** -l for l in ls) <= 1.0 + 1e-12:
            cost = sum(a * b for a, b in zip(f, ls))
            best = cost if best is None else min(best, cost)
    return best


def silu_scalar(v: float) -> float:
    """SiLU(v) = v * sigmoid(v), scalar (for tiny brute-force checks)."""
    return v / (1.0 + math.exp(-v))

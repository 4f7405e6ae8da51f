/*
 * uw.h -- C ABI of libuw: lossless Huffman-coded BF16 MLP weights and the
 * reconstructive GEMM that consumes them, for NVIDIA B200 (sm_100a).
 *
 * The method is Cloudflare's "Unweight: how we compressed an LLM 22% without
 * sacrificing quality":
 *   - section "How to compress model weights effectively": a BF16 weight is
 *     1 sign + 8 exponent + 7 mantissa bits; sign and mantissa stay raw; the
 *     exponent is Huffman coded; the 16 most frequent exponents of a matrix
 *     form its palette; a 64-element row holding any exponent outside the
 *     palette is stored verbatim so the hot loop decides once per row;
 *   - section "Four ways to use compressed weights": full decode, exponent-
 *     only decode, run-time 4-bit palette transcode, and the same transcode
 *     done at load time ("direct palette");
 *   - section "Why no single pipeline wins": the best pipeline depends on the
 *     matrix shape and the batch, so it is measured per matrix and batch;
 *   - section "How the reconstructive matmul works": compressed tiles are
 *     staged on chip, rebuilt to BF16 there and fed straight to the tensor
 *     cores; decoded weights never go back to HBM.
 *
 * Storage layout of one compressed matrix W[rows, cols] (row-major, BF16,
 * rows = output features, cols = input features, cols % 64 == 0):
 *   group       64 consecutive elements of one row (the page's "64-element
 *               row"); group g covers flat elements [64 g, 64 g + 64).
 *   sm          uint8[rows*cols], one byte per element, dense (verbatim groups
 *               included): byte k = (mantissa_k << 1) | sign_{k^1}; each byte
 *               carries its own 7 mantissa bits and the sign of its pair
 *               partner (elements 2j, 2j+1 of a row swap signs).  With this
 *               layout two BF16 words are rebuilt from two sm bytes and two
 *               exponent bytes by one byte permute and one 1-bit rotate.
 *   stream      uint32[stream_words]: canonical Huffman codes of the palette
 *               index of every element of every non-verbatim group, in group
 *               order, packed MSB first (stream bit p = bit 31-(p%32) of word
 *               p/32), followed by 2 zero words.
 *   chunk_bit_off uint32[n_chunks+1]: a chunk is chunk_groups consecutive
 *               groups; entry c is the stream bit where chunk c starts, the
 *               last entry is the total bit count.  Chunks decode in parallel.
 *   vflags      uint32[rows*words_per_row], words_per_row = ceil(cols/64/32):
 *               bit (g%32) of word (row*words_per_row + g/32) is set when
 *               group g of that row is verbatim.
 *   vprefix     uint32[rows*words_per_row+1]: verbatim groups in all earlier
 *               flag words (exclusive prefix); last entry = n_verbatim.
 *   verbatim    uint16[n_verbatim*64]: the raw BF16 words of each verbatim
 *               group, in group order.  The slot of group g of row r is
 *               vprefix[w] + popcount(vflags[w] & ((1<<(g%32))-1)) with
 *               w = r*words_per_row + g/32.
 *   idx4        uint8[rows*cols/2] (optional, from uw_transcode_palette):
 *               palette index per element, element 2j in the low nibble of
 *               byte j of the row, 2j+1 in the high nibble; 0 in verbatim
 *               groups.
 *   pack        (optional, the direct-palette form built at load time by
 *               uw_pack_direct_palette) for the n_tiles = ceil(rows/128) *
 *               cols/64 tiles of 128 rows x 64 columns, in (row block,
 *               column block) order: first one fixed-size 12304-byte body
 *               per tile, body t at byte 12304*t:
 *                 [0, 8192)      sm bytes of the tile: row r, 16-byte chunk
 *                                j at r*64 + 16*(j ^ ((r>>1)&3))
 *                 [8192, 12288)  idx4 bytes of the tile: row r, chunk j at
 *                                8192 + r*32 + 16*(j ^ ((r>>2)&1))
 *                 [12288, 12304) 128-bit verbatim mask, bit r = row r's
 *                                64-element group is verbatim
 *               then, from byte 12304*n_tiles, the verbatim rows of every
 *               tile (64 BF16 words = 128 bytes each) in tile order and, in a
 *               tile, in row order.  Rows past `rows` are zero.  The chunk
 *               order inside each 64-/32-byte row is the one that makes the
 *               GEMM's row-per-thread 16-byte shared-memory reads free of
 *               bank conflicts; fixed-size bodies let the GEMM fetch several
 *               consecutive tiles with one copy whose address it computes.
 *   pack_off    uint32[n_tiles+1]: pack_off[t] = verbatim rows of all tiles
 *               before t, so tile t's verbatim rows start at byte
 *               12304*n_tiles + 128*pack_off[t]; the last entry is n_verbatim
 *               (uw_direct_pack_offsets).
 *
 * Conventions for every call:
 *   - Every call returns a uw_status; nothing throws across the ABI.
 *   - The caller owns all memory.  The library never allocates device
 *     memory; device calls take a caller-provided workspace.
 *   - Device calls are asynchronous on the given stream (a cudaStream_t
 *     passed as void*, NULL = legacy default stream).  They return UW_OK once
 *     launched.  Problems the GPU finds (a corrupt stream, a wait that ran
 *     out of time) are recorded in the workspace's status word and read back
 *     with uw_workspace_status().
 *   - GEMM kernels are launched with programmatic dependent launch: one may
 *     start streaming its (constant) weights while the previous kernel on
 *     the same stream is still running, and waits for that kernel to
 *     complete before it reads x or the SwiGLU gate, or writes y or the
 *     workspace.  A GEMM that follows its own decode kernel (full,
 *     exponent-only and transcode pipelines) is launched plainly, and
 *     uw_pack_direct_palette ends with a plainly launched empty kernel, so a
 *     GEMM never reads weights before the kernel that wrote them is done.
 *     Weights written by a caller's kernel must likewise be followed by a
 *     plain stream operation (another kernel, an event, a copy) before the
 *     GEMM.  Ordering through events, copies or other streams is the usual
 *     full ordering.
 *   - Host calls (uw_build_palette_codebook, uw_encode, uw_validate) are
 *     synchronous and thread-safe.
 *   - Device pointers must be 16-byte aligned; violations give
 *     UW_ERR_INVALID_ARG before anything is launched.
 */
#ifndef UW_H
#define UW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define UW_API __attribute__((visibility("default")))
#else
#define UW_API
#endif

typedef enum {
  UW_OK = 0,
  UW_ERR_INVALID_ARG = 1,        /* NULL/misaligned pointer, bad size or enum */
  UW_ERR_UNSUPPORTED_SHAPE = 2,  /* cols % 64 != 0, batch out of range, ... */
  UW_ERR_CORRUPT = 3,            /* stream or metadata inconsistent */
  UW_ERR_TIMEOUT = 4,            /* a bounded on-GPU wait ran out */
  UW_ERR_CUDA = 5,               /* a CUDA runtime call failed */
  UW_ERR_WORKSPACE_TOO_SMALL = 6,
  UW_ERR_NO_DEVICE = 7           /* no sm_100 device available */
} uw_status;

/* Execution pipelines (section "Four ways to use compressed weights").
 * UW_PIPE_BF16 is the uncompressed comparator: the same GEMM kernel fed an
 * already-BF16 matrix. */
typedef enum {
  UW_PIPE_FULL = 0,       /* Huffman -> BF16 in HBM, then GEMM on BF16 */
  UW_PIPE_EXPONENT = 1,   /* Huffman -> exponent bytes, GEMM rebuilds from sm + exp8 */
  UW_PIPE_TRANSCODE = 2,  /* Huffman -> 4-bit indices at run time, reconstructive GEMM */
  UW_PIPE_DIRECT = 3,     /* 4-bit indices built at load time, reconstructive GEMM */
  UW_PIPE_BF16 = 4        /* uncompressed BF16 matrix (comparator only) */
} uw_pipeline;

#define UW_GROUP 64
#define UW_PALETTE 16
#define UW_MAX_BATCH 512
#define UW_MAX_CODE_LEN 15

/* Palette and canonical Huffman code of one matrix. */
typedef struct {
  uint8_t palette[UW_PALETTE];   /* exponent value of each palette index */
  uint8_t code_len[UW_PALETTE];  /* code length per index, 0 = no code */
  uint16_t code[UW_PALETTE];     /* canonical code value (right aligned) */
  uint64_t freq[UW_PALETTE];     /* count of each index over non-verbatim groups */
  uint8_t n_symbols;             /* indices with a code */
  uint8_t max_len;               /* longest code length (<= 15) */
  uint8_t reserved[6];
} uw_codebook;

/* Sizes of every array of one compressed matrix. */
typedef struct {
  int64_t rows, cols;
  int32_t chunk_groups;     /* groups per chunk (1..16) */
  int32_t words_per_row;    /* vflags words per row */
  int64_t n_groups;         /* rows*cols/64 */
  int64_t n_chunks;         /* ceil(n_groups/chunk_groups) */
  int64_t n_verbatim;       /* verbatim groups */
  int64_t stream_words;     /* including the 2 trailing zero words */
  int64_t total_bits;       /* coded bits (== chunk_bit_off[n_chunks]) */
} uw_layout;

/* One compressed matrix resident on the GPU: device pointers owned by the
 * caller (layout and codebook by value).  idx4 may be NULL until
 * uw_transcode_palette has filled a buffer for it. */
typedef struct {
  uw_layout L;
  uw_codebook cb;
  const uint8_t* sm;
  const uint32_t* stream;
  const uint32_t* chunk_bit_off;
  const uint32_t* vflags;
  const uint32_t* vprefix;
  const uint16_t* verbatim;  /* may be NULL when n_verbatim == 0 */
  const uint8_t* idx4;       /* may be NULL */
  const uint8_t* pack;       /* direct-palette records, may be NULL */
  const uint32_t* pack_off;  /* [n_tiles+1], NULL when pack is NULL */
} uw_matrix;

/* ---------------------------------------------------------------------------
 * Offline (host) calls
 * ------------------------------------------------------------------------- */

/* Palette + canonical Huffman code of a BF16 matrix (section "How to
 * compress model weights effectively").  w_host: host uint16[rows*cols],
 * row-major BF16 bits.  Palette = 16 most frequent exponents over the whole
 * matrix, ties to the smaller value, free slots filled with unused values in
 * ascending order.  Frequencies are counted over non-verbatim groups only;
 * code lengths come from the two-smallest-merge construction with ties broken
 * by (weight, node id), leaves 0..15, merged nodes 16, 17, ... in order.
 * Errors: UW_ERR_INVALID_ARG (NULL), UW_ERR_UNSUPPORTED_SHAPE (cols % 64,
 * rows < 1). */
UW_API uw_status uw_build_palette_codebook(const uint16_t* w_host, int64_t rows, int64_t cols,
                                    uw_codebook* out);

/* Encode a matrix into the storage layout above (sections "How to compress
 * model weights effectively" and "How the reconstructive matmul works").
 * cb: from uw_build_palette_codebook (or any codebook whose codes cover
 * every palette index used outside verbatim groups).  io_layout: filled on
 * return.  When every output pointer is NULL the call only computes the sizes
 * (io_layout) and returns; otherwise every output must be a host buffer of
 * the size io_layout gives (verbatim may be NULL when n_verbatim == 0).
 * Errors: UW_ERR_INVALID_ARG, UW_ERR_UNSUPPORTED_SHAPE (cols % 64, chunk_groups
 * outside 1..16, more than 2^32-1 stream bits), UW_ERR_CORRUPT (codebook does
 * not cover a used symbol). */
UW_API uw_status uw_encode(const uint16_t* w_host, int64_t rows, int64_t cols, const uw_codebook* cb,
                    int32_t chunk_groups, uw_layout* io_layout, uint8_t* sm, uint32_t* stream,
                    uint32_t* chunk_bit_off, uint32_t* vflags, uint32_t* vprefix,
                    uint16_t* verbatim);

/* Verbatim-row offsets of the direct-palette pack of a matrix (section "How
 * the reconstructive matmul works": what the producer stages per tile --
 * sign+mantissa bytes, palette indices, verbatim rows; the byte layout is
 * this library's), computed from its HOST vflags: pack_off[t] = verbatim
 * groups of all tiles before t.  pack_off_host holds n_tiles+1 entries;
 * *pack_bytes (may be NULL) receives the pack's size, 12304*n_tiles +
 * 128*n_verbatim.  Errors: UW_ERR_INVALID_ARG, UW_ERR_CORRUPT
 * (words_per_row), UW_ERR_UNSUPPORTED_SHAPE (pack above 64 GiB). */
UW_API uw_status uw_direct_pack_offsets(const uw_layout* L, const uint32_t* vflags_host,
                                        uint32_t* pack_off_host, uint64_t* pack_bytes);

/* Host-side consistency check (no counterpart on the page: it checks the
 * format of section "How to compress model weights effectively") of a
 * compressed matrix whose pointers are HOST copies: canonical codebook with Kraft sum <= 1, offsets monotone and
 * ending at total_bits, vprefix equal to the running popcount of vflags,
 * sizes consistent.  Run it before uploading data from an untrusted file.
 * Errors: UW_ERR_INVALID_ARG, UW_ERR_CORRUPT. */
UW_API uw_status uw_validate(const uw_matrix* host_mirror);

/* ---------------------------------------------------------------------------
 * Workspace
 * ------------------------------------------------------------------------- */

/* Bytes of device workspace (library plumbing; no counterpart on the page)
 * a device call needs for this matrix, pipeline and batch (batch 0 for the
 * decode/transcode calls).  The workspace holds a
 * 256-byte header (status word), a fixed 64 KB region of split-K tile
 * counters, the split-K partial sums, and for the FULL / EXPONENT /
 * TRANSCODE pipelines the intermediate decoded matrix.  The regions start
 * at the same offsets for every matrix and batch, so calls on different
 * matrices may share one workspace of the largest size they need.  Returns
 * 0 for invalid arguments. */
UW_API size_t uw_workspace_bytes(const uw_layout* L, int32_t pipeline, int32_t batch);

/* Zero a workspace and record its size in its header (library plumbing;
 * synchronizes `stream`).  A workspace must be set up once before its first
 * use; afterwards every call that succeeds leaves its counters at zero
 * again, and a call that fails is cleaned up by uw_workspace_status.  Calls
 * that share one workspace must be ordered on one stream.  Errors:
 * UW_ERR_INVALID_ARG (NULL, misaligned, < 256 bytes), UW_ERR_CUDA. */
UW_API uw_status uw_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Synchronize the stream, read the workspace's sticky status word (the
 * first problem any kernel recorded since the last read) and clear it
 * (library plumbing).  When it is not UW_OK, a kernel gave up part way and
 * may have left split-K tile counters raised, so the whole workspace is
 * zeroed again (the size recorded by uw_workspace_init; a workspace zeroed
 * some other way must be zeroed again by the caller before its next use).
 * Returns that status (UW_OK when none), or UW_ERR_INVALID_ARG / UW_ERR_CUDA
 * for the read itself. */
UW_API uw_status uw_workspace_status(void* workspace, void* stream);

/* Self-test of the bounded waits (no counterpart on the page: a robustness
 * check of this library).  Every wait in these kernels -- on an mbarrier
 * phase or on another CTA's counter -- gives up after a time limit, records
 * UW_ERR_TIMEOUT in the workspace status word and lets the kernel return.
 * This launches one warp that waits on a phase nothing completes and then on
 * a counter nothing increments, each for `limit_us` microseconds (1 ..
 * 1000000): afterwards uw_workspace_status() returns UW_ERR_TIMEOUT and the
 * CUDA context stays usable.  Uses header bytes [64, 80) of the workspace
 * (words 0 and 1 end as 0 when both waits gave up).  Errors:
 * UW_ERR_INVALID_ARG (NULL / misaligned / smaller than 256 bytes / limit out
 * of range), UW_ERR_NO_DEVICE, UW_ERR_CUDA. */
UW_API uw_status uw_selftest_bounded_wait(void* workspace, size_t workspace_bytes, uint32_t limit_us,
                                          void* stream);

/* ---------------------------------------------------------------------------
 * Load-time compression on the GPU (section "Four ways to use compressed
 * weights": the direct palette is prepared when the model is loaded; section
 * "How to compress model weights effectively": the format)
 * ------------------------------------------------------------------------- */

/* Device workspace bytes of the two calls below for a [rows, cols] matrix
 * (0 for an unsupported shape): about 13 bytes per 64-element group. */
UW_API size_t uw_encode_gpu_workspace_bytes(int64_t rows, int64_t cols);

/* uw_build_palette_codebook for a device-resident W (device BF16 [rows,
 * cols], 16-byte aligned): the exponent histogram and the per-index counts
 * over non-verbatim groups are computed on the GPU; the palette and the
 * Huffman code are chosen on the host from those counts by the same
 * routines as the host call, so *out is identical to it.  Synchronizes
 * `stream` (twice).  Errors as uw_build_palette_codebook, plus
 * UW_ERR_WORKSPACE_TOO_SMALL, UW_ERR_NO_DEVICE, UW_ERR_CUDA. */
UW_API uw_status uw_build_palette_codebook_gpu(const uint16_t* w, int64_t rows, int64_t cols,
                                               uw_codebook* out, void* workspace,
                                               size_t workspace_bytes, void* stream);

/* uw_encode for a device-resident W: the same *L and the same sm, stream,
 * chunk_bit_off, vflags, vprefix and verbatim bytes as the host call, written
 * to device buffers (16-byte aligned, sized from *L as for uw_encode).  With
 * every output NULL only *L is filled.  Each call runs the group pass and
 * synchronizes `stream` to read the totals; the writing call synchronizes
 * again at its end.  Errors as uw_encode (UW_ERR_CORRUPT for a codebook that
 * leaves a used palette index without a code, UW_ERR_UNSUPPORTED_SHAPE for
 * 2^32 or more stream bits), plus UW_ERR_WORKSPACE_TOO_SMALL,
 * UW_ERR_NO_DEVICE, UW_ERR_CUDA. */
UW_API uw_status uw_encode_gpu(const uint16_t* w, int64_t rows, int64_t cols, const uw_codebook* cb,
                               int32_t chunk_groups, uw_layout* L, uint8_t* sm, uint32_t* stream,
                               uint32_t* chunk_bit_off, uint32_t* vflags, uint32_t* vprefix,
                               uint16_t* verbatim, void* workspace, size_t workspace_bytes,
                               void* cuda_stream);

/* ---------------------------------------------------------------------------
 * Preprocessing kernels (section "Four ways to use compressed weights")
 * ------------------------------------------------------------------------- */

/* Full Huffman decode (section "Four ways to use compressed weights", full
 * decode): out_bf16[rows*cols] (device, row-major BF16 bits) gets back every
 * original word bit for bit, verbatim groups copied from the verbatim store.
 * Reads sm + stream + offsets + flags + verbatim; writes 2 bytes per
 * element.  Errors: UW_ERR_INVALID_ARG (NULL or misaligned pointers),
 * UW_ERR_WORKSPACE_TOO_SMALL (< 256 bytes), UW_ERR_UNSUPPORTED_SHAPE /
 * UW_ERR_CORRUPT (a layout whose sizes disagree with rows and cols, or a
 * codebook with max_len > 15 or a code length above max_len; found on the
 * host, nothing is launched), UW_ERR_NO_DEVICE, UW_ERR_CUDA;
 * on the device, a chunk whose code lengths do not end exactly at the next
 * chunk's offset (or an invalid code) records UW_ERR_CORRUPT in the status
 * word, and every read stays inside the stream. */
UW_API uw_status uw_decode_full(const uw_matrix* m, uint16_t* out_bf16, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Exponent-only decode (section "Four ways to use compressed weights"):
 * out_exp8[rows*cols] (device) = exponent byte of every element (verbatim
 * groups from the verbatim store); half of the full decode's write traffic.
 * The GEMM recombines it with the raw sm bytes.  Errors as uw_decode_full. */
UW_API uw_status uw_decode_exponent_only(const uw_matrix* m, uint8_t* out_exp8, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Full decode of selected rows (an embedding lookup on a compressed
 * embedding table; section "How to compress model weights effectively"
 * names embeddings among the matrices the page leaves raw): out_bf16
 * [n_rows, cols] (device) row i = row rows[i] of W, bit for bit.  rows:
 * device int32[n_rows]; repeats allowed.  Only the chunks that hold a
 * requested row are decoded.  Errors as uw_decode_full, plus
 * UW_ERR_INVALID_ARG for n_rows < 0 or NULL / misaligned rows; a row id outside
 * [0, rows) is found on the device: that output row is zeros and the
 * status word records UW_ERR_INVALID_ARG. */
UW_API uw_status uw_decode_rows(const uw_matrix* m, const int32_t* rows, int32_t n_rows, uint16_t* out_bf16,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Palette transcode (section "Four ways to use compressed weights"):
 * out_idx4[rows*cols/2] (device) = 4-bit palette index per element in the
 * idx4 layout, 0 in verbatim groups; a quarter of the full decode's write
 * traffic.  Run once at load time this is the "direct palette"
 * preparation; run per call it is the "palette transcode" pipeline.
 * Errors as uw_decode_full. */
UW_API uw_status uw_transcode_palette(const uw_matrix* m, uint8_t* out_idx4, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Load-time assembly of the direct-palette pack (sections "Four ways to use
 * compressed weights", direct palette, and "How the reconstructive matmul
 * works"; layout above) from sm, m->idx4 (must be set) and the verbatim
 * store, so that the direct-palette GEMM streams one contiguous record per
 * tile.  pack_off: device copy of the offsets from uw_direct_pack_offsets;
 * out_pack: device buffer of 16*pack_off[n_tiles] bytes, written by this
 * call (the caller owns it).  Errors: UW_ERR_INVALID_ARG (NULL, misaligned,
 * m->idx4 unset), UW_ERR_UNSUPPORTED_SHAPE, UW_ERR_NO_DEVICE, UW_ERR_CUDA. */
UW_API uw_status uw_pack_direct_palette(const uw_matrix* m, const uint32_t* pack_off,
                                        uint8_t* out_pack, void* stream);

/* ---------------------------------------------------------------------------
 * Reconstructive GEMM (section "How the reconstructive matmul works")
 * ------------------------------------------------------------------------- */

/* Direct-palette reconstructive GEMM (section "How the reconstructive matmul
 * works"; the "direct palette" pipeline of section "Four ways to use
 * compressed weights").
 * y = x W^T with the direct-palette matrix: x is device BF16 [batch, cols]
 * row-major, y is device BF16 [batch, rows] row-major.  W is rebuilt tile by
 * tile on chip from the pack records (sm + 4-bit indices + verbatim rows,
 * chosen once per 64-element row) and fed to tcgen05 MMA with FP32
 * accumulation in tensor memory; y is rounded to nearest-even BF16.
 * m->pack and m->pack_off must be set (uw_pack_direct_palette).  The split of the K
 * loop across CTAs and the order of its reduction depend only on (rows, cols,
 * batch, SM count), so all pipelines give bit-identical y.
 * batch: 1..512; cols <= 32768; ceil(rows/128) * ceil(batch/256) <= 16384
 * output tiles (rows <= 2097152 up to batch 256).  Errors:
 * UW_ERR_INVALID_ARG, UW_ERR_UNSUPPORTED_SHAPE, UW_ERR_WORKSPACE_TOO_SMALL,
 * UW_ERR_CUDA. */
UW_API uw_status uw_gemm_direct_palette(const uw_matrix* m, const uint16_t* x, int32_t batch,
                                 uint16_t* y, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* y = x W^T through any of the four pipelines of section "Four ways to use
 * compressed weights", including its preprocessing kernel (whose output
 * lives in the workspace).  UW_PIPE_BF16 is not accepted here (see
 * uw_gemm_bf16).  Errors as uw_gemm_direct_palette, plus UW_ERR_INVALID_ARG
 * for an unknown pipeline or a DIRECT call without m->pack. */
UW_API uw_status uw_gemm(const uw_matrix* m, int32_t pipeline, const uint16_t* x, int32_t batch,
                  uint16_t* y, void* workspace, size_t workspace_bytes, void* stream);

/* Same as uw_gemm_direct_palette, but always uses the general palette lookup
 * (the one for palettes whose used exponents differ in their top bit)
 * instead of the faster single-table lookup.  Results are identical; this
 * entry point (no counterpart on the page) exists so the general lookup can
 * be tested on any matrix.  Errors as uw_gemm_direct_palette. */
UW_API uw_status uw_gemm_direct_palette_general_lookup(const uw_matrix* m, const uint16_t* x,
                                                       int32_t batch, uint16_t* y, void* workspace,
                                                       size_t workspace_bytes, void* stream);

/* Direct-palette GEMM for callers that cannot allocate device memory (the
 * Unweight page has no counterpart; this is a deployment convenience).
 * Some callers cannot hand the library a workspace -- e.g. an inference
 * engine that gives a kernel plugin only its input and output buffers
 * because it plans all device memory ahead of time.  This call computes the
 * same y as uw_gemm_direct_palette (same kernel, same K split) but keeps the
 * scratch in a 16 MiB array built into the library, so it allocates nothing
 * (no cudaMalloc/cudaFree, no allocating library call).
 *   - Every GPU that loads the library holds that 16 MiB until exit.
 *   - Limit: header + tile counters + split-K partials must fit in it, i.e.
 *     (ceil(rows/128)*ceil(batch/256) + SMs) * batch_tile * 512 bytes plus
 *     64.25 KB, batch_tile = batch rounded up to a multiple of 16 (per 256);
 *     on a 148-SM B200 a 14336 x 4096 matrix fits up to batch 112.  Larger
 *     sizes return UW_ERR_WORKSPACE_TOO_SMALL before anything is launched.
 *   - The first call on a device looks the array's device address up
 *     (cudaGetSymbolAddress); make that first call before any stream
 *     capture.
 *   - Each call zeroes the array's status word and counters on `stream`
 *     before the kernel; all calls share the one array, so calls that may
 *     overlap on the GPU (different streams without ordering) race.
 *   - Device-side problems (a timed-out wait, inconsistent pack offsets) are
 *     recorded in the array's status word, which this call does not report;
 *     use uw_gemm_direct_palette with a workspace to diagnose them. */
UW_API uw_status uw_gemm_direct_palette_noalloc(const uw_matrix* m, const uint16_t* x, int32_t batch,
                                                uint16_t* y, void* stream);

/* Uncompressed comparator (the page's BF16 baseline; the "full decode"
 * pipeline's GEMM step): y = x W^T with W given as device BF16 [rows, cols];
 * the same GEMM kernel, loader reading BF16 tiles.  Workspace:
 * uw_workspace_bytes with UW_PIPE_BF16.  Errors as uw_gemm_direct_palette. */
UW_API uw_status uw_gemm_bf16(const uint16_t* w, int64_t rows, int64_t cols, const uint16_t* x,
                       int32_t batch, uint16_t* y, void* workspace, size_t workspace_bytes,
                       void* stream);

/* ---------------------------------------------------------------------------
 * MLP block
 * ------------------------------------------------------------------------- */

/* h = bf16(SiLU(g) * u) elementwise over n BF16 values (device), computed in
 * FP32: SiLU(v) = v / (1 + exp(-v)).  The glue of a SwiGLU MLP block (the
 * page compresses its gate/up/down matrices; the block itself is not on the
 * page).  Errors: UW_ERR_INVALID_ARG (NULL with n > 0, n < 0),
 * UW_ERR_NO_DEVICE, UW_ERR_CUDA. */
UW_API uw_status uw_swiglu(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t n, void* stream);

/* One SwiGLU MLP block (the three matrices the page compresses, section "How
 * to compress model weights effectively"; the block structure is not on the
 * page): y = W_down (SiLU(W_gate x) * (W_up x)).  gate, up:
 * [ffn, d]; down: [d, ffn]; x: [batch, d]; y: [batch, d] (device BF16).
 * pipelines[3]: pipeline per matrix (gate, up, down), e.g. from uw_autotune.
 * The up GEMM applies SiLU(g)*u in its epilogue and writes h directly.
 * Workspace: uw_mlp_workspace_bytes (0 for invalid arguments).  Errors:
 * UW_ERR_INVALID_ARG (NULL pointers, or shapes that do not chain),
 * UW_ERR_WORKSPACE_TOO_SMALL, and the errors of uw_gemm. */
UW_API size_t uw_mlp_workspace_bytes(const uw_matrix* gate, const uw_matrix* up, const uw_matrix* down,
                              const int32_t* pipelines, int32_t batch);
UW_API uw_status uw_mlp_block(const uw_matrix* gate, const uw_matrix* up, const uw_matrix* down,
                       const int32_t* pipelines, const uint16_t* x, int32_t batch, uint16_t* y,
                       void* workspace, size_t workspace_bytes, void* stream);

/* The MLP part of one decode step through an n_layers stack (section "Why
 * compression is harder than it looks": per-token latency adds up over every
 * layer's matrices): h_0 = x, h_{l+1} = MLP_l(h_l) with MLP_l the block of
 * uw_mlp_block over mats[3l], mats[3l+1], mats[3l+2] (gate, up, down) and
 * pipelines[3l..3l+2]; y = h_{n_layers}.  Attention and residual paths are
 * not part of it: each layer's MLP output is the next layer's input, which
 * keeps the dependency between layers.  Every layer maps d -> d (the same
 * d; ffn may differ).  x, y: device BF16 [batch, d]; mats: host array of
 * 3*n_layers pointers.  All 3*n_layers GEMMs (with the decoders their
 * pipelines need) go onto `stream` back to back; each GEMM may start
 * streaming its weights while the one before it finishes (programmatic
 * dependent launch).  Nothing synchronizes.  Workspace:
 * uw_mlp_stack_workspace_bytes (0 for invalid arguments): the largest
 * block's workspace plus two [batch, d] activation buffers.  Errors:
 * UW_ERR_INVALID_ARG (NULL pointers, n_layers < 1, shapes that do not
 * chain), UW_ERR_WORKSPACE_TOO_SMALL, and the errors of uw_mlp_block; on an
 * error the layers before it are already enqueued. */
UW_API size_t uw_mlp_stack_workspace_bytes(const uw_matrix* const* mats, const int32_t* pipelines,
                                           int32_t n_layers, int32_t batch);
UW_API uw_status uw_mlp_stack(const uw_matrix* const* mats, const int32_t* pipelines, int32_t n_layers,
                              const uint16_t* x, int32_t batch, uint16_t* y, void* workspace,
                              size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Autotuner (sections "Key Points" and "Why no single pipeline wins")
 * ------------------------------------------------------------------------- */

/* Time every pipeline on this matrix at each batch and pick the fastest
 * (sections "Key Points" and "Why no single pipeline wins": the best
 * pipeline depends on the matrix shape and the batch).
 * For each batch b in batches[0..n_batches): warm up, then run reps timed
 * calls (CUDA events on `stream`, preprocessing included), and keep the
 * median.  out_us[i*4 + p] = median microseconds of pipeline p at batches[i]
 * (+INF when the pipeline is unavailable, e.g. DIRECT without m->pack);
 * out_choice[i] = the pipeline with the smallest time.  x/y: device buffers
 * of at least max(batches)*cols / max(batches)*rows BF16 values used as
 * inputs/outputs of the timed calls.  flush/flush_bytes (optional, may be
 * NULL/0): a device buffer larger than L2 that is overwritten before every
 * timed call so the weights are read from HBM as they are in a real decode
 * step.  Synchronizes `stream`.  Workspace: the maximum of
 * uw_workspace_bytes over the four pipelines and batches.  Errors:
 * UW_ERR_INVALID_ARG (NULL outputs, n_batches or reps < 1), errors of the
 * timed calls, UW_ERR_CUDA. */
UW_API uw_status uw_autotune(const uw_matrix* m, const int32_t* batches, int32_t n_batches,
                      int32_t reps, const uint16_t* x, uint16_t* y, void* flush,
                      size_t flush_bytes, void* workspace, size_t workspace_bytes,
                      int32_t* out_choice, float* out_us, void* stream);

/* ---------------------------------------------------------------------------
 * Misc
 * ------------------------------------------------------------------------- */

/* Human-readable name of a status code (library plumbing). */
UW_API const char* uw_status_string(uw_status s);

/* Library version: major*10000 + minor*100 + patch (library plumbing). */
UW_API int32_t uw_version(void);

/* Number of kernel launches the library has issued in this process (all
 * devices; library plumbing); used to count launches inside a timed
 * region. */
UW_API uint64_t uw_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* UW_H */

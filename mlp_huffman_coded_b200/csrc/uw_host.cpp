// Host half of libuw: palette + canonical Huffman codebook, the offline
// encoder and the host-side format validator.
//
// Method: Cloudflare, "Unweight: how we compressed an LLM 22% without
// sacrificing quality", section "How to compress model weights effectively"
// (raw sign/mantissa, Huffman-coded exponent against a top-16 palette,
// verbatim 64-element rows).  The storage layout is documented in uw.h.
#include <algorithm>
#include <array>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <queue>
#include <thread>
#include <utility>
#include <vector>

#include "uw.h"
#include "uw_codebook.h"

namespace {

constexpr int kGroup = UW_GROUP;
constexpr int kPal = UW_PALETTE;

inline int popc32(uint32_t v) { return __builtin_popcount(v); }

// Host threads for the encoder passes: every pass splits the 64-element
// groups into contiguous ranges and combines per-thread results in a fixed
// way, so the output is byte-identical for any thread count.  Small
// matrices use one thread; UW_ENCODE_THREADS sets the count exactly.
int encode_threads(int64_t n_groups) {
  static const int env = [] {
    const char* e = std::getenv("UW_ENCODE_THREADS");
    return e ? std::atoi(e) : 0;
  }();
  if (env > 0) return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(env, n_groups)));
  const int t = static_cast<int>(std::min(16u, std::max(1u, std::thread::hardware_concurrency())));
  const int64_t by_size = n_groups / 16384 + 1;  // >= 1M elements per thread
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(t, by_size)));
}

// fn(thread, g_begin, g_end) over `nt` contiguous ranges of [0, n)
template <class F>
void for_ranges(int nt, int64_t n, F&& fn) {
  if (nt <= 1) {
    fn(0, int64_t(0), n);
    return;
  }
  std::vector<std::thread> pool;
  pool.reserve(nt);
  for (int t = 0; t < nt; ++t)
    pool.emplace_back([&, t] { fn(t, n * t / nt, n * (t + 1) / nt); });
  for (auto& th : pool) th.join();
}

bool shape_ok(int64_t rows, int64_t cols) {
  return rows >= 1 && cols >= kGroup && cols % kGroup == 0 && rows <= (int64_t(1) << 40) / cols;
}

// exponent value -> palette index, 255 when outside the palette
std::array<uint8_t, 256> palette_map(const uint8_t* palette) {
  std::array<uint8_t, 256> m;
  m.fill(255);
  for (int i = 0; i < kPal; ++i) m[palette[i]] = static_cast<uint8_t>(i);
  return m;
}

// Code lengths by the two-smallest-merge construction.  Ties between equal
// weights go to the smaller node id; leaves are the palette indices 0..15 and
// merged nodes are numbered 16, 17, ... in creation order.
void huffman_lengths(const uint64_t* freq, uint8_t* len_out) {
  std::memset(len_out, 0, kPal);
  using Node = std::pair<uint64_t, int>;  // (weight, id)
  std::priority_queue<Node, std::vector<Node>, std::greater<Node>> heap;
  int used = 0, only = -1;
  for (int i = 0; i < kPal; ++i)
    if (freq[i] > 0) {
      heap.push({freq[i], i});
      ++used;
      only = i;
    }
  if (used == 0) return;
  if (used == 1) {
    len_out[only] = 1;
    return;
  }
  std::vector<int> parent(2 * kPal, -1);
  int next_id = kPal;
  while (heap.size() > 1) {
    Node a = heap.top();
    heap.pop();
    Node b = heap.top();
    heap.pop();
    parent[a.second] = next_id;
    parent[b.second] = next_id;
    heap.push({a.first + b.first, next_id});
    ++next_id;
  }
  for (int i = 0; i < kPal; ++i) {
    if (freq[i] == 0) continue;
    int d = 0;
    for (int n = i; parent[n] >= 0; n = parent[n]) ++d;
    len_out[i] = static_cast<uint8_t>(d);
  }
}

// Canonical codes: (length, index) order, consecutive values, shifted left
// whenever the length grows.
void canonical(const uint8_t* len, uint16_t* code) {
  std::vector<std::pair<int, int>> order;
  for (int i = 0; i < kPal; ++i) {
    code[i] = 0;
    if (len[i]) order.push_back({len[i], i});
  }
  std::sort(order.begin(), order.end());
  uint32_t c = 0;
  int prev = order.empty() ? 0 : order[0].first;
  for (auto& li : order) {
    c <<= (li.first - prev);
    code[li.second] = static_cast<uint16_t>(c);
    ++c;
    prev = li.first;
  }
}

}  // namespace

namespace uw {

void choose_palette(const uint64_t* hist, uint8_t* palette) {
  std::array<int, 256> order;
  for (int e = 0; e < 256; ++e) order[e] = e;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    if (hist[a] != hist[b]) return hist[a] > hist[b];
    return a < b;
  });
  for (int i = 0; i < kPal; ++i) palette[i] = static_cast<uint8_t>(order[i]);
}

void finish_codebook(uw_codebook* cb) {
  huffman_lengths(cb->freq, cb->code_len);
  canonical(cb->code_len, cb->code);
  int ns = 0, ml = 0;
  for (int i = 0; i < kPal; ++i) {
    ns += cb->code_len[i] > 0;
    ml = std::max<int>(ml, cb->code_len[i]);
  }
  cb->n_symbols = static_cast<uint8_t>(ns);
  cb->max_len = static_cast<uint8_t>(ml);
}

bool encode_shape_ok(int64_t rows, int64_t cols) { return shape_ok(rows, cols); }

}  // namespace uw

extern "C" uw_status uw_build_palette_codebook(const uint16_t* w, int64_t rows, int64_t cols,
                                                uw_codebook* out) {
  if (!w || !out) return UW_ERR_INVALID_ARG;
  if (!shape_ok(rows, cols)) return UW_ERR_UNSUPPORTED_SHAPE;
  const int64_t n = rows * cols;
  const int64_t n_groups = n / kGroup;
  const int nt = encode_threads(n_groups);
  std::vector<std::array<uint64_t, 256>> part_hist(nt);
  for_ranges(nt, n_groups, [&](int t, int64_t g0, int64_t g1) {
    auto& h = part_hist[t];
    h.fill(0);
    for (int64_t i = g0 * kGroup; i < g1 * kGroup; ++i) ++h[(w[i] >> 7) & 0xFF];
  });
  std::array<uint64_t, 256> hist{};
  for (int t = 0; t < nt; ++t)
    for (int e = 0; e < 256; ++e) hist[e] += part_hist[t][e];
  uw_codebook cb;
  std::memset(&cb, 0, sizeof(cb));
  uw::choose_palette(hist.data(), cb.palette);
  auto pm = palette_map(cb.palette);
  // frequencies over non-verbatim groups only
  std::vector<std::array<uint64_t, kPal>> part_freq(nt);
  for_ranges(nt, n_groups, [&](int t, int64_t g0, int64_t g1) {
    auto& f = part_freq[t];
    f.fill(0);
    for (int64_t g = g0; g < g1; ++g) {
      const uint16_t* p = w + g * kGroup;
      bool verb = false;
      for (int k = 0; k < kGroup; ++k) verb |= pm[(p[k] >> 7) & 0xFF] == 255;
      if (verb) continue;
      for (int k = 0; k < kGroup; ++k) ++f[pm[(p[k] >> 7) & 0xFF]];
    }
  });
  for (int t = 0; t < nt; ++t)
    for (int i = 0; i < kPal; ++i) cb.freq[i] += part_freq[t][i];
  uw::finish_codebook(&cb);
  *out = cb;
  return UW_OK;
}

extern "C" uw_status uw_encode(const uint16_t* w, int64_t rows, int64_t cols, const uw_codebook* cb,
                               int32_t chunk_groups, uw_layout* L, uint8_t* sm, uint32_t* stream,
                               uint32_t* chunk_bit_off, uint32_t* vflags, uint32_t* vprefix,
                               uint16_t* verbatim) {
  if (!w || !cb || !L) return UW_ERR_INVALID_ARG;
  if (!shape_ok(rows, cols) || chunk_groups < 1 || chunk_groups > 16) return UW_ERR_UNSUPPORTED_SHAPE;
  for (int i = 0; i < kPal; ++i)
    if (cb->code_len[i] > UW_MAX_CODE_LEN) return UW_ERR_CORRUPT;
  const int64_t gpr = cols / kGroup;
  const int64_t n_groups = rows * gpr;
  const int32_t wpr = static_cast<int32_t>((gpr + 31) / 32);
  auto pm = palette_map(cb->palette);

  // pass 1: verbatim flags and coded bits per group
  const int nt = encode_threads(n_groups);
  std::vector<uint8_t> verb(n_groups);
  std::vector<uint32_t> gbits(n_groups);
  std::vector<uint64_t> part_bits(nt, 0);
  std::vector<int64_t> part_verb(nt, 0);
  std::atomic<bool> uncovered{false};
  for_ranges(nt, n_groups, [&](int t, int64_t g0, int64_t g1) {
    uint64_t bits = 0;
    int64_t nv = 0;
    for (int64_t g = g0; g < g1; ++g) {
      const uint16_t* p = w + g * kGroup;
      bool v = false;
      for (int k = 0; k < kGroup; ++k) v |= pm[(p[k] >> 7) & 0xFF] == 255;
      verb[g] = v;
      uint32_t b = 0;
      if (!v) {
        for (int k = 0; k < kGroup; ++k) {
          uint8_t len = cb->code_len[pm[(p[k] >> 7) & 0xFF]];
          if (len == 0) uncovered = true;
          b += len;
        }
      } else {
        ++nv;
      }
      gbits[g] = b;
      bits += b;
    }
    part_bits[t] = bits;
    part_verb[t] = nv;
  });
  if (uncovered) return UW_ERR_CORRUPT;
  uint64_t total = 0;
  int64_t n_verb = 0;
  for (int t = 0; t < nt; ++t) {
    total += part_bits[t];
    n_verb += part_verb[t];
  }
  if (total >= (uint64_t(1) << 32)) return UW_ERR_UNSUPPORTED_SHAPE;

  uw_layout lay;
  std::memset(&lay, 0, sizeof(lay));
  lay.rows = rows;
  lay.cols = cols;
  lay.chunk_groups = chunk_groups;
  lay.words_per_row = wpr;
  lay.n_groups = n_groups;
  lay.n_chunks = (n_groups + chunk_groups - 1) / chunk_groups;
  lay.n_verbatim = n_verb;
  lay.total_bits = static_cast<int64_t>(total);
  lay.stream_words = static_cast<int64_t>((total + 31) / 32) + 2;
  *L = lay;
  if (!sm && !stream && !chunk_bit_off && !vflags && !vprefix && !verbatim) return UW_OK;
  if (!sm || !stream || !chunk_bit_off || !vflags || !vprefix || (n_verb > 0 && !verbatim))
    return UW_ERR_INVALID_ARG;

  // sign+mantissa bytes: own mantissa, pair partner's sign
  for_ranges(nt, n_groups, [&](int, int64_t g0, int64_t g1) {
    for (int64_t i = g0 * kGroup; i < g1 * kGroup; i += 2) {
      uint16_t a = w[i], b = w[i + 1];
      sm[i] = static_cast<uint8_t>(((a & 0x7F) << 1) | (b >> 15));
      sm[i + 1] = static_cast<uint8_t>(((b & 0x7F) << 1) | (a >> 15));
    }
  });

  // chunk offsets
  uint64_t pos = 0;
  for (int64_t g = 0; g < n_groups; ++g) {
    if (g % chunk_groups == 0) chunk_bit_off[g / chunk_groups] = static_cast<uint32_t>(pos);
    pos += gbits[g];
  }
  chunk_bit_off[lay.n_chunks] = static_cast<uint32_t>(pos);

  // bitstream, MSB first.  Each thread packs a contiguous range of groups
  // starting at its global bit offset (known from the group bit counts) into
  // words aligned to the global word grid; it owns every word strictly
  // inside its range, and the at most two words it shares with its
  // neighbours are OR-ed in after all threads finish.
  std::memset(stream, 0, lay.stream_words * sizeof(uint32_t));
  std::vector<uint64_t> start_bit(nt + 1, 0);
  {
    uint64_t b = 0;
    for (int t = 0; t < nt; ++t) {
      start_bit[t] = b;
      b += part_bits[t];
    }
    start_bit[nt] = b;
  }
  struct Edge { int64_t word; uint32_t bits; };
  std::vector<std::array<Edge, 2>> edges(nt, {Edge{-1, 0}, Edge{-1, 0}});
  for_ranges(nt, n_groups, [&](int t, int64_t g0, int64_t g1) {
    const uint64_t b0 = start_bit[t], b1 = start_bit[t + 1];
    if (b1 == b0) return;
    const int64_t first_word = static_cast<int64_t>(b0 / 32), last_word = static_cast<int64_t>((b1 - 1) / 32);
    auto put = [&](int64_t wi, uint32_t v) {
      // words this range shares with a neighbour go to the edge list
      const bool shared_first = wi == first_word && (b0 % 32) != 0;
      const bool shared_last = wi == last_word && (b1 % 32) != 0;
      if (shared_first) {
        edges[t][0] = Edge{wi, v};
      } else if (shared_last) {
        edges[t][1] = Edge{wi, v};
      } else {
        stream[wi] = v;
      }
    };
    uint64_t acc = 0;  // pending bits, right aligned
    int nacc = static_cast<int>(b0 % 32);  // leading zero bits: align to the word grid
    int64_t wi = first_word;
    for (int64_t g = g0; g < g1; ++g) {
      if (verb[g]) continue;
      const uint16_t* p = w + g * kGroup;
      for (int k = 0; k < kGroup; ++k) {
        int sym = pm[(p[k] >> 7) & 0xFF];
        acc = (acc << cb->code_len[sym]) | cb->code[sym];
        nacc += cb->code_len[sym];
        if (nacc >= 32) {
          put(wi++, static_cast<uint32_t>(acc >> (nacc - 32)));
          nacc -= 32;
          acc &= (uint64_t(1) << nacc) - 1;
        }
      }
    }
    if (nacc > 0) put(wi++, static_cast<uint32_t>(acc << (32 - nacc)));
  });
  for (int t = 0; t < nt; ++t)
    for (const Edge& e : edges[t])
      if (e.word >= 0) stream[e.word] |= e.bits;

  // verbatim flags, per-word prefix counts, verbatim store
  std::memset(vflags, 0, sizeof(uint32_t) * rows * wpr);
  for (int64_t g = 0; g < n_groups; ++g)
    if (verb[g]) {
      int64_t r = g / gpr, j = g % gpr;
      vflags[r * wpr + j / 32] |= 1u << (j % 32);
    }
  uint32_t run = 0;
  for (int64_t i = 0; i < rows * wpr; ++i) {
    vprefix[i] = run;
    run += popc32(vflags[i]);
  }
  vprefix[rows * wpr] = run;
  int64_t vs = 0;
  for (int64_t g = 0; g < n_groups; ++g)
    if (verb[g]) std::memcpy(verbatim + (vs++) * kGroup, w + g * kGroup, kGroup * sizeof(uint16_t));
  return UW_OK;
}

extern "C" uw_status uw_validate(const uw_matrix* m) {
  if (!m) return UW_ERR_INVALID_ARG;
  const uw_layout& L = m->L;
  if (!shape_ok(L.rows, L.cols) || L.chunk_groups < 1 || L.chunk_groups > 16)
    return UW_ERR_UNSUPPORTED_SHAPE;
  const int64_t gpr = L.cols / kGroup;
  if (L.n_groups != L.rows * gpr || L.words_per_row != (gpr + 31) / 32 ||
      L.n_chunks != (L.n_groups + L.chunk_groups - 1) / L.chunk_groups ||
      L.stream_words != (L.total_bits + 31) / 32 + 2 || L.total_bits < 0 ||
      L.total_bits >= (int64_t(1) << 32))
    return UW_ERR_CORRUPT;
  if (!m->sm || !m->stream || !m->chunk_bit_off || !m->vflags || !m->vprefix ||
      (L.n_verbatim > 0 && !m->verbatim))
    return UW_ERR_INVALID_ARG;
  // codebook: lengths <= 15, Kraft sum <= 1, codes canonical for the lengths
  const uw_codebook& cb = m->cb;
  uint64_t kraft = 0;  // in units of 2^-15
  int ns = 0, ml = 0;
  for (int i = 0; i < kPal; ++i) {
    if (cb.code_len[i] > UW_MAX_CODE_LEN) return UW_ERR_CORRUPT;
    if (cb.code_len[i]) {
      kraft += uint64_t(1) << (UW_MAX_CODE_LEN - cb.code_len[i]);
      ++ns;
      ml = std::max<int>(ml, cb.code_len[i]);
    }
  }
  if (kraft > (uint64_t(1) << UW_MAX_CODE_LEN)) return UW_ERR_CORRUPT;
  if (cb.n_symbols != ns || cb.max_len != ml) return UW_ERR_CORRUPT;
  uint16_t expect[kPal];
  canonical(cb.code_len, expect);
  for (int i = 0; i < kPal; ++i)
    if (cb.code_len[i] && cb.code[i] != expect[i]) return UW_ERR_CORRUPT;
  for (int i = 0; i < kPal; ++i)
    for (int j = i + 1; j < kPal; ++j)
      if (cb.palette[i] == cb.palette[j]) return UW_ERR_CORRUPT;
  // offsets monotone, ending at total_bits; groups of a chunk need at least
  // 64 * (shortest code) bits unless verbatim -- checked loosely as monotone
  if (m->chunk_bit_off[0] != 0) return UW_ERR_CORRUPT;
  for (int64_t c = 0; c < L.n_chunks; ++c)
    if (m->chunk_bit_off[c + 1] < m->chunk_bit_off[c]) return UW_ERR_CORRUPT;
  if (int64_t(m->chunk_bit_off[L.n_chunks]) != L.total_bits) return UW_ERR_CORRUPT;
  // flag words: no bits beyond the row's groups; prefix = running popcount
  const int64_t nw = L.rows * L.words_per_row;
  uint32_t run = 0;
  for (int64_t i = 0; i < nw; ++i) {
    int64_t j = i % L.words_per_row;
    int64_t valid = std::min<int64_t>(32, gpr - 32 * j);
    if (valid < 32 && (m->vflags[i] >> valid) != 0) return UW_ERR_CORRUPT;
    if (m->vprefix[i] != run) return UW_ERR_CORRUPT;
    run += popc32(m->vflags[i]);
  }
  if (m->vprefix[nw] != run || int64_t(run) != L.n_verbatim) return UW_ERR_CORRUPT;
  // a chunk's coded groups need between 64*min_len and 64*max_len bits each
  int minl = 16;
  for (int i = 0; i < kPal; ++i)
    if (cb.code_len[i]) minl = std::min<int>(minl, cb.code_len[i]);
  for (int64_t c = 0; c < L.n_chunks; ++c) {
    int64_t coded = 0;
    for (int64_t g = c * L.chunk_groups; g < std::min<int64_t>((c + 1) * L.chunk_groups, L.n_groups); ++g) {
      int64_t r = g / gpr, j = g % gpr;
      coded += !((m->vflags[r * L.words_per_row + j / 32] >> (j % 32)) & 1);
    }
    int64_t bits = int64_t(m->chunk_bit_off[c + 1]) - m->chunk_bit_off[c];
    if (coded == 0 ? bits != 0 : (ns == 0 || bits < coded * kGroup * minl || bits > coded * kGroup * ml))
      return UW_ERR_CORRUPT;
  }
  return UW_OK;
}

extern "C" const char* uw_status_string(uw_status s) {
  switch (s) {
    case UW_OK: return "ok";
    case UW_ERR_INVALID_ARG: return "invalid argument";
    case UW_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case UW_ERR_CORRUPT: return "corrupt compressed data";
    case UW_ERR_TIMEOUT: return "on-GPU wait timed out";
    case UW_ERR_CUDA: return "CUDA error";
    case UW_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case UW_ERR_NO_DEVICE: return "no sm_100 device";
  }
  return "unknown status";
}

extern "C" int32_t uw_version(void) { return 100; }

extern "C" uw_status uw_direct_pack_offsets(const uw_layout* L, const uint32_t* vflags, uint32_t* off,
                                            uint64_t* pack_bytes) {
  if (!L || !vflags || !off) return UW_ERR_INVALID_ARG;
  if (!shape_ok(L->rows, L->cols)) return UW_ERR_UNSUPPORTED_SHAPE;
  const int64_t kb_n = L->cols / kGroup;
  const int64_t wpr = (kb_n + 31) / 32;
  if (L->words_per_row != wpr) return UW_ERR_CORRUPT;
  const int64_t mt_n = (L->rows + 127) / 128;
  uint64_t rows_before = 0;  // verbatim rows of the tiles so far
  int64_t t = 0;
  for (int64_t mt = 0; mt < mt_n; ++mt) {
    const int64_t r_end = std::min<int64_t>(L->rows, (mt + 1) * 128);
    for (int64_t kb = 0; kb < kb_n; ++kb, ++t) {
      off[t] = static_cast<uint32_t>(rows_before);
      for (int64_t n = mt * 128; n < r_end; ++n) rows_before += (vflags[n * wpr + kb / 32] >> (kb % 32)) & 1;
      if (rows_before >= (uint64_t(1) << 32)) return UW_ERR_UNSUPPORTED_SHAPE;
    }
  }
  off[t] = static_cast<uint32_t>(rows_before);
  const uint64_t bytes = static_cast<uint64_t>(t) * 12304u + rows_before * 128u;
  if (bytes > (uint64_t(1) << 36)) return UW_ERR_UNSUPPORTED_SHAPE;
  if (pack_bytes) *pack_bytes = bytes;
  return UW_OK;
}

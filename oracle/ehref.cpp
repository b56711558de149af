/*
 * ehref.cpp -- CPU oracle for the split-exponent Huffman codec.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the smoke check and the
 * benchmark's CPU-baseline leg.  Plain single-threaded loops in the order the
 * method states them; no blocking, fusion or reordering.
 *
 * The method (sources named in ehref.h):
 *   S1  split every float into its exponent field and its sign+mantissa bits
 *       (DFloat11 article, "方法介绍"; ZipFloat §2.1 for the BF16 bias 127);
 *   S2  histogram the exponent fields of the whole tensor (DFloat11 article,
 *       "方法介绍": the Huffman tree is built from the exponent distribution);
 *   S3  build a Huffman code over the exponent alphabet;
 *   S4  cut the tensor into fixed-size chunks (paper summary, "实验设计") and
 *       record where each chunk's codes start in the bit stream;
 *   S5  pack the codes tightly, in element order (EncodedExponent), and store
 *       sign+mantissa raw in a separate array (PackedSignMantissa);
 *   S6  decode: read codes back chunk by chunk and re-assemble the floats.
 *
 * Readings where the pages leave a step open (each fixes one format):
 *   - chunk size: a parameter here; the product uses 65,536 elements;
 *   - Huffman ties: a node pool keyed (weight, id), leaves have id = symbol,
 *     the k-th internal node id = 256 + k; always merge the two smallest keys
 *     (this is the minimum-variance rule of Schwartz, 1964);
 *   - length limit Lmax (<= 32): when the Huffman depth exceeds it, use
 *     package-merge (Larmore and Hirschberg, 1990) with items ordered by
 *     (weight, leaves before packages, symbol / creation order);
 *   - rank assignment: the multiset of lengths is dealt out in ascending order
 *     to the symbols sorted by (count descending, symbol ascending);
 *   - canonical codes in (length, symbol) order, as in RFC 1951 §3.2.2;
 *   - one present symbol: length 1, code "0"; no present symbol: no code;
 *   - stream: codes MSB-first, bit p in byte p>>3 at bit 7-(p&7), chunks
 *     back to back with no padding, off[c] = first bit of chunk c, the last
 *     byte zero-padded;
 *   - sign+mantissa: BF16 byte (s<<7)|m7; FP8 nibble (s<<3)|m3, element 2i in
 *     the low nibble of byte i, unused high nibble zero;
 *   - BYTES (FP4 block scale factors): the whole byte is the symbol, there is
 *     no sign+mantissa array.
 */
#include "ehref.h"

#include <algorithm>
#include <cstring>
#include <vector>

namespace {

int alphabet_of(int dtype) {
  if (dtype == EHREF_BF16 || dtype == EHREF_BYTES) return 256;
  if (dtype == EHREF_FP8_E4M3) return 16;
  return 0;
}

uint32_t load_elem(int dtype, const void *in, uint64_t i) {
  if (dtype == EHREF_BF16) return ((const uint16_t *)in)[i];
  return ((const uint8_t *)in)[i];
}

void store_elem(int dtype, void *out, uint64_t i, uint32_t x) {
  if (dtype == EHREF_BF16)
    ((uint16_t *)out)[i] = (uint16_t)x;
  else
    ((uint8_t *)out)[i] = (uint8_t)x;
}

/* S1 for one element.  BF16 = s | e8 | m7 ; E4M3 = s | e4 | m3 ; BYTES: the
 * byte is the symbol. */
void split_one(int dtype, uint32_t x, uint8_t *e, uint8_t *sm) {
  if (dtype == EHREF_BYTES) {
    *e = (uint8_t)x;
    *sm = 0;
  } else if (dtype == EHREF_BF16) {
    uint32_t s = (x >> 15) & 1u, ex = (x >> 7) & 0xFFu, m = x & 0x7Fu;
    *e = (uint8_t)ex;
    *sm = (uint8_t)((s << 7) | m);
  } else {
    uint32_t s = (x >> 7) & 1u, ex = (x >> 3) & 0xFu, m = x & 0x7u;
    *e = (uint8_t)ex;
    *sm = (uint8_t)((s << 3) | m);
  }
}

uint32_t merge_one(int dtype, uint32_t e, uint32_t sm) {
  if (dtype == EHREF_BYTES) return e;
  if (dtype == EHREF_BF16) {
    uint32_t s = (sm >> 7) & 1u, m = sm & 0x7Fu;
    return (s << 15) | (e << 7) | m;
  }
  uint32_t s = (sm >> 3) & 1u, m = sm & 0x7u;
  return (s << 7) | (e << 3) | m;
}

/* Bit writer / reader, MSB-first within each byte. */
void put_bit(uint8_t *buf, uint64_t pos, int bit) {
  if (bit) buf[pos >> 3] |= (uint8_t)(0x80u >> (pos & 7));
}
int get_bit(const uint8_t *buf, uint64_t pos) {
  return (buf[pos >> 3] >> (7 - (pos & 7))) & 1;
}

/* Kraft sum times 2^32 over the given lengths (exact integer arithmetic). */
unsigned __int128 kraft_scaled(const uint8_t *len, int A) {
  unsigned __int128 k = 0;
  for (int s = 0; s < A; s++)
    if (len[s]) k += ((unsigned __int128)1) << (32 - len[s]);
  return k;
}

struct Canon {
  /* per length L = 1..32: number of codes, first canonical code, index of
   * its first symbol in the (length, symbol)-sorted list */
  uint64_t count[33], first[33], index[33];
  std::vector<int> sorted;
};

/* Builds the canonical tables; false if the lengths are not a prefix code
 * (Kraft sum above 1) or a length exceeds 32. */
bool canon_tables(const uint8_t *len, int A, Canon *t) {
  std::memset(t->count, 0, sizeof(t->count));
  for (int s = 0; s < A; s++) {
    if (len[s] > 32) return false;
    if (len[s]) t->count[len[s]]++;
  }
  if (kraft_scaled(len, A) > (((unsigned __int128)1) << 32)) return false;
  uint64_t code = 0, idx = 0;
  for (int L = 1; L <= 32; L++) {
    t->first[L] = code;
    t->index[L] = idx;
    code = (code + t->count[L]) << 1;
    idx += t->count[L];
  }
  t->sorted.clear();
  for (int L = 1; L <= 32; L++)
    for (int s = 0; s < A; s++)
      if (len[s] == L) t->sorted.push_back(s);
  return true;
}

}  // namespace

extern "C" {

int ehref_alphabet(int dtype) { return alphabet_of(dtype); }

int ehref_split(int dtype, const void *in, uint64_t n, uint8_t *e,
                uint8_t *sm) {
  if (!alphabet_of(dtype)) return EHREF_EINVAL;
  for (uint64_t i = 0; i < n; i++) split_one(dtype, load_elem(dtype, in, i), &e[i], &sm[i]);
  return EHREF_OK;
}

int ehref_merge(int dtype, const uint8_t *e, const uint8_t *sm, uint64_t n,
                void *out) {
  if (!alphabet_of(dtype)) return EHREF_EINVAL;
  for (uint64_t i = 0; i < n; i++) store_elem(dtype, out, i, merge_one(dtype, e[i], sm[i]));
  return EHREF_OK;
}

int ehref_histogram(int dtype, const void *in, uint64_t n, uint64_t *cnt) {
  int A = alphabet_of(dtype);
  if (!A) return EHREF_EINVAL;
  for (int s = 0; s < A; s++) cnt[s] = 0;
  for (uint64_t i = 0; i < n; i++) {
    uint8_t e, sm;
    split_one(dtype, load_elem(dtype, in, i), &e, &sm);
    cnt[e]++;
  }
  return EHREF_OK;
}

/* S3a: minimum-variance Huffman.  The pool holds every unmerged node; each
 * step removes the two with the smallest (weight, id) and adds their parent.
 * Leaf depth = code length. */
int ehref_huffman_depths(const uint64_t *cnt, int A, uint8_t *depth) {
  if (A < 1 || A > 256) return EHREF_EINVAL;
  struct Node { uint64_t w; uint32_t id; int parent; };
  std::vector<Node> nodes;
  std::vector<int> pool;           /* indices into nodes, unmerged */
  std::vector<int> leaf_node(A, -1);
  for (int s = 0; s < A; s++) {
    depth[s] = 0;
    if (cnt[s]) {
      leaf_node[s] = (int)nodes.size();
      pool.push_back((int)nodes.size());
      nodes.push_back({cnt[s], (uint32_t)s, -1});
    }
  }
  if (pool.size() <= 1) {
    for (int s = 0; s < A; s++)
      if (cnt[s]) depth[s] = 1;
    return pool.empty() ? 0 : 1;
  }
  uint32_t next_id = 256;
  auto less = [&](int a, int b) {
    if (nodes[a].w != nodes[b].w) return nodes[a].w < nodes[b].w;
    return nodes[a].id < nodes[b].id;
  };
  while (pool.size() > 1) {
    /* find the two smallest keys by a linear scan */
    size_t i1 = 0;
    for (size_t i = 1; i < pool.size(); i++)
      if (less(pool[i], pool[i1])) i1 = i;
    size_t i2 = (i1 == 0) ? 1 : 0;
    for (size_t i = 0; i < pool.size(); i++)
      if (i != i1 && less(pool[i], pool[i2])) i2 = i;
    int a = pool[i1], b = pool[i2];
    int p = (int)nodes.size();
    nodes.push_back({nodes[a].w + nodes[b].w, next_id++, -1});
    nodes[a].parent = p;
    nodes[b].parent = p;
    /* remove a and b from the pool (larger index first), add p */
    size_t hi = std::max(i1, i2), lo = std::min(i1, i2);
    pool.erase(pool.begin() + hi);
    pool.erase(pool.begin() + lo);
    pool.push_back(p);
  }
  int maxd = 0;
  for (int s = 0; s < A; s++) {
    if (leaf_node[s] < 0) continue;
    int d = 0;
    for (int v = leaf_node[s]; nodes[v].parent >= 0; v = nodes[v].parent) d++;
    depth[s] = (uint8_t)(d > 255 ? 255 : d);
    maxd = std::max(maxd, d);
  }
  return maxd;
}

/* S3b: package-merge (coin collector).  Every item carries, per symbol, how
 * many leaves of that symbol it contains.  The list for the deepest level is
 * the sorted leaves; each shallower level merges the leaves with the pairs of
 * adjacent items of the level below.  The first 2m-2 items of the top list
 * are selected; a symbol's length is its count over the selected items. */
int ehref_package_merge(const uint64_t *cnt, int A, int Lmax, uint8_t *len) {
  if (A < 1 || A > 256 || Lmax < 1 || Lmax > 32) return EHREF_EINVAL;
  struct Item { uint64_t w; int is_pkg; std::vector<uint32_t> mult; };
  std::vector<Item> leaves;
  std::vector<int> order;
  for (int s = 0; s < A; s++)
    if (cnt[s]) order.push_back(s);
  int m = (int)order.size();
  if (m < 2) return EHREF_EINVAL;
  if (Lmax < 32 && (uint64_t)m > (1ull << Lmax)) return EHREF_EINFEASIBLE;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cnt[a] < cnt[b]; });
  for (int s : order) {
    Item it{cnt[s], 0, std::vector<uint32_t>(A, 0)};
    it.mult[s] = 1;
    leaves.push_back(it);
  }
  std::vector<Item> list = leaves;
  for (int level = Lmax - 1; level >= 1; level--) {
    std::vector<Item> merged = leaves;
    for (size_t i = 0; i + 1 < list.size(); i += 2) {
      Item p{list[i].w + list[i + 1].w, 1, std::vector<uint32_t>(A, 0)};
      for (int s = 0; s < A; s++) p.mult[s] = list[i].mult[s] + list[i + 1].mult[s];
      merged.push_back(p);
    }
    /* stable: leaves keep (weight, symbol) order, packages creation order,
     * and on equal weight a leaf precedes a package */
    std::stable_sort(merged.begin(), merged.end(), [](const Item &a, const Item &b) {
      if (a.w != b.w) return a.w < b.w;
      return a.is_pkg < b.is_pkg;
    });
    list.swap(merged);
  }
  std::vector<uint64_t> total(A, 0);
  for (int i = 0; i < 2 * m - 2; i++)
    for (int s = 0; s < A; s++) total[s] += list[i].mult[s];
  for (int s = 0; s < A; s++) len[s] = (uint8_t)total[s];
  return EHREF_OK;
}

/* S3: the length rule of the format (see the file header). */
int ehref_code_lengths(const uint64_t *cnt, int A, int Lmax, uint8_t *len) {
  if (A < 1 || A > 256 || Lmax < 1 || Lmax > 32) return EHREF_EINVAL;
  int m = 0;
  for (int s = 0; s < A; s++) m += cnt[s] != 0;
  for (int s = 0; s < A; s++) len[s] = 0;
  if (m == 0) return EHREF_OK;
  if (m == 1) {
    for (int s = 0; s < A; s++)
      if (cnt[s]) len[s] = 1;
    return EHREF_OK;
  }
  if (Lmax < 32 && (uint64_t)m > (1ull << Lmax)) return EHREF_EINFEASIBLE;
  std::vector<uint8_t> raw(A, 0);
  int maxd = ehref_huffman_depths(cnt, A, raw.data());
  if (maxd > Lmax) {
    int rc = ehref_package_merge(cnt, A, Lmax, raw.data());
    if (rc) return rc;
  }
  /* rank assignment */
  std::vector<int> lens, syms;
  for (int s = 0; s < A; s++)
    if (cnt[s]) {
      lens.push_back(raw[s]);
      syms.push_back(s);
    }
  std::sort(lens.begin(), lens.end());
  std::stable_sort(syms.begin(), syms.end(), [&](int a, int b) { return cnt[a] > cnt[b]; });
  for (size_t k = 0; k < syms.size(); k++) len[syms[k]] = (uint8_t)lens[k];
  return EHREF_OK;
}

/* Canonical codes: symbols in (length, symbol) order; the first gets 0, each
 * next one (previous + 1) shifted left by the length increase. */
int ehref_canonical_codes(const uint8_t *len, int A, uint32_t *code) {
  if (A < 1 || A > 256) return EHREF_EINVAL;
  std::vector<int> order;
  for (int s = 0; s < A; s++) {
    code[s] = 0;
    if (len[s] > 32) return EHREF_EINVAL;
    if (len[s]) order.push_back(s);
  }
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return len[a] < len[b]; });
  uint64_t c = 0;
  for (size_t k = 0; k < order.size(); k++) {
    if (k > 0) c = (c + 1) << (len[order[k]] - len[order[k - 1]]);
    code[order[k]] = (uint32_t)c;
  }
  return EHREF_OK;
}

uint64_t ehref_sm_bytes(int dtype, uint64_t n) {
  if (dtype == EHREF_BYTES) return 0;
  return dtype == EHREF_BF16 ? n : (n + 1) / 2;
}

int ehref_pack_sm(int dtype, const void *in, uint64_t n, uint8_t *out) {
  if (!alphabet_of(dtype)) return EHREF_EINVAL;
  uint64_t nb = ehref_sm_bytes(dtype, n);
  for (uint64_t b = 0; b < nb; b++) out[b] = 0;
  for (uint64_t i = 0; i < n; i++) {
    uint8_t e, sm;
    split_one(dtype, load_elem(dtype, in, i), &e, &sm);
    if (dtype == EHREF_BF16)
      out[i] = sm;
    else if (dtype == EHREF_FP8_E4M3)
      out[i / 2] |= (uint8_t)(sm << (4 * (i & 1)));
  }
  return EHREF_OK;
}

uint64_t ehref_num_chunks(uint64_t n, uint32_t chunk) {
  return chunk ? (n + chunk - 1) / chunk : 0;
}

/* S4 + S5: append each element's code MSB-first; off[c] = start of chunk c. */
int ehref_encode(int dtype, const void *in, uint64_t n, uint32_t chunk,
                 const uint8_t *len, const uint32_t *code, uint64_t *off,
                 uint8_t *stream, uint64_t cap, uint64_t *total_bits) {
  if (!alphabet_of(dtype) || chunk == 0) return EHREF_EINVAL;
  uint64_t C = ehref_num_chunks(n, chunk);
  uint64_t bits = 0;
  for (uint64_t i = 0; i < n; i++) {
    uint8_t e, sm;
    split_one(dtype, load_elem(dtype, in, i), &e, &sm);
    if (len[e] == 0) return EHREF_EINVAL; /* symbol without a code */
    bits += len[e];
  }
  if ((bits + 7) / 8 > cap) return EHREF_ECAPACITY;
  for (uint64_t b = 0; b < (bits + 7) / 8; b++) stream[b] = 0;
  uint64_t pos = 0;
  for (uint64_t i = 0; i < n; i++) {
    if (i % chunk == 0) off[i / chunk] = pos;
    uint8_t e, sm;
    split_one(dtype, load_elem(dtype, in, i), &e, &sm);
    for (int b = len[e] - 1; b >= 0; b--) put_bit(stream, pos++, (code[e] >> b) & 1u);
  }
  off[C] = pos;
  *total_bits = pos;
  return EHREF_OK;
}

int ehref_value_index(int dtype, const void *in, uint64_t n, uint32_t chunk,
                      const uint8_t *len, uint32_t *index) {
  if (!alphabet_of(dtype) || chunk == 0 || chunk % EHREF_INDEX_STRIDE) return EHREF_EINVAL;
  const uint64_t C = ehref_num_chunks(n, chunk);
  const uint32_t per = chunk / EHREF_INDEX_STRIDE;
  for (uint64_t c = 0; c < C; c++) {
    uint32_t bits = 0;  // from the chunk's first bit
    for (uint64_t j = 0; j < chunk; j++) {
      const uint64_t i = c * chunk + j;
      if (j % EHREF_INDEX_STRIDE == 0) index[c * per + j / EHREF_INDEX_STRIDE] = bits;
      if (i < n) {
        uint8_t e, sm;
        split_one(dtype, load_elem(dtype, in, i), &e, &sm);
        if (len[e] == 0) return EHREF_EINVAL;
        bits += len[e];
      }
    }
    // entries past the last value of a short chunk: the chunk's total bits
    for (uint32_t k = 0; k < per; k++)
      if (c * chunk + (uint64_t)k * EHREF_INDEX_STRIDE >= n) index[c * per + k] = bits;
  }
  return EHREF_OK;
}

int ehref_compress(int dtype, const void *in, uint64_t n, uint32_t chunk,
                   int Lmax, uint8_t *len, uint32_t *code, uint64_t *off,
                   uint8_t *stream, uint64_t cap, uint8_t *sm_packed,
                   uint64_t *total_bits) {
  int A = alphabet_of(dtype);
  if (!A || chunk == 0 || Lmax < 1 || Lmax > 32) return EHREF_EINVAL;
  std::vector<uint64_t> cnt(A);
  int rc = ehref_histogram(dtype, in, n, cnt.data());
  if (rc) return rc;
  rc = ehref_code_lengths(cnt.data(), A, Lmax, len);
  if (rc) return rc;
  rc = ehref_canonical_codes(len, A, code);
  if (rc) return rc;
  rc = ehref_pack_sm(dtype, in, n, sm_packed);
  if (rc) return rc;
  return ehref_encode(dtype, in, n, chunk, len, code, off, stream, cap, total_bits);
}

/* S6: textbook canonical decoding, one bit at a time. */
int ehref_decompress_chunks(int dtype, uint64_t n, uint32_t chunk,
                            const uint8_t *len, const uint32_t *code,
                            const uint64_t *off, const uint8_t *stream,
                            uint64_t stream_bytes, const uint8_t *sm_packed,
                            uint32_t first, uint32_t count, void *out) {
  int A = alphabet_of(dtype);
  if (!A || chunk == 0) return EHREF_EINVAL;
  uint64_t C = ehref_num_chunks(n, chunk);
  if ((uint64_t)first + count > C) return EHREF_EINVAL;
  if (count == 0) return EHREF_OK;
  Canon t;
  if (!canon_tables(len, A, &t)) return EHREF_ECORRUPT;
  /* the stored codes must be the canonical ones */
  std::vector<uint32_t> want(A);
  ehref_canonical_codes(len, A, want.data());
  for (int s = 0; s < A; s++)
    if (len[s] && code[s] != want[s]) return EHREF_ECORRUPT;
  if (off[0] != 0) return EHREF_ECORRUPT;
  for (uint64_t c = 0; c < C; c++)
    if (off[c + 1] < off[c]) return EHREF_ECORRUPT;
  if ((off[C] + 7) / 8 > stream_bytes) return EHREF_ECORRUPT;
  for (uint64_t c = first; c < (uint64_t)first + count; c++) {
    uint64_t pos = off[c], end = off[c + 1];
    uint64_t i0 = c * chunk, i1 = std::min<uint64_t>(n, i0 + chunk);
    for (uint64_t i = i0; i < i1; i++) {
      uint64_t v = 0;
      int sym = -1;
      for (int L = 1; L <= 32; L++) {
        if (pos >= end) return EHREF_ECORRUPT;
        v = (v << 1) | (uint64_t)get_bit(stream, pos++);
        if (t.count[L] && v >= t.first[L] && v - t.first[L] < t.count[L]) {
          sym = t.sorted[t.index[L] + (v - t.first[L])];
          break;
        }
      }
      if (sym < 0) return EHREF_ECORRUPT;
      uint32_t sm = 0;
      if (dtype == EHREF_BF16)
        sm = sm_packed[i];
      else if (dtype == EHREF_FP8_E4M3)
        sm = (sm_packed[i / 2] >> (4 * (i & 1))) & 0xFu;
      store_elem(dtype, out, i - (uint64_t)first * chunk, merge_one(dtype, (uint32_t)sym, sm));
    }
    if (pos != end) return EHREF_ECORRUPT;
  }
  return EHREF_OK;
}

int ehref_decompress(int dtype, uint64_t n, uint32_t chunk, const uint8_t *len,
                     const uint32_t *code, const uint64_t *off,
                     const uint8_t *stream, uint64_t stream_bytes,
                     const uint8_t *sm_packed, void *out) {
  uint64_t C = ehref_num_chunks(n, chunk);
  return ehref_decompress_chunks(dtype, n, chunk, len, code, off, stream,
                                 stream_bytes, sm_packed, 0, (uint32_t)C, out);
}

int ehref_page_encode(int dtype, const void *in, uint64_t n, const uint8_t *len,
                      const uint32_t *code, uint8_t *slot, uint64_t slot_bytes,
                      uint8_t *sm_packed, uint8_t *raw_exps, uint64_t *bits,
                      int *raw) {
  if (!alphabet_of(dtype)) return EHREF_EINVAL;
  int rc = ehref_pack_sm(dtype, in, n, sm_packed);
  if (rc) return rc;
  /* code bits of the page; an exponent without a code forces raw storage */
  uint64_t total = 0;
  bool missing = false;
  for (uint64_t i = 0; i < n; i++) {
    uint8_t e, sm;
    split_one(dtype, load_elem(dtype, in, i), &e, &sm);
    if (len[e] == 0) missing = true;
    total += len[e];
  }
  if (missing || (total + 7) / 8 + 16 > slot_bytes) {
    for (uint64_t i = 0; i < n; i++) {
      uint8_t e, sm;
      split_one(dtype, load_elem(dtype, in, i), &e, &sm);
      raw_exps[i] = e;
    }
    *raw = 1;
    *bits = 0;
    return EHREF_OK;
  }
  for (uint64_t b = 0; b < slot_bytes; b++) slot[b] = 0;
  uint64_t pos = 0;
  for (uint64_t i = 0; i < n; i++) {
    uint8_t e, sm;
    split_one(dtype, load_elem(dtype, in, i), &e, &sm);
    for (int b = len[e] - 1; b >= 0; b--) put_bit(slot, pos++, (code[e] >> b) & 1u);
  }
  *raw = 0;
  *bits = pos;
  return EHREF_OK;
}

int ehref_page_decode(int dtype, uint64_t n, const uint8_t *len,
                      const uint32_t *code, const uint8_t *slot,
                      uint64_t slot_bytes, uint64_t bits, int raw,
                      const uint8_t *raw_exps, const uint8_t *sm_packed,
                      void *out) {
  if (!alphabet_of(dtype)) return EHREF_EINVAL;
  if (raw) {
    for (uint64_t i = 0; i < n; i++) {
      uint32_t sm = 0;
      if (dtype == EHREF_BF16)
        sm = sm_packed[i];
      else if (dtype == EHREF_FP8_E4M3)
        sm = (sm_packed[i / 2] >> (4 * (i & 1))) & 0xFu;
      store_elem(dtype, out, i, merge_one(dtype, raw_exps[i], sm));
    }
    return EHREF_OK;
  }
  /* one coded chunk: offsets [0, bits] */
  uint64_t off[2] = {0, bits};
  if ((bits + 7) / 8 > slot_bytes) return EHREF_ECORRUPT;
  return ehref_decompress_chunks(dtype, n, n ? (uint32_t)n : 1u, len, code, off, slot,
                                 slot_bytes, sm_packed, 0, n ? 1u : 0u, out);
}

/* ---- stored form (see ehref.h) ---- */

uint32_t ehref_crc32(const uint8_t *data, uint64_t len) {
  /* bit by bit, lowest bit first, with the reflected polynomial */
  uint32_t crc = 0xFFFFFFFFu;
  for (uint64_t i = 0; i < len; i++) {
    crc ^= data[i];
    for (int b = 0; b < 8; b++) {
      if (crc & 1u)
        crc = (crc >> 1) ^ 0xEDB88320u;
      else
        crc >>= 1;
    }
  }
  return ~crc;
}

static void le_store(uint8_t *p, uint64_t v, int bytes) {
  for (int i = 0; i < bytes; i++) p[i] = (uint8_t)(v >> (8 * i));
}

int ehref_container_write(int dtype, uint64_t n, uint32_t chunk, int lmax,
                          const uint8_t *len, const uint32_t *code,
                          const uint64_t *chunk_bit_off, const uint8_t *stream,
                          uint64_t bits, const uint8_t *sm_packed,
                          const uint32_t *index, uint8_t *out, uint64_t out_cap,
                          uint64_t *size) {
  const int A = alphabet_of(dtype);
  if (!A || chunk == 0 || chunk % 128 != 0 || lmax < 1 || lmax > 32 || !size) return EHREF_EINVAL;
  const uint64_t C = ehref_num_chunks(n, chunk);
  /* section contents, in order */
  uint64_t slen[6];
  const uint8_t *sptr[6];
  slen[0] = (uint64_t)A;              sptr[0] = len;
  slen[1] = 4 * (uint64_t)A;          sptr[1] = (const uint8_t *)code;
  slen[2] = 8 * (C + 1);              sptr[2] = (const uint8_t *)chunk_bit_off;
  slen[3] = (bits + 7) / 8;           sptr[3] = stream;
  slen[4] = ehref_sm_bytes(dtype, n); sptr[4] = sm_packed;
  slen[5] = index ? 4 * C * (chunk / 128) : 0;
  sptr[5] = (const uint8_t *)index;
  /* offsets: from 192, each section at the next multiple of 16 */
  uint64_t soff[6], pos = 192;
  for (int i = 0; i < 6; i++) {
    soff[i] = pos;
    pos += slen[i];
    while (pos % 16) pos++;
  }
  *size = pos;
  if (!out) return EHREF_OK;
  if (out_cap < pos) return EHREF_ECAPACITY;
  for (uint64_t i = 0; i < pos; i++) out[i] = 0;
  out[0] = 'E'; out[1] = 'X'; out[2] = 'H'; out[3] = 'F';
  le_store(out + 4, 1, 2);
  out[6] = (uint8_t)dtype;
  out[7] = (uint8_t)lmax;
  le_store(out + 8, chunk, 4);
  le_store(out + 12, index ? 1 : 0, 4);
  le_store(out + 16, n, 8);
  le_store(out + 24, C, 8);
  le_store(out + 32, bits, 8);
  for (int i = 0; i < 6; i++) {
    for (uint64_t j = 0; j < slen[i]; j++) out[soff[i] + j] = sptr[i][j];
    uint8_t *entry = out + 40 + 24 * i;
    le_store(entry, soff[i], 8);
    le_store(entry + 8, slen[i], 8);
    le_store(entry + 16, ehref_crc32(out + soff[i], slen[i]), 4);
  }
  le_store(out + 184, ehref_crc32(out, 184), 4);
  return EHREF_OK;
}

}  // extern "C"

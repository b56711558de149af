// eh_container.cu -- serialisation of one compressed tensor (host code).
//
// The weights a deployment decompresses are compressed once, offline, and
// stored (the DFloat11 article, "方法介绍", and the ZipFloat paper, §4.2:
// model weights are compressed ahead of time and decompressed on the GPU).
// This file defines the stored form: one self-describing byte container per
// tensor, every part guarded by a CRC-32, written from and read into host
// memory.  Layout (all integers little-endian):
//
//   0    "EXHF"                       magic
//   4    u16 version (1)
//   6    u8  dtype, u8 max_code_len
//   8    u32 chunk_elems
//   12   u32 flags (bit 0: value index present)
//   16   u64 n, u64 n_chunks, u64 exp_stream_bits
//   40   6 section entries {u64 offset, u64 length, u32 crc32, u32 0}:
//        code_len, code, chunk_bit_off, exp_stream, sign_mant, value_index
//   184  u32 crc32 of bytes [0, 184), u32 0
//   192  the sections in that order, each at a 16-byte aligned offset,
//        zero bytes between them and after the last up to a multiple of 16
//        (checked on reading, so that no byte of a container goes unchecked).
//
// Section contents: code_len A bytes; code A u32; chunk_bit_off n_chunks+1
// u64; exp_stream ceil(exp_stream_bits/8) bytes; sign_mant the packed
// sign/mantissa bytes; value_index n_chunks * chunk_elems/128 u32 (length 0
// when absent).  CRC-32 is the IEEE 802.3 / zlib one (reflected polynomial
// 0xEDB88320, initial and final value 0xFFFFFFFF).
#include <cstring>

#include "eh_internal.cuh"

namespace {

constexpr uint32_t kVersion = 1;
constexpr uint64_t kHeaderBytes = 192;
constexpr int kSections = 6;

struct Crc32Table {
  uint32_t t[256];
  Crc32Table() {
    for (uint32_t i = 0; i < 256; i++) {
      uint32_t c = i;
      for (int k = 0; k < 8; k++) c = (c & 1u) ? 0xEDB88320u ^ (c >> 1) : c >> 1;
      t[i] = c;
    }
  }
};
const Crc32Table kCrc;

uint32_t crc32(const uint8_t *p, uint64_t len) {
  uint32_t c = 0xFFFFFFFFu;
  for (uint64_t i = 0; i < len; i++) c = kCrc.t[(c ^ p[i]) & 0xFFu] ^ (c >> 8);
  return c ^ 0xFFFFFFFFu;
}

void put16(uint8_t *p, uint32_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
void put32(uint8_t *p, uint32_t v) { for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i)); }
void put64(uint8_t *p, uint64_t v) { for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i)); }
uint32_t get16(const uint8_t *p) { return (uint32_t)p[0] | ((uint32_t)p[1] << 8); }
uint32_t get32(const uint8_t *p) {
  uint32_t v = 0;
  for (int i = 0; i < 4; i++) v |= (uint32_t)p[i] << (8 * i);
  return v;
}
uint64_t get64(const uint8_t *p) {
  uint64_t v = 0;
  for (int i = 0; i < 8; i++) v |= (uint64_t)p[i] << (8 * i);
  return v;
}
uint64_t up16(uint64_t x) { return (x + 15) & ~uint64_t(15); }

bool plan_valid(int dtype, uint32_t chunk, uint32_t lmax) {
  return (dtype == EH_BF16 || dtype == EH_FP8_E4M3 || dtype == EH_BYTES) && chunk >= 1024 && chunk <= 65536 &&
         chunk % 1024 == 0 && lmax >= 1 && lmax <= EH_MAX_CODE_LEN;
}

// Section lengths of a tensor (the value index only when present).
void section_lengths(int dtype, uint32_t chunk, uint64_t n, uint64_t bits, bool index, uint64_t len[kSections]) {
  const uint64_t A = eh::alphabet_of(dtype);
  const uint64_t C = (n + chunk - 1) / chunk;
  len[0] = A;
  len[1] = 4 * A;
  len[2] = 8 * (C + 1);
  len[3] = (bits + 7) / 8;
  len[4] = dtype == EH_BYTES ? 0 : (dtype == EH_BF16 ? n : (n + 1) / 2);
  len[5] = index ? 4 * C * (chunk / EH_INDEX_STRIDE) : 0;
}

uint64_t layout(const uint64_t len[kSections], uint64_t off[kSections]) {
  uint64_t pos = kHeaderBytes;
  for (int i = 0; i < kSections; i++) {
    off[i] = pos;
    pos = up16(pos + len[i]);
  }
  return pos;
}

}  // namespace

extern "C" {

eh_status eh_container_size(const eh_plan_t *plan, uint64_t n, uint64_t exp_stream_bits, int with_index,
                            uint64_t *bytes) {
  if (!plan || !bytes || !plan_valid(plan->dtype, plan->chunk_elems, plan->max_code_len)) return EH_ERR_INVALID_ARG;
  if (n > (1ull << 40) || exp_stream_bits > n * plan->max_code_len) return EH_ERR_INVALID_ARG;
  uint64_t len[kSections], off[kSections];
  section_lengths(plan->dtype, plan->chunk_elems, n, exp_stream_bits, with_index != 0, len);
  *bytes = layout(len, off);
  return EH_OK;
}

eh_status eh_container_write(const eh_plan_t *plan, const eh_compressed_t *c, void *dst, uint64_t dst_bytes) {
  if (!plan || !c || !dst || !plan_valid(plan->dtype, plan->chunk_elems, plan->max_code_len))
    return EH_ERR_INVALID_ARG;
  if (c->dtype != plan->dtype || c->n > (1ull << 40) || c->exp_stream_bits > c->n * plan->max_code_len)
    return EH_ERR_INVALID_ARG;
  const uint64_t C = (c->n + plan->chunk_elems - 1) / plan->chunk_elems;
  if (c->n_chunks != C) return EH_ERR_INVALID_ARG;
  const bool index = c->value_index != nullptr;
  uint64_t len[kSections], off[kSections];
  section_lengths(plan->dtype, plan->chunk_elems, c->n, c->exp_stream_bits, index, len);
  const uint64_t total = layout(len, off);
  if (dst_bytes < total) return EH_ERR_NOMEM;
  const void *src[kSections] = {c->code_len, c->code, c->chunk_bit_off, c->exp_stream, c->sign_mant, c->value_index};
  for (int i = 0; i < kSections; i++)
    if (len[i] && !src[i]) return EH_ERR_INVALID_ARG;
  if (len[3] > c->exp_stream_cap) return EH_ERR_INVALID_ARG;
  uint8_t *o = (uint8_t *)dst;
  std::memset(o, 0, total);
  std::memcpy(o, "EXHF", 4);
  put16(o + 4, kVersion);
  o[6] = (uint8_t)plan->dtype;
  o[7] = (uint8_t)plan->max_code_len;
  put32(o + 8, plan->chunk_elems);
  put32(o + 12, index ? 1u : 0u);
  put64(o + 16, c->n);
  put64(o + 24, C);
  put64(o + 32, c->exp_stream_bits);
  for (int i = 0; i < kSections; i++) {
    if (len[i]) std::memcpy(o + off[i], src[i], len[i]);
    uint8_t *e = o + 40 + 24 * i;
    put64(e, off[i]);
    put64(e + 8, len[i]);
    put32(e + 16, crc32(o + off[i], len[i]));
  }
  put32(o + 184, crc32(o, 184));
  return EH_OK;
}

eh_status eh_container_read(const void *src, uint64_t src_bytes, eh_plan_t *plan, eh_compressed_t *view) {
  if (!src || !plan || !view) return EH_ERR_INVALID_ARG;
  const uint8_t *s = (const uint8_t *)src;
  if (src_bytes < kHeaderBytes || std::memcmp(s, "EXHF", 4) != 0) return EH_ERR_CORRUPT;
  if (get32(s + 184) != crc32(s, 184) || get16(s + 4) != kVersion) return EH_ERR_CORRUPT;
  const int dtype = s[6];
  const uint32_t lmax = s[7], chunk = get32(s + 8), flags = get32(s + 12);
  const uint64_t n = get64(s + 16), C = get64(s + 24), bits = get64(s + 32);
  if (!plan_valid(dtype, chunk, lmax) || (flags & ~1u) || n > (1ull << 40) || C != (n + chunk - 1) / chunk ||
      bits > n * lmax)
    return EH_ERR_CORRUPT;
  uint64_t len[kSections], off[kSections];
  section_lengths(dtype, chunk, n, bits, (flags & 1u) != 0, len);
  const uint64_t total = layout(len, off);
  if (src_bytes < total) return EH_ERR_CORRUPT;
  if (get32(s + 188) != 0) return EH_ERR_CORRUPT;
  for (int i = 0; i < kSections; i++) {
    const uint8_t *e = s + 40 + 24 * i;
    if (get64(e) != off[i] || get64(e + 8) != len[i] || get32(e + 20) != 0) return EH_ERR_CORRUPT;
    if (get32(e + 16) != crc32(s + off[i], len[i])) return EH_ERR_CORRUPT;
    // the padding after the section is zero: every byte of a container is checked
    const uint64_t pad_end = i + 1 < kSections ? off[i + 1] : total;
    for (uint64_t k = off[i] + len[i]; k < pad_end; k++)
      if (s[k]) return EH_ERR_CORRUPT;
  }
  plan->dtype = dtype;
  plan->chunk_elems = chunk;
  plan->max_code_len = lmax;
  plan->reserved = 0;
  std::memset(view, 0, sizeof(*view));
  view->dtype = dtype;
  view->n = n;
  view->n_chunks = (uint32_t)C;
  view->code_len = const_cast<uint8_t *>(s + off[0]);
  view->code = (uint32_t *)const_cast<uint8_t *>(s + off[1]);
  view->chunk_bit_off = (uint64_t *)const_cast<uint8_t *>(s + off[2]);
  view->exp_stream = const_cast<uint8_t *>(s + off[3]);
  view->exp_stream_cap = len[3];
  view->sign_mant = len[4] ? const_cast<uint8_t *>(s + off[4]) : nullptr;
  view->exp_stream_bits = bits;
  view->value_index = len[5] ? (uint32_t *)const_cast<uint8_t *>(s + off[5]) : nullptr;
  return EH_OK;
}

}  // extern "C"

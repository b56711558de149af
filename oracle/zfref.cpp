/*
 * zfref.cpp -- CPU oracle for the ZipFloat comparison codec (BF16).
 *
 * TEST INFRASTRUCTURE ONLY.  Plain loops over each block in the order the
 * ZipFloat page states the steps (§3.2 then §3.3); the format and its readings
 * are listed in zfref.h.
 */
#include "zfref.h"

#include "ehref.h"

namespace {

inline uint32_t exp_field(uint16_t x) { return (x >> 7) & 0xFFu; }

}  // namespace

extern "C" {

uint64_t zfref_blocks(uint64_t n) { return (n + ZFREF_BLOCK - 1) / ZFREF_BLOCK; }

int zfref_block_base(const uint16_t *in, uint32_t count, uint32_t *md, uint32_t *lb) {
  if (!in || !md || !lb || count == 0 || count > ZFREF_BLOCK) return EHREF_EINVAL;
  // §3.2: the most frequent exponent (MD) of the block
  uint32_t hist[256] = {0};
  for (uint32_t i = 0; i < count; i++) hist[exp_field(in[i])]++;
  uint32_t best = 0;
  for (uint32_t e = 1; e < 256; e++)
    if (hist[e] > hist[best]) best = e;  // strict: ties keep the smaller field
  *md = best;
  // the dominant range starts Delta* = 6 below MD (the page's fixed offset)
  *lb = (best + 256 - 6) & 0xFFu;
  return EHREF_OK;
}

int zfref_compress(const uint16_t *in, uint64_t n, uint8_t *sign_mant, uint32_t *meta, uint32_t *dense,
                   uint32_t *sparse_off, uint16_t *sparse, uint64_t sparse_cap, uint64_t *n_records) {
  if (!n_records || (n && (!in || !sign_mant || !meta || !dense || !sparse_off))) return EHREF_EINVAL;
  const uint64_t B = zfref_blocks(n);
  uint64_t rec = 0;
  for (uint64_t b = 0; b < B; b++) {
    const uint64_t i0 = b * ZFREF_BLOCK;
    const uint32_t count = (uint32_t)((n - i0) < ZFREF_BLOCK ? (n - i0) : ZFREF_BLOCK);
    uint32_t md, lb;
    zfref_block_base(in + i0, count, &md, &lb);
    // Eq. 4: remapped exponent r = e - l_b (8 bits)
    uint32_t *planes = dense + b * 3 * 64;
    for (uint32_t w = 0; w < 3 * 64; w++) planes[w] = 0;
    sparse_off[b] = (uint32_t)rec;
    uint32_t nnz = 0;
    for (uint32_t i = 0; i < count; i++) {
      const uint16_t x = in[i0 + i];
      const uint32_t r = (exp_field(x) + 256 - lb) & 0xFFu;
      // dense part: the low three bits, one bit plane each
      for (uint32_t p = 0; p < 3; p++)
        if ((r >> p) & 1u) planes[p * 64 + i / 32] |= 1u << (i % 32);
      // sparse part: a record for a non-zero high part
      if (r >> 3) {
        if (rec >= sparse_cap || !sparse) return EHREF_ECAPACITY;
        sparse[rec++] = (uint16_t)((i << 5) | (r >> 3));
        nnz++;
      }
      sign_mant[i0 + i] = (uint8_t)(((x >> 8) & 0x80u) | (x & 0x7Fu));
    }
    meta[b] = lb | (nnz << 8);
  }
  *n_records = rec;
  return EHREF_OK;
}

int zfref_decompress(uint64_t n, const uint8_t *sign_mant, const uint32_t *meta, const uint32_t *dense,
                     const uint32_t *sparse_off, const uint16_t *sparse, uint64_t n_records, uint16_t *out) {
  if (n && (!sign_mant || !meta || !dense || !sparse_off || !out)) return EHREF_EINVAL;
  const uint64_t B = zfref_blocks(n);
  for (uint64_t b = 0; b < B; b++) {
    const uint64_t i0 = b * ZFREF_BLOCK;
    const uint32_t count = (uint32_t)((n - i0) < ZFREF_BLOCK ? (n - i0) : ZFREF_BLOCK);
    const uint32_t lb = meta[b] & 0xFFu, nnz = meta[b] >> 8;
    if (nnz > count || (uint64_t)sparse_off[b] + nnz > n_records || (nnz && !sparse)) return EHREF_ECORRUPT;
    uint8_t high[ZFREF_BLOCK] = {0};
    uint32_t prev = 0;
    for (uint32_t k = 0; k < nnz; k++) {
      const uint16_t rcd = sparse[sparse_off[b] + k];
      const uint32_t i = rcd >> 5;
      if (i >= count || (k && i <= prev)) return EHREF_ECORRUPT;
      high[i] = (uint8_t)(rcd & 31u);
      prev = i;
    }
    const uint32_t *planes = dense + b * 3 * 64;
    for (uint32_t i = 0; i < count; i++) {
      uint32_t r = (uint32_t)high[i] << 3;
      for (uint32_t p = 0; p < 3; p++) r |= ((planes[p * 64 + i / 32] >> (i % 32)) & 1u) << p;
      const uint32_t e = (r + lb) & 0xFFu;  // inverse of Eq. 4
      const uint32_t sm = sign_mant[i0 + i];
      out[i0 + i] = (uint16_t)(((sm & 0x80u) << 8) | (e << 7) | (sm & 0x7Fu));
    }
  }
  return EHREF_OK;
}

}  // extern "C"

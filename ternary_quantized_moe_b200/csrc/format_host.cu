// format_host.cu -- host packers/unpackers for the two ternary containers.
//
// PQ2_0 ("Scion-35B-A3B" model card, Weight Representation: 2-bit slots and one
// fp16 scale per 128 weights, 34 bytes) and PTQ1_0 ("Scion-FlashNext-176B-A6B"
// model card, Weight Representation: base-3 trits and one fp16 scale, 28 bytes).
// Bit orders follow the container specification in include/scion.h.
#include <string.h>

#include "scion_internal.cuh"

extern "C" size_t scion_block_bytes(int fmt) {
  if (fmt == SCION_PQ2_0) return scion::kPq2Block;
  if (fmt == SCION_PTQ1_0) return scion::kPtq1Block;
  return 0;
}

extern "C" int scion_pack_pq2(const int8_t* codes, const uint16_t* scales, int64_t n_groups, uint8_t* out) {
  if (!codes || !scales || !out || n_groups < 0) return SCION_EINVAL;
  for (int64_t g = 0; g < n_groups; ++g) {
    const int8_t* c = codes + g * 128;
    uint8_t* o = out + g * scion::kPq2Block;
    for (int i = 0; i < 32; ++i) {
      unsigned b = 0;
      for (int j = 0; j < 4; ++j) {
        int v = c[4 * i + j];
        if (v < -1 || v > 1) return SCION_EINVAL;
        b |= unsigned(v + 1) << (2 * j);
      }
      o[i] = uint8_t(b);
    }
    o[32] = uint8_t(scales[g] & 0xff);
    o[33] = uint8_t(scales[g] >> 8);
  }
  return SCION_OK;
}

extern "C" int scion_pack_ptq1(const int8_t* codes, const uint16_t* scales, int64_t n_groups, uint8_t* out) {
  if (!codes || !scales || !out || n_groups < 0) return SCION_EINVAL;
  for (int64_t g = 0; g < n_groups; ++g) {
    const int8_t* c = codes + g * 128;
    uint8_t* o = out + g * scion::kPtq1Block;
    for (int i = 0; i < 128; ++i)
      if (c[i] < -1 || c[i] > 1) return SCION_EINVAL;
    for (int q = 0; q < 26; ++q) {
      // quintet bytes q < 25 hold 5 trits, byte 25 holds the last 3; lowest weight = lowest digit
      int n = q < 25 ? 5 : 3, v = 0;
      for (int j = n - 1; j >= 0; --j) v = v * 3 + (c[5 * q + j] + 1);
      o[q] = uint8_t(v);
    }
    o[26] = uint8_t(scales[g] & 0xff);
    o[27] = uint8_t(scales[g] >> 8);
  }
  return SCION_OK;
}

extern "C" int scion_unpack(int fmt, const uint8_t* in, int64_t n_groups, int8_t* codes, uint16_t* scales) {
  if (!in || !codes || !scales || n_groups < 0) return SCION_EINVAL;
  if (fmt != SCION_PQ2_0 && fmt != SCION_PTQ1_0) return SCION_EINVAL;
  int st = SCION_OK;
  for (int64_t g = 0; g < n_groups; ++g) {
    int8_t* c = codes + g * 128;
    if (fmt == SCION_PQ2_0) {
      const uint8_t* b = in + g * scion::kPq2Block;
      for (int i = 0; i < 128; ++i) {
        int f = (b[i >> 2] >> (2 * (i & 3))) & 3;
        if (f == 3) st = SCION_EFORMAT;
        c[i] = int8_t(f == 3 ? 0 : f - 1);
      }
      scales[g] = uint16_t(b[32] | (b[33] << 8));
    } else {
      const uint8_t* b = in + g * scion::kPtq1Block;
      for (int q = 0; q < 26; ++q) {
        int n = q < 25 ? 5 : 3, v = b[q];
        bool bad = v >= (q < 25 ? 243 : 27);
        if (bad) st = SCION_EFORMAT;
        for (int j = 0; j < n; ++j) {
          c[5 * q + j] = int8_t(bad ? 0 : v % 3 - 1);
          v /= 3;
        }
      }
      scales[g] = uint16_t(b[26] | (b[27] << 8));
    }
  }
  return st;
}

/*
 * CPU oracle for IQ2_KS / IQ2_K 2-bit reconstruction.
 *
 * TEST INFRASTRUCTURE ONLY: called from tests/, the package's smoke check and
 * the benchmark's CPU-baseline leg; never from the product path. It shares no
 * code, header, table or constant with the CUDA library.
 *
 * What it computes (mlx-iqk 0.1.1 PKG-INFO, section "Format"):
 *   a 2-bit weight reconstructs as  d * float(scale_index) * values[4*alphabet + code],
 *   every step float32, left to right, in the CPU dequantizer's order:
 *       t = d * (float)scale_index;   w = t * values[4*alphabet + code];
 *   IQ2_KS: qs 2-bit code per weight (little-endian in uint32 words); per 32
 *           weights scl (low 4 bits of the signed scale index), sch (its high
 *           bit), sex (alphabet bit); dv one fp16 scale per row.
 *   IQ2_K:  qs as above; per 16 weights scl (4-bit offset-8 signed index) and
 *           sex; dv one fp16 scale per 256 weights.
 * Readings where the page is silent (stated once here, used everywhere):
 *   - IQ2_KS signed index is offset-16: idx = (low4 | high<<4) - 16 in [-16, 15],
 *     by analogy with IQ2_K's stated offset-8 (idx = nibble - 8 in [-8, 7]).
 *   - scl/sch/sex packing: sub-block j of a row lives in word/byte/halfword
 *     (j >> 3) (IQ2_KS), (j >> 3) / (j >> 4) (IQ2_K scl / sex), lowest bits first,
 *     following the page's "little-endian" for qs.
 * Build with -ffp-contract=off and without fast-math so each product rounds once.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* IEEE binary16 bit pattern -> binary32, exact for every input. */
float oracle_half_to_float(uint16_t h) {
  uint32_t sign = (uint32_t)(h >> 15) << 31;
  uint32_t ex = (h >> 10) & 0x1fu;
  uint32_t man = h & 0x3ffu;
  uint32_t bits;
  if (ex == 0) {
    /* zero or subnormal: man * 2^-24, exact in binary32 */
    float f = (float)man * (1.0f / 16777216.0f);
    memcpy(&bits, &f, 4);
    bits |= sign;
  } else if (ex == 31) {
    bits = sign | 0x7f800000u | (man << 13);
  } else {
    bits = sign | ((ex + 112u) << 23) | (man << 13);
  }
  float out;
  memcpy(&out, &bits, 4);
  return out;
}

/* binary32 -> bfloat16 bit pattern, round to nearest even; NaN stays NaN. */
uint16_t oracle_float_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

void oracle_f32_to_bf16_array(const float* in, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; i++) out[i] = oracle_float_to_bf16(in[i]);
}

void oracle_half_to_float_array(const uint16_t* in, float* out, int64_t n) {
  for (int64_t i = 0; i < n; i++) out[i] = oracle_half_to_float(in[i]);
}

/* The three decoded fields of weight k within one IQ2_KS row. */
void oracle_fields_iq2_ks(const uint32_t* qs, const uint32_t* scl, const uint8_t* sch,
                          const uint8_t* sex, int64_t k, int32_t* code, int32_t* idx,
                          int32_t* alpha) {
  int64_t j = k >> 5; /* 32-weight sub-block */
  uint32_t c = (qs[k >> 4] >> (2 * (k & 15))) & 3u;
  uint32_t lo = (scl[j >> 3] >> (4 * (j & 7))) & 15u;
  uint32_t hi = ((uint32_t)sch[j >> 3] >> (j & 7)) & 1u;
  uint32_t a = ((uint32_t)sex[j >> 3] >> (j & 7)) & 1u;
  *code = (int32_t)c;
  *idx = (int32_t)(lo | (hi << 4)) - 16;
  *alpha = (int32_t)a;
}

/* The three decoded fields of weight k within one IQ2_K row. */
void oracle_fields_iq2_k(const uint32_t* qs, const uint32_t* scl, const uint16_t* sex, int64_t k,
                         int32_t* code, int32_t* idx, int32_t* alpha) {
  int64_t j = k >> 4; /* 16-weight sub-block */
  uint32_t c = (qs[k >> 4] >> (2 * (k & 15))) & 3u;
  uint32_t nib = (scl[j >> 3] >> (4 * (j & 7))) & 15u;
  uint32_t a = ((uint32_t)sex[j >> 4] >> (j & 15)) & 1u;
  *code = (int32_t)c;
  *idx = (int32_t)nib - 8;
  *alpha = (int32_t)a;
}

/* One reconstructed weight: the page's float32 chain, two rounded products. */
static float reconstruct(float d, int32_t idx, int32_t alpha, int32_t code, const float* values) {
  float t = d * (float)idx;
  float w = t * values[4 * alpha + code];
  return w;
}

/* Dequantize one IQ2_KS matrix [rows, cols] (cols % 256 == 0) to float32. */
int oracle_dequant_iq2_ks(int64_t rows, int64_t cols, const uint32_t* qs, const uint32_t* scl,
                          const uint8_t* sch, const uint8_t* sex, const uint16_t* dv,
                          const float* values, float* out) {
  if (rows < 0 || cols <= 0 || cols % 256) return -2;
  for (int64_t r = 0; r < rows; r++) {
    const uint32_t* q = qs + r * (cols / 16);
    const uint32_t* s = scl + r * (cols / 256);
    const uint8_t* h = sch + r * (cols / 256);
    const uint8_t* x = sex + r * (cols / 256);
    float d = oracle_half_to_float(dv[r]);
    for (int64_t k = 0; k < cols; k++) {
      int32_t c, idx, a;
      oracle_fields_iq2_ks(q, s, h, x, k, &c, &idx, &a);
      out[r * cols + k] = reconstruct(d, idx, a, c, values);
    }
  }
  return 0;
}

/* Dequantize one IQ2_K matrix [rows, cols] (cols % 256 == 0) to float32. */
int oracle_dequant_iq2_k(int64_t rows, int64_t cols, const uint32_t* qs, const uint32_t* scl,
                         const uint16_t* sex, const uint16_t* dv, const float* values,
                         float* out) {
  if (rows < 0 || cols <= 0 || cols % 256) return -2;
  for (int64_t r = 0; r < rows; r++) {
    const uint32_t* q = qs + r * (cols / 16);
    const uint32_t* s = scl + r * (cols / 128);
    const uint16_t* x = sex + r * (cols / 256);
    const uint16_t* dr = dv + r * (cols / 256);
    for (int64_t k = 0; k < cols; k++) {
      int32_t c, idx, a;
      oracle_fields_iq2_k(q, s, x, k, &c, &idx, &a);
      float d = oracle_half_to_float(dr[k >> 8]);
      out[r * cols + k] = reconstruct(d, idx, a, c, values);
    }
  }
  return 0;
}

/*
 * Address-floor checksum of one row (the deleted-decode measurement arm):
 * every byte of every stream of the row folded into one little-endian 32-bit
 * XOR, byte i of a stream landing in byte (i & 3) of the word. A kernel that
 * skips any load cannot reproduce it.
 */
static uint32_t fold_bytes(const uint8_t* p, int64_t n) {
  uint32_t h = 0;
  for (int64_t i = 0; i < n; i++) h ^= (uint32_t)p[i] << (8 * (i & 3));
  return h;
}

void oracle_floor_xor(int64_t rows, int64_t n_streams, const uint8_t* const* streams,
                      const int64_t* row_bytes, uint32_t* out) {
  for (int64_t r = 0; r < rows; r++) {
    uint32_t h = 0;
    for (int64_t s = 0; s < n_streams; s++) h ^= fold_bytes(streams[s] + r * row_bytes[s], row_bytes[s]);
    out[r] = h;
  }
}

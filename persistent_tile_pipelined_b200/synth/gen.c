/*
 * Seeded synthetic inputs: one counter-based generator that both the GPU engine's
 * uploads and the CPU oracle consume, so the two sides see bit-identical bf16 data.
 * It holds none of the decode arithmetic: it only turns (seed, tensor id, index) into
 * numbers.
 *
 * Definition (every value is a pure function of seed, tensor_id and its index):
 *   mix64      the SplitMix64 output function (Steele, Lea & Flood, "Fast splittable
 *              pseudorandom number generators", OOPSLA 2014): two xor-shift-multiply
 *              rounds and a final xor-shift.
 *   key        mix64(seed + G) ^ mix64(tensor_id * G + C)        G = 0x9E3779B97F4A7C15
 *   draw(i)    mix64(key + (i + 1) * G)                            (SplitMix64 stream)
 *   normal     Box-Muller on the pair (draw(2p), draw(2p+1)):
 *                u1 = ((d0 >> 11) + 1) * 2^-53  in (0, 1]
 *                u2 =  (d1 >> 11)      * 2^-53  in [0, 1)
 *                z[2p] = sqrt(-2 ln u1) cos(2 pi u2),  z[2p+1] = sqrt(-2 ln u1) sin(2 pi u2)
 *              value = mean + std * z, computed in double
 *   bf16       double -> float (C conversion, round to nearest even) -> bf16 by round to
 *              nearest even on the upper 16 bits.
 *   e4m3 blocks  data preparation of a block-scaled FP8 weight (what an FP8 checkpoint
 *              holds): the values std * z of a [N][K] matrix, one fp32 scale per 128 x 128
 *              block = (float)(block max |value| / 448) (1 for an all-zero block), and each
 *              value divided by its block's scale, rounded to the nearest E4M3 number (ties
 *              to even, saturated at +-448) and stored as its E4M3 byte.
 *   mxfp4 rows bytes of an [N] x pitch matrix of FP4 weight rows (K elements each): the
 *              row's first K/2 bytes are draws' bytes (byte b of the matrix is byte b % 8
 *              of draw(b / 8)), the next K/32 bytes are scale exponents lo + (that byte & 1),
 *              the rest of the row is zero.  Random codes, not a quantised matrix: every
 *              E2M1 pair (and, with lo = 119, scales of 2^-8 or 2^-7) is equally likely.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL
#define KEYC 0x632BE59BD9B4E019ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t tensor_id) {
  return mix64(seed + GOLDEN) ^ mix64(tensor_id * GOLDEN + KEYC);
}

static inline uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GOLDEN); }

static inline void normal_pair(uint64_t key, uint64_t p, double* z0, double* z1) {
  const double two53 = 1.0 / 9007199254740992.0; /* 2^-53 */
  uint64_t d0 = draw(key, 2 * p), d1 = draw(key, 2 * p + 1);
  double u1 = (double)((d0 >> 11) + 1) * two53;
  double u2 = (double)(d1 >> 11) * two53;
  double r = sqrt(-2.0 * log(u1));
  double a = 6.283185307179586476925286766559 * u2;
  *z0 = r * cos(a);
  *z1 = r * sin(a);
}

static inline uint16_t float_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* quiet NaN */
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

uint64_t synth_u64(uint64_t seed, uint64_t tensor_id, uint64_t index) {
  return draw(stream_key(seed, tensor_id), index);
}

void synth_normal_f64(uint64_t seed, uint64_t tensor_id, int64_t n, double mean, double std,
                      double* out) {
  uint64_t key = stream_key(seed, tensor_id);
  int64_t pairs = (n + 1) / 2;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < pairs; ++p) {
    double z0, z1;
    normal_pair(key, (uint64_t)p, &z0, &z1);
    out[2 * p] = mean + std * z0;
    if (2 * p + 1 < n) out[2 * p + 1] = mean + std * z1;
  }
}

void synth_normal_f32(uint64_t seed, uint64_t tensor_id, int64_t n, double mean, double std,
                      float* out) {
  uint64_t key = stream_key(seed, tensor_id);
  int64_t pairs = (n + 1) / 2;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < pairs; ++p) {
    double z0, z1;
    normal_pair(key, (uint64_t)p, &z0, &z1);
    out[2 * p] = (float)(mean + std * z0);
    if (2 * p + 1 < n) out[2 * p + 1] = (float)(mean + std * z1);
  }
}

void synth_normal_bf16(uint64_t seed, uint64_t tensor_id, int64_t n, double mean, double std,
                       uint16_t* out) {
  uint64_t key = stream_key(seed, tensor_id);
  int64_t pairs = (n + 1) / 2;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < pairs; ++p) {
    double z0, z1;
    normal_pair(key, (uint64_t)p, &z0, &z1);
    out[2 * p] = float_to_bf16_rne((float)(mean + std * z0));
    if (2 * p + 1 < n) out[2 * p + 1] = float_to_bf16_rne((float)(mean + std * z1));
  }
}

/* The E4M3 byte of the E4M3 number nearest to v (ties to even; |v| saturates at 448). */
static uint8_t e4m3_rne(double v) {
  uint8_t sgn = (v < 0) ? 0x80 : 0;
  double a = fabs(v);
  if (a >= 448.0) return sgn | 0x7E;
  if (a < ldexp(1.0, -6)) {                     /* subnormal range: steps of 2^-9 */
    double m = nearbyint(a / ldexp(1.0, -9));
    if (m >= 8.0) return sgn | 0x08;            /* rounded up to 2^-6 */
    return sgn | (uint8_t)m;
  }
  int e;
  frexp(a, &e);                                 /* a in [2^(e-1), 2^e) */
  int E = e - 1;                                /* -6 .. 8 */
  double r = nearbyint(ldexp(a, 3 - E));        /* 8 .. 16: 1 + m/8 in eighths */
  if (r >= 16.0) {
    r = 8.0;
    E += 1;
  }
  if (E > 8 || (E == 8 && r > 14.0)) return sgn | 0x7E;
  return sgn | (uint8_t)((E + 7) << 3) | (uint8_t)(r - 8.0);
}

void synth_e4m3_blocks(uint64_t seed, uint64_t tensor_id, int64_t N, int64_t K, double std,
                       uint8_t* codes, float* scales) {
  int64_t NB = (N + 127) / 128, KB = (K + 127) / 128;
  uint64_t key = stream_key(seed, tensor_id);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t nb = 0; nb < NB; ++nb) {
    int64_t n0 = nb * 128, n1 = n0 + 128 < N ? n0 + 128 : N;
    for (int64_t kb = 0; kb < KB; ++kb) {
      int64_t k0 = kb * 128, k1 = k0 + 128 < K ? k0 + 128 : K;
      double amax = 0.0;
      for (int64_t n = n0; n < n1; ++n)
        for (int64_t k = k0; k < k1; ++k) {
          int64_t i = n * K + k;
          double z0, z1;
          normal_pair(key, (uint64_t)(i / 2), &z0, &z1);
          double v = std * ((i & 1) ? z1 : z0);
          if (fabs(v) > amax) amax = fabs(v);
        }
      float sc = amax > 0.0 ? (float)(amax / 448.0) : 1.0f;
      scales[nb * KB + kb] = sc;
      for (int64_t n = n0; n < n1; ++n)
        for (int64_t k = k0; k < k1; ++k) {
          int64_t i = n * K + k;
          double z0, z1;
          normal_pair(key, (uint64_t)(i / 2), &z0, &z1);
          double v = std * ((i & 1) ? z1 : z0);
          codes[i] = e4m3_rne(v / (double)sc);
        }
    }
  }
}

void synth_mxfp4_rows(uint64_t seed, uint64_t tensor_id, int64_t N, int64_t K, int64_t pitch,
                      int32_t lo, uint8_t* out) {
  uint64_t key = stream_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    uint8_t* row = out + n * pitch;
    for (int64_t j = 0; j < pitch; ++j) {
      const uint64_t b = (uint64_t)(n * pitch + j);
      const uint8_t v = (uint8_t)(draw(key, b / 8) >> (8 * (b % 8)));
      if (j < K / 2) row[j] = v;
      else if (j < K / 2 + K / 32) row[j] = (uint8_t)(lo + (v & 1));
      else row[j] = 0;
    }
  }
}

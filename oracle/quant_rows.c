/*
 * Row quantizers of the CPU oracle in plain C -- TEST INFRASTRUCTURE ONLY.
 *
 * The same rules, step for step, as mxfp8_quantize / nvfp4_quantize followed
 * by their dequantize in moe_oracle.py (which define them and are pinned by
 * the CPU tests); this file only makes a full-size expert's weights take well
 * under a second instead of seconds, and the CPU tests check it against the
 * numpy functions bit for bit.  It shares nothing with the CUDA library.
 *
 *   MXFP8 (TransformerEngine PR "DeepSeekV3Layer", Performance, MXFP8 rows):
 *     per 32 consecutive elements of a row, X = 2^(floor(log2 amax) - 8) with
 *     the e8m0 code clamped to [0, 254] (an all-zero block: X = 1); each
 *     element is v / X rounded to the nearest e4m3 value, ties to the even
 *     code, saturating at 448; the value it stands for is code * X.
 *   NVFP4 (sglang PR "Mistral Large 3 NVFP4 TRTLLM MoE support",
 *     Modifications: W4A4 NVFP4): per 16 consecutive elements, with the
 *     tensor's fp32 global encode scale g, each step one fp32 operation:
 *     t = (amax / 6) * g; sb = e4m3(t) (nearest, ties to even, saturating);
 *     sb == 0 gives zeros; else r = g / sb and q = e2m1(v * r) (nearest, ties
 *     to even, saturating at 6); the value is q * sb / g (in double).
 *
 * Inputs are doubles holding bf16 values; outputs are doubles.  Rows are
 * independent, so they are split over OpenMP threads.
 */
#include <math.h>
#include <stdint.h>

static double e4m3_mag[127];  /* codes 0x00 .. 0x7E, ascending */
static const double e2m1_mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
static int tables_ready = 0;

static void init_tables(void) {
  if (tables_ready) return;
  for (int c = 0; c < 127; ++c) {
    const int ef = c >> 3, m = c & 7;
    e4m3_mag[c] = ef == 0 ? (m / 8.0) * ldexp(1.0, -6) : (1.0 + m / 8.0) * ldexp(1.0, ef - 7);
  }
  tables_ready = 1;
}

/* Index of the table entry nearest to a (0 <= a <= table[n-1]); halfway
 * between two entries, the even index. */
static int nearest(double a, const double* table, int n) {
  int lo = 0, hi = n;  /* first index with table[i] >= a */
  while (lo < hi) {
    const int mid = (lo + hi) / 2;
    if (table[mid] < a) lo = mid + 1; else hi = mid;
  }
  int up = lo < n ? lo : n - 1;
  int down = up > 0 ? up - 1 : 0;
  const double d_down = a - table[down], d_up = table[up] - a;
  if (d_up < d_down || (d_up == d_down && up % 2 == 0)) return up;
  return down;
}

/* signed e4m3 value nearest to v, saturating at +-448 */
static double e4m3_round(double v) {
  double a = fabs(v);
  if (a > 448.0) a = 448.0;
  const double m = e4m3_mag[nearest(a, e4m3_mag, 127)];
  return signbit(v) ? -m : m;
}

static double e2m1_round(double v) {
  double a = fabs(v);
  if (a > 6.0) a = 6.0;
  const double m = e2m1_mag[nearest(a, e2m1_mag, 8)];
  return signbit(v) ? -m : m;
}

void oracle_mxfp8_qdq_rows(const double* in, double* out, int64_t rows, int64_t cols) {
  init_tables();
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < cols; b += 32) {
      const double* v = in + r * cols + b;
      double* o = out + r * cols + b;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i) amax = fabs(v[i]) > amax ? fabs(v[i]) : amax;
      int code = 127;
      if (amax != 0.0) {
        int e;
        frexp(amax, &e);  /* amax = m * 2^e, m in [0.5, 1): floor(log2 amax) = e - 1 */
        code = (e - 1) - 8 + 127;
        if (code < 0) code = 0;
        if (code > 254) code = 254;
      }
      const double X = ldexp(1.0, code - 127);
      for (int i = 0; i < 32; ++i) o[i] = e4m3_round(v[i] / X) * X;
    }
  }
}

void oracle_nvfp4_qdq_rows(const double* in, double* out, int64_t rows, int64_t cols, float g) {
  init_tables();
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < cols; b += 16) {
      const double* v = in + r * cols + b;
      double* o = out + r * cols + b;
      float amax = 0.0f;
      for (int i = 0; i < 16; ++i) {
        const float a = fabsf((float)v[i]);
        amax = a > amax ? a : amax;
      }
      volatile float q6 = amax / 6.0f;  /* one fp32 operation each */
      volatile float t = q6 * g;
      const double sb = e4m3_round((double)t);
      if (sb == 0.0) {
        for (int i = 0; i < 16; ++i) o[i] = 0.0;
        continue;
      }
      volatile float rr = g / (float)sb;
      for (int i = 0; i < 16; ++i) {
        volatile float s = (float)v[i] * rr;
        o[i] = e2m1_round((double)s) * sb / (double)g;
      }
    }
  }
}

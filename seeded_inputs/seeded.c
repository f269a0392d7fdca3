/* Host-side fast path of the seeded input generator (same definition as the
 * numpy code in __init__.py: SplitMix64 counter streams, Box-Muller with ln and
 * cos(2*pi*t) built from IEEE add/mul/div/sqrt only). Compile with
 * -ffp-contract=off so that no multiply-add is fused: the bits must match the
 * numpy and CUDA implementations exactly. */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SG 0x9E3779B97F4A7C15ULL
#define SM1 0xBF58476D1CE4E5B9ULL
#define SM2 0x94D049BB133111EBULL

static const double kCos[10] = {0x1.0000000000000p+0, -0x1.0000000000000p-1, 0x1.5555555555555p-5,
                                -0x1.6c16c16c16c17p-10, 0x1.a01a01a01a01ap-16, -0x1.27e4fb7789f5cp-22,
                                0x1.1eed8eff8d898p-29, -0x1.93974a8c07c9dp-37, 0x1.ae7f3e733b81fp-45,
                                -0x1.6827863b97d97p-53};
static const double kSin[10] = {0x1.0000000000000p+0, -0x1.5555555555555p-3, 0x1.1111111111111p-7,
                                -0x1.a01a01a01a01ap-13, 0x1.71de3a556c734p-19, -0x1.ae64567f544e4p-26,
                                0x1.6124613a86d09p-33, -0x1.ae7f3e733b81fp-41, 0x1.952c77030ad4ap-49,
                                -0x1.2f49b46814157p-57};
static const double kAtanh[11] = {0x1.0000000000000p+0, 0x1.5555555555555p-2, 0x1.999999999999ap-3,
                                  0x1.2492492492492p-3, 0x1.c71c71c71c71cp-4, 0x1.745d1745d1746p-4,
                                  0x1.3b13b13b13b14p-4, 0x1.1111111111111p-4, 0x1.e1e1e1e1e1e1ep-5,
                                  0x1.af286bca1af28p-5, 0x1.8618618618618p-5};
static const double kLn2 = 0x1.62e42fefa39efp-1;
static const double kTwoPi = 0x1.921fb54442d18p+2;
static const double kInvSqrt2 = 0x1.6a09e667f3bcdp-1;

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * SM1;
  z = (z ^ (z >> 27)) * SM2;
  return z ^ (z >> 31);
}

static double det_log(double u) {
  int e;
  double m = frexp(u, &e);
  if (m < kInvSqrt2) { m = m * 2.0; e -= 1; }
  double s = (m - 1.0) / (m + 1.0);
  double s2 = s * s;
  double p = kAtanh[10];
  for (int k = 9; k >= 0; --k) p = p * s2 + kAtanh[k];
  return (double)e * kLn2 + (2.0 * s) * p;
}

static double det_cos2pi(double t) {
  if (t > 0.5) t = 1.0 - t;
  int neg = t > 0.25;
  if (neg) t = 0.5 - t;
  int use_sin = t > 0.125;
  double x = (use_sin ? 0.25 - t : t) * kTwoPi;
  double x2 = x * x, r;
  if (use_sin) {
    double p = kSin[9];
    for (int k = 8; k >= 0; --k) p = p * x2 + kSin[k];
    r = x * p;
  } else {
    double p = kCos[9];
    for (int k = 8; k >= 0; --k) p = p * x2 + kCos[k];
    r = p;
  }
  return neg ? -r : r;
}

uint64_t seeded_stream_key(uint64_t seed, uint64_t stream) { return mix64(seed * SG + stream * SM1 + SG); }

static inline uint16_t bf16_rne(float f) {
  uint32_t b;
  memcpy(&b, &f, 4);
  return (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

void seeded_normal(uint64_t seed, uint64_t stream, uint64_t start, uint64_t count, float std,
                   int as_bf16, void* out) {
  const uint64_t key = seeded_stream_key(seed, stream);
  const double sd = (double)std;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (int64_t)count; ++j) {
    uint64_t i = start + (uint64_t)j;
    uint64_t d0 = mix64(key + (2 * i + 1) * SG);
    uint64_t d1 = mix64(key + (2 * i + 2) * SG);
    double u1 = (double)((d0 >> 11) + 1) * 0x1p-53;
    double u2 = (double)(d1 >> 11) * 0x1p-53;
    double z = sqrt(-2.0 * det_log(u1)) * det_cos2pi(u2);
    float v = (float)(z * sd);
    if (as_bf16) ((uint16_t*)out)[j] = bf16_rne(v);
    else ((float*)out)[j] = v;
  }
}

/*
 * lbq_oracle.c -- the oracle: a plain fp64 CPU statement of what the low-bit
 * GEMV/GEMM computes. TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU
 * baseline); never linked into or called by the product path, and independent
 * of it (own layouts, own fp16 rounding, own generator, own transform).
 *
 * Sources, cited by page and section:
 *   pptc.cn ternary-27B article §5.1: ternarise with s = mean|w| and
 *     t = clip(round(w / s), -1, 1); §1.2: three states, log2(3) bits/weight.
 *   mhpq.cn "27B in 5.9 GB" article §2.1: one shared scale per block of 64/128
 *     weights, dequantised weight = trit * scale; §3.2: the scale is fp16.
 *   neodrop.ai round-up, part 2: Q1_0 weights are +1 or -1 (one bit each).
 *   feinterview.poetries.top "27B in 12 GB" article, section on what fits in
 *     12 GB: random Hadamard rotation before low-bit coding (QuIP#/QTIP line).
 * Readings where the pages are silent (block layout, digit order, tie rules,
 * scale rounding, the sign generator) are stated next to the code below.
 *
 * Parity pins live in tests/test_oracle_pins.py; every function here is pinned
 * there against something other than itself.
 */
#include "lbq_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ fp16 -- */

/* IEEE 754 binary16, round to nearest, ties to even, from binary64.
 * Written from the format's definition: 1 sign bit, 5 exponent bits (bias 15),
 * 10 fraction bits; subnormals are multiples of 2^-24. */
uint16_t orc_f16_from_f64(double v) {
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  double a = fabs(v);
  if (isnan(a)) return (uint16_t)(sign | 0x7e00u);
  if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u); /* 65504 + half an ulp (16) ties to even -> inf */
  if (a < 6.103515625e-05) {                           /* below 2^-14: subnormal grid 2^-24 */
    double m = rint(a * 16777216.0);                  /* exact scaling, rint = RNE */
    return (uint16_t)(sign | (uint16_t)m);            /* m == 1024 encodes 2^-14 correctly */
  }
  int e;
  double f = frexp(a, &e);       /* a = f * 2^e, f in [0.5, 1) */
  double m = rint(ldexp(f, 11)); /* 1.fraction * 2^10 in [1024, 2048] */
  if (m == 2048.0) {
    m = 1024.0;
    e += 1;
  }
  int E = e - 1 + 15;
  if (E >= 31) return (uint16_t)(sign | 0x7c00u);
  return (uint16_t)(sign | (uint16_t)(E << 10) | (uint16_t)((int)m - 1024));
}

double orc_f16_to_f64(uint16_t h) {
  int s = (h >> 15) & 1, E = (h >> 10) & 31, F = h & 1023;
  double v;
  if (E == 0)
    v = ldexp((double)F, -24);
  else if (E == 31)
    v = F ? NAN : INFINITY;
  else
    v = ldexp((double)(F + 1024), E - 25);
  return s ? -v : v;
}

/* bf16 is the top half of an IEEE binary32. */
double orc_bf16_to_f64(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* ---------------------------------------------------------------- layout -- */

/* Format 1 (ternary): 128-weight blocks of 28 bytes = 26 code bytes + fp16 scale,
 *   rows padded to 16 bytes. Format 2 (sign): K/8 code bytes per row, one fp16
 *   scale per 128, scale rows padded with zeros to a multiple of 8 entries.
 *   Format 3 (2-bit): K/4 code bytes per row, one fp16 scale per 32. */
int orc_layout(int fmt, int64_t K, int64_t* code_stride, int64_t* scale_stride,
               int64_t* block) {
  int64_t cs, ss, blk;
  if (K < 128 || K % 128) return -1;
  if (fmt == 1) {
    cs = (K / 128) * 28;
    cs = (cs + 15) / 16 * 16;
    ss = 0;
    blk = 128;
  } else if (fmt == 2) {
    cs = K / 8;
    ss = (K / 128 + 7) / 8 * 8; /* scale rows padded to 8 entries (16 bytes), pad = 0 */
    blk = 128;
  } else if (fmt == 3) {
    if (K % 512) return -1;
    cs = K / 4;
    ss = K / 32;
    blk = 32;
  } else {
    return -1;
  }
  if (code_stride) *code_stride = cs;
  if (scale_stride) *scale_stride = ss;
  if (block) *block = blk;
  return 0;
}

/* ------------------------------------------------------------ quantisers -- */

/* Block scale of the ternary and sign formats: the absolute mean of the block
 * (pptc.cn §5.1 uses |W|.mean() for the whole tensor; mhpq.cn §2.1 takes one
 * scale per block), summed in fp64 in increasing k, divided by the block size,
 * rounded once to fp16 (mhpq.cn §3.2: fp16 scales). Reading: no epsilon; a mean
 * above the largest finite fp16 saturates to 65504 rather than becoming inf. */
static uint16_t absmean_scale(const float* w, int n) {
  double acc = 0.0;
  for (int k = 0; k < n; ++k) acc += fabs((double)w[k]);
  double m = acc / (double)n;
  if (m > 65504.0) m = 65504.0;
  return orc_f16_from_f64(m);
}

/* t = clip(round(w / s), -1, 1) with round-half-even (torch.round, as in the
 * pptc.cn §5.1 pseudo-code), evaluated in fp64. A zero scale gives t = 0. */
static int ternarise(float w, double s) {
  if (s == 0.0) return 0;
  double r = rint((double)w / s);
  if (r > 1.0) r = 1.0;
  if (r < -1.0) r = -1.0;
  return (int)r;
}

/* 2-bit levels (q - 1.5) * s, q = 0..3: the nearest level, ties to the upper
 * one, i.e. q = clip(floor(w / s) + 2, 0, 3). Scale s = max|w| / 1.5 so that the
 * largest weight lands on the outer level. A zero scale gives q = 2. */
static int quant2(float w, double s) {
  if (s == 0.0) return 2;
  double q = floor((double)w / s) + 2.0;
  if (q < 0.0) q = 0.0;
  if (q > 3.0) q = 3.0;
  return (int)q;
}

static uint16_t q2_scale(const float* w) {
  double mx = 0.0;
  for (int k = 0; k < 32; ++k) {
    double a = fabs((double)w[k]);
    if (a > mx) mx = a;
  }
  double m = mx / 1.5;
  if (m > 65504.0) m = 65504.0;
  return orc_f16_from_f64(m);
}

int orc_pack(int fmt, const float* W, int64_t K, int64_t N, uint8_t* codes,
             uint16_t* scales) {
  int64_t cs, ss, blk;
  if (!W || !codes || N < 1 || orc_layout(fmt, K, &cs, &ss, &blk)) return -1;
  if (fmt != 1 && !scales) return -1;
  memset(codes, 0, (size_t)(N * cs));
  if (scales) memset(scales, 0, sizeof(uint16_t) * (size_t)(N * ss));
  for (int64_t n = 0; n < N; ++n) {
    const float* wr = W + n * K;
    uint8_t* cr = codes + n * cs;
    for (int64_t b = 0; b < K / blk; ++b) {
      const float* wb = wr + b * blk;
      if (fmt == 1) {
        /* 5 trits per byte, little-endian base 3 of d = t + 1 (pptc.cn §1.2:
         * log2 3 bits per weight; 3^5 = 243 <= 256). Byte 25 carries weights
         * 125..127 and two zero trits (d = 1) as padding. */
        uint16_t h = absmean_scale(wb, 128);
        double s = orc_f16_to_f64(h);
        uint8_t* blkp = cr + b * 28;
        for (int j = 0; j < 26; ++j) {
          int v = 0, p = 1;
          for (int i = 0; i < 5; ++i) {
            int k = 5 * j + i;
            int d = (k < 128) ? ternarise(wb[k], s) + 1 : 1;
            v += d * p;
            p *= 3;
          }
          blkp[j] = (uint8_t)v;
        }
        blkp[26] = (uint8_t)(h & 0xff);
        blkp[27] = (uint8_t)(h >> 8);
      } else if (fmt == 2) {
        /* bit i of byte j = weight 8j+i, set iff w >= 0 (so -0.0 and +0.0 -> +1) */
        scales[n * ss + b] = absmean_scale(wb, 128);
        for (int k = 0; k < 128; ++k)
          if (wb[k] >= 0.0f) cr[(b * 128 + k) / 8] |= (uint8_t)(1u << (k % 8));
      } else {
        uint16_t h = q2_scale(wb);
        double s = orc_f16_to_f64(h);
        scales[n * ss + b] = h;
        for (int k = 0; k < 32; ++k) {
          int q = quant2(wb[k], s);
          cr[(b * 32 + k) / 4] |= (uint8_t)(q << (2 * (k % 4)));
        }
      }
    }
  }
  return 0;
}

int orc_unpack(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t K,
               int64_t N, int8_t* out, double* block_scales) {
  int64_t cs, ss, blk;
  if (!codes || !out || N < 1 || orc_layout(fmt, K, &cs, &ss, &blk)) return -1;
  if (fmt != 1 && !scales) return -1;
  int64_t nb = K / blk;
  for (int64_t n = 0; n < N; ++n) {
    const uint8_t* cr = codes + n * cs;
    int8_t* orow = out + n * K;
    for (int64_t b = 0; b < nb; ++b) {
      double s;
      if (fmt == 1) {
        const uint8_t* blkp = cr + b * 28;
        s = orc_f16_to_f64((uint16_t)(blkp[26] | (blkp[27] << 8)));
        for (int j = 0; j < 26; ++j) {
          int v = blkp[j];
          if (v > 242) return -2;
          for (int i = 0; i < 5; ++i) {
            int d = v % 3;
            v /= 3;
            int k = 5 * j + i;
            if (k < 128)
              orow[b * 128 + k] = (int8_t)(d - 1);
            else if (d != 1)
              return -2;
          }
        }
      } else if (fmt == 2) {
        s = orc_f16_to_f64(scales[n * ss + b]);
        for (int k = 0; k < 128; ++k) {
          int64_t kk = b * 128 + k;
          orow[kk] = (cr[kk / 8] >> (kk % 8)) & 1 ? 1 : -1;
        }
      } else {
        s = orc_f16_to_f64(scales[n * ss + b]);
        for (int k = 0; k < 32; ++k) {
          int64_t kk = b * 32 + k;
          orow[kk] = (int8_t)((cr[kk / 4] >> (2 * (kk % 4))) & 3);
        }
      }
      if (block_scales) block_scales[n * nb + b] = s;
    }
  }
  return 0;
}

int orc_dequant(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t K,
                int64_t N, double* What) {
  int64_t cs, ss, blk;
  if (!What || orc_layout(fmt, K, &cs, &ss, &blk)) return -1;
  int8_t* t = (int8_t*)malloc((size_t)(N * K));
  double* s = (double*)malloc(sizeof(double) * (size_t)(N * (K / blk)));
  if (!t || !s) {
    free(t);
    free(s);
    return -3;
  }
  int rc = orc_unpack(fmt, codes, scales, K, N, t, s);
  if (rc == 0) {
    for (int64_t n = 0; n < N; ++n)
      for (int64_t k = 0; k < K; ++k) {
        double sc = s[n * (K / blk) + k / blk];
        double c = (double)t[n * K + k];
        What[n * K + k] = (fmt == 3) ? sc * (c - 1.5) : sc * c;
      }
  }
  free(t);
  free(s);
  return rc;
}

/* ------------------------------------------------------------- rotation -- */

/* SplitMix64 (Steele, Lea & Flood, OOPSLA 2014; Vigna's reference generator):
 * a Weyl sequence with increment 0x9e3779b97f4a7c15, each state value passed
 * through the "variant 13" 64-bit finaliser. */
static uint64_t splitmix64_next(uint64_t* state) {
  uint64_t z = (*state += 0x9e3779b97f4a7c15ULL);
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

int orc_splitmix64(uint64_t seed, int64_t n, uint64_t* out) {
  if (!out || n < 0) return -1;
  uint64_t st = seed;
  for (int64_t i = 0; i < n; ++i) out[i] = splitmix64_next(&st);
  return 0;
}

/* Random diagonal of the rotation: one +-1 per input coordinate (reading: the
 * page says only "random Hadamard rotation"; the sign source is ours). */
int orc_rht_signs(uint64_t seed, int64_t K, int8_t* D) {
  if (!D || K < 0) return -1;
  uint64_t st = seed;
  for (int64_t k = 0; k < K; ++k) D[k] = (splitmix64_next(&st) >> 63) ? -1 : 1;
  return 0;
}

/* Sylvester Hadamard matrix in natural order: H[i][j] = (-1)^popcount(i & j). */
static int hadamard_entry(int i, int j) { return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1; }

/* x'[512c+i] = (1/sqrt 512) sum_j H[i][j] D[512c+j] x[512c+j]: the dense
 * matrix-vector product per 512-block, no fast transform. */
int orc_hadamard(const double* x, const int8_t* D, int64_t M, int64_t K, double* out) {
  if (!x || !D || !out || M < 1 || K < 512 || K % 512) return -1;
  const double norm = 1.0 / sqrt(512.0);
  for (int64_t m = 0; m < M; ++m)
    for (int64_t c = 0; c < K / 512; ++c) {
      const double* xb = x + m * K + c * 512;
      const int8_t* db = D + c * 512;
      double* ob = out + m * K + c * 512;
      for (int i = 0; i < 512; ++i) {
        double acc = 0.0;
        for (int j = 0; j < 512; ++j) acc += (double)hadamard_entry(i, j) * (double)db[j] * xb[j];
        ob[i] = acc * norm;
      }
    }
  return 0;
}

/* ---------------------------------------------------------------- product -- */

typedef struct {
  int fmt;
  const uint8_t* codes;
  const uint16_t* scales;
  int64_t K, N, M, cs, ss;
  const double* xin;
  double *Y, *Bnd;
  int64_t n0, n1;
  int rc;
} gemm_job;

static void* gemm_rows(void* arg) {
  gemm_job* j = (gemm_job*)arg;
  double* wrow = (double*)malloc(sizeof(double) * (size_t)j->K);
  if (!wrow) {
    j->rc = -3;
    return NULL;
  }
  for (int64_t n = j->n0; n < j->n1 && j->rc == 0; ++n) {
    j->rc = orc_dequant(j->fmt, j->codes + n * j->cs, j->scales ? j->scales + n * j->ss : NULL,
                        j->K, 1, wrow);
    for (int64_t m = 0; m < j->M && j->rc == 0; ++m) {
      const double* xr = j->xin + m * j->K;
      double acc = 0.0, bacc = 0.0;
      for (int64_t k = 0; k < j->K; ++k) {
        double p = wrow[k] * xr[k];
        acc += p;
        bacc += fabs(p);
      }
      j->Y[m * j->N + n] = acc;
      if (j->Bnd) j->Bnd[m * j->N + n] = bacc;
    }
  }
  free(wrow);
  return NULL;
}

int orc_gemm(int fmt, const uint8_t* codes, const uint16_t* scales, int64_t K, int64_t N,
             const uint16_t* X, int64_t M, const int8_t* D, double* Y, double* Bnd,
             int nthreads) {
  int64_t cs, ss, blk;
  if (!codes || !X || !Y || N < 1 || M < 1 || orc_layout(fmt, K, &cs, &ss, &blk)) return -1;
  if (fmt != 1 && !scales) return -1;
  if (fmt == 3 && !D) return -1;
  double* xin = (double*)malloc(sizeof(double) * (size_t)(M * K));
  if (!xin) return -3;
  for (int64_t i = 0; i < M * K; ++i) xin[i] = orc_bf16_to_f64(X[i]);
  if (fmt == 3) {
    double* rot = (double*)malloc(sizeof(double) * (size_t)(M * K));
    if (!rot) {
      free(xin);
      return -3;
    }
    orc_hadamard(xin, D, M, K, rot);
    free(xin);
    xin = rot;
  }
  if (nthreads < 1) nthreads = 1;
  if (nthreads > N) nthreads = (int)N;
  gemm_job* jobs = (gemm_job*)calloc((size_t)nthreads, sizeof(gemm_job));
  pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  int rc = 0;
  if (!jobs || !th) rc = -3;
  for (int t = 0; t < nthreads && rc == 0; ++t) {
    gemm_job j = {fmt, codes, scales, K, N, M, cs, ss, xin, Y, Bnd,
                  N * t / nthreads, N * (t + 1) / nthreads, 0};
    jobs[t] = j;
  }
  if (rc == 0) {
    if (nthreads == 1) {
      gemm_rows(&jobs[0]);
    } else {
      for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, gemm_rows, &jobs[t]);
      for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    }
    for (int t = 0; t < nthreads; ++t)
      if (jobs[t].rc) rc = jobs[t].rc;
  }
  free(jobs);
  free(th);
  free(xin);
  return rc;
}

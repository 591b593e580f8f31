/*
 * bonsai_oracle.c - plain CPU oracle for the weight-only low-bit linear layer.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  The CUDA library never
 * includes, links or calls it, and it includes nothing from the CUDA side.
 *
 * What it computes, from the pages:
 *   - every quantised weight is w = scale_g * t with t in {-1,+1} (binary) or
 *     {-1,0,+1} (ternary), one FP16 scale shared by a group of 128 weights
 *     ["Cómo Bonsai Ternary 4B revoluciona la difusión texto-imagen",
 *     section "Representación y almacenamiento de los pesos ternarios";
 *     "Introducing 1-bit and Ternary Bonsai Image 4B: Image Generation for
 *     Local Devices", section "量化数学：1.125 和 1.71 是怎么来的"];
 *   - the group runs over 128 consecutive weights of one output row, along
 *     the input dimension K (the reading the rest of the design supports);
 *   - ternary weights are stored as INT2, two bits per weight ["Cómo
 *     Bonsai Ternary 4B ...", same section]; binary weights as one bit per
 *     weight (1 + 16/128 = 1.125 effective bits, "Introducing 1-bit and
 *     Ternary Bonsai Image 4B ...", same section);
 *   - out[m,n] = sum_k A[m,k] * w[n,k] with FP16 activations A [M,K] and an
 *     FP16 result [M,N].
 *
 * How: codes are unpacked, each weight is formed as the IEEE product t*s in
 * double and rounded to FP16, and every output is one double accumulation
 * over k in ascending order, rounded once to FP16 (round to nearest even).
 * The FP16 <-> double conversions below are written from the IEEE 754
 * binary16 definition (1 sign bit, 5 exponent bits with bias 15, 10
 * fraction bits, subnormals, inf and NaN).
 *
 * The bit layout of a packed word is this project's own format; the pages
 * only fix the number of bits per weight.  It is defined at oracle_pack.
 * A third, denser ternary format (five trits per byte, 1.75 bits per weight
 * with its alignment padding; the pages' 1.71-bit figure is log2(3) +
 * 16/128, and INT2 storage spends 2 bits) is this project's own too; it is
 * defined at pack_b3_group.
 *
 * 4-bit group-affine weights.  The pages name "4-bit HQQ" for the text
 * encoder ("Cómo Bonsai Ternary 4B revoluciona la difusión texto-imagen",
 * section "Arquitectura de despliegue y eficiencia en tiempo de ejecución")
 * and give nothing more.  This project reads it
 * as HQQ's published scheme: an unsigned 4-bit q per weight, and per group of
 * 64 weights along K an FP16 scale s and FP16 zero z, the weight being
 * evaluated in FP16 as w = fp16(fp16(q - z) * s).  The group size, the zero
 * as an FP16 value and the packing (oracle_hqq4_pack) are this reading's
 * choices; none of it is pinned by the pages: parity unpinned for the
 * oracle_hqq4_* functions (their FP16 arithmetic and layout are checked by
 * the tests, the reading is not).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_SHAPE 2
#define ORACLE_ERR_BAD_CODE 4
#define ORACLE_ERR_NOMEM 5

#define MODE_BINARY 1
#define MODE_TERNARY 2
#define MODE_TERNARY_B3 3
#define GROUP 128
#define B3_GROUP_BYTES 26  /* ceil(128 / 5) */
#define B3_BLOCK_GROUPS 4  /* groups per 16-byte-aligned block */
#define B3_BLOCK_BYTES 112 /* 4 x 26 data bytes + 8 zero bytes */

/* ---------------------------------------------------------------- FP16 -- */

/* binary16 bit pattern -> exact double value. */
double oracle_half_to_double(uint16_t h) {
  int negative = (h >> 15) & 1;
  int expo = (h >> 10) & 0x1f;
  int frac = h & 0x3ff;
  double v;
  if (expo == 0) {
    v = ldexp((double)frac, -24); /* zero or subnormal: frac * 2^-24 */
  } else if (expo == 31) {
    v = frac ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + frac), expo - 25); /* (1.frac) * 2^(expo-15) */
  }
  return negative ? -v : v;
}

/* double -> nearest binary16, ties to the even significand. */
uint16_t oracle_double_to_half(double x) {
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  if (isnan(x)) return (uint16_t)(sign | 0x7e00);
  double a = fabs(x);
  if (isinf(a)) return (uint16_t)(sign | 0x7c00);
  /* Write a = q * 2^(e-10): normal binades have q in [1024, 2048); below
   * 2^-14 the spacing is fixed at 2^-24, i.e. e = -14 with q < 1024. */
  int e;
  if (a < 0x1p-14) {
    e = -14;
  } else {
    frexp(a, &e); /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;       /* a in [2^e, 2^(e+1)) */
  }
  double q = ldexp(a, 10 - e); /* exact: scaling by a power of two */
  double qi = floor(q);
  double rest = q - qi; /* exact */
  if (rest > 0.5 || (rest == 0.5 && fmod(qi, 2.0) != 0.0)) qi += 1.0;
  if (qi >= 2048.0) { /* rounding carried into the next binade */
    qi = 1024.0;
    e += 1;
  }
  if (e > 15) return (uint16_t)(sign | 0x7c00); /* overflow -> inf */
  if (qi < 1024.0) return (uint16_t)(sign | (uint16_t)qi); /* subnormal */
  return (uint16_t)(sign | ((e + 15) << 10) | ((int)qi - 1024));
}

void oracle_half_to_double_array(const uint16_t* h, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_half_to_double(h[i]);
}

void oracle_double_to_half_array(const double* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_double_to_half(x[i]);
}

/* ------------------------------------------------------------- format -- */

/* Weights per 32-bit word (binary and INT2 ternary). */
static int per_word(int mode) { return mode == MODE_BINARY ? 32 : 16; }

static int check_mode_shape(int64_t N, int64_t K, int mode) {
  if (mode != MODE_BINARY && mode != MODE_TERNARY && mode != MODE_TERNARY_B3) return ORACLE_ERR_ARG;
  if (N < 0 || K < 0) return ORACLE_ERR_SHAPE;
  if (K % GROUP != 0) return ORACLE_ERR_SHAPE;
  return ORACLE_OK;
}

/* Bytes of one packed row.  Base-3: one 112-byte block per 4 groups of 128
 * (the last block of a row may hold fewer groups). */
static int64_t row_bytes(int64_t K, int mode) {
  if (mode == MODE_TERNARY_B3) return (K / GROUP + B3_BLOCK_GROUPS - 1) / B3_BLOCK_GROUPS * B3_BLOCK_BYTES;
  return K / per_word(mode) * 4;
}

/* Byte offset of group g within its row (base-3 format). */
static int64_t b3_group_offset(int64_t g) {
  return g / B3_BLOCK_GROUPS * B3_BLOCK_BYTES + g % B3_BLOCK_GROUPS * B3_GROUP_BYTES;
}

/* Bytes of packed weights for an [N,K] matrix (scales not included). */
int64_t oracle_packed_bytes(int64_t N, int64_t K, int mode) {
  if (check_mode_shape(N, K, mode) != ORACLE_OK) return -1;
  return N * row_bytes(K, mode);
}

/* Base-3 format.  A group of 128 ternary weights t[0..127] of one row
 * becomes 26 bytes.  Byte j (0 <= j < 26) holds the five weights at
 * positions j, j+26, j+52, j+78 and j+104 of the group as the base-3 number
 *
 *     v[j] = sum_{i=0..4} q(26 i + j) * 3^(4-i),   q(k) = t[k] + 1,
 *
 * with q(k) = 0 for the two positions past the group (k = 128, 129, the
 * last digit of v[24] and v[25]), stored as the byte
 *
 *     byte[j] = ceil(256 * v[j] / 243),   so that   v[j] = floor(243 * byte[j] / 256).
 *
 * So the weight at position 26 i + j is the i-th base-3 digit of v[j], most
 * significant first, minus one.  The 13 byte values that are no ceil(256 v /
 * 243) and non-zero padding digits are not codes.  Groups follow each other
 * along K in blocks of four: block b of a row is 112 bytes at offset 112 b,
 * group 4b + r at byte 26 r of it; the block's last 8 bytes, and the group
 * slots past the row's last group, are zero.  (The blocks keep every 4-group
 * run on a 16-byte boundary, where a tensor-memory-access copy can start.
 * Storing 256 v / 243 rounded up makes the digits of a byte come out,
 * most significant first, as the bits above 8 of repeated multiplications
 * by 3; taking byte j's digits from positions 26 apart makes the same digit
 * of bytes j and j+1 two neighbouring weights.) */
static const int kPow3[5] = {81, 27, 9, 3, 1}; /* 3^(4-i) */

static int pack_b3_group(const int8_t* t, uint8_t* out) {
  for (int j = 0; j < B3_GROUP_BYTES; ++j) {
    int value = 0;
    for (int i = 0; i < 5; ++i) {
      const int k = 26 * i + j;
      int q = 0;
      if (k < GROUP) {
        if (t[k] < -1 || t[k] > 1) return ORACLE_ERR_BAD_CODE;
        q = t[k] + 1;
      }
      value += q * kPow3[i];
    }
    out[j] = (uint8_t)((256 * value + 242) / 243); /* ceil(256 v / 243) */
  }
  return ORACLE_OK;
}

static int unpack_b3_group(const uint8_t* in, int8_t* t) {
  for (int j = 0; j < B3_GROUP_BYTES; ++j) {
    const int value = (243 * in[j]) / 256; /* floor(243 byte / 256) */
    if ((256 * value + 242) / 243 != in[j]) return ORACLE_ERR_BAD_CODE;
    for (int i = 0; i < 5; ++i) {
      const int q = (value / kPow3[i]) % 3;
      const int k = 26 * i + j;
      if (k < GROUP) t[k] = (int8_t)(q - 1);
      else if (q != 0) return ORACLE_ERR_BAD_CODE;
    }
  }
  return ORACLE_OK;
}

static int pack_b3(const int8_t* codes, int64_t N, int64_t K, uint8_t* packed) {
  const int64_t rb = row_bytes(K, MODE_TERNARY_B3), groups = K / GROUP;
  for (int64_t n = 0; n < N; ++n) {
    uint8_t* row = packed + n * rb;
    memset(row, 0, (size_t)rb);
    for (int64_t g = 0; g < groups; ++g) {
      int rc = pack_b3_group(codes + n * K + g * GROUP, row + b3_group_offset(g));
      if (rc != ORACLE_OK) return rc;
    }
  }
  return ORACLE_OK;
}

static int unpack_b3(const uint8_t* packed, int64_t N, int64_t K, int8_t* codes) {
  const int64_t rb = row_bytes(K, MODE_TERNARY_B3), groups = K / GROUP;
  for (int64_t n = 0; n < N; ++n) {
    const uint8_t* row = packed + n * rb;
    for (int64_t g = 0; g < groups; ++g) {
      int rc = unpack_b3_group(row + b3_group_offset(g), codes + n * K + g * GROUP);
      if (rc != ORACLE_OK) return rc;
    }
    /* every byte outside the groups is padding and must be zero */
    for (int64_t b = 0; b < rb; ++b) {
      const int64_t r = b % B3_BLOCK_BYTES / B3_GROUP_BYTES, g = b / B3_BLOCK_BYTES * B3_BLOCK_GROUPS + r;
      const int in_group = r < B3_BLOCK_GROUPS && g < groups;
      if (!in_group && row[b] != 0) return ORACLE_ERR_BAD_CODE;
    }
  }
  return ORACLE_OK;
}

/* Bit position of weight i of a word.
 *
 * Both formats pair weights (2p, 2p+1) of a word: weight 2p lives in the
 * low 16-bit half, weight 2p+1 in the high half, at the same offset.
 *
 * binary  (32 weights/word): weight i -> bit 16*(i%2) + 15 - i/2.
 *         Bit set <=> t = -1, clear <=> t = +1.
 * ternary (16 weights/word): weight i -> 2-bit field whose low bit is at
 *         16*(i%2) + 14 - 2*(i/2) (the magnitude, |t|) and whose high bit,
 *         one above, is the sign.  t=0 -> 00, t=+1 -> 01, t=-1 -> 11;
 *         the pattern 10 is not a code.
 * Words run along K: word j of row n holds k = j*per_word .. +per_word-1,
 * rows of N words each laid out one after the other (row-major [N, K/pw]).
 */
static int binary_bit(int i) { return 16 * (i & 1) + 15 - (i >> 1); }
static int ternary_low_bit(int i) { return 16 * (i & 1) + 14 - 2 * (i >> 1); }

int oracle_pack(const int8_t* codes, int64_t N, int64_t K, int mode, uint32_t* packed) {
  int rc = check_mode_shape(N, K, mode);
  if (rc != ORACLE_OK) return rc;
  if (mode == MODE_TERNARY_B3) return pack_b3(codes, N, K, (uint8_t*)packed);
  const int pw = per_word(mode);
  const int64_t words = K / pw;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t j = 0; j < words; ++j) {
      uint32_t word = 0;
      for (int i = 0; i < pw; ++i) {
        int t = codes[n * K + j * pw + i];
        if (mode == MODE_BINARY) {
          if (t == -1) word |= 1u << binary_bit(i);
          else if (t != 1) return ORACLE_ERR_BAD_CODE;
        } else {
          uint32_t field;
          if (t == 0) field = 0u;
          else if (t == 1) field = 1u;
          else if (t == -1) field = 3u;
          else return ORACLE_ERR_BAD_CODE;
          word |= field << ternary_low_bit(i);
        }
      }
      packed[n * words + j] = word;
    }
  }
  return ORACLE_OK;
}

int oracle_unpack(const uint32_t* packed, int64_t N, int64_t K, int mode, int8_t* codes) {
  int rc = check_mode_shape(N, K, mode);
  if (rc != ORACLE_OK) return rc;
  if (mode == MODE_TERNARY_B3) return unpack_b3((const uint8_t*)packed, N, K, codes);
  const int pw = per_word(mode);
  const int64_t words = K / pw;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t j = 0; j < words; ++j) {
      uint32_t word = packed[n * words + j];
      for (int i = 0; i < pw; ++i) {
        int t;
        if (mode == MODE_BINARY) {
          t = ((word >> binary_bit(i)) & 1u) ? -1 : 1;
        } else {
          uint32_t field = (word >> ternary_low_bit(i)) & 3u;
          if (field == 0u) t = 0;
          else if (field == 1u) t = 1;
          else if (field == 3u) t = -1;
          else return ORACLE_ERR_BAD_CODE; /* 10: sign without magnitude */
        }
        codes[n * K + j * pw + i] = (int8_t)t;
      }
    }
  }
  return ORACLE_OK;
}

/* --------------------------------------------------------- dequantise -- */

/* w[n,k] = fp16(t[n,k] * s[n, k/128]); scales are row-major [N, K/128]. */
static void dequant_row(const int8_t* t_row, const uint16_t* s_row, int64_t K, uint16_t* w_row) {
  for (int64_t k = 0; k < K; ++k) {
    double s = oracle_half_to_double(s_row[k / GROUP]);
    w_row[k] = oracle_double_to_half((double)t_row[k] * s);
  }
}

int oracle_dequant(const uint32_t* packed, const uint16_t* scales, int64_t N, int64_t K,
                   int mode, uint16_t* w) {
  int rc = check_mode_shape(N, K, mode);
  if (rc != ORACLE_OK) return rc;
  int8_t* t = (int8_t*)malloc((size_t)(N * K > 0 ? N * K : 1));
  if (!t) return ORACLE_ERR_NOMEM;
  rc = oracle_unpack(packed, N, K, mode, t);
  if (rc == ORACLE_OK) {
    for (int64_t n = 0; n < N; ++n) dequant_row(t + n * K, scales + n * (K / GROUP), K, w + n * K);
  }
  free(t);
  return rc;
}

/* --------------------------------------------------------------- GEMM -- */

typedef struct {
  const double* a; /* [M,K] activations as doubles */
  const double* w; /* [N,K] dequantised weights as doubles */
  int64_t M, N, K;
  int64_t m_begin, m_end;
  uint16_t* out;  /* [M,N] fp16, may be NULL */
  double* acc;    /* [M,N] double sums, may be NULL */
  double* absacc; /* [M,N] sum of |a*w|, may be NULL */
} gemm_job;

static void* gemm_rows(void* arg) {
  gemm_job* j = (gemm_job*)arg;
  for (int64_t m = j->m_begin; m < j->m_end; ++m) {
    const double* a = j->a + m * j->K;
    for (int64_t n = 0; n < j->N; ++n) {
      const double* w = j->w + n * j->K;
      double sum = 0.0, sum_abs = 0.0;
      for (int64_t k = 0; k < j->K; ++k) {
        double p = a[k] * w[k]; /* exact: two 11-bit significands */
        sum += p;
        sum_abs += fabs(p);
      }
      if (j->out) j->out[m * j->N + n] = oracle_double_to_half(sum);
      if (j->acc) j->acc[m * j->N + n] = sum;
      if (j->absacc) j->absacc[m * j->N + n] = sum_abs;
    }
  }
  return NULL;
}

/* Dequantise the whole weight matrix into doubles (unpack, then t*s rounded
 * to fp16 exactly as oracle_dequant, then widened). */
static int weights_as_double(const uint32_t* packed, const uint16_t* scales, int64_t N, int64_t K,
                             int mode, double** w_out) {
  uint16_t* w16 = (uint16_t*)malloc((size_t)(N * K > 0 ? N * K : 1) * sizeof(uint16_t));
  double* w = (double*)malloc((size_t)(N * K > 0 ? N * K : 1) * sizeof(double));
  if (!w16 || !w) {
    free(w16);
    free(w);
    return ORACLE_ERR_NOMEM;
  }
  int rc = oracle_dequant(packed, scales, N, K, mode, w16);
  if (rc == ORACLE_OK) oracle_half_to_double_array(w16, N * K, w);
  free(w16);
  if (rc != ORACLE_OK) {
    free(w);
    return rc;
  }
  *w_out = w;
  return ORACLE_OK;
}

static int gemm_with_weights(const uint16_t* A, double* w, int64_t M, int64_t N, int64_t K, uint16_t* out,
                             double* acc, double* absacc, int nthreads);

/* out = A * W^T, one double accumulation per output.  Rows of the output are
 * split across nthreads worker threads (each output is still one sequential
 * sum, so the thread count does not change any result). */
int oracle_gemm(const uint16_t* A, const uint32_t* packed, const uint16_t* scales, int64_t M,
                int64_t N, int64_t K, int mode, uint16_t* out, double* acc, double* absacc,
                int nthreads) {
  int rc = check_mode_shape(N, K, mode);
  if (rc != ORACLE_OK) return rc;
  if (M < 0) return ORACLE_ERR_SHAPE;
  double* w = NULL;
  rc = weights_as_double(packed, scales, N, K, mode, &w);
  if (rc != ORACLE_OK) return rc;
  return gemm_with_weights(A, w, M, N, K, out, acc, absacc, nthreads);
}

/* The same product for FP16 weights given directly, [N,K] row-major. */
int oracle_gemm_w16(const uint16_t* A, const uint16_t* w16, int64_t M, int64_t N, int64_t K, uint16_t* out,
                    double* acc, double* absacc, int nthreads) {
  if (M < 0 || N < 0 || K < 0) return ORACLE_ERR_SHAPE;
  double* w = (double*)malloc((size_t)(N * K > 0 ? N * K : 1) * sizeof(double));
  if (!w) return ORACLE_ERR_NOMEM;
  oracle_half_to_double_array(w16, N * K, w);
  return gemm_with_weights(A, w, M, N, K, out, acc, absacc, nthreads);
}

/* Takes ownership of w. */
static int gemm_with_weights(const uint16_t* A, double* w, int64_t M, int64_t N, int64_t K, uint16_t* out,
                             double* acc, double* absacc, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  double* a = (double*)malloc((size_t)(M * K > 0 ? M * K : 1) * sizeof(double));
  if (!a) {
    free(w);
    return ORACLE_ERR_NOMEM;
  }
  oracle_half_to_double_array(A, M * K, a);

  if (nthreads > M) nthreads = M > 0 ? (int)M : 1;
  gemm_job* jobs = (gemm_job*)calloc((size_t)nthreads, sizeof(gemm_job));
  pthread_t* tids = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !tids) {
    free(jobs);
    free(tids);
    free(a);
    free(w);
    return ORACLE_ERR_NOMEM;
  }
  for (int i = 0; i < nthreads; ++i) {
    jobs[i] = (gemm_job){a, w, M, N, K, M * i / nthreads, M * (i + 1) / nthreads, out, acc, absacc};
  }
  int started = 0;
  for (int i = 1; i < nthreads; ++i) {
    if (pthread_create(&tids[i], NULL, gemm_rows, &jobs[i]) != 0) break;
    started = i;
  }
  gemm_rows(&jobs[0]);
  for (int i = started + 1; i < nthreads; ++i) gemm_rows(&jobs[i]); /* threads that failed to start */
  for (int i = 1; i <= started; ++i) pthread_join(tids[i], NULL);
  free(jobs);
  free(tids);
  free(a);
  free(w);
  return ORACLE_OK;
}

/* The same sums for a list of (m, n) output positions, each computed on its
 * own: only the needed weight rows are unpacked.  Used to check full-size
 * problems at sampled positions. */
int oracle_gemm_entries(const uint16_t* A, const uint32_t* packed, const uint16_t* scales,
                        int64_t M, int64_t N, int64_t K, int mode, const int64_t* ms,
                        const int64_t* ns, int64_t count, uint16_t* out, double* acc,
                        double* absacc) {
  int rc = check_mode_shape(N, K, mode);
  if (rc != ORACLE_OK) return rc;
  const int64_t words = row_bytes(K, mode) / 4;
  int8_t* t = (int8_t*)malloc((size_t)(K > 0 ? K : 1));
  uint16_t* w16 = (uint16_t*)malloc((size_t)(K > 0 ? K : 1) * sizeof(uint16_t));
  if (!t || !w16) {
    free(t);
    free(w16);
    return ORACLE_ERR_NOMEM;
  }
  rc = ORACLE_OK;
  for (int64_t i = 0; i < count && rc == ORACLE_OK; ++i) {
    int64_t m = ms[i], n = ns[i];
    if (m < 0 || m >= M || n < 0 || n >= N) {
      rc = ORACLE_ERR_ARG;
      break;
    }
    rc = oracle_unpack(packed + n * words, 1, K, mode, t);
    if (rc != ORACLE_OK) break;
    dequant_row(t, scales + n * (K / GROUP), K, w16);
    double sum = 0.0, sum_abs = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      double p = oracle_half_to_double(A[m * K + k]) * oracle_half_to_double(w16[k]);
      sum += p;
      sum_abs += fabs(p);
    }
    if (out) out[i] = oracle_double_to_half(sum);
    if (acc) acc[i] = sum;
    if (absacc) absacc[i] = sum_abs;
  }
  free(t);
  free(w16);
  return rc;
}

/* ---------------------------------------------- 4-bit group-affine (HQQ) -- */

#define HQQ_GROUP 64

/* Packing (this project's): words run along K, 8 weights per word; weight i
 * of word j (k = 8 j + i) is the nibble at bit 16 (i % 2) + 4 (i / 2), so
 * weights 2p and 2p+1 sit at the same offset of the two 16-bit halves.  Rows
 * of K/8 words, row-major [N, K/8].  q must be in 0..15. */
static int hqq4_bit(int i) { return 16 * (i & 1) + 4 * (i >> 1); }

static int hqq4_check(int64_t N, int64_t K) {
  if (N < 0 || K < 0) return ORACLE_ERR_SHAPE;
  if (K % GROUP != 0) return ORACLE_ERR_SHAPE; /* whole 128-weight tiles, two affine groups each */
  return ORACLE_OK;
}

int oracle_hqq4_pack(const uint8_t* q, int64_t N, int64_t K, uint32_t* packed) {
  int rc = hqq4_check(N, K);
  if (rc != ORACLE_OK) return rc;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K / 8; ++j) {
      uint32_t word = 0;
      for (int i = 0; i < 8; ++i) {
        const uint8_t v = q[n * K + 8 * j + i];
        if (v > 15) return ORACLE_ERR_BAD_CODE;
        word |= (uint32_t)v << hqq4_bit(i);
      }
      packed[n * (K / 8) + j] = word;
    }
  return ORACLE_OK;
}

int oracle_hqq4_unpack(const uint32_t* packed, int64_t N, int64_t K, uint8_t* q) {
  int rc = hqq4_check(N, K);
  if (rc != ORACLE_OK) return rc;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K / 8; ++j) {
      const uint32_t word = packed[n * (K / 8) + j];
      for (int i = 0; i < 8; ++i) q[n * K + 8 * j + i] = (uint8_t)((word >> hqq4_bit(i)) & 15u);
    }
  return ORACLE_OK;
}

/* w[n,k] = fp16(fp16(q - z) * s) with s = scales[n, k/64], z = zeros[n, k/64]:
 * both steps are exact in double (a small integer minus an FP16 value; the
 * product of two FP16 values) and rounded once each to FP16, which is the
 * IEEE FP16 subtraction and multiplication. */
int oracle_hqq4_dequant(const uint32_t* packed, const uint16_t* scales, const uint16_t* zeros, int64_t N,
                        int64_t K, uint16_t* w) {
  int rc = hqq4_check(N, K);
  if (rc != ORACLE_OK) return rc;
  uint8_t* q = (uint8_t*)malloc((size_t)(N * K > 0 ? N * K : 1));
  if (!q) return ORACLE_ERR_NOMEM;
  rc = oracle_hqq4_unpack(packed, N, K, q);
  const int64_t groups = K / HQQ_GROUP;
  for (int64_t n = 0; rc == ORACLE_OK && n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      const double s = oracle_half_to_double(scales[n * groups + k / HQQ_GROUP]);
      const double z = oracle_half_to_double(zeros[n * groups + k / HQQ_GROUP]);
      const uint16_t d = oracle_double_to_half((double)q[n * K + k] - z);
      w[n * K + k] = oracle_double_to_half(oracle_half_to_double(d) * s);
    }
  free(q);
  return rc;
}

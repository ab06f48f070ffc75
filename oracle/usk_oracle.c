/*
 * usk_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, sequential CPU restatement of the UltraSketchLLM sketch
 * (build, decode, reference products).  Only the test suite, the smoke check
 * and the CPU-baseline leg of the benchmark may load this file's library; the
 * product path never does.  It shares no code, header, table or constant
 * generator with the CUDA library: every constant below is written out here
 * from its published definition.
 *
 * Sources (page title + section):
 *  - "UltraSketchLLM: Sub-1-Bit LLM Compression via Sketch and Hardware-Friendly
 *    Operators" (gist.science/es/paper/2506.17255), Resumen Tecnico:
 *      Metodologia §1 "Diseno de Sketch AbsMaxMin"  -- one value kept per hashed
 *        bucket, chosen by magnitude;
 *      Metodologia §4 "Mapeo de Operadores de Matriz" -- decompression is
 *        W_hat = S . P^T, i.e. every weight reads back its bucket;
 *      Resultados Experimentales "Eficiencia de Compresion" -- 0.5 bit/weight.
 *    The lay part of the same page, §2 "La Solucion: El Sketch": a hash drops
 *    weights into buckets and a bucket keeps only its largest member.
 *  - The pages give no hash family, tie-break, block geometry or rounding.  The
 *    readings used here (winner = max of |w|*importance, ties to the smallest
 *    row-major index, 64-row scale blocks, 64x256 hash tiles, octet-structured
 *    multiply-shift hash keyed by SplitMix64) are the frozen format of this
 *    library; each one is written where it is used.
 *  - SplitMix64: Steele, Lea, Flood, "Fast splittable pseudorandom number
 *    generators" (OOPSLA 2014); constants as in Vigna's public-domain
 *    splitmix64.c.
 *  - Multiply-shift hashing: Dietzfelbinger et al., "A reliable randomized
 *    algorithm for the closest-pair problem" (J. Algorithms 1997).
 *  - Range reduction by a 32x32->64 multiply: Lemire, "A fast alternative to
 *    the modulo reduction" (2016).
 *  - IEEE 754-2008 binary16 / binary32, round to nearest, ties to even.
 *
 * Build: gcc -std=c99 -O2 -ffp-contract=off -fPIC -shared (no fast-math), so
 * every float operation below is one correctly rounded IEEE operation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Status values returned by the oracle (same meanings as the library's). */
#define ORC_OK 0
#define ORC_ERR_NULL 1
#define ORC_ERR_SHAPE 2
#define ORC_ERR_DTYPE 3
#define ORC_ERR_NONFINITE 8
#define ORC_ERR_IMPORTANCE 11
#define ORC_ERR_SCALE_OVERFLOW 12

/* Format geometry. */
#define ROWS_PER_BLOCK 64   /* scale block and hash-tile height            */
#define TILE_COLS 256       /* hash-tile width; K % 256 == 0, so all tiles are full */
#define WEIGHTS_PER_BUCKET 16
#define OCTET 8             /* columns that share one hash evaluation      */
#define CLASSES 32          /* bucket classes per slot                     */

/* ---------------------------------------------------------------- numbers */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 is the top half of a binary32. */
float orc_bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* binary16 -> binary32, from the IEEE 754 encoding. */
float orc_f16_to_f32(uint16_t h) {
  int sign = (h >> 15) & 1, e = (h >> 10) & 31, man = h & 1023;
  double v;
  if (e == 31) return man ? f32_from_bits(0x7fc00000u) : (sign ? -INFINITY : INFINITY);
  if (e == 0) v = ldexp((double)man, -24);              /* subnormal: man * 2^-24 */
  else v = ldexp((double)(1024 + man), e - 25);         /* (1.man) * 2^(e-15)     */
  return (float)(sign ? -v : v);
}

/* binary32 -> binary16, round to nearest, ties to even, from the definition:
 * find the binary16 quantum for |f|, round |f| / quantum to an integer (ties
 * to even), and encode.  Every double step below is exact. */
uint16_t orc_f32_to_f16(float f) {
  uint32_t u = bits_from_f32(f);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  if (isnan(f)) return (uint16_t)(sign | 0x7e00u);
  double a = fabs((double)f);
  if (isinf(f) || a >= 65520.0) return (uint16_t)(sign | 0x7c00u); /* 65520 = 65504 + half ulp */
  if (a == 0.0) return sign;
  int ex;
  frexp(a, &ex);                              /* a = fr * 2^ex, fr in [0.5, 1) */
  int e = ex - 1;                             /* a in [2^e, 2^(e+1))           */
  double q = (e < -14) ? ldexp(1.0, -24) : ldexp(1.0, e - 10);
  double n = nearbyint(a / q);                /* ties to even (default mode)   */
  double r = n * q;
  if (r == 0.0) return sign;
  if (r < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)n); /* subnormal */
  frexp(r, &ex);
  e = ex - 1;
  if (e > 15) return (uint16_t)(sign | 0x7c00u);
  uint16_t man = (uint16_t)((r / ldexp(1.0, e) - 1.0) * 1024.0);
  return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | man);
}

/* ------------------------------------------------------------- hashing */

/* SplitMix64: output n (n = 1, 2, ...) of the generator seeded with `seed` is
 * mix(seed + n * gamma). */
uint64_t orc_splitmix64(uint64_t seed, uint64_t n) {
  uint64_t z = seed + n * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* Tiles per 64-row block of a K-column matrix. */
static int64_t tiles_per_row(int64_t K) { return K / TILE_COLS; }

/* Hash key of tile `tile_id`: A (odd multiplier) and C (offset) of the affine
 * multiply-shift hash are the low and high halves of SplitMix64 output
 * tile_id + 1. */
void orc_tile_hash_params(uint64_t seed, uint64_t tile_id, uint32_t* A, uint32_t* C) {
  uint64_t z = orc_splitmix64(seed, tile_id + 1);
  *A = (uint32_t)z | 1u;
  *C = (uint32_t)(z >> 32);
}

/* Global code index of weight (i, j) in an M x K matrix.
 * Row block rb = i / 64 (row r inside it), tile tc = j / 256 (column c inside
 * it).  The 8 columns of octet o = c / 8 (o in 0..31) share one hash value:
 *   m     = r * 32 + o                           (octet's index in the tile)
 *   h     = A * m + C  (mod 2^32)                (multiply-shift, keyed per tile)
 *   slot  = floor(h * 4 / 2^32)                  (4 slots per class)
 *   class = (o + r) mod 32
 *   sub   = c mod 8
 *   b     = (slot * 32 + class) * 8 + sub        (bucket inside the tile, 0..1023)
 * A tile holds 64*256 weights and 1024 buckets (16 weights per bucket); its
 * codes are stored from rb * (4K) + 1024 * tc.  Every (class, sub) pair owns
 * exactly one octet column per row, i.e. 64 members spread over 4 slots. */
int64_t orc_bucket_index(int64_t K, uint64_t seed, int64_t i, int64_t j) {
  int64_t rb = i / ROWS_PER_BLOCK, r = i % ROWS_PER_BLOCK;
  int64_t tc = j / TILE_COLS, c = j % TILE_COLS;
  int64_t T = tiles_per_row(K);
  int64_t o = c / OCTET, sub = c % OCTET;
  uint32_t A, C;
  orc_tile_hash_params(seed, (uint64_t)(rb * T + tc), &A, &C);
  uint32_t m = (uint32_t)(r * (TILE_COLS / OCTET) + o);
  uint32_t h = A * m + C;
  int64_t slot = (int64_t)(((uint64_t)h * 4u) >> 32);
  int64_t cls = (o + r) % CLASSES;
  int64_t b = (slot * CLASSES + cls) * OCTET + sub;
  return rb * (4 * K) + 1024 * tc + b;
}

/* ------------------------------------------------------------- shapes */

static int check_shape(int64_t M, int64_t K) {
  if (M < 0 || K < 0) return ORC_ERR_SHAPE;
  if (M % ROWS_PER_BLOCK != 0 || K % 256 != 0) return ORC_ERR_SHAPE;
  if (K > (1LL << 20) || M > (1LL << 22)) return ORC_ERR_SHAPE;
  return ORC_OK;
}

static float load_elem(const void* p, int dtype, int64_t idx) {
  if (dtype == 0) return ((const float*)p)[idx];
  return orc_bf16_to_f32(((const uint16_t*)p)[idx]);
}

/* -------------------------------------------------------------- build */

/* Build the sketch of W [M, K] (row stride ldw elements; dtype 0 = fp32,
 * 1 = bf16 bit patterns) with per-column importance imp [K] (NULL = all ones).
 *
 * Per bucket the kept member is the one with the largest selection key
 * k = fp32(|w|) * imp_j (one IEEE fp32 multiply); equal keys go to the member
 * with the smallest row-major index.  The bucket keeps that member's signed
 * value v (0 for a bucket with no member).  Per 64-row block the scale is
 * s16 = binary16(max |v| / 127) and each code is
 * clamp(round_half_even(v / float(s16)), -127, 127), or 0 when s16 == 0.
 *
 * Outputs: codes [M*K/16] int8, scales [M/64] binary16 bits.  Optional:
 * winner [M*K/16] (row-major flat index i*K + j of each bucket's kept member,
 * -1 if empty) and value [M*K/16] (the kept fp32 value).
 *
 * The scan below visits the weights of each tile in row-major order and keeps
 * a running best per bucket, which is the sequential hash-and-update the pages
 * describe; the maximum does not depend on the order. */
int orc_build_rows(const void* W, int dtype, int64_t M, int64_t K, int64_t ldw,
                   const float* imp, uint64_t seed, int64_t rb0, int8_t* codes,
                   uint16_t* scales, int64_t* winner, float* value);

int orc_build(const void* W, int dtype, int64_t M, int64_t K, int64_t ldw,
              const float* imp, uint64_t seed, int8_t* codes, uint16_t* scales,
              int64_t* winner, float* value) {
  return orc_build_rows(W, dtype, M, K, ldw, imp, seed, 0, codes, scales, winner, value);
}

/* Same as orc_build for the M rows starting at row block rb0 of a larger
 * matrix: W holds rows [64*rb0, 64*rb0 + M), the hash uses their true row
 * blocks, codes/scales/winner/value are those rows' slices (winner indices are
 * relative to W). */
int orc_build_rows(const void* W, int dtype, int64_t M, int64_t K, int64_t ldw,
                   const float* imp, uint64_t seed, int64_t rb0, int8_t* codes,
                   uint16_t* scales, int64_t* winner, float* value) {
  int st = check_shape(M, K);
  if (st) return st;
  if (rb0 < 0) return ORC_ERR_SHAPE;
  if (dtype != 0 && dtype != 1) return ORC_ERR_DTYPE;
  if (M == 0) return ORC_OK;
  if (!codes || !scales) return ORC_ERR_NULL;
  if (K == 0) {
    for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) scales[rb] = 0;
    return ORC_OK;
  }
  if (!W || ldw < K) return ORC_ERR_NULL;
  if (imp) {
    for (int64_t j = 0; j < K; ++j) {
      uint32_t u = bits_from_f32(imp[j]);
      if ((u >> 31) || !isfinite(imp[j])) return ORC_ERR_IMPORTANCE;
    }
  }
  int64_t nb = M * K / WEIGHTS_PER_BUCKET;
  int64_t per_block = 4 * K;             /* buckets per 64-row block */
  float* bestkey = (float*)malloc(sizeof(float) * (size_t)per_block);
  int64_t* bestidx = (int64_t*)malloc(sizeof(int64_t) * (size_t)per_block);
  float* val = (float*)malloc(sizeof(float) * (size_t)per_block);
  if (!bestkey || !bestidx || !val) { free(bestkey); free(bestidx); free(val); return ORC_ERR_NULL; }
  int status = ORC_OK;
  for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) {
    for (int64_t b = 0; b < per_block; ++b) { bestkey[b] = -1.0f; bestidx[b] = -1; }
    /* selection: a running best per bucket */
    for (int64_t r = 0; r < ROWS_PER_BLOCK; ++r) {
      int64_t i = rb * ROWS_PER_BLOCK + r;
      for (int64_t j = 0; j < K; ++j) {
        float w = load_elem(W, dtype, i * ldw + j);
        if (!isfinite(w)) status = ORC_ERR_NONFINITE;
        float k = fabsf(w) * (imp ? imp[j] : 1.0f);
        int64_t b = orc_bucket_index(K, seed, i + rb0 * ROWS_PER_BLOCK, j) - (rb + rb0) * per_block;
        int64_t flat = i * K + j;
        /* strictly larger key wins; an equal key never displaces the earlier
         * (smaller-index) member because the scan is in row-major order */
        if (k > bestkey[b] || bestidx[b] < 0) { bestkey[b] = k; bestidx[b] = flat; }
      }
    }
    /* kept values and the block maximum */
    float mx = 0.0f;
    for (int64_t b = 0; b < per_block; ++b) {
      float v = 0.0f;
      if (bestidx[b] >= 0) {
        int64_t i = bestidx[b] / K, j = bestidx[b] % K;
        v = load_elem(W, dtype, i * ldw + j);
      }
      val[b] = v;
      if (fabsf(v) > mx) mx = fabsf(v);
    }
    /* scale */
    uint16_t s16 = orc_f32_to_f16(mx / 127.0f);
    if ((s16 & 0x7c00u) == 0x7c00u) status = status ? status : ORC_ERR_SCALE_OVERFLOW;
    scales[rb] = s16;
    float s = orc_f16_to_f32(s16);
    /* quantization */
    for (int64_t b = 0; b < per_block; ++b) {
      int8_t code = 0;
      if (s != 0.0f) {
        float q = nearbyintf(val[b] / s);
        if (q > 127.0f) q = 127.0f;
        if (q < -127.0f) q = -127.0f;
        code = (int8_t)q;           /* NaN never reaches here for finite input */
        if (isnan(q)) code = 0;
      }
      int64_t g = rb * per_block + b;
      codes[g] = code;
      if (winner) winner[g] = bestidx[b];
      if (value) value[g] = val[b];
    }
  }
  (void)nb;
  free(bestkey); free(bestidx); free(val);
  return status;
}

/* ------------------------------------------------------------- decode */

/* W_hat [M, K] fp32: every weight reads its bucket's code and its block scale,
 * w_hat = float(code) * float(s16) (exact in fp32). */
int orc_decode(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K,
               uint64_t seed, float* What) {
  int st = check_shape(M, K);
  if (st) return st;
  if (M == 0 || K == 0) return ORC_OK;
  if (!codes || !scales || !What) return ORC_ERR_NULL;
  for (int64_t i = 0; i < M; ++i) {
    float s = orc_f16_to_f32(scales[i / ROWS_PER_BLOCK]);
    for (int64_t j = 0; j < K; ++j)
      What[i * K + j] = (float)codes[orc_bucket_index(K, seed, i, j)] * s;
  }
  return ORC_OK;
}

/* Reference product y[t][i] = sum_j w_hat[i][j] * x[t][j] in float64, for the
 * rows listed in rows[0..nrows) (rows == NULL: all M rows, nrows ignored).
 * x [batch, K] has dtype 0 = fp32, 1 = bf16 bits.  y is [batch, nrows] (or
 * [batch, M]).  The decoded weight is rebuilt from its bucket for every term,
 * exactly as W_hat = S . P^T reads it back. */
int orc_gemv_f64(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K,
                 uint64_t seed, const void* x, int xdtype, int64_t batch,
                 const int64_t* rows, int64_t nrows, double* y) {
  int st = check_shape(M, K);
  if (st) return st;
  if (xdtype != 0 && xdtype != 1) return ORC_ERR_DTYPE;
  if (batch < 0) return ORC_ERR_SHAPE;
  int64_t nr = rows ? nrows : M;
  if (nr == 0 || batch == 0) return ORC_OK;
  if (!y) return ORC_ERR_NULL;
  if (K == 0) {
    for (int64_t q = 0; q < batch * nr; ++q) y[q] = 0.0;
    return ORC_OK;
  }
  if (!codes || !scales || !x) return ORC_ERR_NULL;
  double* wrow = (double*)malloc(sizeof(double) * (size_t)K);
  if (!wrow) return ORC_ERR_NULL;
  for (int64_t q = 0; q < nr; ++q) {
    int64_t i = rows ? rows[q] : q;
    if (i < 0 || i >= M) { free(wrow); return ORC_ERR_SHAPE; }
    float s = orc_f16_to_f32(scales[i / ROWS_PER_BLOCK]);
    for (int64_t j = 0; j < K; ++j)
      wrow[j] = (double)((float)codes[orc_bucket_index(K, seed, i, j)] * s);
    for (int64_t t = 0; t < batch; ++t) {
      double acc = 0.0;
      for (int64_t j = 0; j < K; ++j) acc += wrow[j] * (double)load_elem(x, xdtype, t * K + j);
      y[t * nr + q] = acc;
    }
  }
  free(wrow);
  return ORC_OK;
}

/* Storage of a sketch in bytes: codes (1 byte per 16 weights) and scales
 * (2 bytes per 64-row block). */
void orc_storage_bytes(int64_t M, int64_t K, int64_t* code_bytes, int64_t* scale_bytes) {
  *code_bytes = M * K / WEIGHTS_PER_BUCKET;
  *scale_bytes = 2 * (M / ROWS_PER_BLOCK);
}

/* Element-wise conversions over arrays (for exhaustive pins). */
void orc_f32_to_f16_array(const float* in, uint16_t* out, int64_t n) {
  for (int64_t q = 0; q < n; ++q) out[q] = orc_f32_to_f16(in[q]);
}
void orc_f16_to_f32_array(const uint16_t* in, float* out, int64_t n) {
  for (int64_t q = 0; q < n; ++q) out[q] = orc_f16_to_f32(in[q]);
}

/* ================================================================ format 2
 *
 * The multi-row AbsMaxMin sketch ("UltraSketchLLM" explainer, Resumen Tecnico,
 * Metodologia §1 "Diseno de Sketch AbsMaxMin"): a bucket stores the member
 * with the SMALLEST absolute value, decompression takes the MAX over several
 * independently hashed sketch rows, and the rebuilt weight is the original one
 * or one of smaller magnitude.  Readings (the pages give no more detail):
 *  - depth D in {1, 2, 4} hash rows share the tile's 1024 buckets, so the
 *    storage stays one int8 code per 16 weights (Resultados, 0.5 bit/weight):
 *    row rho owns buckets [rho*1024/D, (rho+1)*1024/D) of the tile;
 *  - row rho of tile tile_id is keyed by SplitMix64 output tile_id*D + rho + 1,
 *    slot = floor(4h / 2^32) as in format 1, class = (o + r) mod (32/D),
 *    bucket = rho*1024/D + (slot*(32/D) + class)*8 + c mod 8.  With D = 1 this
 *    is exactly the format-1 hash;
 *  - the kept member has the smallest |w|, ties to the smallest row-major
 *    index; an empty bucket keeps 0.  No importance weighting (a weighted key
 *    would break the magnitude bound);
 *  - scale as format 1: s16 = binary16(max over the block's buckets of |v| / 127);
 *  - code = sign(v) * min(127, floor(|v| / s)) (toward zero), so that
 *    |code * s| <= |v| and the bound survives quantisation;
 *  - decode: the code of largest magnitude among the weight's D buckets (ties
 *    to the lowest row), times s. */

static int amm_depth_ok(int depth) { return depth == 1 || depth == 2 || depth == 4; }

/* Global code index of weight (i, j) in hash row rho of a depth-D sketch. */
int64_t orc_amm_bucket_index(int64_t K, uint64_t seed, int depth, int rho, int64_t i, int64_t j) {
  int64_t rb = i / ROWS_PER_BLOCK, r = i % ROWS_PER_BLOCK;
  int64_t tc = j / TILE_COLS, c = j % TILE_COLS;
  int64_t T = tiles_per_row(K);
  int64_t o = c / OCTET, sub = c % OCTET;
  int64_t nclass = CLASSES / depth, per_row = 1024 / depth;
  uint32_t A, C;
  orc_tile_hash_params(seed, (uint64_t)((rb * T + tc) * depth + rho), &A, &C);
  uint32_t m = (uint32_t)(r * (TILE_COLS / OCTET) + o);
  uint32_t h = A * m + C;
  int64_t slot = (int64_t)(((uint64_t)h * 4u) >> 32);
  int64_t cls = (o + r) % nclass;
  int64_t b = rho * per_row + (slot * nclass + cls) * OCTET + sub;
  return rb * (4 * K) + 1024 * tc + b;
}

/* Largest n in [0, 127] with n * s <= a (a >= 0, s > 0); every product and
 * comparison below is exact in double (an 8-bit integer times a binary16). */
static int floor_code(double a, double s) {
  double n = floor(a / s);
  if (n > 127.0) n = 127.0;
  while (n < 127.0 && (n + 1.0) * s <= a) n += 1.0;
  while (n > 0.0 && n * s > a) n -= 1.0;
  return (int)n;
}

/* Build a depth-D AbsMaxMin sketch of W [M, K] (rows starting at row block rb0
 * of a larger matrix, as orc_build_rows).  Outputs as orc_build_rows: codes,
 * scales, optional winner (flat index into W, -1 if empty) and value. */
int orc_amm_build_rows(const void* W, int dtype, int64_t M, int64_t K, int64_t ldw,
                       uint64_t seed, int depth, int64_t rb0, int8_t* codes,
                       uint16_t* scales, int64_t* winner, float* value) {
  int st = check_shape(M, K);
  if (st) return st;
  if (rb0 < 0) return ORC_ERR_SHAPE;
  if (dtype != 0 && dtype != 1) return ORC_ERR_DTYPE;
  if (!amm_depth_ok(depth)) return ORC_ERR_SHAPE;
  if (M == 0) return ORC_OK;
  if (!codes || !scales) return ORC_ERR_NULL;
  if (K == 0) {
    for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) scales[rb] = 0;
    return ORC_OK;
  }
  if (!W || ldw < K) return ORC_ERR_NULL;
  int64_t per_block = 4 * K;
  float* bestmag = (float*)malloc(sizeof(float) * (size_t)per_block);
  int64_t* bestidx = (int64_t*)malloc(sizeof(int64_t) * (size_t)per_block);
  float* val = (float*)malloc(sizeof(float) * (size_t)per_block);
  if (!bestmag || !bestidx || !val) { free(bestmag); free(bestidx); free(val); return ORC_ERR_NULL; }
  int status = ORC_OK;
  for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) {
    for (int64_t b = 0; b < per_block; ++b) { bestmag[b] = 0.0f; bestidx[b] = -1; }
    /* every weight updates its bucket in each hash row: keep the smallest |w|;
     * the row-major scan keeps the earlier member on equal magnitudes */
    for (int64_t r = 0; r < ROWS_PER_BLOCK; ++r) {
      int64_t i = rb * ROWS_PER_BLOCK + r;
      for (int64_t j = 0; j < K; ++j) {
        float w = load_elem(W, dtype, i * ldw + j);
        if (!isfinite(w)) status = ORC_ERR_NONFINITE;
        float mag = fabsf(w);
        for (int rho = 0; rho < depth; ++rho) {
          int64_t b = orc_amm_bucket_index(K, seed, depth, rho, i + rb0 * ROWS_PER_BLOCK, j) -
                      (rb + rb0) * per_block;
          if (bestidx[b] < 0 || mag < bestmag[b]) { bestmag[b] = mag; bestidx[b] = i * K + j; }
        }
      }
    }
    float mx = 0.0f;
    for (int64_t b = 0; b < per_block; ++b) {
      float v = 0.0f;
      if (bestidx[b] >= 0) {
        int64_t i = bestidx[b] / K, j = bestidx[b] % K;
        v = load_elem(W, dtype, i * ldw + j);
      }
      val[b] = v;
      if (fabsf(v) > mx) mx = fabsf(v);
    }
    uint16_t s16 = orc_f32_to_f16(mx / 127.0f);
    if ((s16 & 0x7c00u) == 0x7c00u) status = status ? status : ORC_ERR_SCALE_OVERFLOW;
    scales[rb] = s16;
    double s = (double)orc_f16_to_f32(s16);
    for (int64_t b = 0; b < per_block; ++b) {
      int code = 0;
      if (s != 0.0 && isfinite(s) && isfinite(val[b])) {
        code = floor_code(fabs((double)val[b]), s);
        if (val[b] < 0.0f) code = -code;
      }
      int64_t g = rb * per_block + b;
      codes[g] = (int8_t)code;
      if (winner) winner[g] = bestidx[b];
      if (value) value[g] = val[b];
    }
  }
  free(bestmag); free(bestidx); free(val);
  return status;
}

/* Code of weight (i, j): the largest-magnitude code over the D rows (ties to
 * the lowest row). */
static int amm_code(const int8_t* codes, int64_t K, uint64_t seed, int depth, int64_t i, int64_t j) {
  int best = codes[orc_amm_bucket_index(K, seed, depth, 0, i, j)];
  for (int rho = 1; rho < depth; ++rho) {
    int c = codes[orc_amm_bucket_index(K, seed, depth, rho, i, j)];
    if (abs(c) > abs(best)) best = c;
  }
  return best;
}

/* W_hat [M, K] of a depth-D sketch: w_hat = float(code) * float(s16). */
int orc_amm_decode(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K,
                   uint64_t seed, int depth, float* What) {
  int st = check_shape(M, K);
  if (st) return st;
  if (!amm_depth_ok(depth)) return ORC_ERR_SHAPE;
  if (M == 0 || K == 0) return ORC_OK;
  if (!codes || !scales || !What) return ORC_ERR_NULL;
  for (int64_t i = 0; i < M; ++i) {
    float s = orc_f16_to_f32(scales[i / ROWS_PER_BLOCK]);
    for (int64_t j = 0; j < K; ++j) What[i * K + j] = (float)amm_code(codes, K, seed, depth, i, j) * s;
  }
  return ORC_OK;
}

/* Reference product of a depth-D sketch in float64 (arguments as orc_gemv_f64). */
int orc_amm_gemv_f64(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K,
                     uint64_t seed, int depth, const void* x, int xdtype, int64_t batch,
                     const int64_t* rows, int64_t nrows, double* y) {
  int st = check_shape(M, K);
  if (st) return st;
  if (!amm_depth_ok(depth)) return ORC_ERR_SHAPE;
  if (xdtype != 0 && xdtype != 1) return ORC_ERR_DTYPE;
  if (batch < 0) return ORC_ERR_SHAPE;
  int64_t nr = rows ? nrows : M;
  if (nr == 0 || batch == 0) return ORC_OK;
  if (!y) return ORC_ERR_NULL;
  if (K == 0) {
    for (int64_t q = 0; q < batch * nr; ++q) y[q] = 0.0;
    return ORC_OK;
  }
  if (!codes || !scales || !x) return ORC_ERR_NULL;
  double* wrow = (double*)malloc(sizeof(double) * (size_t)K);
  if (!wrow) return ORC_ERR_NULL;
  for (int64_t q = 0; q < nr; ++q) {
    int64_t i = rows ? rows[q] : q;
    if (i < 0 || i >= M) { free(wrow); return ORC_ERR_SHAPE; }
    float s = orc_f16_to_f32(scales[i / ROWS_PER_BLOCK]);
    for (int64_t j = 0; j < K; ++j)
      wrow[j] = (double)((float)amm_code(codes, K, seed, depth, i, j) * s);
    for (int64_t t = 0; t < batch; ++t) {
      double acc = 0.0;
      for (int64_t j = 0; j < K; ++j) acc += wrow[j] * (double)load_elem(x, xdtype, t * K + j);
      y[t * nr + q] = acc;
    }
  }
  free(wrow);
  return ORC_OK;
}

/* ================================================================ format 3
 *
 * The column-shared projection ("UltraSketchLLM" explainer, Resumen Tecnico,
 * Metodologia §4 "Mapeo de Operadores de Matriz Amigables con el Hardware"):
 * compression is a modified matrix product of W with a projection matrix P
 * whose reduction is a MIN over absolute values, and decompression is the plain
 * product W_hat = S . P^T.  Readings (the pages give no more detail):
 *  - P is one-hot per input column and shared by every row: within each
 *    256-column tile tc, a seeded bijection sigma_tc of [0, 256) lists the
 *    columns, and bucket b' in [0, 16) of the tile holds the 16 columns
 *    sigma_tc(16 b' + k), k = 0..15 (every bucket exactly 16 members);
 *    global bucket b = 16 tc + b', K/16 buckets per row;
 *  - sigma_tc: z = SplitMix64 output tc + 1 of the seed, A = (z & 255) | 1,
 *    B = (z >> 8) & 255, C = ((z >> 16) & 255) | 1; for u in [0, 256):
 *    v1 = (A u + B) mod 256, v2 = v1 xor (v1 >> 4), v3 = (C v2) mod 256,
 *    sigma(u) = v3 xor (v3 >> 3) -- each step is a bijection of 8-bit values;
 *  - S[i][b] = the signed value of row i's member of bucket b with the smallest
 *    |w| (the MIN reduction), ties to the smallest column; no importance;
 *  - scale and codes as format 2 (binary16 of max|v|/127 per 64-row block,
 *    codes toward zero); storage row-major: codes[i * K/16 + b];
 *  - decode: w_hat[i][j] = code[i][bucket of column j] * s. */

/* sigma_tc(u) of tile column tc. */
int orc_cs_sigma(uint64_t seed, int64_t tc, int u) {
  uint64_t z = orc_splitmix64(seed, (uint64_t)tc + 1);
  unsigned A = (unsigned)(z & 255u) | 1u, B = (unsigned)((z >> 8) & 255u), C = (unsigned)((z >> 16) & 255u) | 1u;
  unsigned v1 = (A * (unsigned)u + B) & 255u;
  unsigned v2 = v1 ^ (v1 >> 4);
  unsigned v3 = (C * v2) & 255u;
  return (int)(v3 ^ (v3 >> 3));
}

/* Bucket (global, in [0, K/16)) of column j: the position of j's in-tile
 * column in sigma's list, divided by 16 (found by searching the list). */
int64_t orc_cs_bucket(int64_t K, uint64_t seed, int64_t j) {
  int64_t tc = j / TILE_COLS, c = j % TILE_COLS;
  (void)K;
  for (int u = 0; u < TILE_COLS; ++u)
    if (orc_cs_sigma(seed, tc, u) == c) return tc * (TILE_COLS / WEIGHTS_PER_BUCKET) + u / WEIGHTS_PER_BUCKET;
  return -1; /* not reached: sigma is a bijection */
}

int orc_cs_build(const void* W, int dtype, int64_t M, int64_t K, int64_t ldw, uint64_t seed,
                 int8_t* codes, uint16_t* scales, int64_t* winner, float* value) {
  int st = check_shape(M, K);
  if (st) return st;
  if (dtype != 0 && dtype != 1) return ORC_ERR_DTYPE;
  if (M == 0) return ORC_OK;
  if (!codes || !scales) return ORC_ERR_NULL;
  if (K == 0) {
    for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) scales[rb] = 0;
    return ORC_OK;
  }
  if (!W || ldw < K) return ORC_ERR_NULL;
  int64_t nb = K / WEIGHTS_PER_BUCKET;  /* buckets per row */
  int64_t* bucket_of = (int64_t*)malloc(sizeof(int64_t) * (size_t)K);
  float* val = (float*)malloc(sizeof(float) * (size_t)(ROWS_PER_BLOCK * nb));
  int64_t* idx = (int64_t*)malloc(sizeof(int64_t) * (size_t)(ROWS_PER_BLOCK * nb));
  if (!bucket_of || !val || !idx) { free(bucket_of); free(val); free(idx); return ORC_ERR_NULL; }
  for (int64_t j = 0; j < K; ++j) bucket_of[j] = orc_cs_bucket(K, seed, j);
  int status = ORC_OK;
  for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) {
    float mx = 0.0f;
    for (int64_t r = 0; r < ROWS_PER_BLOCK; ++r) {
      int64_t i = rb * ROWS_PER_BLOCK + r;
      float* vr = val + r * nb;
      int64_t* ir = idx + r * nb;
      for (int64_t b = 0; b < nb; ++b) ir[b] = -1;
      /* scan the row in column order: the first member of smallest |w| stays */
      for (int64_t j = 0; j < K; ++j) {
        float w = load_elem(W, dtype, i * ldw + j);
        if (!isfinite(w)) status = ORC_ERR_NONFINITE;
        int64_t b = bucket_of[j];
        if (ir[b] < 0 || fabsf(w) < fabsf(vr[b])) { vr[b] = w; ir[b] = j; }
      }
      for (int64_t b = 0; b < nb; ++b)
        if (fabsf(vr[b]) > mx) mx = fabsf(vr[b]);
    }
    uint16_t s16 = orc_f32_to_f16(mx / 127.0f);
    if ((s16 & 0x7c00u) == 0x7c00u) status = status ? status : ORC_ERR_SCALE_OVERFLOW;
    scales[rb] = s16;
    double s = (double)orc_f16_to_f32(s16);
    for (int64_t r = 0; r < ROWS_PER_BLOCK; ++r) {
      int64_t i = rb * ROWS_PER_BLOCK + r;
      for (int64_t b = 0; b < nb; ++b) {
        float v = val[r * nb + b];
        int code = 0;
        if (s != 0.0 && isfinite(s) && isfinite(v)) {
          code = floor_code(fabs((double)v), s);
          if (v < 0.0f) code = -code;
        }
        codes[i * nb + b] = (int8_t)code;
        if (winner) winner[i * nb + b] = i * K + idx[r * nb + b];
        if (value) value[i * nb + b] = v;
      }
    }
  }
  free(bucket_of); free(val); free(idx);
  return status;
}

/* W_hat [M, K] of a format-3 sketch. */
int orc_cs_decode(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                  float* What) {
  int st = check_shape(M, K);
  if (st) return st;
  if (M == 0 || K == 0) return ORC_OK;
  if (!codes || !scales || !What) return ORC_ERR_NULL;
  int64_t nb = K / WEIGHTS_PER_BUCKET;
  for (int64_t j = 0; j < K; ++j) {
    int64_t b = orc_cs_bucket(K, seed, j);
    for (int64_t i = 0; i < M; ++i)
      What[i * K + j] = (float)codes[i * nb + b] * orc_f16_to_f32(scales[i / ROWS_PER_BLOCK]);
  }
  return ORC_OK;
}

/* Reference product of a format-3 sketch in float64, from the definition
 * y[t][i] = sum_j w_hat[i][j] x[t][j] (arguments as orc_gemv_f64). */
int orc_cs_gemv_f64(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                    const void* x, int xdtype, int64_t batch, const int64_t* rows, int64_t nrows, double* y) {
  int st = check_shape(M, K);
  if (st) return st;
  if (xdtype != 0 && xdtype != 1) return ORC_ERR_DTYPE;
  if (batch < 0) return ORC_ERR_SHAPE;
  int64_t nr = rows ? nrows : M;
  if (nr == 0 || batch == 0) return ORC_OK;
  if (!y) return ORC_ERR_NULL;
  if (K == 0) {
    for (int64_t q = 0; q < batch * nr; ++q) y[q] = 0.0;
    return ORC_OK;
  }
  if (!codes || !scales || !x) return ORC_ERR_NULL;
  int64_t nb = K / WEIGHTS_PER_BUCKET;
  int64_t* bucket_of = (int64_t*)malloc(sizeof(int64_t) * (size_t)K);
  if (!bucket_of) return ORC_ERR_NULL;
  for (int64_t j = 0; j < K; ++j) bucket_of[j] = orc_cs_bucket(K, seed, j);
  for (int64_t q = 0; q < nr; ++q) {
    int64_t i = rows ? rows[q] : q;
    if (i < 0 || i >= M) { free(bucket_of); return ORC_ERR_SHAPE; }
    float s = orc_f16_to_f32(scales[i / ROWS_PER_BLOCK]);
    for (int64_t t = 0; t < batch; ++t) {
      double acc = 0.0;
      for (int64_t j = 0; j < K; ++j)
        acc += (double)((float)codes[i * nb + bucket_of[j]] * s) * (double)load_elem(x, xdtype, t * K + j);
      y[t * nr + q] = acc;
    }
  }
  free(bucket_of);
  return ORC_OK;
}

/* ================================================================ format 4
 *
 * The format-1 sketch with 4-bit codes ("UltraSketchLLM" explainer, Resultados
 * Experimentales: 0.5 bit/weight with 4-bit quantisation): a bucket holds 8
 * weights instead of 16, so a 64 x 256 tile owns 2048 buckets and a code is a
 * signed 4-bit integer; storage stays M*K/16 bytes.  Readings:
 *  - hash as format 1 with 8 slots: slot = floor(8h / 2^32), class = (o + r) mod
 *    32, bucket b = (slot*32 + class)*8 + c mod 8 in [0, 2048);
 *  - selection as format 1 (largest fp32(|w|) * importance, ties to the
 *    smallest row-major index, empty bucket 0);
 *  - scale s16 = binary16(max |v| / 7); code = clamp(round_half_even(v / s), -7, 7);
 *  - storage: bucket b of tile (rb, tc) is nibble b mod 2 (0 = low) of byte
 *    rb*4K + 1024*tc + b/2; a nibble is two's complement. */

/* Bucket of weight (i, j) within its 64-row block: 2048 tc + b, in [0, 8K). */
int64_t orc_q4_bucket(int64_t K, uint64_t seed, int64_t i, int64_t j) {
  int64_t rb = i / ROWS_PER_BLOCK, r = i % ROWS_PER_BLOCK;
  int64_t tc = j / TILE_COLS, c = j % TILE_COLS;
  int64_t o = c / OCTET, sub = c % OCTET;
  uint32_t A, C;
  orc_tile_hash_params(seed, (uint64_t)(rb * tiles_per_row(K) + tc), &A, &C);
  uint32_t h = A * (uint32_t)(r * (TILE_COLS / OCTET) + o) + C;
  int64_t slot = (int64_t)(((uint64_t)h * 8u) >> 32);
  int64_t cls = (o + r) % CLASSES;
  return 2048 * tc + (slot * CLASSES + cls) * OCTET + sub;
}

/* Signed value of the 4-bit code of block bucket q (row block rb). */
static int q4_code(const int8_t* codes, int64_t K, int64_t rb, int64_t q) {
  uint8_t byte = (uint8_t)codes[rb * 4 * K + q / 2];
  int nib = (q % 2) ? (byte >> 4) : (byte & 15);
  return nib >= 8 ? nib - 16 : nib;
}

int orc_q4_build_rows(const void* W, int dtype, int64_t M, int64_t K, int64_t ldw, const float* imp,
                      uint64_t seed, int64_t rb0, int8_t* codes, uint16_t* scales, int64_t* winner,
                      float* value) {
  int st = check_shape(M, K);
  if (st) return st;
  if (rb0 < 0) return ORC_ERR_SHAPE;
  if (dtype != 0 && dtype != 1) return ORC_ERR_DTYPE;
  if (M == 0) return ORC_OK;
  if (!codes || !scales) return ORC_ERR_NULL;
  if (K == 0) {
    for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) scales[rb] = 0;
    return ORC_OK;
  }
  if (!W || ldw < K) return ORC_ERR_NULL;
  if (imp) {
    for (int64_t j = 0; j < K; ++j) {
      uint32_t u = bits_from_f32(imp[j]);
      if ((u >> 31) || !isfinite(imp[j])) return ORC_ERR_IMPORTANCE;
    }
  }
  int64_t per_block = 8 * K;  /* buckets per 64-row block */
  float* bestkey = (float*)malloc(sizeof(float) * (size_t)per_block);
  int64_t* bestidx = (int64_t*)malloc(sizeof(int64_t) * (size_t)per_block);
  float* val = (float*)malloc(sizeof(float) * (size_t)per_block);
  if (!bestkey || !bestidx || !val) { free(bestkey); free(bestidx); free(val); return ORC_ERR_NULL; }
  int status = ORC_OK;
  for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) {
    for (int64_t b = 0; b < per_block; ++b) { bestkey[b] = -1.0f; bestidx[b] = -1; }
    for (int64_t r = 0; r < ROWS_PER_BLOCK; ++r) {
      int64_t i = rb * ROWS_PER_BLOCK + r;
      for (int64_t j = 0; j < K; ++j) {
        float w = load_elem(W, dtype, i * ldw + j);
        if (!isfinite(w)) status = ORC_ERR_NONFINITE;
        float k = fabsf(w) * (imp ? imp[j] : 1.0f);
        int64_t b = orc_q4_bucket(K, seed, i + rb0 * ROWS_PER_BLOCK, j);
        if (k > bestkey[b] || bestidx[b] < 0) { bestkey[b] = k; bestidx[b] = i * K + j; }
      }
    }
    float mx = 0.0f;
    for (int64_t b = 0; b < per_block; ++b) {
      float v = 0.0f;
      if (bestidx[b] >= 0) v = load_elem(W, dtype, (bestidx[b] / K) * ldw + bestidx[b] % K);
      val[b] = v;
      if (fabsf(v) > mx) mx = fabsf(v);
    }
    uint16_t s16 = orc_f32_to_f16(mx / 7.0f);
    if ((s16 & 0x7c00u) == 0x7c00u) status = status ? status : ORC_ERR_SCALE_OVERFLOW;
    scales[rb] = s16;
    float s = orc_f16_to_f32(s16);
    for (int64_t q = 0; q < 4 * K; ++q) codes[rb * 4 * K + q] = 0;
    for (int64_t b = 0; b < per_block; ++b) {
      int code = 0;
      if (s != 0.0f) {
        float qv = nearbyintf(val[b] / s);
        if (qv > 7.0f) qv = 7.0f;
        if (qv < -7.0f) qv = -7.0f;
        code = isnan(qv) ? 0 : (int)qv;
      }
      uint8_t* byte = (uint8_t*)&codes[rb * 4 * K + b / 2];
      *byte = (uint8_t)(*byte | (((unsigned)code & 15u) << (4 * (b % 2))));
      if (winner) winner[rb * per_block + b] = bestidx[b];
      if (value) value[rb * per_block + b] = val[b];
    }
  }
  free(bestkey); free(bestidx); free(val);
  return status;
}

int orc_q4_decode(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                  float* What) {
  int st = check_shape(M, K);
  if (st) return st;
  if (M == 0 || K == 0) return ORC_OK;
  if (!codes || !scales || !What) return ORC_ERR_NULL;
  for (int64_t i = 0; i < M; ++i) {
    int64_t rb = i / ROWS_PER_BLOCK;
    float s = orc_f16_to_f32(scales[rb]);
    for (int64_t j = 0; j < K; ++j)
      What[i * K + j] = (float)q4_code(codes, K, rb, orc_q4_bucket(K, seed, i, j)) * s;
  }
  return ORC_OK;
}

int orc_q4_gemv_f64(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                    const void* x, int xdtype, int64_t batch, const int64_t* rows, int64_t nrows, double* y) {
  int st = check_shape(M, K);
  if (st) return st;
  if (xdtype != 0 && xdtype != 1) return ORC_ERR_DTYPE;
  if (batch < 0) return ORC_ERR_SHAPE;
  int64_t nr = rows ? nrows : M;
  if (nr == 0 || batch == 0) return ORC_OK;
  if (!y) return ORC_ERR_NULL;
  if (K == 0) {
    for (int64_t q = 0; q < batch * nr; ++q) y[q] = 0.0;
    return ORC_OK;
  }
  if (!codes || !scales || !x) return ORC_ERR_NULL;
  double* wrow = (double*)malloc(sizeof(double) * (size_t)K);
  if (!wrow) return ORC_ERR_NULL;
  for (int64_t q = 0; q < nr; ++q) {
    int64_t i = rows ? rows[q] : q;
    if (i < 0 || i >= M) { free(wrow); return ORC_ERR_SHAPE; }
    int64_t rb = i / ROWS_PER_BLOCK;
    float s = orc_f16_to_f32(scales[rb]);
    for (int64_t j = 0; j < K; ++j)
      wrow[j] = (double)((float)q4_code(codes, K, rb, orc_q4_bucket(K, seed, i, j)) * s);
    for (int64_t t = 0; t < batch; ++t) {
      double acc = 0.0;
      for (int64_t j = 0; j < K; ++j) acc += wrow[j] * (double)load_elem(x, xdtype, t * K + j);
      y[t * nr + q] = acc;
    }
  }
  free(wrow);
  return ORC_OK;
}

/* ================================================================ rates
 *
 * Importance-aware space allocation ("UltraSketchLLM" explainer, Resumen
 * Tecnico, Metodologia §2: rows or layers of higher importance E[a^2] receive
 * larger sketch spaces, more buckets).  Reading: the space is chosen per sketch
 * (a layer); format 1 takes S = 2, 4 or 8 hash slots per class, i.e. 512, 1024
 * or 2048 buckets per 64 x 256 tile (32, 16 or 8 weights per bucket; 0.25, 0.5
 * or 1 bit/weight with 8-bit codes).  S = 4 is format 1 exactly.
 *  - slot = floor(S h / 2^32); bucket b = (slot*32 + class)*8 + c mod 8;
 *  - storage: codes[rb*S*K + 256*S*tc + b];
 *  - selection, scale (max|v| / 127) and codes as format 1. */

int64_t orc_rate_bucket(int64_t K, uint64_t seed, int slots, int64_t i, int64_t j) {
  int64_t rb = i / ROWS_PER_BLOCK, r = i % ROWS_PER_BLOCK;
  int64_t tc = j / TILE_COLS, c = j % TILE_COLS;
  int64_t o = c / OCTET, sub = c % OCTET;
  uint32_t A, C;
  orc_tile_hash_params(seed, (uint64_t)(rb * tiles_per_row(K) + tc), &A, &C);
  uint32_t h = A * (uint32_t)(r * (TILE_COLS / OCTET) + o) + C;
  int64_t slot = (int64_t)(((uint64_t)h * (uint64_t)slots) >> 32);
  int64_t b = (slot * CLASSES + (o + r) % CLASSES) * OCTET + sub;
  return rb * slots * K + 256 * slots * tc + b;
}

/* Selection, scale and codes of row block rb at `slots` slots per class: the
 * block's slots*K codes go to out[0 .. slots*K), its scale to *scale16.  The
 * caller has checked the shape, the dtype and the importance. */
static int rate_build_block(const void* W, int dtype, int64_t K, int64_t ldw, const float* imp, uint64_t seed,
                            int slots, int64_t rb, float* bestkey, int64_t* bestidx, int8_t* out,
                            uint16_t* scale16) {
  int status = ORC_OK;
  int64_t per_block = slots * K;
  for (int64_t b = 0; b < per_block; ++b) { bestkey[b] = -1.0f; bestidx[b] = -1; }
  for (int64_t r = 0; r < ROWS_PER_BLOCK; ++r) {
    int64_t i = rb * ROWS_PER_BLOCK + r;
    for (int64_t j = 0; j < K; ++j) {
      float w = load_elem(W, dtype, i * ldw + j);
      if (!isfinite(w)) status = ORC_ERR_NONFINITE;
      float k = fabsf(w) * (imp ? imp[j] : 1.0f);
      int64_t b = orc_rate_bucket(K, seed, slots, i, j) - rb * per_block;
      if (k > bestkey[b] || bestidx[b] < 0) { bestkey[b] = k; bestidx[b] = i * K + j; }
    }
  }
  float mx = 0.0f;
  for (int64_t b = 0; b < per_block; ++b) {
    float v = bestidx[b] >= 0 ? load_elem(W, dtype, (bestidx[b] / K) * ldw + bestidx[b] % K) : 0.0f;
    bestkey[b] = v;  /* reuse as the kept value */
    if (fabsf(v) > mx) mx = fabsf(v);
  }
  uint16_t s16 = orc_f32_to_f16(mx / 127.0f);
  if ((s16 & 0x7c00u) == 0x7c00u) status = status ? status : ORC_ERR_SCALE_OVERFLOW;
  *scale16 = s16;
  float s = orc_f16_to_f32(s16);
  for (int64_t b = 0; b < per_block; ++b) {
    int code = 0;
    if (s != 0.0f) {
      float q = nearbyintf(bestkey[b] / s);
      if (q > 127.0f) q = 127.0f;
      if (q < -127.0f) q = -127.0f;
      code = isnan(q) ? 0 : (int)q;
    }
    out[b] = (int8_t)code;
  }
  return status;
}

/* Argument checks shared by the rate builds; ORC_OK when the build may go on. */
static int rate_check_imp(int64_t K, const float* imp) {
  if (imp) {
    for (int64_t j = 0; j < K; ++j) {
      uint32_t u = bits_from_f32(imp[j]);
      if ((u >> 31) || !isfinite(imp[j])) return ORC_ERR_IMPORTANCE;
    }
  }
  return ORC_OK;
}

int orc_rate_build(const void* W, int dtype, int64_t M, int64_t K, int64_t ldw, const float* imp,
                   uint64_t seed, int slots, int8_t* codes, uint16_t* scales) {
  int st = check_shape(M, K);
  if (st) return st;
  if (dtype != 0 && dtype != 1) return ORC_ERR_DTYPE;
  if (slots != 2 && slots != 4 && slots != 8) return ORC_ERR_SHAPE;
  if (M == 0) return ORC_OK;
  if (!codes || !scales) return ORC_ERR_NULL;
  if (K == 0) {
    for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) scales[rb] = 0;
    return ORC_OK;
  }
  if (!W || ldw < K) return ORC_ERR_NULL;
  st = rate_check_imp(K, imp);
  if (st) return st;
  int64_t per_block = slots * K;
  float* bestkey = (float*)malloc(sizeof(float) * (size_t)per_block);
  int64_t* bestidx = (int64_t*)malloc(sizeof(int64_t) * (size_t)per_block);
  if (!bestkey || !bestidx) { free(bestkey); free(bestidx); return ORC_ERR_NULL; }
  int status = ORC_OK;
  for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) {
    int bs = rate_build_block(W, dtype, K, ldw, imp, seed, slots, rb, bestkey, bestidx, codes + rb * per_block,
                              &scales[rb]);
    if (bs == ORC_ERR_NONFINITE || (bs && !status)) status = bs;
  }
  free(bestkey); free(bestidx);
  return status;
}

int orc_rate_gemv_f64(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed, int slots,
                      const void* x, int xdtype, int64_t batch, const int64_t* rows, int64_t nrows, double* y) {
  int st = check_shape(M, K);
  if (st) return st;
  if (slots != 2 && slots != 4 && slots != 8) return ORC_ERR_SHAPE;
  if (xdtype != 0 && xdtype != 1) return ORC_ERR_DTYPE;
  int64_t nr = rows ? nrows : M;
  if (nr == 0 || batch <= 0) return ORC_OK;
  if (!y) return ORC_ERR_NULL;
  if (K == 0) {
    for (int64_t q = 0; q < batch * nr; ++q) y[q] = 0.0;
    return ORC_OK;
  }
  if (!codes || !scales || !x) return ORC_ERR_NULL;
  double* wrow = (double*)malloc(sizeof(double) * (size_t)K);
  if (!wrow) return ORC_ERR_NULL;
  for (int64_t q = 0; q < nr; ++q) {
    int64_t i = rows ? rows[q] : q;
    if (i < 0 || i >= M) { free(wrow); return ORC_ERR_SHAPE; }
    float s = orc_f16_to_f32(scales[i / ROWS_PER_BLOCK]);
    for (int64_t j = 0; j < K; ++j) wrow[j] = (double)((float)codes[orc_rate_bucket(K, seed, slots, i, j)] * s);
    for (int64_t t = 0; t < batch; ++t) {
      double acc = 0.0;
      for (int64_t j = 0; j < K; ++j) acc += wrow[j] * (double)load_elem(x, xdtype, t * K + j);
      y[t * nr + q] = acc;
    }
  }
  free(wrow);
  return ORC_OK;
}

/* ================================================================ per-row-block rates
 *
 * Importance-aware space allocation at row-block granularity (Metodologia §2:
 * rows of higher importance E[a^2] receive larger sketch spaces).  Reading:
 * each 64-row block rb carries its own slot count S_rb in {2, 4, 8}; its codes
 * are the S_rb-slot format-1 codes of that block (same hash tile ids rb*T + tc),
 * stored at byte offset off_rb = K * (S_0 + ... + S_{rb-1}) -- the row blocks in
 * matrix order, each block's slots*K codes contiguous.  Total code bytes
 * K * sum(S_rb). */

/* off[rb] for every row block; returns the total code bytes, -1 on a bad slot count. */
int64_t orc_vr_offsets(int64_t M, int64_t K, const uint32_t* slots, int64_t* off) {
  int64_t acc = 0;
  for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) {
    if (slots[rb] != 2 && slots[rb] != 4 && slots[rb] != 8) return -1;
    if (off) off[rb] = acc;
    acc += (int64_t)slots[rb] * K;
  }
  return acc;
}

int64_t orc_vr_bucket(int64_t K, uint64_t seed, const uint32_t* slots, int64_t i, int64_t j) {
  int64_t rb = i / ROWS_PER_BLOCK, off = 0;
  for (int64_t q = 0; q < rb; ++q) off += (int64_t)slots[q] * K;
  int S = (int)slots[rb];
  return off + (orc_rate_bucket(K, seed, S, i, j) - rb * S * K);
}

int orc_vr_build(const void* W, int dtype, int64_t M, int64_t K, int64_t ldw, const float* imp, uint64_t seed,
                 const uint32_t* slots, int8_t* codes, uint16_t* scales) {
  int st = check_shape(M, K);
  if (st) return st;
  if (dtype != 0 && dtype != 1) return ORC_ERR_DTYPE;
  if (M == 0) return ORC_OK;
  if (!slots || !codes || !scales) return ORC_ERR_NULL;
  if (orc_vr_offsets(M, K, slots, NULL) < 0) return ORC_ERR_SHAPE;
  if (K == 0) {
    for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) scales[rb] = 0;
    return ORC_OK;
  }
  if (!W || ldw < K) return ORC_ERR_NULL;
  st = rate_check_imp(K, imp);
  if (st) return st;
  float* bestkey = (float*)malloc(sizeof(float) * (size_t)(8 * K));
  int64_t* bestidx = (int64_t*)malloc(sizeof(int64_t) * (size_t)(8 * K));
  if (!bestkey || !bestidx) { free(bestkey); free(bestidx); return ORC_ERR_NULL; }
  int status = ORC_OK;
  int64_t off = 0;
  for (int64_t rb = 0; rb < M / ROWS_PER_BLOCK; ++rb) {
    int S = (int)slots[rb];
    int bs = rate_build_block(W, dtype, K, ldw, imp, seed, S, rb, bestkey, bestidx, codes + off, &scales[rb]);
    if (bs == ORC_ERR_NONFINITE || (bs && !status)) status = bs;
    off += (int64_t)S * K;
  }
  free(bestkey); free(bestidx);
  return status;
}

int orc_vr_gemv_f64(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                    const uint32_t* slots, const void* x, int xdtype, int64_t batch, const int64_t* rows,
                    int64_t nrows, double* y) {
  int st = check_shape(M, K);
  if (st) return st;
  if (xdtype != 0 && xdtype != 1) return ORC_ERR_DTYPE;
  int64_t nr = rows ? nrows : M;
  if (nr == 0 || batch <= 0) return ORC_OK;
  if (!y || !slots) return ORC_ERR_NULL;
  if (orc_vr_offsets(M, K, slots, NULL) < 0) return ORC_ERR_SHAPE;
  if (K == 0) {
    for (int64_t q = 0; q < batch * nr; ++q) y[q] = 0.0;
    return ORC_OK;
  }
  if (!codes || !scales || !x) return ORC_ERR_NULL;
  double* wrow = (double*)malloc(sizeof(double) * (size_t)K);
  if (!wrow) return ORC_ERR_NULL;
  for (int64_t q = 0; q < nr; ++q) {
    int64_t i = rows ? rows[q] : q;
    if (i < 0 || i >= M) { free(wrow); return ORC_ERR_SHAPE; }
    float s = orc_f16_to_f32(scales[i / ROWS_PER_BLOCK]);
    for (int64_t j = 0; j < K; ++j) wrow[j] = (double)((float)codes[orc_vr_bucket(K, seed, slots, i, j)] * s);
    for (int64_t t = 0; t < batch; ++t) {
      double acc = 0.0;
      for (int64_t j = 0; j < K; ++j) acc += wrow[j] * (double)load_elem(x, xdtype, t * K + j);
      y[t * nr + q] = acc;
    }
  }
  free(wrow);
  return ORC_OK;
}

/* ------------------------------------------------- all-core baseline mode */

/* The same format-1 build and float64 product, spread over `nthreads` host
 * threads (OpenMP; 0 = all the runtime offers) for the CPU baseline and for
 * whole-model checks.  Nothing is recomputed differently: row blocks are
 * independent in the method (a bucket's members all lie in one 64-row block,
 * Metodologia §1 of the explainer, and the scale is per block), so each run of
 * row blocks is handed, unchanged, to the sequential orc_build_rows /
 * orc_gemv_f64 above.  The result is therefore identical to the single-thread
 * call; the status is the one the sequential scan would return (a non-finite
 * weight anywhere wins over a scale overflow).  Compiled without OpenMP the
 * loops simply run on one thread. */
#ifdef _OPENMP
#include <omp.h>
#endif

int orc_threads(int nthreads) {
#ifdef _OPENMP
  return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
  (void)nthreads;
  return 1;
#endif
}

int orc_build_mt(const void* W, int dtype, int64_t M, int64_t K, int64_t ldw,
                 const float* imp, uint64_t seed, int8_t* codes, uint16_t* scales,
                 int nthreads) {
  int st = check_shape(M, K);
  if (st) return st;
  if (dtype != 0 && dtype != 1) return ORC_ERR_DTYPE;
  if (M == 0 || K == 0) return orc_build_rows(W, dtype, M, K, ldw, imp, seed, 0, codes, scales, NULL, NULL);
  if (!W || !codes || !scales || ldw < K) return ORC_ERR_NULL;
  const int64_t RB = M / ROWS_PER_BLOCK;
  const size_t esz = dtype == 0 ? 4 : 2;
  int any_nonfinite = 0, any_overflow = 0, any_other = 0;
  int64_t rb;
  (void)nthreads;
#pragma omp parallel for schedule(dynamic, 1) num_threads(orc_threads(nthreads)) \
    reduction(| : any_nonfinite, any_overflow, any_other)
  for (rb = 0; rb < RB; ++rb) {
    const char* wrb = (const char*)W + (size_t)(rb * ROWS_PER_BLOCK) * (size_t)ldw * esz;
    int s = orc_build_rows(wrb, dtype, ROWS_PER_BLOCK, K, ldw, imp, seed, rb, codes + rb * 4 * K, scales + rb,
                           NULL, NULL);
    if (s == ORC_ERR_NONFINITE) any_nonfinite = 1;
    else if (s == ORC_ERR_SCALE_OVERFLOW) any_overflow = 1;
    else if (s != ORC_OK) any_other = s;
  }
  if (any_other) return any_other; /* argument errors: the same for every row block */
  if (any_nonfinite) return ORC_ERR_NONFINITE;
  if (any_overflow) return ORC_ERR_SCALE_OVERFLOW;
  return ORC_OK;
}

/* y [batch, M] = W_hat x^T in float64 over all rows, rows spread over threads in
 * runs of 64; each run is one orc_gemv_f64 call on its row list. */
int orc_gemv_f64_mt(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K,
                    uint64_t seed, const void* x, int xdtype, int64_t batch, double* y,
                    int nthreads) {
  int st = check_shape(M, K);
  if (st) return st;
  if (xdtype != 0 && xdtype != 1) return ORC_ERR_DTYPE;
  if (batch < 0) return ORC_ERR_SHAPE;
  if (M == 0 || batch == 0) return ORC_OK;
  if (!y) return ORC_ERR_NULL;
  const int64_t RB = M / ROWS_PER_BLOCK;
  int err = 0;
  int64_t rb;
  (void)nthreads;
#pragma omp parallel for schedule(dynamic, 1) num_threads(orc_threads(nthreads)) reduction(| : err)
  for (rb = 0; rb < RB; ++rb) {
    int64_t rows[ROWS_PER_BLOCK];
    double part[ROWS_PER_BLOCK * 16];
    for (int64_t r = 0; r < ROWS_PER_BLOCK; ++r) rows[r] = rb * ROWS_PER_BLOCK + r;
    for (int64_t t0 = 0; t0 < batch; t0 += 16) {
      const int64_t nb = batch - t0 < 16 ? batch - t0 : 16;
      const char* xt = (const char*)x + (size_t)(t0 * K) * (size_t)(xdtype == 0 ? 4 : 2);
      int s = orc_gemv_f64(codes, scales, M, K, seed, xt, xdtype, nb, rows, ROWS_PER_BLOCK, part);
      if (s) { err |= s; continue; }
      for (int64_t t = 0; t < nb; ++t)
        for (int64_t r = 0; r < ROWS_PER_BLOCK; ++r) y[(t0 + t) * M + rows[r]] = part[t * ROWS_PER_BLOCK + r];
    }
  }
  return err ? ORC_ERR_NULL : ORC_OK;
}

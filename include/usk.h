/*
 * usk.h -- C ABI of libusk: UltraSketchLLM sketch weights on NVIDIA B200 (sm_100a).
 *
 * The library compresses a weight matrix W [M, K] into a hashed sketch at
 * 0.5 bit per weight (one int8 code per 16 weights plus one binary16 scale per
 * 64-row block) and multiplies the sketch with activations without ever
 * materialising the decompressed matrix.
 *
 * Source of the method: "UltraSketchLLM: Sub-1-Bit LLM Compression via Sketch
 * and Hardware-Friendly Operators" (explainer pages gist.science/es|nl/paper/
 * 2506.17255), Resumen Tecnico:
 *   - Metodologia §1 "Diseno de Sketch AbsMaxMin": weights are hashed into a
 *     smaller shared bucket state and a bucket keeps a single value chosen by
 *     magnitude (the lay section §2 "El Sketch": it keeps its largest member);
 *   - Metodologia §2 "Asignacion consciente de la importancia": importance
 *     decides what is preserved (here: it weights the selection key);
 *   - Metodologia §4 "Mapeo de Operadores de Matriz": compression is one fused
 *     select-and-update kernel; decompression is W_hat = S . P^T, i.e. each
 *     weight reads its bucket back;
 *   - Resultados Experimentales "Eficiencia de Compresion": 0.5 bit/weight.
 *
 * FORMAT (version 1).  The pages fix none of the following; this is the
 * library's frozen reading.
 *   Geometry: M % 64 == 0, K % 256 == 0.  Row block rb = rows [64 rb, 64 rb+64)
 *   carries one binary16 scale.  Hash tile (rb, tc) = that row block x columns
 *   [256 tc, 256 tc + 256); it owns 1024 buckets.
 *   Hash of weight (i, j): r = i % 64, c = j % 256, octet o = c / 8,
 *     z = SplitMix64 output number tile_id + 1 of `seed`, tile_id = rb*(K/256)+tc,
 *     A = low32(z) | 1, C = high32(z), h = A*(32 r + o) + C  (mod 2^32),
 *     slot = h >> 30, class = (o + r) mod 32,
 *     bucket b = (slot*32 + class)*8 + c % 8   in [0, 1024).
 *   Code storage: codes[rb*4K + 1024*tc + b] (int8), scales[rb] (binary16).
 *   Selection: key = fp32(|w|) * importance[j] (one fp32 multiply, RN); each
 *   bucket keeps the signed value v of its member with the largest key, ties to
 *   the smallest row-major index; an empty bucket keeps 0.
 *   Scale: s16 = binary16_rn(max_b |v_b| / 127) over the row block.
 *   Code: clamp(rint_half_even(v / float(s16)), -127, 127); 0 when s16 == 0.
 *   Decode: w_hat = float(code) * float(s16) (exact in fp32).
 *
 * FORMAT 2 (multi-row AbsMaxMin; Metodologia §1: the sketch state keeps the
 * member of SMALLEST absolute value per bucket, several independently hashed
 * sketch rows are kept, decompression takes the MAX, so every rebuilt weight
 * is the original or one of smaller magnitude).  Same geometry, scales and
 * storage size as format 1 (0.5 bit/weight); depth D in {1, 2, 4}:
 *   Hash row rho in [0, D) of tile tile_id: z = SplitMix64 output number
 *     tile_id*D + rho + 1, A, C, h and slot as above, class = (o + r) mod (32/D),
 *     b = rho*(1024/D) + (slot*(32/D) + class)*8 + c % 8   (D = 1: the format-1 hash).
 *   Selection: every weight updates its bucket in each hash row; a bucket keeps
 *   the signed value of its member with the smallest |w|, ties to the smallest
 *   row-major index; an empty bucket keeps 0.  No importance weighting.
 *   Code: sign(v) * min(127, floor(|v| / float(s16))) (toward zero, so
 *   |code * s16| <= |v|); 0 when s16 == 0.
 *   Decode: w_hat = float(c) * float(s16), c = the code of largest magnitude
 *   among the weight's D buckets, ties to the lowest row.  |w_hat| <= |w|.
 *
 * FORMAT 3 (column-shared projection; Metodologia §4: compression is a matrix
 * product with a projection P whose reduction is a MIN over |w|, decompression
 * the plain product W_hat = S . P^T).  P is one-hot per input column and shared
 * by all rows; same geometry, scales and storage size (0.5 bit/weight):
 *   Column list of tile tc: z = SplitMix64 output number tc + 1 of `seed`,
 *     A = (z & 255) | 1, B = (z >> 8) & 255, C = ((z >> 16) & 255) | 1,
 *     sigma(u) = v3 ^ (v3 >> 3), v3 = (C * v2) mod 256, v2 = v1 ^ (v1 >> 4),
 *     v1 = (A u + B) mod 256, for u in [0, 256) (a bijection).
 *   Bucket b' in [0, 16) of the tile holds columns 256 tc + sigma(16 b' + k),
 *   k = 0..15; global bucket b = 16 tc + b'.
 *   Selection: per row and bucket the member with the smallest |w|, ties to the
 *   smallest column; no importance.  Scale and codes as format 2.
 *   Code storage: row-major, codes[i * K/16 + b].
 *   Decode: w_hat[i][j] = float(codes[i][bucket of j]) * float(s16); the product
 *   is computed as y = S (P^T x): bucket sums of x, then a dense code product.
 *   usk_gemm does not take format 3 (USK_ERR_PARAMS); usk_gemv covers batch 1..15.
 *
 * RATES (Metodologia §2, importance-aware space): format 1 takes slots = 2, 4
 *   (default) or 8 hash slots per class -- slot = floor(slots * h / 2^32),
 *   256 * slots buckets per tile (32, 16 or 8 weights per bucket; 0.25, 0.5 or
 *   1 bit/weight), codes[(rb * K/256 + tc) * 256 * slots + b]; everything else
 *   as format 1.  usk_plan_slots chooses slot counts per layer from importance.
 *
 * PER-ROW-BLOCK RATES (Metodologia §2 at row granularity: rows of higher
 *   importance get larger spaces): a format-1 sketch whose 64-row block rb has
 *   its own slot count S_rb in {2, 4, 8}.  Block rb's codes are exactly those
 *   of row block rb of the uniform S_rb sketch (same hash tiles rb*K/256 + tc),
 *   stored from byte off_rb = K * (S_0 + ... + S_{rb-1}) on: codes[off_rb +
 *   256*S_rb*tc + b].  Total code bytes K * sum(S_rb).  The per-block table
 *   lives in a usk_rate_map (usk_rate_map_plan fills it from the slot counts).
 *
 * FORMAT 4 (format 1 with 4-bit codes; Resultados: 0.5 bit/weight with 4-bit
 * quantisation): 8 weights per bucket, 2048 buckets per tile, same storage size.
 *   Hash as format 1 with 8 slots: slot = h >> 29, b = (slot*32 + class)*8 + c % 8.
 *   Selection as format 1 (importance allowed).  Scale s16 = binary16_rn(max|v| / 7);
 *   code = clamp(rint_half_even(v / float(s16)), -7, 7), two's complement nibble.
 *   Storage: bucket b of tile (rb, tc) is nibble b % 2 (0 = low) of byte
 *   codes[rb*4K + 1024*tc + b/2].
 *
 * CONVENTIONS
 *   - All array pointers are DEVICE pointers owned by the caller; the library
 *     allocates no memory and keeps no state beyond cached kernel attributes.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and reentrant.
 *   - Argument errors are returned synchronously and nothing is launched.
 *     A failed launch returns USK_ERR_CUDA.
 *   - Conditions found on the device (non-finite weights, bad importance, scale
 *     overflow, a wait that gave up) are OR-ed as USK_FLAG_* bits into
 *     *d_status when d_status is not NULL; the caller reads it after a sync.
 *     The library never clears it.
 */
#ifndef USK_H_
#define USK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define USK_API __attribute__((visibility("default")))
#else
#define USK_API
#endif

#define USK_FORMAT_MAXKEY 1     /* format 1: one hash row, largest key kept   */
#define USK_FORMAT_ABSMAXMIN 2  /* format 2: multi-row AbsMaxMin              */
#define USK_FORMAT_COLSHARED 3  /* format 3: column-shared projection, W_hat = S . P^T */
#define USK_FORMAT_Q4 4         /* format 4: format 1 with 4-bit codes, 8 weights per bucket */
#define USK_FORMAT_VERSION 4    /* highest format this library builds and reads */
#define USK_ROWS_PER_BLOCK 64
#define USK_TILE_COLS 256
#define USK_WEIGHTS_PER_BUCKET 16
#define USK_MAX_M (1 << 21)   /* rows */
#define USK_MAX_K (1 << 16)   /* columns */
#define USK_GEMV_MAX_BATCH 15
#define USK_GEMM_MIN_BATCH 16
#define USK_GEMM_MAX_BATCH 256

typedef enum {
  USK_OK = 0,
  USK_ERR_NULL = 1,            /* a required pointer is NULL                     */
  USK_ERR_SHAPE = 2,           /* M % 64, K % 256, negative or above the limits   */
  USK_ERR_DTYPE = 3,           /* unknown usk_dtype                              */
  USK_ERR_BATCH = 4,           /* batch outside the call's range                 */
  USK_ERR_WORKSPACE = 5,       /* workspace missing or too small                 */
  USK_ERR_PARAMS = 6,          /* params NULL, unknown format, bad depth, slots, flags or rate map */
  USK_ERR_CUDA = 7,            /* a CUDA runtime call or a launch failed         */
  USK_ERR_NONFINITE = 8,       /* (flag decoding) non-finite weight              */
  USK_ERR_TIMEOUT = 9,         /* (flag decoding) a bounded device wait gave up  */
  USK_ERR_ALIGN = 10,          /* pointer or stride misaligned (16-byte rule)    */
  USK_ERR_IMPORTANCE = 11,     /* (flag decoding) importance < 0, -0 or non-finite */
  USK_ERR_SCALE_OVERFLOW = 12  /* (flag decoding) max|v|/127 above binary16 range */
} usk_status;

/* Bits OR-ed into *d_status by the device. */
#define USK_FLAG_NONFINITE_W (1u << 0)
#define USK_FLAG_BAD_IMPORTANCE (1u << 1)
#define USK_FLAG_SCALE_OVERFLOW (1u << 2)
#define USK_FLAG_TIMEOUT (1u << 3)
#define USK_FLAG_RATE_MAP (1u << 4) /* a rate-map entry out of range: that row block was skipped */

typedef enum { USK_F32 = 0, USK_BF16 = 1 } usk_dtype;

/* Per-row-block rate table of a format-1 sketch (see PER-ROW-BLOCK RATES).
 * offset and order are DEVICE arrays of M/64 entries owned by the caller:
 *   offset[rb]  byte offset of row block rb's codes (K * slots of the blocks above);
 *   order       the row blocks at 2 slots, then those at 4, then those at 8,
 *               each group in increasing row-block order (the kernels take one
 *               group per launch);
 *   count[g]    host value: row blocks at 2 (g = 0), 4 (g = 1) and 8 (g = 2) slots;
 *   code_bytes  host value: K * sum of the slots (the codes array's size).
 * order must be a permutation of the row blocks grouped by slot count, as
 * usk_rate_map_plan produces.  The library checks the counts against M on the
 * host; on the device an order entry outside [0, M/64), an offset whose block
 * would end past code_bytes, or a block whose extent (offset[rb + 1] -
 * offset[rb], or code_bytes - offset[rb] for the last) is not K times its
 * group's slot count skips that row block (its outputs are not written; the
 * other row block of a usk_gemm tile is still computed) and sets
 * USK_FLAG_RATE_MAP.  A duplicated entry is not detected: the block it
 * replaces is neither built nor multiplied. */
typedef struct {
  const int64_t* offset;
  const int32_t* order;
  int64_t count[3];
  int64_t code_bytes;
} usk_rate_map;

/* Build parameters.  version: USK_FORMAT_MAXKEY, USK_FORMAT_ABSMAXMIN,
 * USK_FORMAT_COLSHARED or USK_FORMAT_Q4; flags must be 0; depth = hash rows: 0
 * or 1 for formats 1, 3 and 4, 1, 2 or 4 for format 2; slots: 0, 2, 4 or 8 for
 * format 1, 0 or 8 for format 4, 0 or 4 otherwise.  Anything else:
 * USK_ERR_PARAMS. */
typedef struct {
  uint32_t version;
  uint32_t flags;
  uint64_t seed;
  uint32_t depth;
  uint32_t slots;  /* hash slots per class; 0 = the format's default (see RATES) */
  const usk_rate_map* rates; /* per-row-block rates (format 1, slots 0, depth <= 1); NULL = uniform */
} usk_params;

/* A built sketch (device pointers, caller-owned).  version / depth as built
 * (version 0 is read as format 1; depth 0 as 1). */
typedef struct {
  int64_t M, K;
  uint64_t seed;
  const int8_t* codes;     /* [M*K/16], 16-byte aligned */
  const uint16_t* scales;  /* [M/64] binary16 bits      */
  uint32_t version;
  uint32_t depth;
  uint32_t slots;          /* as built (0 = the format's default) */
  uint32_t pad;
  const usk_rate_map* rates; /* as built; NULL = one rate for the whole sketch */
} usk_sketch;

/* Storage of a sketch: code_bytes = M*K/16, scale_bytes = 2*M/64.
 * Errors: USK_ERR_SHAPE, USK_ERR_NULL (an output pointer). */
USK_API usk_status usk_sizes(int64_t M, int64_t K, size_t* code_bytes, size_t* scale_bytes);

/* Storage of a sketch of a given format and slot count: code_bytes =
 * M*K*slots/64 for format 1 (M*K/16 for the other formats and the defaults),
 * scale_bytes = 2*M/64.  Errors: USK_ERR_SHAPE, USK_ERR_NULL, USK_ERR_PARAMS. */
USK_API usk_status usk_sizes_ex(int64_t M, int64_t K, uint32_t version, uint32_t slots, size_t* code_bytes,
                                size_t* scale_bytes);

/* Importance-aware space allocation (Metodologia §2 "Asignacion de Espacio
 * Consciente de la Importancia": units of higher importance E[a^2] receive
 * larger sketch spaces).  For n units (e.g. the linear layers of a model) with
 * weights[i] > 0 weights and importance[i] >= 0 (finite), writes slots[i] in
 * {2, 4, 8} (format-1 rates of 0.25, 0.5 and 1 bit/weight) such that
 * sum(weights[i] * slots[i] / 8) <= budget_bits * sum(weights).  Procedure:
 * every unit starts at 2 slots; the steps 2 -> 4 and 4 -> 8 of all units are
 * visited in decreasing importance gained per bit -- with a unit's distortion
 * taken as importance x weights / slots this is importance for 2 -> 4 and
 * importance / 4 for 4 -> 8 -- ties to the 2 -> 4 step, then to the lower index;
 * a step is taken when the unit is at its starting level and the budget holds.
 * budget_bits in [0.25, 1].  Host only (no GPU).  Errors: USK_ERR_NULL,
 * USK_ERR_SHAPE (n < 0), USK_ERR_PARAMS (budget, weights or importance). */
USK_API usk_status usk_plan_slots(int64_t n, const int64_t* weights, const double* importance, double budget_bits,
                                  uint32_t* slots);

/* Rate table of a per-row-block-rate sketch, on the host: from slots[M/64]
 * (each 2, 4 or 8) writes offset[M/64] (byte offsets, matrix order),
 * order[M/64] (row blocks grouped by slot count 2, 4, 8, increasing within a
 * group), count[3] and *code_bytes = K * sum(slots).  All HOST arrays; the
 * caller copies offset and order to the device for a usk_rate_map.  Host only.
 * Errors: USK_ERR_SHAPE, USK_ERR_NULL, USK_ERR_PARAMS (a slot count). */
USK_API usk_status usk_rate_map_plan(int64_t M, int64_t K, const uint32_t* slots, int64_t* offset, int32_t* order,
                                     int64_t* count, int64_t* code_bytes);

/* Build the sketch of W (Metodologia §1 and §4: fused select-and-update).
 *   W          [M, K] row-major, row stride ldw elements (ldw >= K); fp32 or
 *              bf16 per wdtype.  W and every row start must be 16-byte aligned
 *              (ldw % 4 == 0 for fp32, % 8 == 0 for bf16).
 *   importance [K] fp32 per input column, or NULL for all ones.  Values must
 *              be finite with the sign bit clear (else USK_FLAG_BAD_IMPORTANCE).
 *              Formats 2 and 3 take no importance: non-NULL is USK_ERR_PARAMS.
 *   params     format, depth and seed of the hash.
 *   codes      int8 output, 16-byte aligned: M*K/16 bytes (usk_sizes_ex for
 *              other formats and slot counts; rate-map code_bytes with
 *              params->rates).   scales [M/64] output.
 *   params->rates  per-row-block rates: still one launch; each row block uses
 *              its own slot count.
 *   d_status   optional device word for USK_FLAG_* bits.
 * M == 0 is a no-op; K == 0 writes zero scales.  Codes and scales are
 * bit-identical for any launch geometry. */
USK_API usk_status usk_build(const void* W, usk_dtype wdtype, int64_t M, int64_t K, int64_t ldw,
                     const float* importance, const usk_params* params, int8_t* codes,
                     uint16_t* scales, uint32_t* d_status, void* stream);

/* y = W_hat x for batch 1..15 (Metodologia §4: W_hat = S . P^T applied on the
 * fly: every weight is rehashed and its bucket gathered; W_hat is never stored).
 *   x  [batch, K] row-major, fp32 or bf16 per xdtype, 16-byte aligned.
 *   y  [batch, M] fp32 output (y[t*M + i] = sum_j w_hat[i][j] x[t][j]).
 * Paths, chosen from the shape (measured on B200):
 *   - bf16 x on uniform 4-slot single-row sketches (format 1, or format 2 at
 *     depth 1) of more than 2 x SMs row blocks (e.g. 28672 rows) and
 *     batch * K <= 16384: integer tensor path over row slabs (int8 codes x x
 *     split into byte digit planes, exact integer sums, one rounding at the end);
 *   - bf16 x at batch 2..8, or batch 1 with K <= 4096 and M <= 4096, and every
 *     multi-row or 4-bit sketch at batch <= 8: bf16 tensor path with the x
 *     fragments read straight from global memory (each hash row gathered, the
 *     code of largest magnitude kept; exact products, fp32 accumulation);
 *   - other bf16 x at batch 1 on single-row sketches: integer tensor path with
 *     thread-block clusters along K (digit planes as above);
 *   - fp32 x, batch 9..15, and the rest: bf16 tensor path with x staged in
 *     shared memory; fp32 x is split into two bf16 terms (|error| <= 2^-16 |x|
 *     per element).
 * A sketch with a rate map: one launch, each row block at its slot count, bf16
 * paths (direct x at batch <= 8 with bf16 x, else staged).
 * batch == 0 or M == 0 is a no-op; K == 0 writes y = 0.  Deterministic for a
 * given shape (the summation order is fixed). */
USK_API usk_status usk_gemv(const usk_sketch* sketch, const void* x, usk_dtype xdtype, int64_t batch,
                    float* y, uint32_t* d_status, void* stream);

/* usk_gemv with launch flags.  USK_GEMV_PDL: launch as a programmatic
 * dependent of the previous kernel in the stream; the kernel prefetches the
 * sketch codes (and reads a rate map's order and offset tables) before
 * waiting for that kernel, so the caller guarantees that no kernel still
 * running in the stream writes this sketch's codes, scales or rate-map tables
 * (x and y may be produced / consumed by neighbouring kernels).  Other bits:
 * USK_ERR_PARAMS. */
#define USK_GEMV_PDL 1u
USK_API usk_status usk_gemv_ex(const usk_sketch* sketch, const void* x, usk_dtype xdtype, int64_t batch,
                               float* y, uint32_t flags, uint32_t* d_status, void* stream);

/* Several independent products in one launch (Metodologia §4, as usk_gemv):
 * y[l] = W_hat_l x[l] for l < n, n in 0..16, batch 0..8, bf16 x only.
 * A persistent kernel streams every 64-row x 1024-column piece of every
 * sketch through shared memory with bulk copies a few pieces ahead of the
 * math, so the copies of one piece (and of the next sketch) overlap the math
 * of others; a row whose K spans several pieces is summed through the
 * workspace in a fixed order (deterministic for a given list of shapes).
 *   sketches  n sketches (host array), one format, depth and slot count among
 *             them: format 1 (any slot count), 2 or 4; no rate map; format 3
 *             is usk_gemv only (USK_ERR_PARAMS).
 *   x, y      HOST arrays of n DEVICE pointers: x[l] [batch, K_l] bf16,
 *             16-byte aligned; y[l] [batch, M_l] fp32.  The products must be
 *             independent: no y[l] may overlap another y or any x.
 *   ws        caller-owned device workspace of at least the bytes
 *             usk_gemv_multi_ws_bytes returns for the same list and batch
 *             (0 when every K <= 1024; ws may then be NULL), 16-byte aligned,
 *             zero-filled before its first use.  It starts with one arrival
 *             counter per split row block, which every call that completes
 *             without USK_FLAG_TIMEOUT returns to zero, then the partial sums,
 *             which need no clearing; so calls that follow one another in a
 *             stream can share it, while calls that may run at the same time
 *             need one each.  After a timeout, fill it with zeros again.
 *   flags     USK_GEMV_PDL as in usk_gemv_ex: the first pieces' codes are
 *             fetched before the previous kernel in the stream completes (x,
 *             y and ws only after it).  Other bits: USK_ERR_PARAMS.
 * Errors: USK_ERR_SHAPE (n), USK_ERR_BATCH, USK_ERR_DTYPE (fp32 x),
 * USK_ERR_PARAMS, USK_ERR_NULL, USK_ERR_ALIGN, USK_ERR_WORKSPACE (ws missing or
 * smaller than required).  Sketches with M == 0 are skipped; K == 0 writes
 * y[l] = 0. */
USK_API usk_status usk_gemv_multi_ws_bytes(int64_t n, const usk_sketch* sketches, int64_t batch, size_t* ws_bytes);
USK_API usk_status usk_gemv_multi(int64_t n, const usk_sketch* sketches, const void* const* x, usk_dtype xdtype,
                                  int64_t batch, float* const* y, void* ws, size_t ws_bytes, uint32_t flags,
                                  uint32_t* d_status, void* stream);

/* usk_gemv_multi for callers that may not allocate device memory: the same
 * products, with the scratch the call needs (the arrival counters and partial
 * sums of split rows) held in a fixed array inside the library instead of a
 * caller workspace.  Meant for code that runs where allocation is not an
 * option -- a plug-in or an inference engine that hands this library only
 * its input and output buffers and owns every other byte of device memory,
 * or a real-time loop that must not call cudaMalloc after start-up (it can
 * synchronise the device and its time is unbounded).  The paper has no
 * counterpart; this is a calling convention of the library.
 *   Arguments, results, formats and errors as usk_gemv_multi, without ws.
 *   The fixed array holds USK_GEMV_MULTI_STATIC_BYTES bytes on every device
 *   that loads the library, from load until the process exits.  A list whose
 *   workspace (usk_gemv_multi_ws_bytes for the same list and batch) is larger
 *   is refused with USK_ERR_WORKSPACE before anything is launched (for
 *   instance one 4096 x 4096 sketch at batch 8 on a 148-SM B200, whose rows
 *   split into 4 pieces: 512 KiB of partial sums plus the counters).
 *   The call allocates nothing: it makes no cudaMalloc, cudaFree or other
 *   allocating call.  Its first call on a device looks up the array's device
 *   address (cudaGetSymbolAddress, with that device current); make that first
 *   call before any stream capture.  Each call first clears the counters on
 *   `stream` (cudaMemsetAsync), then launches.
 *   Every call shares the one array: calls that may overlap on the GPU (other
 *   streams, other threads, concurrent graph branches) race on it and give
 *   wrong results; keep them in one stream order. */
#define USK_GEMV_MULTI_STATIC_BYTES (512u * 1024u)
USK_API usk_status usk_gemv_multi_static(int64_t n, const usk_sketch* sketches, const void* const* x,
                                         usk_dtype xdtype, int64_t batch, float* const* y, uint32_t flags,
                                         uint32_t* d_status, void* stream);

/* y = W_hat x for batch 16..256 (multiple of 16) on the tcgen05 tensor cores:
 * decoded bf16 tiles of W_hat are written to tensor memory and multiplied with
 * bf16 x tiles (copied into shared memory by the tensor memory accelerator),
 * fp32 accumulation in tensor memory.
 *   x_bf16 [batch, K] bf16, 16-byte aligned.  y [batch, M] fp32.
 *   ws / ws_bytes: unused by this version (may be NULL / 0).
 * A sketch with a rate map: one launch; a 128-row tile takes two row blocks of
 * the same slot count; the launch is planned for the 8-slot layout, so K is
 * limited as for a uniform 8-slot sketch (USK_ERR_SHAPE beyond it).
 * M == 0 is a no-op; K == 0 writes y = 0. */
USK_API usk_status usk_gemm(const usk_sketch* sketch, const uint16_t* x_bf16, int64_t batch, float* y,
                    void* ws, size_t ws_bytes, uint32_t* d_status, void* stream);

/* usk_gemm with launch flags (Metodologia §4, as usk_gemm).  USK_GEMM_PDL:
 * launch as a programmatic dependent of the previous kernel in the stream.
 * Before waiting for that kernel a block sets up, copies its share of the
 * sketch codes (and reads a rate map's order and offset tables), widens them
 * and decodes the first tiles into tensor memory; x, the scales, y and
 * d_status are touched only after the wait.  So the caller guarantees that no
 * kernel still running in the stream writes this sketch's codes or rate-map
 * tables (x and y may be produced / consumed by neighbouring kernels).  The
 * results are those of usk_gemm.  Other bits: USK_ERR_PARAMS. */
#define USK_GEMM_PDL 1u
USK_API usk_status usk_gemm_ex(const usk_sketch* sketch, const uint16_t* x_bf16, int64_t batch, float* y,
                               uint32_t flags, uint32_t* d_status, void* stream);

/* Test hook: override the launch geometry (0 = default).  build_cluster is the
 * number of thread blocks per row block in usk_build (1..8); gemv_tiles_per_block
 * the number of hash tiles per thread block in usk_gemv.  Results are
 * bit-identical for every geometry; only the split of the work changes.
 * Process-wide; not thread-safe with concurrent calls. */
USK_API void usk_debug_set_geometry(int build_cluster, int gemv_tiles_per_block);

/* Test hook: choose the usk_gemv path (0 = automatic, 1 = bf16 tensor path,
 * 2 = integer path with thread-block clusters where eligible, 3 = integer
 * row-slab path where eligible: bf16 x and batch * K <= 16384; single-row
 * sketches only), 4 = bf16 path with x fragments from global memory (bf16 x,
 * batch <= 8).  Every path gives results within the products' tolerance;
 * process-wide. */
USK_API void usk_debug_set_gemv_path(int path);

/* Test hook: rows per thread block of the row-slab path (16, 32 or 64) and of
 * the format-3 product (64 or 256); any other value restores the automatic
 * choice.  Results stay within the products' tolerance; process-wide. */
USK_API void usk_debug_set_gemv_rows(int rows);

/* Test hook: thread blocks along K per 128-row tile of usk_gemm (1..16, used
 * where that many tiles per block fit; 0 = the library's choice).  Results
 * stay within the products' tolerance; process-wide. */
USK_API void usk_debug_set_gemm_splits(int splits);

/* Test hook: MMA issuer warps of usk_gemm (1, 2 or 4, at most the default for
 * the batch: 4 up to 64, 2 up to 128, 1 above; 0 = the library's choice).
 * Results stay within the products' tolerance; process-wide. */
USK_API void usk_debug_set_gemm_issuers(int issuers);

/* Test hook for the failure path (host-made; no device fault): kernel = 1 makes
 * usk_build, 2 usk_gemm, 3 usk_gemv, 4 usk_gemv_multi skip one bulk or tensor
 * copy in thread block (0, 0) (for the usk_gemv path without copies: the
 * partial sums of block 1 of row block 0), so a bounded wait gives up after
 * about 1 s and sets
 * USK_FLAG_TIMEOUT; the kernel still completes and the context stays usable.
 * 0 switches it off.  Process-wide. */
USK_API void usk_debug_inject_timeout(int kernel);

/* Static description of a status value. */
USK_API const char* usk_status_str(usk_status status);

/* Format version compiled into the library. */
USK_API uint32_t usk_format_version(void);

#ifdef __cplusplus
}
#endif

#endif /* USK_H_ */

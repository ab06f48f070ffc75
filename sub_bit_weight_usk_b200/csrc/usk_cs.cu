// usk_cs.cu -- the column-shared projection sketch (format 3): build and
// y = W_hat x for batch 1..15 as y = S (P^T x).
//
// "UltraSketchLLM" explainer, Resumen Tecnico, Metodologia §4 "Mapeo de
// Operadores de Matriz Amigables con el Hardware": compression is a matrix
// product with a projection matrix P whose reduction is a MIN over absolute
// values, decompression the plain product W_hat = S . P^T, which turns the
// irregular hash-and-gather access into coalesced, matrix-shaped traffic.
//
// Format 3 (include/usk.h): P is one-hot per input column and shared by all
// rows.  Inside 256-column tile tc a seeded bijection sigma_tc of [0, 256) lists
// the columns; bucket b' of the tile holds sigma_tc(16 b' + k), k = 0..15.  S
// keeps per row and bucket the member of smallest |w| (ties: smallest column);
// codes toward zero; row-major codes [M][K/16], one binary16 scale per 64 rows.
//
// Design (B200, sm_100a):
//  * build: the format-1 skeleton (64 x 256 weight tiles by 2-D tensor copies
//    into a double-buffered ring, a cluster per row block, the scale exchange
//    through distributed shared memory).  The selection needs no atomics: a
//    thread owns (row, bucket) pairs, reads the bucket's 16 members through the
//    tile's sigma table and keeps the minimum of packed (|w|, column, sign) keys
//    in registers.  Lanes of the second row of a warp walk the members from the
//    middle so the two rows read different columns (fewer bank conflicts).
//  * product: P^T x is a bucket sum of x -- K/16 values per batch row -- so the
//    dense part S z streams one int8 code per 16 weights from HBM with coalesced
//    16-byte loads, no gathers.  One thread block per (R rows, tpb tiles), R =
//    64 or 256; the blocks along K form a cluster.  Each block first issues
//    its code loads, then builds z for its 16 tpb buckets from x (16/tpb threads
//    per bucket, added in a fixed order), then every thread dots its row's codes
//    with z (broadcast shared-memory reads); the lanes of a row combine by
//    shuffles and the blocks' partials meet in the first block (st.async onto a
//    transaction-counted mbarrier, added in rank order: deterministic).  Tall
//    matrices take 256-row blocks, which amortise the bucket sums over more
//    rows (at 64 rows the kernel was measured instruction-bound, 78 % issue, on
//    28672 x 8192); smaller ones keep 64-row blocks with fewer registers.
#include <cooperative_groups.h>

#include "usk_common.cuh"

namespace cg = cooperative_groups;

namespace usk {

// sigma_tc(u): seeded bijection of [0, 256) (every step is invertible on 8 bits).
__device__ __forceinline__ uint32_t cs_sigma(uint3 key, uint32_t u) {
  const uint32_t v1 = (key.x * u + key.y) & 255u;
  const uint32_t v2 = v1 ^ (v1 >> 4);
  const uint32_t v3 = (key.z * v2) & 255u;
  return v3 ^ (v3 >> 3);
}

__host__ __device__ __forceinline__ uint3 cs_key(uint64_t seed, uint64_t tc) {
  const uint64_t z = splitmix64(seed, tc + 1);
  return make_uint3(static_cast<uint32_t>(z & 255u) | 1u, static_cast<uint32_t>((z >> 8) & 255u),
                    static_cast<uint32_t>((z >> 16) & 255u) | 1u);
}

// ============================================================ build

constexpr int kCsThreads = 256;

struct BuildCsArgs {
  const void* W;
  int64_t ldw;
  int64_t K;
  uint64_t seed;
  int8_t* codes;
  uint16_t* scales;
  uint32_t* status;
  int T, C, tpc, nbuf;
  int inject;  // test hook: block (0, 0) skips the copy of its first tile
};

struct BuildCsLayout {
  uint32_t wbuf, sig, vals, bars, misc, total;
};

__host__ __device__ inline BuildCsLayout build_cs_layout(bool bf16, int tpc, int nbuf) {
  const uint32_t tile = kRowsPerBlock * kTileCols * (bf16 ? 2u : 4u);
  BuildCsLayout L;
  L.wbuf = 0;
  L.sig = L.wbuf + nbuf * tile;                                      // u8 [tpc][256]
  L.vals = L.sig + static_cast<uint32_t>(tpc) * 256u;               // [tpc][64][16] kept values
  L.bars = (L.vals + static_cast<uint32_t>(tpc) * 1024u * (bf16 ? 2u : 4u) + 7u) & ~7u;
  L.misc = L.bars + 64u;
  L.total = L.misc + 64u;
  return L;
}

template <bool BF16>
__global__ void __launch_bounds__(kCsThreads, 2)
    build_cs_kernel(const BuildCsArgs a, const __grid_constant__ CUtensorMap wmap) {
  constexpr uint32_t kRowBytes = kTileCols * (BF16 ? 2 : 4);
  constexpr uint32_t kTileBytes = kRowsPerBlock * kRowBytes;
  extern __shared__ __align__(128) uint8_t smraw_unaligned[];
  const BuildCsLayout L = build_cs_layout(BF16, a.tpc, a.nbuf);
  const uint32_t s0 = (smem_u32(smraw_unaligned) + 1023u) & ~1023u;
  uint8_t* smraw = smraw_unaligned + (s0 - smem_u32(smraw_unaligned));
  uint32_t* misc = reinterpret_cast<uint32_t*>(smraw + L.misc);
  uint8_t* sig_all = smraw + L.sig;

  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int rb = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nt = (a.T - crank + a.C - 1) / a.C;  // this block's tiles: crank, crank + C, ...

  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  if (tid == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap)) : "memory");
  auto issue = [&](int i) {
    const int tc = crank + a.C * i;
    const int buf = i % a.nbuf;
    const uint32_t bar = s0 + L.bars + 8 * buf;
    mbar_arrive_expect_tx(bar, kTileBytes);
    tma_load_2d(s0 + L.wbuf + buf * kTileBytes, &wmap, tc * kTileCols, rb * kRowsPerBlock, bar);
  };
  if (tid == 0) {
    for (int b = 0; b < a.nbuf; ++b) mbar_init(s0 + L.bars + 8 * b, 1);
    mbar_fence_init();
    misc[0] = 0u;
    for (int i = 0; i < a.nbuf && i < nt; ++i)
      if (!(a.inject && i == 0 && crank == 0 && rb == 0)) issue(i);
  }
  // the column lists of this block's tiles, while the first weights stream in
  for (int q = tid; q < nt * 256; q += kCsThreads) {
    const int i = q >> 8;
    sig_all[q] = static_cast<uint8_t>(cs_sigma(cs_key(a.seed, static_cast<uint64_t>(crank + a.C * i)), q & 255));
  }
  __syncthreads();

  uint32_t flags = 0;
  uint32_t vmax = 0;
  using ValT = typename std::conditional<BF16, uint16_t, uint32_t>::type;
  ValT* vals_all = reinterpret_cast<ValT*>(smraw + L.vals);
  // pair p = tid + 256 e: row r = p / 16, bucket b' = p % 16; a warp covers 2 rows
  const int bq = tid & 15;
  const int kofs = (lane >> 4) * 8;  // second row of the warp starts half-way round

  for (int i = 0; i < nt; ++i) {
    const int buf = i % a.nbuf;
    if (!mbar_wait(s0 + L.bars + 8 * buf, (i / a.nbuf) & 1)) flags |= USK_FLAG_TIMEOUT;
    const uint8_t* wt = smraw + L.wbuf + buf * kTileBytes;
    const uint8_t* sig = sig_all + i * 256 + 16 * bq;
    ValT* vals = vals_all + i * 1024;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = (tid >> 4) + 16 * e;
      if (BF16) {
        const uint16_t* wrow = reinterpret_cast<const uint16_t*>(wt + r * kRowBytes);
        uint32_t best = 0xFFFFFFFFu, nf = 0u;
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
          const uint32_t c = sig[(kk + kofs) & 15];
          const uint32_t b16 = wrow[c];
          nf |= (b16 & 0x7F80u) + 0x80u;  // exponent all ones -> bit 15
          best = min(best, ((b16 & 0x7FFFu) << 16) | (c << 1) | (b16 >> 15));
        }
        if (nf & 0x8000u) flags |= USK_FLAG_NONFINITE_W;
        const uint32_t vb = ((best >> 16) & 0x7FFFu) | ((best & 1u) << 15);
        vals[r * 16 + bq] = static_cast<ValT>(vb);
        vmax = max(vmax, (vb & 0x7FFFu) << 16);
      } else {
        const uint32_t* wrow = reinterpret_cast<const uint32_t*>(wt + r * kRowBytes);
        uint64_t best = ~0ull;
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
          const uint32_t c = sig[(kk + kofs) & 15];
          const uint32_t wb = wrow[c];
          if ((wb & 0x7F800000u) == 0x7F800000u) flags |= USK_FLAG_NONFINITE_W;
          best = min(best, (static_cast<uint64_t>(wb & 0x7FFFFFFFu) << 32) | (c << 1) | (wb >> 31));
        }
        const uint32_t vb = static_cast<uint32_t>(best >> 32) | (static_cast<uint32_t>(best & 1u) << 31);
        vals[r * 16 + bq] = static_cast<ValT>(vb);
        vmax = max(vmax, vb & 0x7FFFFFFFu);
      }
    }
    __syncthreads();  // tile i resolved; its weight buffer is free
    if (tid == 0 && i + a.nbuf < nt) issue(i + a.nbuf);
  }

  // ---- row-block maximum through distributed shared memory (as format 1)
  vmax = __reduce_max_sync(0xFFFFFFFFu, vmax);
  if (lane == 0) atomicMax(&misc[0], vmax);
  __syncthreads();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if (warp == 0 && lane < a.C && lane != crank) atomicMax(cluster.map_shared_rank(&misc[0], lane), misc[0]);
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  const float mx = __uint_as_float(misc[0]);
  const __half s16 = __float2half_rn(mx / 127.0f);
  const float sc = __half2float(s16);
  if (crank == 0 && tid == 0) {
    a.scales[rb] = __half_as_ushort(s16);
    if (isinf(sc)) flags |= USK_FLAG_SCALE_OVERFLOW;
  }
  // codes toward zero (as format 2); one 16-byte store per (row, tile):
  // codes[(64 rb + r) * K/16 + 16 tc + b']
  const int64_t nbk = a.K / 16;
  for (int q = tid; q < nt * 64; q += kCsThreads) {
    const int i = q >> 6, r = q & 63;
    const int tc = crank + a.C * i;
    const ValT* v16 = vals_all + i * 1024 + r * 16;
    uint32_t w4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t vb = v16[e];
      const float v = BF16 ? __uint_as_float(vb << 16) : __uint_as_float(vb);
      int code = 0;
      if (sc != 0.0f) {
        const float m = fabsf(v);
        float t = fminf(truncf(m / sc), 127.0f);
        if (t * sc > m) t -= 1.0f;
        code = static_cast<int>(t);
        if (v < 0.0f) code = -code;
      }
      w4[e >> 2] |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * (e & 3));
    }
    int8_t* dst = a.codes + (static_cast<int64_t>(rb) * 64 + r) * nbk + 16 * static_cast<int64_t>(tc);
    *reinterpret_cast<uint4*>(dst) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
  report(a.status, flags);
}

template <bool BF16>
static cudaError_t launch_build_cs_t(BuildCsArgs a, int64_t RB, cudaStream_t stream, int cluster_override) {
  auto mk = [&](int C, int nbuf) {
    a.C = C < a.T ? C : a.T;
    a.tpc = (a.T + a.C - 1) / a.C;
    a.nbuf = nbuf;
    return build_cs_layout(BF16, a.tpc, nbuf).total + 1024u;  // + alignment slack
  };
  uint32_t smem;
  if (cluster_override > 0) {
    smem = mk(cluster_override, 2);
    if (smem > 220u * 1024u) smem = mk(cluster_override, 1);
  } else {
    smem = mk(4, 2);
    if (smem > 112u * 1024u && a.T > 4) smem = mk(8, 2);
    if (smem > 112u * 1024u && a.T > 8) smem = mk(16, 2);
    if (smem > 220u * 1024u) smem = mk(a.C, 1);
  }
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap wmap;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(RB * kRowsPerBlock)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(a.ldw) * (BF16 ? 2u : 4u)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileCols), static_cast<cuuint32_t>(kRowsPerBlock)};
  const cuuint32_t estride[2] = {1, 1};
  if (encode(&wmap, BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
             const_cast<void*>(a.W), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  auto kern = build_cs_kernel<BF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (a.C > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.C, static_cast<unsigned>(RB), 1);
  cfg.blockDim = dim3(kCsThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, wmap);
}

cudaError_t launch_build_cs(const void* W, bool bf16, int64_t M, int64_t K, int64_t ldw, uint64_t seed,
                            int8_t* codes, uint16_t* scales, uint32_t* status, cudaStream_t stream,
                            int cluster_override, int inject) {
  BuildCsArgs a;
  a.W = W; a.ldw = ldw; a.K = K; a.seed = seed;
  a.codes = codes; a.scales = scales; a.status = status;
  a.T = static_cast<int>(K / kTileCols);
  a.C = a.tpc = a.nbuf = 0;
  a.inject = inject;
  const int64_t RB = M / kRowsPerBlock;
  return bf16 ? launch_build_cs_t<true>(a, RB, stream, cluster_override)
              : launch_build_cs_t<false>(a, RB, stream, cluster_override);
}

// ============================================================ product

struct GemvCsArgs {
  const int8_t* codes;
  const uint16_t* scales;
  const void* x;
  float* y;
  int64_t M, K;
  uint64_t seed;
  uint32_t* status;
  int T, C, tpb;  // tiles per row, blocks along K (cluster size), tiles per block (power of two)
  int R;          // rows per block: 64 or 256
  int pdl;
  int inject;  // test hook: block 1 of the first row group skips its partial sums
};

constexpr int kCsMaxTiles = 16;  // tiles per block
constexpr int kCsMaxBatch = 15;

struct GemvCsLayout {
  uint32_t ctile, z, push, bars, total;
};

// 256-row blocks stage their codes (256 rows x 128 bytes, 128-byte swizzle) at
// the 1024-byte aligned start; then z, the first block's receive area and two
// mbarriers (partial sums, code tile).
__host__ __device__ inline GemvCsLayout gemv_cs_layout(int tpb, int batch, int C, int R) {
  GemvCsLayout L;
  L.ctile = 0;
  L.z = R == 256 ? 256u * 128u : 0u;                                        // fp32 [batch][16 tpb]
  L.push = L.z + static_cast<uint32_t>(batch * 16 * tpb) * 4u;             // fp32 [C][batch][R] (rank 0)
  L.bars = (L.push + static_cast<uint32_t>(C * batch * R) * 4u + 7u) & ~7u;
  L.total = L.bars + 16u;
  return L;
}

__device__ __forceinline__ uint32_t cs_mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cs_st_async_f32(uint32_t remote_addr, float v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(remote_addr),
               "r"(__float_as_uint(v)), "r"(remote_bar)
               : "memory");
}

// TPR threads per row.  4: 64-row blocks of up to 16 tiles; thread (row r,
// part q) loads tiles q, q + 4, ... of its row (16 codes each, the four lanes of
// a row read adjacent 16-byte pieces).  1: 256-row blocks of 8 tiles; the block's
// codes (256 rows x 128 bytes, rows K/16 bytes apart) arrive by one 2-D tensor
// copy into 128-byte-swizzled shared memory -- as per-thread loads each warp
// instruction touched 32 separate lines and issuing them took 1.4 us (traced)
// -- and thread r reads row r's 8 pieces conflict-free.  The bucket sums use
// four threads per bucket, four members each, all loads in flight at once.
template <int B, bool XF32, int TPR>
__global__ void __launch_bounds__(kCsThreads) gemv_cs_kernel(const GemvCsArgs a,
                                                             const __grid_constant__ CUtensorMap cmap) {
  constexpr int R = kCsThreads / TPR, tpr = TPR;
  constexpr int kCsChunks = TPR == 4 ? 4 : 8;  // 16-code pieces per thread
  extern __shared__ __align__(128) uint8_t sm_raw[];
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int t0 = crank * a.tpb;
  const int nt = min(a.tpb, a.T - t0);
  const GemvCsLayout L = gemv_cs_layout(a.tpb, B, a.C, R);
  const uint32_t raw_s = smem_u32(sm_raw);
  const uint32_t s0 = (raw_s + 1023u) & ~1023u;  // the swizzled code tile wants 1024-byte alignment
  uint8_t* sm = sm_raw + (s0 - raw_s);
  const uint32_t push_bar = s0 + L.bars, code_bar = push_bar + 8u;
  float* zs = reinterpret_cast<float*>(sm + L.z);
  float* push = reinterpret_cast<float*>(sm + L.push);
  const int nbk = 16 * a.tpb;  // z row stride
  const uint32_t part_bytes = static_cast<uint32_t>(B * R) * 4u;

  // ---- code loads first (never written by a programmatic-dependent neighbour)
  const int r = tid / tpr, q = tid % tpr;
  const int64_t row = static_cast<int64_t>(blockIdx.y) * R + r;
  const bool row_ok = row < a.M;
  const int8_t* crow = a.codes + row * (a.K / 16) + 16 * static_cast<int64_t>(t0);
  uint4 cv[kCsChunks];
  if constexpr (TPR == 4) {
#pragma unroll
    for (int u = 0; u < kCsChunks; ++u) {
      const int tl = q + tpr * u;
      cv[u] = make_uint4(0u, 0u, 0u, 0u);
      if (row_ok && tl < nt) cv[u] = ldg_nc128(crow + 16 * tl);
    }
  } else if (tid == 0) {
    // rows and columns outside the matrix are filled with zeros by the copy
    mbar_init(code_bar, 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(code_bar, 256u * 128u);
    tma_load_2d(s0 + L.ctile, &cmap, 16 * t0, static_cast<int>(blockIdx.y) * R, code_bar);
  }
  if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0 && a.C > 1) {
    mbar_init(push_bar, 1);
    mbar_fence_init();
    if (crank == 0) mbar_arrive_expect_tx(push_bar, static_cast<uint32_t>(a.C - 1) * part_bytes);
  }
  if (a.C > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  // ---- z = P^T x for this block's buckets: four threads per bucket, members
  // 4 m4 .. 4 m4 + 3 each, added in member order, then the quarters in order
  for (int bb = tid >> 2; bb < nt * 16; bb += kCsThreads / 4) {
    const int m4 = tid & 3;
    const int tl = bb >> 4, bp = bb & 15;
    const uint3 key = cs_key(a.seed, static_cast<uint64_t>(t0 + tl));
    const int64_t col0 = static_cast<int64_t>(t0 + tl) * kTileCols;
    uint32_t c[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) c[k] = cs_sigma(key, static_cast<uint32_t>(16 * bp + 4 * m4 + k));
    float xv[B][4];
#pragma unroll
    for (int t = 0; t < B; ++t)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int64_t idx = static_cast<int64_t>(t) * a.K + col0 + c[k];
        if (XF32) xv[t][k] = __ldg(static_cast<const float*>(a.x) + idx);
        else xv[t][k] = __uint_as_float(static_cast<uint32_t>(__ldg(static_cast<const unsigned short*>(a.x) + idx)) << 16);
      }
#pragma unroll
    for (int t = 0; t < B; ++t) {
      const float sq = ((xv[t][0] + xv[t][1]) + xv[t][2]) + xv[t][3];
      const float s1 = __shfl_xor_sync(0xFFFFFFFFu, sq, 1);
      const float pair = (m4 & 1) ? (s1 + sq) : (sq + s1);     // (q0 + q1), (q2 + q3)
      const float p2 = __shfl_xor_sync(0xFFFFFFFFu, pair, 2);
      const float tot = (m4 & 2) ? (p2 + pair) : (pair + p2);  // (q0 + q1) + (q2 + q3)
      if (m4 == 0) zs[t * nbk + bb] = tot;
    }
  }
  __syncthreads();
  if (a.C > 1 && crank != 0) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");

  if constexpr (TPR == 1) {
    if (!mbar_wait(code_bar, 0)) report(a.status, USK_FLAG_TIMEOUT);  // bounded (about 1 s)
#pragma unroll
    for (int u = 0; u < kCsChunks; ++u)  // piece u of row r, 128-byte swizzle
      cv[u] = lds128(s0 + L.ctile + static_cast<uint32_t>(r) * 128u + (static_cast<uint32_t>(u ^ (r & 7)) * 16u));
  }
  // ---- S z: 16 codes per tile against the tile's 16 bucket sums
  float acc[B];
#pragma unroll
  for (int t = 0; t < B; ++t) acc[t] = 0.0f;
#pragma unroll
  for (int u = 0; u < kCsChunks; ++u) {
    const int tl = q + tpr * u;
    if (tl < nt) {
      const uint32_t ws[4] = {cv[u].x, cv[u].y, cv[u].z, cv[u].w};
      float cf[16];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t lo = i8pair_to_bf16x2<0x4140>(ws[e]), hi = i8pair_to_bf16x2<0x4342>(ws[e]);
        cf[4 * e + 0] = bf16lo(lo);
        cf[4 * e + 1] = bf16hi(lo);
        cf[4 * e + 2] = bf16lo(hi);
        cf[4 * e + 3] = bf16hi(hi);
      }
#pragma unroll
      for (int t = 0; t < B; ++t) {
        const float4* zt = reinterpret_cast<const float4*>(zs + t * nbk + 16 * tl);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 z4 = zt[e];
          acc[t] = fmaf(cf[4 * e + 0], z4.x, acc[t]);
          acc[t] = fmaf(cf[4 * e + 1], z4.y, acc[t]);
          acc[t] = fmaf(cf[4 * e + 2], z4.z, acc[t]);
          acc[t] = fmaf(cf[4 * e + 3], z4.w, acc[t]);
        }
      }
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the tpr lanes of a row, in part order
  for (int w = 1; w < tpr; w <<= 1) {
#pragma unroll
    for (int t = 0; t < B; ++t) {
      const float o = __shfl_xor_sync(0xFFFFFFFFu, acc[t], w);
      acc[t] = (q & w) ? (o + acc[t]) : (acc[t] + o);
    }
  }
  const float s = row_ok ? __half2float(__ushort_as_half(a.scales[row / kRowsPerBlock])) : 0.0f;
  // one scale per block when the block is one row block
  const float sblk = R == kRowsPerBlock ? __half2float(__ushort_as_half(a.scales[blockIdx.y])) : 0.0f;
  if (a.C == 1) {
    if (q == 0 && row_ok) {
#pragma unroll
      for (int t = 0; t < B; ++t) a.y[static_cast<int64_t>(t) * a.M + row] = acc[t] * s;
    }
    return;
  }
  if (crank != 0) {
    if (a.inject && crank == 1 && blockIdx.y == 0) return;  // test hook: the first block's wait gives up
    if (q == 0) {
      const uint32_t bar0 = cs_mapa(push_bar, 0);
#pragma unroll
      for (int t = 0; t < B; ++t)
        cs_st_async_f32(cs_mapa(s0 + L.push + (static_cast<uint32_t>((crank * B + t) * R + r)) * 4u, 0), acc[t],
                        bar0);
    }
    return;
  }
  if (q == 0) {
#pragma unroll
    for (int t = 0; t < B; ++t) push[t * R + r] = acc[t];
  }
  if (!mbar_wait(push_bar, 0)) report(a.status, USK_FLAG_TIMEOUT);  // bounded (about 1 s)
  __syncthreads();
  for (int qq = tid; qq < B * R; qq += kCsThreads) {
    const int64_t orow = static_cast<int64_t>(blockIdx.y) * R + qq % R;
    if (orow < a.M) {
      float tot = 0.0f;
      for (int c = 0; c < a.C; ++c) tot += push[c * B * R + qq];
      const float so = R == kRowsPerBlock ? sblk : __half2float(__ushort_as_half(a.scales[orow / kRowsPerBlock]));
      a.y[static_cast<int64_t>(qq / R) * a.M + orow] = tot * so;
    }
  }
}

template <int B, bool XF32>
static cudaError_t launch_gemv_cs_t(GemvCsArgs a, cudaStream_t stream) {
  const size_t smem = gemv_cs_layout(a.tpb, B, a.C, a.R).total + 1024;  // + alignment slack
  auto kern = a.R == 64 ? gemv_cs_kernel<B, XF32, 4> : gemv_cs_kernel<B, XF32, 1>;
  CUtensorMap cmap = {};
  if (a.R == 256) {
    // codes [M][K/16] bytes; one 128-byte x 256-row box per block, 128-byte swizzle
    const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(a.K / 16), static_cast<cuuint64_t>(a.M)};
    const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(a.K / 16)};
    const cuuint32_t box[2] = {128u, 256u};
    const cuuint32_t estride[2] = {1, 1};
    if (encode(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(a.codes), gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (a.C > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.C, static_cast<unsigned>((a.M + a.R - 1) / a.R), 1);
  cfg.blockDim = dim3(kCsThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, a, cmap);
}

template <bool XF32>
static cudaError_t launch_gemv_cs_b(const GemvCsArgs& a, int batch, cudaStream_t stream) {
  switch (batch) {
    case 1: return launch_gemv_cs_t<1, XF32>(a, stream);
    case 2: return launch_gemv_cs_t<2, XF32>(a, stream);
    case 3: return launch_gemv_cs_t<3, XF32>(a, stream);
    case 4: return launch_gemv_cs_t<4, XF32>(a, stream);
    case 5: return launch_gemv_cs_t<5, XF32>(a, stream);
    case 6: return launch_gemv_cs_t<6, XF32>(a, stream);
    case 7: return launch_gemv_cs_t<7, XF32>(a, stream);
    case 8: return launch_gemv_cs_t<8, XF32>(a, stream);
    case 9: return launch_gemv_cs_t<9, XF32>(a, stream);
    case 10: return launch_gemv_cs_t<10, XF32>(a, stream);
    case 11: return launch_gemv_cs_t<11, XF32>(a, stream);
    case 12: return launch_gemv_cs_t<12, XF32>(a, stream);
    case 13: return launch_gemv_cs_t<13, XF32>(a, stream);
    case 14: return launch_gemv_cs_t<14, XF32>(a, stream);
    default: return launch_gemv_cs_t<15, XF32>(a, stream);
  }
}

// Blocks along K for rows-per-block R (64 or 256) and tiles per block tpb: tpb
// is at most 16 (R = 64) or 8 (R = 256); it doubles, then R drops to 64, until
// the cluster has at most 16 blocks.
static void cs_geometry(GemvCsArgs& a, int R, int tpb) {
  a.R = (R == 256 && a.T >= 8) ? 256 : 64;
  a.tpb = a.R == 256 ? 8 : tpb;  // 256-row blocks copy 128 bytes (8 tiles) of each row
  for (;;) {
    const int cap = a.R == 64 ? 16 : 8;
    if (a.tpb > cap) a.tpb = cap;
    if ((a.T + a.tpb - 1) / a.tpb <= 16) break;
    if (a.tpb < cap) a.tpb *= 2;
    else if (a.R > 64) a.R = 64, a.tpb = 16;
    else break;
  }
  a.C = (a.T + a.tpb - 1) / a.tpb;
}

// Geometry: tpb_override (rounded down to a power of two; 256-row blocks always
// take 8 tiles) and rows_override (64 or 256) if given; else 256-row blocks for
// tall matrices (at least two row blocks of 64 per SM: the bucket sums of x are
// amortised over more rows, the codes arrive by one tensor copy per block and
// the grid stays within one wave) and from batch 4 when there is at least one
// row block per SM, 64-row blocks of 4 tiles otherwise -- measured on B200.
cudaError_t launch_gemv_cs(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                           const void* x, bool xf32, int batch, float* y, uint32_t* status, bool pdl,
                           cudaStream_t stream, int tpb_override, int rows_override, int inject) {
  GemvCsArgs a;
  a.codes = codes; a.scales = scales; a.x = x; a.y = y;
  a.M = M; a.K = K; a.seed = seed; a.status = status;
  a.T = static_cast<int>(K / kTileCols);
  a.pdl = pdl ? 1 : 0;
  a.inject = inject;
  if (batch < 1 || batch > kCsMaxBatch) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int tpb_given = 0;
  if (tpb_override > 0) {
    tpb_given = 1;
    while (tpb_given * 2 <= tpb_override && tpb_given < kCsMaxTiles) tpb_given *= 2;
  }
  const bool tall = M / kRowsPerBlock >= 2 * sms;
  const bool wide = tall || (batch >= 4 && M / kRowsPerBlock >= sms);
  const int R = (rows_override == 64 || rows_override == 256) ? rows_override : (wide ? 256 : 64);
  cs_geometry(a, R, tpb_given ? tpb_given : 4);
  // the first block's receive area: 64-row blocks when it would not fit
  if (gemv_cs_layout(a.tpb, batch, a.C, a.R).total > 200u * 1024u) cs_geometry(a, 64, a.tpb);
  if (a.C > 16) return cudaErrorInvalidValue;
  return xf32 ? launch_gemv_cs_b<true>(a, batch, stream) : launch_gemv_cs_b<false>(a, batch, stream);
}

}  // namespace usk

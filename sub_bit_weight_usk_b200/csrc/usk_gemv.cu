// usk_gemv.cu -- y = W_hat x for small batches, W_hat rebuilt on the fly.
//
// "UltraSketchLLM" explainer, Metodologia §4: decompression is the product
// W_hat = S . P^T with a one-hot projection P, i.e. every weight (i, j) reads
// the code of the bucket its index hashes to.  P is never materialised: the
// hash is recomputed in registers, one evaluation per octet of 8 columns.
//
// Design (B200, sm_100a):
//  * One thread block per (64-row block, contiguous range of hash tiles); the
//    blocks of a row block form a cluster and sum their partial products
//    through distributed shared memory in a fixed order (deterministic).
//  * The block stages its tiles' int8 codes as bf16 in shared memory (exact:
//    |code| <= 127), in the global bucket order [slot][class][sub], so the 8
//    buckets of one (row, octet) are one 16-byte word.
//  * Each warp owns one of the 8 column phases of every tile and all 64 rows;
//    lane (g, t) = (lane / 4, lane % 4) gathers the octet o = o0 + 2t of rows
//    g and g + 8 of each 16-row group with one 16-byte shared load each.
//    Because class = (o + r) mod 32, the 8 lanes of every quarter warp touch 8
//    distinct 16-byte bank groups: the gathers are conflict-free.
//  * The gathered bf16 pairs are already the A fragment of mma.sync m16n8k16
//    (the reduction dimension is permuted consistently for A and x, which the
//    sum does not see), and x is the B fragment: the tensor core does the
//    multiply-add and the reduction over columns, fp32 accumulation, exact
//    products.  Batch rows fill the MMA's n dimension; fp32 x is split into
//    hi + lo bf16 rows of the same n tile.
#include <cooperative_groups.h>

#include "usk_common.cuh"

namespace cg = cooperative_groups;

namespace usk {

struct GemvArgs {
  const int8_t* codes;
  const uint16_t* scales;
  const void* x;
  float* y;
  int64_t M, K;
  uint64_t seed;
  int T;      // tiles per row block
  int C;      // blocks per row block (cluster size)
  int tpc;    // tiles per block (the last block of a row block may have fewer)
  int batch;  // 1..15
  uint32_t* status;
  RbMap map;  // grid row -> row block and code offset
  int64_t g1, g2;  // per-row-block rates: first grid rows of the 4- and 8-slot groups
};

constexpr int kGemvThreads = 256;

// Shared memory (bytes):
//   key table  [tpc][depth] uint2, padded to 16
//   codes      [tpc][1024] bf16 (2 KiB per tile)
//   x slice    [nvalid rows][tpc * 512 + 16] bf16 (rows padded by 16 B: conflict-free)
//   block sums [batch][64] fp32
// The per-warp partials [8][NB * 8][64] fp32 alias the first three areas after
// the main loop.
struct GemvLayout {
  uint32_t keys, codes, xs, xrow, stage_end, parts, cta, total;
};

__host__ __device__ inline GemvLayout gemv_layout(int tpc, int nb, int batch, bool xf32, int depth, uint32_t tile_bf) {
  GemvLayout L;
  const uint32_t nvalid = static_cast<uint32_t>(xf32 ? 2 * batch : batch);
  L.keys = 0;
  L.codes = (static_cast<uint32_t>(tpc * depth) * 8u + 15u) / 16u * 16u;
  L.xs = L.codes + static_cast<uint32_t>(tpc) * tile_bf;
  L.xrow = static_cast<uint32_t>(tpc) * 512u + 16u;
  L.stage_end = L.xs + nvalid * L.xrow;
  L.parts = 0;
  const uint32_t parts_end = 8u * static_cast<uint32_t>(nb) * 8u * 64u * 4u;
  L.cta = ((L.stage_end > parts_end ? L.stage_end : parts_end) + 15u) / 16u * 16u;
  L.total = L.cta + static_cast<uint32_t>(batch) * 64u * 4u;
  return L;
}

__device__ __forceinline__ uint32_t pack_bf16x2_from_i8(int lo, int hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(static_cast<float>(lo), static_cast<float>(hi));
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }

// D = hash rows (1: format 1 or format 2 at depth 1; 2, 4: the multi-row
// AbsMaxMin sketch, each row gathered from its own 2048/D-byte segment of the
// tile and reduced to the code of largest magnitude)
// VAR: code layout (CodeFmt; D == 1 unless VAR == 0).
template <int NB, bool XF32, int D, int VAR>
__device__ __forceinline__ void gemv_body(const GemvArgs& a, int64_t grid_row) {
  using F = CodeFmt<VAR>;
  constexpr bool Q4 = F::kNibble;
  constexpr uint32_t kNc = 32u / D;  // classes per slot in one hash row
  constexpr uint32_t kTileBf = F::kTileBf;
  constexpr uint32_t kShift = F::kShift;
  extern __shared__ __align__(16) uint8_t sm[];
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  int rb;
  int64_t code_base;
  if (!rb_resolve(a.map, grid_row, static_cast<int64_t>(a.T) * F::kTileBytes, rb, code_base)) {
    if (threadIdx.x == 0 && crank == 0) report(a.status, USK_FLAG_RATE_MAP);
    return;  // the whole cluster (same grid row) leaves before any cluster barrier
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = crank * a.tpc;
  const int nt = min(a.tpc, a.T - t0);  // >= 1 by construction of C
  const int nvalid = XF32 ? 2 * a.batch : a.batch;
  const GemvLayout L = gemv_layout(a.tpc, NB, a.batch, XF32, D, kTileBf);
  uint2* keytab = reinterpret_cast<uint2*>(sm + L.keys);
  const uint32_t sm_s = smem_u32(sm);

  // ---- stage: hash keys, codes (int8 -> bf16) and the x slice, all loads in flight at once
  if (tid < nt * D) keytab[tid] = row_key(a.seed, static_cast<uint64_t>(rb) * a.T + t0 + tid / D, D, tid % D);
  {
    const int8_t* csrc = a.codes + code_base + static_cast<int64_t>(t0) * F::kTileBytes;
    const int ncode = nt * static_cast<int>(F::kTileBytes / 16u);  // 16-byte code chunks
    const int xchunks_row = XF32 ? nt * 64 : nt * 32;            // 16-byte x chunks per batch row
    const int nx = a.batch * xchunks_row;
    const int total = ncode + nx;
    constexpr int kR = 8;  // loads in flight per thread per round
    for (int base = 0; base < total; base += kR * kGemvThreads) {
      uint4 v[kR];
#pragma unroll
      for (int u = 0; u < kR; ++u) {
        const int q = base + u * kGemvThreads + tid;
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        if (q < ncode) {
          v[u] = ldg_nc128(csrc + 16 * q);
        } else if (q < total) {
          const int qx = q - ncode, n = qx / xchunks_row, c = qx % xchunks_row;
          const char* xrow = static_cast<const char*>(a.x) + (static_cast<int64_t>(n) * a.K +
                                                                static_cast<int64_t>(t0) * kTileCols) * (XF32 ? 4 : 2);
          v[u] = ldg_nc128(xrow + 16 * c);
        }
      }
#pragma unroll
      for (int u = 0; u < kR; ++u) {
        const int q = base + u * kGemvThreads + tid;
        if (q < ncode) {
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
          if constexpr (Q4) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint32_t o4[4];
              i4x8_to_bf16x8(w[e], o4);
              sts128(sm_s + L.codes + 64u * q + 16u * e, make_uint4(o4[0], o4[1], o4[2], o4[3]));
            }
          } else {
            uint32_t o[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              o[2 * e] = pack_bf16x2_from_i8(static_cast<int8_t>(w[e] & 0xFF), static_cast<int8_t>((w[e] >> 8) & 0xFF));
              o[2 * e + 1] = pack_bf16x2_from_i8(static_cast<int8_t>((w[e] >> 16) & 0xFF), static_cast<int8_t>(w[e] >> 24));
            }
            const uint32_t dst = sm_s + L.codes + 32u * q;
            sts128(dst, make_uint4(o[0], o[1], o[2], o[3]));
            sts128(dst + 16, make_uint4(o[4], o[5], o[6], o[7]));
          }
        } else if (q < total) {
          const int qx = q - ncode, n = qx / xchunks_row, c = qx % xchunks_row;
          if (!XF32) {
            sts128(sm_s + L.xs + n * L.xrow + 16u * c, v[u]);
          } else {
            // 4 floats -> hi row n and lo row n + batch (x = hi + lo + O(2^-16 |x|))
            const float f0 = __uint_as_float(v[u].x), f1 = __uint_as_float(v[u].y);
            const float f2 = __uint_as_float(v[u].z), f3 = __uint_as_float(v[u].w);
            const __nv_bfloat162 h01 = __floats2bfloat162_rn(f0, f1), h23 = __floats2bfloat162_rn(f2, f3);
            const float2 g01 = __bfloat1622float2(h01), g23 = __bfloat1622float2(h23);
            const __nv_bfloat162 l01 = __floats2bfloat162_rn(f0 - g01.x, f1 - g01.y);
            const __nv_bfloat162 l23 = __floats2bfloat162_rn(f2 - g23.x, f3 - g23.y);
            const uint32_t hi_dst = sm_s + L.xs + n * L.xrow + 8u * c;
            const uint32_t lo_dst = sm_s + L.xs + (n + a.batch) * L.xrow + 8u * c;
            asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(hi_dst), "r"(bf16x2_bits(h01)), "r"(bf16x2_bits(h23))
                         : "memory");
            asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(lo_dst), "r"(bf16x2_bits(l01)), "r"(bf16x2_bits(l23))
                         : "memory");
          }
        }
      }
    }
  }
  __syncthreads();

  // ---- main loop
  const int g = lane >> 2, t = lane & 3;
  const int o = 8 * (warp >> 1) + (warp & 1) + 2 * t;  // this lane's octet in every tile
  const uint32_t c0 = static_cast<uint32_t>(o + g) & (kNc - 1u);
  uint32_t cls16[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) cls16[k] = ((c0 + 8u * k) & (kNc - 1u)) * 16u;
  const uint32_t codes_s = sm_s + L.codes;

  float d[4][NB][4];
#pragma unroll
  for (int mb = 0; mb < 4; ++mb)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) d[mb][nb][e] = 0.0f;

  for (int tt = 0; tt < nt; ++tt) {
    // B fragments (x) of this tile for the lane's octet: n = 8 nb + g
    uint32_t bq[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int n = nb * 8 + g;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (n < nvalid) v = lds128(sm_s + L.xs + n * L.xrow + (tt * 32 + o) * 16);
      bq[nb][0] = v.x; bq[nb][1] = v.y; bq[nb][2] = v.z; bq[nb][3] = v.w;
    }
    const uint32_t tile_s = codes_s + tt * kTileBf;
    uint2 hk[D];
    uint32_t h[D];
#pragma unroll
    for (int rho = 0; rho < D; ++rho) {
      hk[rho] = keytab[tt * D + rho];
      h[rho] = hk[rho].x * (32u * g + o) + hk[rho].y;
    }
#pragma unroll
    for (int mb = 0; mb < 4; ++mb) {
      uint4 q0 = make_uint4(0u, 0u, 0u, 0u), q1 = q0;
#pragma unroll
      for (int rho = 0; rho < D; ++rho) {
        const uint32_t h0 = h[rho] + mb * (hk[rho].x * 512u);
        const uint32_t h1 = h0 + hk[rho].x * 256u;
        const uint32_t seg = tile_s + static_cast<uint32_t>(rho) * (2048u / D);
        const uint4 u0 = lds128(seg + (h0 >> kShift) * (kNc * 16u) + cls16[(2 * mb) & 3]);
        const uint4 u1 = lds128(seg + (h1 >> kShift) * (kNc * 16u) + cls16[(2 * mb + 1) & 3]);
        q0 = rho == 0 ? u0 : absmax_sel(q0, u0);
        q1 = rho == 0 ? u1 : absmax_sel(q1, u1);
      }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        mma_bf16_16816(d[mb][nb], q0.x, q1.x, q0.y, q1.y, bq[nb][0], bq[nb][1]);
        mma_bf16_16816(d[mb][nb], q0.z, q1.z, q0.w, q1.w, bq[nb][2], bq[nb][3]);
      }
    }
  }
  __syncthreads();  // the stage area is reused for the partials below

  // ---- per-warp partials -> block sums (fixed order over warps)
  float* part = reinterpret_cast<float*>(sm + L.parts);
  float* cta_part = reinterpret_cast<float*>(sm + L.cta);
#pragma unroll
  for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int n = nb * 8 + 2 * t;
      const int r0 = 16 * mb + g;
      float* pw = part + static_cast<size_t>(warp) * (NB * 8) * 64;
      pw[n * 64 + r0] = d[mb][nb][0];
      pw[(n + 1) * 64 + r0] = d[mb][nb][1];
      pw[n * 64 + r0 + 8] = d[mb][nb][2];
      pw[(n + 1) * 64 + r0 + 8] = d[mb][nb][3];
    }
  }
  __syncthreads();
  for (int q = tid; q < a.batch * 64; q += kGemvThreads) {
    const int n = q >> 6, r = q & 63;
    float acc = 0.0f;
    for (int w = 0; w < 8; ++w) acc += part[(static_cast<size_t>(w) * (NB * 8) + n) * 64 + r];
    if (XF32) {
      float lo = 0.0f;
      for (int w = 0; w < 8; ++w) lo += part[(static_cast<size_t>(w) * (NB * 8) + n + a.batch) * 64 + r];
      acc += lo;
    }
    cta_part[q] = acc;
  }
  cluster.sync();

  // ---- cluster reduction (fixed order over blocks) and the row-block scale;
  // block c finishes outputs c, c + C, ...
  {
    const float s = __half2float(__ushort_as_half(a.scales[rb]));
    for (int q = crank * kGemvThreads + tid; q < a.batch * 64; q += a.C * kGemvThreads) {
      float acc = 0.0f;
      for (int c = 0; c < a.C; ++c) acc += *cluster.map_shared_rank(&cta_part[q], c);
      const int n = q >> 6, r = q & 63;
      a.y[static_cast<int64_t>(n) * a.M + static_cast<int64_t>(rb) * 64 + r] = acc * s;
    }
  }
  cluster.sync();  // keep shared memory alive until every peer has read it
}

// ---------------------------------------------------------------- launch

struct GemvGeometry {
  int T, C, tpc;
};

static GemvGeometry gemv_geometry(int64_t K, int tpc_override) {
  GemvGeometry g;
  g.T = static_cast<int>(K / kTileCols);
  int tpc = tpc_override > 0 ? tpc_override : 4;
  if ((g.T + tpc - 1) / tpc > 8) tpc = (g.T + 7) / 8;  // cluster of at most 8 blocks
  if (tpc > g.T) tpc = g.T;
  g.tpc = tpc;
  g.C = (g.T + tpc - 1) / tpc;
  return g;
}

template <int NB, bool XF32, int D, int VAR>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const GemvArgs a) {
  gemv_body<NB, XF32, D, VAR>(a, blockIdx.y);
}

// Per-row-block rates in one launch: grid row g is entry g of the rate map's
// order list (grouped by slot count), so its code layout follows from g.
template <int NB, bool XF32>
__global__ void __launch_bounds__(kGemvThreads) gemv_vr_kernel(const GemvArgs a) {
  const int64_t g = blockIdx.y;
  if (g < a.g1) gemv_body<NB, XF32, 1, 2>(a, g);
  else if (g < a.g2) gemv_body<NB, XF32, 1, 0>(a, g);
  else gemv_body<NB, XF32, 1, 3>(a, g);
}

template <int NB, bool XF32, int D, int VAR>
static cudaError_t launch_gemv_t(const GemvArgs& a, int64_t nrb, cudaStream_t stream) {
  // a rate map: one launch over every row block, shared memory for 8 slots
  const bool vr = a.map.order != nullptr;
  const size_t smem =
      gemv_layout(a.tpc, NB, a.batch, XF32, D, vr ? CodeFmt<3>::kTileBf : CodeFmt<VAR>::kTileBf).total;
  auto kern = vr ? gemv_vr_kernel<NB, XF32> : gemv_kernel<NB, XF32, D, VAR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.C, static_cast<unsigned>(nrb), 1);
  cfg.blockDim = dim3(kGemvThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

cudaError_t launch_gemv_i8(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                           const uint16_t* x, int batch, float* y, uint32_t* status, int T, int C, int tpc, bool pdl,
                           cudaStream_t stream, int inject);

bool slab_supported(int64_t K, int batch);
cudaError_t launch_gemv_slab(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                             const uint16_t* x, int batch, float* y, uint32_t* status, bool pdl,
                             cudaStream_t stream, int rows_override, int inject);

bool gemv_bf_supported(int64_t K, int batch, int tpc_override);
cudaError_t launch_gemv_bf(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                           const uint16_t* x, int batch, float* y, uint32_t* status, bool pdl, cudaStream_t stream,
                           int tpc_override, int inject, int depth, int var, const RbMap& map, int64_t nrb,
                           int64_t g1, int64_t g2);

template <int D, int VAR>
static cudaError_t launch_staged(const GemvArgs& a, bool xf32, int64_t RB, cudaStream_t stream) {
  const int rows = xf32 ? 2 * a.batch : a.batch;
  const int nb = (rows + 7) / 8;
  if (!xf32) {
    if (nb == 1) return launch_gemv_t<1, false, D, VAR>(a, RB, stream);
    return launch_gemv_t<2, false, D, VAR>(a, RB, stream);
  }
  switch (nb) {
    case 1: return launch_gemv_t<1, true, D, VAR>(a, RB, stream);
    case 2: return launch_gemv_t<2, true, D, VAR>(a, RB, stream);
    case 3: return launch_gemv_t<3, true, D, VAR>(a, RB, stream);
    default: return launch_gemv_t<4, true, D, VAR>(a, RB, stream);
  }
}

// path: 0 = automatic, 1 = bf16 tensor path (staged x), 2 = integer path with
// clusters, 3 = integer row-slab path (bf16 x, batch * K <= 16384), 4 = bf16
// path with x fragments from global memory (bf16 x, batch <= 8).  depth = hash
// rows of the sketch: the integer paths read single-row sketches only.
cudaError_t launch_gemv(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                        const void* x, bool xf32, int batch, float* y, uint32_t* status, bool pdl, int path,
                        cudaStream_t stream, int tpc_override, int rows_override, int inject, int depth, int var,
                        const RbMap& map, int64_t nrb, int64_t g1, int64_t g2) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // automatic choice (measured on B200, graphs of back-to-back calls):
  //  * tall matrices (more than two row blocks per SM): integer row slabs;
  //  * batch >= 2, or batch 1 up to 4096 x 4096: bf16 with direct x fragments;
  //  * batch 1 with longer K or taller M: the integer cluster kernel (half the
  //    shared-memory gather bytes; its x preparation is amortised over more tiles)
  // the integer paths read uniform format-1 layouts of 4 slots
  const bool single = depth == 1 && var == 0 && map.order == nullptr;
  const bool slab = single && (path == 3 || (path == 0 && M / kRowsPerBlock > 2 * sms));
  if (!xf32 && slab && slab_supported(K, batch))
    return launch_gemv_slab(codes, scales, M, K, seed, static_cast<const uint16_t*>(x), batch, y, status, pdl,
                            stream, rows_override, inject);
  // multi-row sketches: the direct path unless the staged one is asked for
  const bool direct =
      path == 4 || (!single && path != 1) || (path == 0 && (batch > 1 || (K <= 4096 && M <= 4096)));
  if (!xf32 && direct && gemv_bf_supported(K, batch, tpc_override))
    return launch_gemv_bf(codes, scales, M, K, seed, static_cast<const uint16_t*>(x), batch, y, status, pdl, stream,
                          tpc_override, inject, depth, var, map, nrb, g1, g2);
  const GemvGeometry geo = gemv_geometry(K, tpc_override);
  // the integer cluster path takes 8 tiles per block by default: its x
  // preparation is per block (measured, batch 1: 11008 x 4096 7.5 us at 8
  // tiles against 9.3 us at 4; 4096 x 11008 the same)
  const GemvGeometry geo8 = gemv_geometry(K, tpc_override > 0 ? tpc_override : 8);
  const bool i8_ok = single && !xf32 && batch <= 4 && batch * geo8.tpc * 32 <= 1024;
  if (i8_ok && path != 1)
    return launch_gemv_i8(codes, scales, M, K, seed, static_cast<const uint16_t*>(x), batch, y, status, geo8.T,
                          geo8.C, geo8.tpc, pdl, stream, inject);
  GemvArgs a;
  a.codes = codes; a.scales = scales; a.x = x; a.y = y;
  a.M = M; a.K = K; a.seed = seed;
  a.T = geo.T; a.C = geo.C; a.tpc = geo.tpc; a.batch = batch;
  a.status = status;
  a.map = map;
  a.map.RB = M / kRowsPerBlock;
  a.g1 = g1;
  a.g2 = g2;
  const int64_t RB = nrb;
  if (map.order != nullptr) return launch_staged<1, 0>(a, xf32, RB, stream);  // covers every layout
  if (var == 1) return launch_staged<1, 1>(a, xf32, RB, stream);
  if (var == 2) return launch_staged<1, 2>(a, xf32, RB, stream);
  if (var == 3) return launch_staged<1, 3>(a, xf32, RB, stream);
  if (depth == 2) return launch_staged<2, 0>(a, xf32, RB, stream);
  if (depth == 4) return launch_staged<4, 0>(a, xf32, RB, stream);
  return launch_staged<1, 0>(a, xf32, RB, stream);
}

}  // namespace usk

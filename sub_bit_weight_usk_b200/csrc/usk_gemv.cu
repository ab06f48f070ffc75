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
};

constexpr int kGemvThreads = 256;

// smem: key table [tpc] uint2 (padded to 16 B) | codes bf16 [tpc][1024];
// the partial sums later alias the code area.
__host__ __device__ constexpr size_t gemv_stage_bytes(int tpc) {
  return static_cast<size_t>((tpc * 8 + 15) / 16 * 16) + static_cast<size_t>(tpc) * 2048;
}
__host__ __device__ constexpr size_t gemv_part_bytes(int nb) {
  return static_cast<size_t>(8) * (nb * 8) * 64 * 4;  // [warp][n][row] fp32
}
__host__ __device__ constexpr size_t gemv_smem_bytes(int tpc, int nb, int batch) {
  return (gemv_stage_bytes(tpc) > gemv_part_bytes(nb) ? gemv_stage_bytes(tpc) : gemv_part_bytes(nb)) +
         static_cast<size_t>(batch) * 64 * 4;
}

__device__ __forceinline__ uint32_t pack_bf16x2_from_i8(int lo, int hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(static_cast<float>(lo), static_cast<float>(hi));
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int NB, bool XF32>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(const GemvArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int rb = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = crank * a.tpc;
  const int nt = min(a.tpc, a.T - t0);  // >= 1 by construction of C
  uint2* keytab = reinterpret_cast<uint2*>(sm);
  const size_t code_off = static_cast<size_t>((a.tpc * 8 + 15) / 16 * 16);
  uint8_t* scodes = sm + code_off;
  float* part = reinterpret_cast<float*>(sm);  // aliases the stage area after the main loop
  float* cta_part = reinterpret_cast<float*>(
      sm + (gemv_stage_bytes(a.tpc) > gemv_part_bytes(NB) ? gemv_stage_bytes(a.tpc) : gemv_part_bytes(NB)));

  // ---- stage: hash keys and codes (int8 -> bf16) of this block's tiles
  if (tid < nt) keytab[tid] = tile_key(a.seed, static_cast<uint64_t>(rb) * a.T + t0 + tid);
  {
    const int8_t* src = a.codes + static_cast<int64_t>(rb) * 4 * a.K + 1024 * static_cast<int64_t>(t0);
    const int n16 = nt * 64;  // 16-code chunks
    for (int q = tid; q < n16; q += kGemvThreads) {
      const uint4 v = ldg_nc128(src + 16 * q);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c0 = static_cast<int8_t>(w[e] & 0xFF), c1 = static_cast<int8_t>((w[e] >> 8) & 0xFF);
        const int c2 = static_cast<int8_t>((w[e] >> 16) & 0xFF), c3 = static_cast<int8_t>(w[e] >> 24);
        o[2 * e] = pack_bf16x2_from_i8(c0, c1);
        o[2 * e + 1] = pack_bf16x2_from_i8(c2, c3);
      }
      uint4* dst = reinterpret_cast<uint4*>(scodes + 32 * q);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
  __syncthreads();

  // ---- main loop
  const int g = lane >> 2, t = lane & 3;
  const int o = 8 * (warp >> 1) + (warp & 1) + 2 * t;  // this lane's octet in every tile
  const uint32_t c0 = static_cast<uint32_t>(o + g) & 31u;
  uint32_t cls16[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) cls16[k] = ((c0 + 8u * k) & 31u) * 16u;
  const uint32_t codes_s = smem_u32(scodes);

  float d[4][NB][4];
#pragma unroll
  for (int mb = 0; mb < 4; ++mb)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) d[mb][nb][e] = 0.0f;

  for (int tt = 0; tt < nt; ++tt) {
    const uint2 hk = keytab[tt];
    const int64_t col = static_cast<int64_t>(t0 + tt) * kTileCols + 8 * o;
    // B fragments (x) of this tile for the lane's octet: n = 8 nb + g
    uint32_t bq[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int n = nb * 8 + g;
      if (!XF32) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (n < a.batch) v = ldg_nc128(static_cast<const uint16_t*>(a.x) + n * a.K + col);
        bq[nb][0] = v.x; bq[nb][1] = v.y; bq[nb][2] = v.z; bq[nb][3] = v.w;
      } else {
        // rows n < batch carry hi = bf16(x); rows batch <= n < 2 batch carry lo = bf16(x - hi)
        bq[nb][0] = bq[nb][1] = bq[nb][2] = bq[nb][3] = 0u;
        if (n < 2 * a.batch) {
          const int src_row = n < a.batch ? n : n - a.batch;
          const float* xp = static_cast<const float*>(a.x) + src_row * a.K + col;
          const uint4 u0 = ldg_nc128(xp), u1 = ldg_nc128(xp + 4);
          const float xf[8] = {__uint_as_float(u0.x), __uint_as_float(u0.y), __uint_as_float(u0.z),
                               __uint_as_float(u0.w), __uint_as_float(u1.x), __uint_as_float(u1.y),
                               __uint_as_float(u1.z), __uint_as_float(u1.w)};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 hi = __floats2bfloat162_rn(xf[2 * e], xf[2 * e + 1]);
            uint32_t r;
            if (n < a.batch) {
              r = *reinterpret_cast<uint32_t*>(&hi);
            } else {
              const float2 hf = __bfloat1622float2(hi);
              __nv_bfloat162 lo = __floats2bfloat162_rn(xf[2 * e] - hf.x, xf[2 * e + 1] - hf.y);
              r = *reinterpret_cast<uint32_t*>(&lo);
            }
            bq[nb][e] = r;
          }
        }
      }
    }
    const uint32_t tile_s = codes_s + tt * 2048u;
    uint32_t h = hk.x * (32u * g + o) + hk.y;
    const uint32_t d512 = hk.x * 512u, d256 = hk.x * 256u;
#pragma unroll
    for (int mb = 0; mb < 4; ++mb) {
      const uint32_t h0 = h + mb * d512;
      const uint32_t h1 = h0 + d256;
      const uint4 q0 = lds128(tile_s + (h0 >> 30) * 512u + cls16[(2 * mb) & 3]);
      const uint4 q1 = lds128(tile_s + (h1 >> 30) * 512u + cls16[(2 * mb + 1) & 3]);
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        mma_bf16_16816(d[mb][nb], q0.x, q1.x, q0.y, q1.y, bq[nb][0], bq[nb][1]);
        mma_bf16_16816(d[mb][nb], q0.z, q1.z, q0.w, q1.w, bq[nb][2], bq[nb][3]);
      }
    }
  }
  __syncthreads();  // stage area is reused for the partials below

  // ---- per-warp partials -> block partial (fixed order over warps)
  const int nvalid = XF32 ? 2 * a.batch : a.batch;
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
  (void)nvalid;
  cluster.sync();

  // ---- cluster reduction (fixed order over blocks) and the row-block scale
  if (crank == 0) {
    const float s = __half2float(__ushort_as_half(a.scales[rb]));
    for (int q = tid; q < a.batch * 64; q += kGemvThreads) {
      float acc = 0.0f;
      for (int c = 0; c < a.C; ++c) acc += *cluster.map_shared_rank(&cta_part[q], c);
      const int n = q >> 6, r = q & 63;
      a.y[static_cast<int64_t>(n) * a.M + static_cast<int64_t>(rb) * 64 + r] = acc * s;
    }
  }
  cluster.sync();  // keep shared memory alive until block 0 has read it
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

template <int NB, bool XF32>
static cudaError_t launch_gemv_t(const GemvArgs& a, int64_t RB, cudaStream_t stream) {
  const size_t smem = gemv_smem_bytes(a.tpc, NB, a.batch);
  auto kern = gemv_kernel<NB, XF32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.C, static_cast<unsigned>(RB), 1);
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

cudaError_t launch_gemv(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                        const void* x, bool xf32, int batch, float* y, cudaStream_t stream, int tpc_override) {
  const GemvGeometry geo = gemv_geometry(K, tpc_override);
  GemvArgs a;
  a.codes = codes; a.scales = scales; a.x = x; a.y = y;
  a.M = M; a.K = K; a.seed = seed;
  a.T = geo.T; a.C = geo.C; a.tpc = geo.tpc; a.batch = batch;
  const int64_t RB = M / kRowsPerBlock;
  const int rows = xf32 ? 2 * batch : batch;
  const int nb = (rows + 7) / 8;
  if (!xf32) {
    if (nb == 1) return launch_gemv_t<1, false>(a, RB, stream);
    return launch_gemv_t<2, false>(a, RB, stream);
  }
  switch (nb) {
    case 1: return launch_gemv_t<1, true>(a, RB, stream);
    case 2: return launch_gemv_t<2, true>(a, RB, stream);
    case 3: return launch_gemv_t<3, true>(a, RB, stream);
    default: return launch_gemv_t<4, true>(a, RB, stream);
  }
}

}  // namespace usk

// usk_build_amm.cu -- construction of the multi-row AbsMaxMin sketch (format 2).
//
// "UltraSketchLLM" explainer, Resumen Tecnico, Metodologia §1 "Diseno de Sketch
// AbsMaxMin": a bucket stores the member with the smallest absolute value, and
// several independently hashed sketch rows are kept so that decompression can
// take the largest of the row values; every rebuilt weight is then the
// original or one of smaller magnitude.  Metodologia §4: selection and update
// fused in one kernel.
//
// Format 2 (include/usk.h): depth D in {1, 2, 4} hash rows share a tile's 1024
// buckets (row rho owns 1024/D of them), so the storage stays one int8 code per
// 16 weights.  Row rho of tile t is keyed by SplitMix64 output t*D + rho + 1;
// class = (octet + row) mod (32/D).  Codes are toward zero, so |code * s| <= |v|.
//
// Design (B200, sm_100a): the thread-block cluster per row block, the 2-D
// tensor copies of 64 x 256 weight tiles into a double-buffered shared-memory
// ring and the scale exchange through distributed shared memory are those of
// the format-1 kernel.  Selection per weight and hash row:
//   - bf16 weights: ONE shared-memory atomicMin of the packed word
//       (|w| bits << 16) | (l << 1) | sign
//     which orders by |w|, then by the tile-local row-major index l, and carries
//     the sign, so the bucket ends up holding its winner;
//   - fp32 weights: pass 1 atomicMin of the |w| bits; pass 2 the members whose
//     magnitude equals the bucket minimum atomicMin (l << 1) | sign; the value
//     is the minimum magnitude with that sign.
//  Bucket words are laid out [rho][slot][sub][class]: for a fixed sub the 32
//  lanes of a warp (one row, 32 octets) hit 32/D classes of each row segment.
#include <cooperative_groups.h>

#include "usk_common.cuh"

namespace cg = cooperative_groups;

namespace usk {

constexpr int kAmmThreads = 256;

struct BuildAmmArgs {
  const void* W;
  int64_t ldw;
  int64_t K;
  uint64_t seed;
  int8_t* codes;
  uint16_t* scales;
  uint32_t* status;
  int T;       // tiles per row block = K / 256
  int C;       // thread blocks per row block (cluster size)
  int tpc;     // max tiles per block
  int nbuf;    // weight-tile buffers (1 or 2)
  int inject;  // test hook: block (0, 0) skips the copy of its first tile
};

struct BuildAmmLayout {
  uint32_t wbuf, keys, win, vals, bars, misc, total;
};

__host__ __device__ inline BuildAmmLayout build_amm_layout(bool bf16, int tpc, int nbuf) {
  const uint32_t tile = kRowsPerBlock * kTileCols * (bf16 ? 2u : 4u);
  BuildAmmLayout L;
  L.wbuf = 0;
  L.keys = L.wbuf + nbuf * tile;                 // fp32 only: u32 [2][1024] minimum magnitudes
  L.win = L.keys + (bf16 ? 0u : 2u * 4096u);     // u32 [2][1024] packed winners
  L.vals = L.win + 2u * 4096u;                   // [tpc][1024] kept values (bf16 or fp32 bits)
  L.bars = (L.vals + static_cast<uint32_t>(tpc) * 1024u * (bf16 ? 2u : 4u) + 7u) & ~7u;
  L.misc = L.bars + 64u;
  L.total = L.misc + 64u;
  return L;
}

// word offset of the bucket of (row r, octet o) in hash row rho, sub 0
template <int D>
__device__ __forceinline__ uint32_t amm_word(uint2 hk, uint32_t r, uint32_t o, int rho) {
  constexpr uint32_t kNc = 32u / D;
  const uint32_t h = hk.x * (32u * r + o) + hk.y;
  return static_cast<uint32_t>(rho) * (1024u / D) + (h >> 30) * 8u * kNc + ((o + r) & (kNc - 1u));
}

template <bool BF16, int D>
__global__ void __launch_bounds__(kAmmThreads, 2)
    build_amm_kernel(const BuildAmmArgs a, const __grid_constant__ CUtensorMap wmap) {
  constexpr uint32_t kNc = 32u / D;                 // classes per slot in one hash row
  constexpr uint32_t kRowBytes = kTileCols * (BF16 ? 2 : 4);
  constexpr uint32_t kTileBytes = kRowsPerBlock * kRowBytes;
  extern __shared__ __align__(128) uint8_t smraw_unaligned[];
  const BuildAmmLayout L = build_amm_layout(BF16, a.tpc, a.nbuf);
  const uint32_t s0 = (smem_u32(smraw_unaligned) + 1023u) & ~1023u;
  uint8_t* smraw = smraw_unaligned + (s0 - smem_u32(smraw_unaligned));
  uint32_t* misc = reinterpret_cast<uint32_t*>(smraw + L.misc);

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
  {
    uint32_t* win32 = reinterpret_cast<uint32_t*>(smraw + L.win);
    for (int q = tid; q < 2048; q += kAmmThreads) win32[q] = 0xFFFFFFFFu;
    if (!BF16) {
      uint32_t* k32 = reinterpret_cast<uint32_t*>(smraw + L.keys);
      for (int q = tid; q < 2048; q += kAmmThreads) k32[q] = 0xFFFFFFFFu;
    }
  }
  __syncthreads();

  uint32_t flags = 0;
  uint32_t vmax = 0;  // max |v| bits (fp32 encoding) over the winners this thread compacts
  using ValT = typename std::conditional<BF16, uint16_t, uint32_t>::type;
  ValT* vals_all = reinterpret_cast<ValT*>(smraw + L.vals);

  for (int i = 0; i < nt; ++i) {
    const int tc = crank + a.C * i;
    const int buf = i % a.nbuf;
    uint2 hk[D];
#pragma unroll
    for (int rho = 0; rho < D; ++rho)
      hk[rho] = tile_key(a.seed, (static_cast<uint64_t>(rb) * a.T + tc) * D + rho);
    if (!mbar_wait(s0 + L.bars + 8 * buf, (i / a.nbuf) & 1)) flags |= USK_FLAG_TIMEOUT;

    const uint32_t wt = s0 + L.wbuf + buf * kTileBytes;
    const uint32_t win_s = s0 + L.win + (i & 1) * 4096u;
    const uint32_t keys_s = s0 + L.keys + (i & 1) * 4096u;

    if (BF16) {
      uint32_t nf = 0u;
#pragma unroll 2
      for (int q = 0; q < 8; ++q) {
        const uint32_t r = warp + 8 * q;
        const uint32_t l0 = r * kTileCols + lane * 8;
        const uint4 v = lds128(wt + r * kRowBytes + lane * 16);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) nf |= (wv[e] & 0x7F807F80u) + 0x00800080u;  // exponent all ones -> bit 15
        uint32_t off[D];
#pragma unroll
        for (int rho = 0; rho < D; ++rho) off[rho] = 4u * amm_word<D>(hk[rho], r, lane, rho);
        static_for<8>([&](auto S) {
          constexpr int s = decltype(S)::value;
          const uint32_t b16 = (s & 1) ? (wv[s >> 1] >> 16) : (wv[s >> 1] & 0xFFFFu);
          const uint32_t p = ((b16 & 0x7FFFu) << 16) | ((l0 + s) << 1) | (b16 >> 15);
#pragma unroll
          for (int rho = 0; rho < D; ++rho) atoms_min_u32_off<4 * kNc * s>(win_s + off[rho], p);
        });
      }
      if (nf & 0x80008000u) flags |= USK_FLAG_NONFINITE_W;
    } else {
      // pass 1: minimum magnitude per bucket
#pragma unroll 2
      for (int q = 0; q < 8; ++q) {
        const uint32_t r = warp + 8 * q;
        const uint4 v0 = lds128(wt + r * kRowBytes + lane * 32), v1 = lds128(wt + r * kRowBytes + lane * 32 + 16);
        const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t off[D];
#pragma unroll
        for (int rho = 0; rho < D; ++rho) off[rho] = 4u * amm_word<D>(hk[rho], r, lane, rho);
        static_for<8>([&](auto S) {
          constexpr int s = decltype(S)::value;
          if ((wv[s] & 0x7F800000u) == 0x7F800000u) flags |= USK_FLAG_NONFINITE_W;
#pragma unroll
          for (int rho = 0; rho < D; ++rho) atoms_min_u32_off<4 * kNc * s>(keys_s + off[rho], wv[s] & 0x7FFFFFFFu);
        });
      }
      __syncthreads();
      // pass 2: the members at the minimum keep the smallest index and its sign
#pragma unroll 2
      for (int q = 0; q < 8; ++q) {
        const uint32_t r = warp + 8 * q;
        const uint32_t l0 = r * kTileCols + lane * 8;
        const uint4 v0 = lds128(wt + r * kRowBytes + lane * 32), v1 = lds128(wt + r * kRowBytes + lane * 32 + 16);
        const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int rho = 0; rho < D; ++rho) {
          const uint32_t off = 4u * amm_word<D>(hk[rho], r, lane, rho);
          uint32_t kmin[8];
          static_for<8>([&](auto S) {
            constexpr int s = decltype(S)::value;
            kmin[s] = lds32_off<4 * kNc * s>(keys_s + off);
          });
          static_for<8>([&](auto S) {
            constexpr int s = decltype(S)::value;
            atoms_min_u32_off_if_eq<4 * kNc * s>(win_s + off, ((l0 + s) << 1) | (wv[s] >> 31), wv[s] & 0x7FFFFFFFu,
                                                 kmin[s]);
          });
        }
      }
    }
    __syncthreads();  // tile i resolved; its weight buffer is free
    if (tid == 0 && i + a.nbuf < nt) issue(i + a.nbuf);

    // compact the winners into this tile's value array and reset the slot
    {
      ValT* vals = vals_all + i * 1024;
      uint32_t* win32 = reinterpret_cast<uint32_t*>(smraw + L.win + (i & 1) * 4096u);
      uint32_t* k32 = reinterpret_cast<uint32_t*>(smraw + L.keys + (i & 1) * 4096u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kidx = tid + kAmmThreads * e;
        const uint32_t p = win32[kidx];
        uint32_t vb, mag;
        if (BF16) {
          vb = (p == 0xFFFFFFFFu) ? 0u : (((p >> 16) & 0x7FFFu) | ((p & 1u) << 15));
          mag = (vb & 0x7FFFu) << 16;
        } else {
          vb = (p == 0xFFFFFFFFu) ? 0u : (k32[kidx] | ((p & 1u) << 31));
          mag = vb & 0x7FFFFFFFu;
          k32[kidx] = 0xFFFFFFFFu;
        }
        win32[kidx] = 0xFFFFFFFFu;
        vals[kidx] = static_cast<ValT>(vb);
        vmax = max(vmax, mag);
      }
    }
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
  // codes toward zero: t = trunc(|v| / s) can exceed floor(|v| / s) by one only
  // when the quotient rounds up onto an integer; t * s is exact (8-bit integer
  // times a binary16), so one comparison with |v| settles it
  for (int i = 0; i < nt; ++i) {
    const int tc = crank + a.C * i;
    const ValT* vals = vals_all + i * 1024;
    const uint32_t b0 = 4u * tid;                   // 4 consecutive buckets of the tile
    const uint32_t rho = b0 / (1024u / D), bin = b0 % (1024u / D);
    const uint32_t slot = (bin >> 3) / kNc, cls = (bin >> 3) % kNc;
    const uint32_t base = rho * (1024u / D) + (slot * 8u + (bin & 7u)) * kNc + cls;
    uint32_t packed = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t vb = vals[base + kNc * e];
      const float v = BF16 ? __uint_as_float(vb << 16) : __uint_as_float(vb);
      int code = 0;
      if (sc != 0.0f) {
        const float m = fabsf(v);
        float t = fminf(truncf(m / sc), 127.0f);
        if (t * sc > m) t -= 1.0f;
        code = static_cast<int>(t);
        if (v < 0.0f) code = -code;
      }
      packed |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * e);
    }
    int8_t* dst = a.codes + static_cast<int64_t>(rb) * 4 * a.K + 1024 * static_cast<int64_t>(tc) + b0;
    *reinterpret_cast<uint32_t*>(dst) = packed;
  }
  report(a.status, flags);
}

// ---------------------------------------------------------------- launch

template <bool BF16, int D>
static cudaError_t launch_build_amm_t(BuildAmmArgs a, int64_t RB, cudaStream_t stream, int cluster_override) {
  auto mk = [&](int C, int nbuf) {
    a.C = C < a.T ? C : a.T;
    a.tpc = (a.T + a.C - 1) / a.C;
    a.nbuf = nbuf;
    return build_amm_layout(BF16, a.tpc, nbuf).total + 1024u;  // + alignment slack
  };
  uint32_t smem;
  if (cluster_override > 0) {
    smem = mk(cluster_override, 2);
    if (smem > 220u * 1024u) smem = mk(cluster_override, 1);
  } else {
    // 4 blocks per row block; larger clusters only to keep two blocks per SM when K is long
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
  auto kern = build_amm_kernel<BF16, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (a.C > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.C, static_cast<unsigned>(RB), 1);
  cfg.blockDim = dim3(kAmmThreads, 1, 1);
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

cudaError_t launch_build_amm(const void* W, bool bf16, int64_t M, int64_t K, int64_t ldw, uint64_t seed, int depth,
                             int8_t* codes, uint16_t* scales, uint32_t* status, cudaStream_t stream,
                             int cluster_override, int inject) {
  BuildAmmArgs a;
  a.W = W; a.ldw = ldw; a.K = K; a.seed = seed;
  a.codes = codes; a.scales = scales; a.status = status;
  a.T = static_cast<int>(K / kTileCols);
  a.C = a.tpc = a.nbuf = 0;
  a.inject = inject;
  const int64_t RB = M / kRowsPerBlock;
  switch (depth) {
    case 1: return bf16 ? launch_build_amm_t<true, 1>(a, RB, stream, cluster_override)
                        : launch_build_amm_t<false, 1>(a, RB, stream, cluster_override);
    case 2: return bf16 ? launch_build_amm_t<true, 2>(a, RB, stream, cluster_override)
                        : launch_build_amm_t<false, 2>(a, RB, stream, cluster_override);
    case 4: return bf16 ? launch_build_amm_t<true, 4>(a, RB, stream, cluster_override)
                        : launch_build_amm_t<false, 4>(a, RB, stream, cluster_override);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace usk

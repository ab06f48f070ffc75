// usk_build.cu -- sketch construction (the fused select-and-update kernel).
//
// "UltraSketchLLM" explainer, Metodologia §4 (compression: selection and
// update fused into one kernel) and §1 (AbsMaxMin: a bucket keeps one value
// chosen by magnitude).  The selection key is fp32(|w|) * importance[j]; the
// winner is the largest key, ties to the smallest row-major index, so the
// result does not depend on the order of the scatter.
//
// Design (B200, sm_100a):
//  * One thread block per (row block, group of hash tiles); the blocks of one
//    row block form a thread-block cluster so that the row-block scale is an
//    exchange of per-block maxima through distributed shared memory: no
//    workspace and one launch.
//  * A tile (64 x 256 weights, 1024 buckets) is read once from HBM with 16-byte
//    coalesced loads and kept in registers (64 weights per thread) while three
//    passes resolve the winners with 32-bit shared-memory atomics, which run
//    about four times faster than 64-bit ones on this part:
//      pass 1  atomicMax of the key bits per bucket (order-preserving: keys are
//              non-negative fp32, whose bit patterns sort like the values);
//      pass 2  members whose key equals the bucket maximum atomicMin their
//              tile-local row-major index;
//      pass 3  the member holding that index writes its signed value.
//  * Bucket key arrays are laid out [slot][sub][class] so that the 32 lanes of
//    a warp (one row, 32 octets, 32 distinct classes) hit 32 distinct banks.
#include <cooperative_groups.h>

#include "usk_common.cuh"

namespace cg = cooperative_groups;

namespace usk {

struct BuildArgs {
  const void* W;
  int64_t ldw;
  int64_t K;
  const float* imp;
  uint64_t seed;
  int8_t* codes;
  uint16_t* scales;
  uint32_t* status;
  int T;  // tiles per row block = K / 256
  int C;  // thread blocks per row block (cluster size)
};

constexpr int kBuildThreads = 512;
constexpr int kUnits = kRowsPerBlock * kTileCols / 8 / kBuildThreads;  // octets per thread per tile (4)
constexpr int kRowStep = kBuildThreads / 32;                            // rows between a thread's octets (16)

// The 64 weights (8 octets) one thread owns in a tile, kept in registers.
template <bool BF16>
struct TileRegs;

template <>
struct TileRegs<true> {
  uint32_t u[kUnits][4];
  __device__ __forceinline__ void load(int q, const void* p) {
    uint4 v = ldg_nc128(p);
    u[q][0] = v.x; u[q][1] = v.y; u[q][2] = v.z; u[q][3] = v.w;
  }
  __device__ __forceinline__ float get(int q, int s) const {
    return (s & 1) ? bf16hi(u[q][s >> 1]) : bf16lo(u[q][s >> 1]);
  }
  // value stored per bucket: the raw bf16 bits (exact)
  __device__ __forceinline__ uint16_t stored(int q, int s) const {
    return static_cast<uint16_t>((s & 1) ? (u[q][s >> 1] >> 16) : (u[q][s >> 1] & 0xFFFFu));
  }
  // Opaque to the compiler: keys are recomputed in each pass instead of being
  // kept live across the barriers (64 extra registers otherwise).
  __device__ __forceinline__ void fence() {
#pragma unroll
    for (int q = 0; q < kUnits; ++q)
#pragma unroll
      for (int i = 0; i < 4; ++i) asm volatile("" : "+r"(u[q][i]));
  }
};

template <>
struct TileRegs<false> {
  float f[kUnits][8];
  __device__ __forceinline__ void load(int q, const void* p) {
    uint4 a = ldg_nc128(p);
    uint4 b = ldg_nc128(static_cast<const char*>(p) + 16);
    f[q][0] = __uint_as_float(a.x); f[q][1] = __uint_as_float(a.y);
    f[q][2] = __uint_as_float(a.z); f[q][3] = __uint_as_float(a.w);
    f[q][4] = __uint_as_float(b.x); f[q][5] = __uint_as_float(b.y);
    f[q][6] = __uint_as_float(b.z); f[q][7] = __uint_as_float(b.w);
  }
  __device__ __forceinline__ float get(int q, int s) const { return f[q][s]; }
  __device__ __forceinline__ uint32_t stored(int q, int s) const { return __float_as_uint(f[q][s]); }
  __device__ __forceinline__ void fence() {
#pragma unroll
    for (int q = 0; q < kUnits; ++q)
#pragma unroll
      for (int i = 0; i < 8; ++i) asm volatile("" : "+f"(f[q][i]));
  }
};

template <bool BF16>
using ValT = typename std::conditional<BF16, uint16_t, uint32_t>::type;

template <bool BF16>
__device__ __forceinline__ float stored_to_f32(ValT<BF16> v);
template <>
__device__ __forceinline__ float stored_to_f32<true>(uint16_t v) { return __uint_as_float(static_cast<uint32_t>(v) << 16); }
template <>
__device__ __forceinline__ float stored_to_f32<false>(uint32_t v) { return __uint_as_float(v); }

// Shared memory: keys[1024] u32 | widx[1024] u32 | misc[4] u32 | vals[tpc][1024]
__host__ __device__ constexpr size_t build_smem_bytes(int tiles_per_block, bool bf16) {
  return (2 * 1024 + 4) * 4 + static_cast<size_t>(tiles_per_block) * 1024 * (bf16 ? 2 : 4);
}

template <bool BF16, bool HAS_IMP>
__global__ void __launch_bounds__(kBuildThreads, 2) build_kernel(const BuildArgs a) {
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t* keys = sm;
  uint32_t* widx = sm + 1024;
  uint32_t* misc = sm + 2048;  // [0] block max |v| bits, [1] non-finite screen
  ValT<BF16>* vals_all = reinterpret_cast<ValT<BF16>*>(sm + 2048 + 4);

  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int rb = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t flags = 0;
  uint32_t vmax = 0;  // running max of |v| bits over this thread's winners

  int nt = 0;
  for (int tc = crank; tc < a.T; tc += a.C, ++nt) {
    ValT<BF16>* vals = vals_all + nt * 1024;
    for (int q = tid; q < 1024; q += kBuildThreads) {
      keys[q] = 0u;
      widx[q] = 0xFFFFFFFFu;
      vals[q] = 0;
    }
    if (tid == 0) misc[1] = 0u;

    // Issue the tile's loads before the barrier so that their latency overlaps it.
    const int64_t col0 = static_cast<int64_t>(tc) * kTileCols + lane * 8;
    TileRegs<BF16> w;
#pragma unroll
    for (int q = 0; q < kUnits; ++q) {
      const int64_t row = static_cast<int64_t>(rb) * kRowsPerBlock + warp + kRowStep * q;
      const char* p = static_cast<const char*>(a.W) + (row * a.ldw + col0) * (BF16 ? 2 : 4);
      w.load(q, p);
    }
    float imp[8];
    if (HAS_IMP) {
      const uint4 i0 = ldg_nc128(a.imp + col0);
      const uint4 i1 = ldg_nc128(a.imp + col0 + 4);
      const uint32_t ib[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        // importance must be finite with the sign bit clear
        if ((ib[s] >> 31) || (ib[s] & 0x7F800000u) == 0x7F800000u) flags |= USK_FLAG_BAD_IMPORTANCE;
        imp[s] = __uint_as_float(ib[s]);
      }
    }
    const uint2 hk = tile_key(a.seed, static_cast<uint64_t>(rb) * a.T + tc);
    uint32_t kb[kUnits];  // shared byte offset of (slot, sub 0, class) for each owned octet
#pragma unroll
    for (int q = 0; q < kUnits; ++q) {
      const uint32_t r = warp + kRowStep * q;
      const uint32_t h = hk.x * (32u * r + lane) + hk.y;
      kb[q] = ((h >> 30) * 256u + ((lane + r) & 31u)) * 4u;
    }
    const uint32_t keys_s = smem_u32(keys), widx_s = smem_u32(widx);
    __syncthreads();

    // pass 1: per-bucket maximum of the key bits
#pragma unroll
    for (int q = 0; q < kUnits; ++q) {
      const uint32_t base = keys_s + kb[q];
      static_for<8>([&](auto S) {
        constexpr int s = decltype(S)::value;
        const float f = w.get(q, s);
        const float k = HAS_IMP ? fabsf(f) * imp[s] : fabsf(f);
        atoms_max_u32_off<128 * s>(base, __float_as_uint(k));
      });
    }
    __syncthreads();

    // Non-finite screen: a NaN or Inf weight forces a key >= +Inf bits in its
    // bucket (an fp32 overflow of |w| * importance can too; the exact check
    // below separates the two).
    {
      const uint2 v = reinterpret_cast<const uint2*>(keys)[tid];
      if (max(v.x, v.y) >= 0x7F800000u) misc[1] = 1u;
    }

    // pass 2: members that reach the maximum compete on their index
    w.fence();
    uint32_t cand = 0u;
#pragma unroll
    for (int q = 0; q < kUnits; ++q) {
      const uint32_t kbase = keys_s + kb[q], wbase = widx_s + kb[q];
      const uint32_t l0 = static_cast<uint32_t>((warp + kRowStep * q) * kTileCols + lane * 8);
      static_for<8>([&](auto S) {
        constexpr int s = decltype(S)::value;
        const float f = w.get(q, s);
        const float k = HAS_IMP ? fabsf(f) * imp[s] : fabsf(f);
        if (__float_as_uint(k) == lds32_off<128 * s>(kbase)) {
          atoms_min_u32_off<128 * s>(wbase, l0 + s);
          cand |= 1u << (q * 8 + s);
        }
      });
    }
    __syncthreads();
    if (misc[1]) {
#pragma unroll
      for (int q = 0; q < kUnits; ++q)
#pragma unroll
        for (int s = 0; s < 8; ++s)
          if ((__float_as_uint(w.get(q, s)) & 0x7F800000u) == 0x7F800000u) flags |= USK_FLAG_NONFINITE_W;
    }

    // pass 3: the winning member writes its signed value
    w.fence();
    if (cand) {
#pragma unroll
      for (int q = 0; q < kUnits; ++q) {
        const uint32_t wbase = widx_s + kb[q];
        const uint32_t l0 = static_cast<uint32_t>((warp + kRowStep * q) * kTileCols + lane * 8);
        static_for<8>([&](auto S) {
          constexpr int s = decltype(S)::value;
          if ((cand >> (q * 8 + s)) & 1u) {
            if (lds32_off<128 * s>(wbase) == l0 + s) {
              vals[(kb[q] >> 2) + 32 * s] = w.stored(q, s);
              vmax = max(vmax, __float_as_uint(fabsf(w.get(q, s))));
            }
          }
        });
      }
    }
    __syncthreads();
  }

  // block maximum of |v|, then the row-block maximum across the cluster
  vmax = __reduce_max_sync(0xFFFFFFFFu, vmax);
  if (tid == 0) misc[0] = 0u;
  __syncthreads();
  if (lane == 0) atomicMax(&misc[0], vmax);
  cluster.sync();
  uint32_t mbits = 0u;
  for (int c = 0; c < a.C; ++c) mbits = max(mbits, *cluster.map_shared_rank(&misc[0], c));

  const float m = __uint_as_float(mbits);
  const __half s16 = __float2half_rn(m / 127.0f);
  const float s = __half2float(s16);
  if (crank == 0 && tid == 0) {
    a.scales[rb] = __half_as_ushort(s16);
    if (isinf(s)) flags |= USK_FLAG_SCALE_OVERFLOW;
  }

  // quantize this block's tiles; each thread writes 4 consecutive codes
  nt = 0;
  for (int tc = crank; tc < a.T; tc += a.C, ++nt) {
    const ValT<BF16>* vals = vals_all + nt * 1024;
    const uint32_t b0 = 2u * tid;
    const uint32_t base = (b0 >> 8) * 256u + (b0 & 7u) * 32u + ((b0 >> 3) & 31u);
    uint32_t packed = 0u;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float v = stored_to_f32<BF16>(vals[base + 32u * e]);
      int code = 0;
      if (s != 0.0f) code = static_cast<int>(fminf(fmaxf(rintf(v / s), -127.0f), 127.0f));
      packed |= (static_cast<uint32_t>(code) & 0xFFu) << (8 * e);
    }
    int8_t* dst = a.codes + static_cast<int64_t>(rb) * 4 * a.K + 1024 * static_cast<int64_t>(tc) + b0;
    *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(packed);
  }
  report(a.status, flags);
  cluster.sync();  // keep this block's shared memory alive until every peer has read it
}

// ---------------------------------------------------------------- launch

static int build_cluster_size(int T) { return T < 8 ? T : 8; }

template <bool BF16, bool HAS_IMP>
static cudaError_t launch_build_t(const BuildArgs& a, int64_t RB, cudaStream_t stream) {
  const int tpc = (a.T + a.C - 1) / a.C;
  const size_t smem = build_smem_bytes(tpc, BF16);
  auto kern = build_kernel<BF16, HAS_IMP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.C, static_cast<unsigned>(RB), 1);
  cfg.blockDim = dim3(kBuildThreads, 1, 1);
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

cudaError_t launch_build(const void* W, bool bf16, int64_t M, int64_t K, int64_t ldw, const float* imp,
                         uint64_t seed, int8_t* codes, uint16_t* scales, uint32_t* status,
                         cudaStream_t stream, int cluster_override) {
  BuildArgs a;
  a.W = W; a.ldw = ldw; a.K = K; a.imp = imp; a.seed = seed;
  a.codes = codes; a.scales = scales; a.status = status;
  a.T = static_cast<int>(K / kTileCols);
  a.C = cluster_override > 0 ? (cluster_override < a.T ? cluster_override : a.T) : build_cluster_size(a.T);
  const int64_t RB = M / kRowsPerBlock;
  if (bf16) return imp ? launch_build_t<true, true>(a, RB, stream) : launch_build_t<true, false>(a, RB, stream);
  return imp ? launch_build_t<false, true>(a, RB, stream) : launch_build_t<false, false>(a, RB, stream);
}

}  // namespace usk

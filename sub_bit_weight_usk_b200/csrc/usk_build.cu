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
//    row block form a thread-block cluster, so the row-block scale is an
//    exchange of per-block maxima through distributed shared memory: no
//    workspace, one launch.
//  * Weight tiles (64 x 256) stream from HBM into shared memory with one 2-D
//    tensor copy each (the tensor memory accelerator, tensor map over W),
//    completing on mbarriers, double buffered, so the copy of tile i+1
//    overlaps the selection of tile i.
//  * Selection uses order-preserving 32-bit keys and shared-memory atomics
//    (64-bit shared atomics run about four times slower on this part):
//      - bf16 weights, unit importance: ONE pass.  The packed word
//        (|w| bits << 16) | (16384 - l) << 1 | sign  orders by |w|, then by
//        the smaller tile-local row-major index l, and carries the sign, so
//        one atomicMax per weight leaves the winner itself in the bucket.
//      - with importance (or fp32 weights): pass 1 atomicMax of the fp32 key
//        bits; pass 2 the members equal to the maximum atomicMin the packed
//        (l, value) word, which keeps the smallest index and its value.
//  * Bucket arrays are laid out [slot][sub][class]: the 32 lanes of a warp
//    (one row, 32 octets, 32 distinct classes) hit 32 distinct banks.
#include <cooperative_groups.h>

#include "usk_common.cuh"

namespace cg = cooperative_groups;

namespace usk {

constexpr int kBuildThreads = 256;

struct BuildArgs {
  const void* W;
  int64_t ldw;
  int64_t K;
  const float* imp;
  uint64_t seed;
  int8_t* codes;
  uint16_t* scales;
  uint32_t* status;
  int T;     // tiles per row block = K / 256
  int C;     // thread blocks per row block (cluster size)
  int tpc;   // max tiles per block
  int nbuf;  // weight-tile buffers (1 or 2)
  int inject;  // test hook: block (0, 0) skips the copy of its first tile
  RbMap map;   // grid row -> row block and code offset
  int64_t g1, g2;  // per-row-block rates: first grid rows of the 4- and 8-slot groups
};

// Shared-memory layout (byte offsets from a 128-byte aligned base).
struct BuildLayout {
  uint32_t wbuf, keys, win, vals, bars, misc, total;
};

// nbk: buckets per tile (256 x hash slots per class)
__host__ __device__ inline BuildLayout build_layout(bool bf16, bool has_imp, int tpc, int nbuf, uint32_t nbk) {
  const bool single = bf16 && !has_imp;
  const uint32_t tile = kRowsPerBlock * kTileCols * (bf16 ? 2u : 4u);
  BuildLayout L;
  L.wbuf = 0;
  L.keys = L.wbuf + nbuf * tile;
  L.win = L.keys + (single ? 0u : 2u * 4u * nbk);
  L.vals = L.win + ((single || bf16) ? 2u * 4u * nbk : 2u * 8u * nbk);
  L.bars = (L.vals + static_cast<uint32_t>(tpc) * nbk * (bf16 ? 2u : 4u) + 7u) & ~7u;
  L.misc = L.bars + 64u;
  L.total = L.misc + 64u;
  return L;
}

// VAR: code layout (CodeFmt): 2, 4 or 8 hash slots per class (slot = h >> kShift,
// 256 x slots buckets per tile) and 8-bit codes, or 8 slots with 4-bit codes
// (scale max |v| / 7, codes clamp(rint(v / s), -7, 7) packed two per byte).
template <bool BF16, bool HAS_IMP, int VAR>
__device__ __forceinline__ void build_body(const BuildArgs& a, const CUtensorMap* wmap, int64_t grid_row) {
  using F = CodeFmt<VAR>;
  constexpr bool Q4 = F::kNibble;
  constexpr bool kSingle = BF16 && !HAS_IMP;
  constexpr uint32_t kRowBytes = kTileCols * (BF16 ? 2 : 4);
  constexpr uint32_t kTileBytes = kRowsPerBlock * kRowBytes;
  constexpr uint32_t kBk = F::kBuckets;          // buckets per tile
  constexpr uint32_t kShift = F::kShift;         // slot = h >> kShift
  constexpr uint32_t kWinBytes = (kSingle || BF16) ? 4u * kBk : 8u * kBk;  // one tile's winner words
  extern __shared__ __align__(128) uint8_t smraw_unaligned[];
  const BuildLayout L = build_layout(BF16, HAS_IMP, a.tpc, a.nbuf, kBk);
  const uint32_t s0 = (smem_u32(smraw_unaligned) + 1023u) & ~1023u;  // tensor copies want 128 B; use 1 KiB
  uint8_t* smraw = smraw_unaligned + (s0 - smem_u32(smraw_unaligned));
  uint32_t* misc = reinterpret_cast<uint32_t*>(smraw + L.misc);

  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  int rb;
  int64_t code_base;
  if (!rb_resolve(a.map, grid_row, static_cast<int64_t>(a.T) * F::kTileBytes, rb, code_base)) {
    if (threadIdx.x == 0 && crank == 0) report(a.status, USK_FLAG_RATE_MAP);
    return;  // the whole cluster (same grid row) leaves before any cluster barrier
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nt = (a.T - crank + a.C - 1) / a.C;  // this block's tiles: crank, crank + C, ...

  // first half of a split cluster barrier; its wait, before the first remote
  // access, guarantees that every block of the cluster has started
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  if (tid == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(wmap)) : "memory");

  // importance of this lane's 8 columns, one tile ahead (the loads of tile 0
  // go out before the weight copies fill the memory queues)
  uint4 ipre0 = make_uint4(0u, 0u, 0u, 0u), ipre1 = ipre0;
  auto load_imp = [&](int i) {
    if (HAS_IMP && i < nt) {
      const int64_t col0 = static_cast<int64_t>(crank + a.C * i) * kTileCols + lane * 8;
      ipre0 = ldg_nc128(a.imp + col0);
      ipre1 = ldg_nc128(a.imp + col0 + 4);
    }
  };
  load_imp(0);
  auto issue = [&](int i) {  // one tensor copy of tile i of this block into buffer i % nbuf
    const int tc = crank + a.C * i;
    const int buf = i % a.nbuf;
    const uint32_t bar = s0 + L.bars + 8 * buf;
    mbar_arrive_expect_tx(bar, kTileBytes);
    tma_load_2d(s0 + L.wbuf + buf * kTileBytes, wmap, tc * kTileCols, rb * kRowsPerBlock, bar);
  };
  // ---- init: the first tile copies go out first, then the winner and key
  // words of both slots are cleared while the weights stream in
  if (tid == 0) {
    for (int b = 0; b < a.nbuf; ++b) mbar_init(s0 + L.bars + 8 * b, 1);
    mbar_fence_init();
    misc[0] = 0u;
    for (int i = 0; i < a.nbuf && i < nt; ++i)
      if (!(a.inject && i == 0 && crank == 0 && rb == 0)) issue(i);
  }
  {
    uint32_t* win32 = reinterpret_cast<uint32_t*>(smraw + L.win);
    const uint32_t init = kSingle ? 0u : 0xFFFFFFFFu;
    for (uint32_t q = tid; q < 2u * kWinBytes / 4u; q += kBuildThreads) win32[q] = init;
    if (!kSingle) {
      uint32_t* k32 = reinterpret_cast<uint32_t*>(smraw + L.keys);
      for (uint32_t q = tid; q < 2u * kBk; q += kBuildThreads) k32[q] = 0u;
    }
  }
  __syncthreads();

  uint32_t flags = 0;
  uint32_t vmax = 0;  // max |v| bits over the winners this thread converts
  using ValT = typename std::conditional<BF16, uint16_t, uint32_t>::type;
  ValT* vals_all = reinterpret_cast<ValT*>(smraw + L.vals);

  for (int i = 0; i < nt; ++i) {
    const int tc = crank + a.C * i;
    const int buf = i % a.nbuf;
    const uint2 hk = tile_key(a.seed, static_cast<uint64_t>(rb) * a.T + tc);
    float imp[8];
    if (HAS_IMP) {
      const uint32_t ib[8] = {ipre0.x, ipre0.y, ipre0.z, ipre0.w, ipre1.x, ipre1.y, ipre1.z, ipre1.w};
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        if ((ib[s] >> 31) || (ib[s] & 0x7F800000u) == 0x7F800000u) flags |= USK_FLAG_BAD_IMPORTANCE;
        imp[s] = __uint_as_float(ib[s]);
      }
      load_imp(i + 1);
    }
    if (!mbar_wait(s0 + L.bars + 8 * buf, (i / a.nbuf) & 1)) flags |= USK_FLAG_TIMEOUT;

    const uint32_t wt = s0 + L.wbuf + buf * kTileBytes;
    const uint32_t win_s = s0 + L.win + (i & 1) * kWinBytes;
    const uint32_t keys_s = s0 + L.keys + (i & 1) * (4u * kBk);

    if (BF16 && HAS_IMP) {
      // pass 1: key maxima; the tile's weight words stay in registers for pass 2,
      // and a per-word test flags Inf/NaN weights exactly (exponent field all
      // ones <=> (bits & 0x7F80) + 0x80 reaches 0x8000, per half word)
      uint4 wq[8];
      uint32_t nf = 0u;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t r = warp + 8 * q;
        const uint32_t h = hk.x * (32u * r + lane) + hk.y;
        const uint32_t off = ((h >> kShift) * 256u + ((lane + r) & 31u)) * 4u;
        wq[q] = lds128(wt + r * kRowBytes + lane * 16);
        const uint32_t wv[4] = {wq[q].x, wq[q].y, wq[q].z, wq[q].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) nf |= (wv[e] & 0x7F807F80u) + 0x00800080u;
        static_for<8>([&](auto S) {
          constexpr int s = decltype(S)::value;
          const float f = (s & 1) ? __uint_as_float(wv[s >> 1] & 0xFFFF0000u) : __uint_as_float(wv[s >> 1] << 16);
          atoms_max_u32_off<128 * s>(keys_s + off, __float_as_uint(fabsf(f) * imp[s]));
        });
      }
      if (nf & 0x80008000u) flags |= USK_FLAG_NONFINITE_W;
      __syncthreads();
      // pass 2: members whose key equals the bucket maximum keep the smallest
      // index and its value (predicated reductions, no divergent branches)
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t r = warp + 8 * q;
        const uint32_t h = hk.x * (32u * r + lane) + hk.y;
        const uint32_t off = ((h >> kShift) * 256u + ((lane + r) & 31u)) * 4u;
        const uint32_t l0 = r * kTileCols + lane * 8;
        const uint32_t wv[4] = {wq[q].x, wq[q].y, wq[q].z, wq[q].w};
        uint32_t kmax[8];
        static_for<8>([&](auto S) {
          constexpr int s = decltype(S)::value;
          kmax[s] = lds32_off<128 * s>(keys_s + off);
        });
        static_for<8>([&](auto S) {
          constexpr int s = decltype(S)::value;
          const uint32_t bits = (s & 1) ? (wv[s >> 1] >> 16) : (wv[s >> 1] & 0xFFFFu);
          const uint32_t k = __float_as_uint(fabsf(__uint_as_float(bits << 16)) * imp[s]);
          atoms_min_u32_off_if_eq<128 * s>(win_s + off, ((l0 + s) << 16) | bits, k, kmax[s]);
        });
      }
    } else {
      // pass 1 (and the only pass for bf16 with unit importance)
  #pragma unroll 2
      for (int q = 0; q < 8; ++q) {
        const uint32_t r = warp + 8 * q;
        const uint32_t h = hk.x * (32u * r + lane) + hk.y;
        const uint32_t off = ((h >> kShift) * 256u + ((lane + r) & 31u)) * 4u;
        const uint32_t l0 = r * kTileCols + lane * 8;
        if (BF16) {
          const uint4 v = lds128(wt + r * kRowBytes + lane * 16);
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
          static_for<8>([&](auto S) {
            constexpr int s = decltype(S)::value;
            const uint32_t b16 = (s & 1) ? (wv[s >> 1] >> 16) : (wv[s >> 1] & 0xFFFFu);
            if (kSingle) {
              const uint32_t p = ((b16 & 0x7FFFu) << 16) | ((16384u - (l0 + s)) << 1) | (b16 >> 15);
              atoms_max_u32_off<128 * s>(win_s + off, p);
            } else {
              const float k = fabsf(__uint_as_float(b16 << 16)) * imp[s];
              atoms_max_u32_off<128 * s>(keys_s + off, __float_as_uint(k));
            }
          });
        } else {
          const uint4 v0 = lds128(wt + r * kRowBytes + lane * 32), v1 = lds128(wt + r * kRowBytes + lane * 32 + 16);
          const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
          static_for<8>([&](auto S) {
            constexpr int s = decltype(S)::value;
            const float f = __uint_as_float(wv[s]);
            const float k = HAS_IMP ? fabsf(f) * imp[s] : fabsf(f);
            atoms_max_u32_off<128 * s>(keys_s + off, __float_as_uint(k));
          });
        }
      }

      if (!kSingle) {
        __syncthreads();
        // Non-finite screen: a NaN or Inf weight forces a key >= +Inf bits in
        // its bucket; an fp32 overflow of |w| * importance can too, so the exact
        // per-weight check runs only when the screen fires (rare).
        bool screen;
        {
          uint32_t m = 0u;
#pragma unroll
          for (uint32_t part = 0; part < (kBk + 1023u) / 1024u; ++part) {  // every key word of the tile
            if (tid + part * kBuildThreads >= kBk / 4u) break;
            const uint4 mx = lds128(keys_s + 16u * (tid + part * kBuildThreads));
            m = max(m, max(max(mx.x, mx.y), max(mx.z, mx.w)));
          }
          screen = __syncthreads_or(m >= 0x7F800000u) != 0;
        }
        // pass 2: members whose key equals the bucket maximum keep the smallest
        // index and its value (predicated reductions, no divergent branches)
  #pragma unroll 2
        for (int q = 0; q < 8; ++q) {
          const uint32_t r = warp + 8 * q;
          const uint32_t h = hk.x * (32u * r + lane) + hk.y;
          const uint32_t off = ((h >> kShift) * 256u + ((lane + r) & 31u)) * 4u;
          const uint32_t l0 = r * kTileCols + lane * 8;
          uint32_t wv[8];
          if (BF16) {
            const uint4 v = lds128(wt + r * kRowBytes + lane * 16);
            wv[0] = v.x; wv[1] = v.y; wv[2] = v.z; wv[3] = v.w;
            wv[4] = wv[5] = wv[6] = wv[7] = 0u;
          } else {
            const uint4 v0 = lds128(wt + r * kRowBytes + lane * 32), v1 = lds128(wt + r * kRowBytes + lane * 32 + 16);
            wv[0] = v0.x; wv[1] = v0.y; wv[2] = v0.z; wv[3] = v0.w; wv[4] = v1.x; wv[5] = v1.y; wv[6] = v1.z; wv[7] = v1.w;
          }
          uint32_t kmax[8];
          static_for<8>([&](auto S) {
            constexpr int s = decltype(S)::value;
            kmax[s] = lds32_off<128 * s>(keys_s + off);
          });
          static_for<8>([&](auto S) {
            constexpr int s = decltype(S)::value;
            uint32_t bits;
            if (BF16) bits = (s & 1) ? (wv[s >> 1] >> 16) : (wv[s >> 1] & 0xFFFFu);
            else bits = wv[s];
            const float f = BF16 ? __uint_as_float(bits << 16) : __uint_as_float(bits);
            const uint32_t k = __float_as_uint(HAS_IMP ? fabsf(f) * imp[s] : fabsf(f));
            if (BF16) atoms_min_u32_off_if_eq<128 * s>(win_s + off, ((l0 + s) << 16) | bits, k, kmax[s]);
            else atoms_min_u64_off_if_eq<256 * s>(win_s + 2 * off, (static_cast<uint64_t>(l0 + s) << 32) | bits, k, kmax[s]);
            if (screen && (__float_as_uint(f) & 0x7F800000u) == 0x7F800000u) flags |= USK_FLAG_NONFINITE_W;
          });
        }
      }
    }
    __syncthreads();  // tile i resolved; its weight buffer is free
    if (tid == 0 && i + a.nbuf < nt) issue(i + a.nbuf);

    // compact this tile's winners into its value array and reset the slot
    // (reused by tile i + 2, after the barrier of tile i + 1)
    {
      ValT* vals = vals_all + i * kBk;
      uint32_t* win32 = reinterpret_cast<uint32_t*>(smraw + L.win + (i & 1) * kWinBytes);
      uint64_t* win64 = reinterpret_cast<uint64_t*>(smraw + L.win + (i & 1) * kWinBytes);
      uint32_t* k32 = reinterpret_cast<uint32_t*>(smraw + L.keys + (i & 1) * (4u * kBk));
#pragma unroll
      for (int e = 0; e < static_cast<int>(kBk / kBuildThreads); ++e) {  // 2, 4 or 8 words per thread
        const int kidx = tid + kBuildThreads * e;  // consecutive lanes, consecutive words: no bank conflicts
        uint32_t vb, mag;
        if (kSingle) {
          const uint32_t p = win32[kidx];
          vb = ((p >> 16) & 0x7FFFu) | ((p & 1u) << 15);
          mag = (vb & 0x7FFFu) << 16;
          win32[kidx] = 0u;
        } else if (BF16) {
          const uint32_t p = win32[kidx];
          vb = (p == 0xFFFFFFFFu) ? 0u : (p & 0xFFFFu);
          mag = (vb & 0x7FFFu) << 16;
          win32[kidx] = 0xFFFFFFFFu;
          k32[kidx] = 0u;
        } else {
          const uint64_t p = win64[kidx];
          vb = (p == ~0ull) ? 0u : static_cast<uint32_t>(p);
          mag = vb & 0x7FFFFFFFu;
          win64[kidx] = ~0ull;
          k32[kidx] = 0u;
        }
        if (kSingle && (mag & 0x7F800000u) == 0x7F800000u) flags |= USK_FLAG_NONFINITE_W;
        vals[kidx] = static_cast<ValT>(vb);
        vmax = max(vmax, mag);
      }
    }
  }

  // ---- row-block maximum: every block pushes its maximum into every peer's
  // word (remote atomicMax), then one cluster barrier; afterwards each block
  // reads only its own shared memory, so no block waits for its peers to exit.
  vmax = __reduce_max_sync(0xFFFFFFFFu, vmax);
  if (lane == 0) atomicMax(&misc[0], vmax);
  __syncthreads();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");  // every block has started
  if (warp == 0 && lane < a.C && lane != crank) atomicMax(cluster.map_shared_rank(&misc[0], lane), misc[0]);
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  const float mx = __uint_as_float(misc[0]);
  const __half s16 = __float2half_rn(mx / (Q4 ? 7.0f : 127.0f));
  const float sc = __half2float(s16);
  if (crank == 0 && tid == 0) {
    a.scales[rb] = __half_as_ushort(s16);
    if (isinf(sc)) flags |= USK_FLAG_SCALE_OVERFLOW;
  }
  for (int i = 0; i < nt; ++i) {
    const int tc = crank + a.C * i;
    const ValT* vals = vals_all + i * kBk;
    // kPer = slots consecutive buckets per thread (same slot and class, subs
    // b0 % 8 .. + kPer - 1): 8-bit codes -> kPer bytes; 4-bit codes -> 8 nibbles
    constexpr uint32_t kPer = F::kSlots;
    const uint32_t b0 = kPer * tid;
    const uint32_t base = (b0 >> 8) * 256u + (b0 & 7u) * 32u + ((b0 >> 3) & 31u);
    uint64_t packed = 0u;
#pragma unroll
    for (int e = 0; e < static_cast<int>(kPer); ++e) {
      const uint32_t vb = vals[base + 32u * e];
      const float v = BF16 ? __uint_as_float(vb << 16) : __uint_as_float(vb);
      constexpr float kQmax = Q4 ? 7.0f : 127.0f;
      int code = 0;
      if (sc != 0.0f) code = static_cast<int>(fminf(fmaxf(rintf(v / sc), -kQmax), kQmax));
      packed |= Q4 ? (static_cast<uint64_t>(static_cast<uint32_t>(code) & 0xFu) << (4 * e))
                   : (static_cast<uint64_t>(static_cast<uint32_t>(code) & 0xFFu) << (8 * e));
    }
    int8_t* dst = a.codes + code_base + static_cast<int64_t>(tc) * F::kTileBytes + (Q4 ? 4u : kPer) * tid;
    if (Q4 || kPer == 4) *reinterpret_cast<uint32_t*>(dst) = static_cast<uint32_t>(packed);
    else if (kPer == 2) *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(packed);
    else *reinterpret_cast<uint64_t*>(dst) = packed;
  }
  report(a.status, flags);
}

template <bool BF16, bool HAS_IMP, int VAR>
__global__ void __launch_bounds__(kBuildThreads, 2) build_kernel(const BuildArgs a, const __grid_constant__ CUtensorMap wmap) {
  build_body<BF16, HAS_IMP, VAR>(a, &wmap, blockIdx.y);
}

// Per-row-block rates in one launch: grid row g is entry g of the rate map's
// order list (grouped by slot count), so its group -- and the compile-time code
// layout -- follows from g; every block of a cluster shares g.
template <bool BF16, bool HAS_IMP>
__global__ void __launch_bounds__(kBuildThreads, 2) build_vr_kernel(const BuildArgs a, const __grid_constant__ CUtensorMap wmap) {
  const int64_t g = blockIdx.y;
  if (g < a.g1) build_body<BF16, HAS_IMP, 2>(a, &wmap, g);
  else if (g < a.g2) build_body<BF16, HAS_IMP, 0>(a, &wmap, g);
  else build_body<BF16, HAS_IMP, 3>(a, &wmap, g);
}

// ---------------------------------------------------------------- launch

struct BuildPlan {
  int C, tpc, nbuf;
  uint32_t smem;
};

static BuildPlan plan_build(int T, bool bf16, bool has_imp, int cluster_override, uint32_t nbk) {
  auto mk = [&](int C, int nbuf) {
    BuildPlan p;
    p.C = C < T ? C : T;
    p.tpc = (T + p.C - 1) / p.C;
    p.nbuf = nbuf;
    p.smem = build_layout(bf16, has_imp, p.tpc, nbuf, nbk).total + 1024;  // + alignment slack
    return p;
  };
  if (cluster_override > 0) {
    BuildPlan p = mk(cluster_override, 2);
    if (p.smem > 220u * 1024u) p = mk(cluster_override, 1);
    return p;
  }
  // 4 blocks per row block measured fastest at 4096 x 4096 and 28672 x 8192;
  // larger clusters only to keep two blocks per SM when K is long
  BuildPlan p = mk(4, 2);
  if (p.smem > 112u * 1024u && T > 4) p = mk(8, 2);
  if (p.smem > 112u * 1024u && T > 8) p = mk(16, 2);
  if (p.smem > 220u * 1024u) p = mk(p.C, 1);
  return p;
}

template <bool BF16, bool HAS_IMP, int VAR>
static cudaError_t launch_build_t(BuildArgs a, int64_t nrb, cudaStream_t stream, int cluster_override) {
  // a rate map: one launch over every row block, shared memory planned for 8 slots
  const bool vr = a.map.order != nullptr;
  const BuildPlan p =
      plan_build(a.T, BF16, HAS_IMP, cluster_override, vr ? CodeFmt<3>::kBuckets : CodeFmt<VAR>::kBuckets);
  // tensor map over W [M, K] (row stride ldw), one 64 x 256 box per tile
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap wmap;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.map.RB * kRowsPerBlock)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(a.ldw) * (BF16 ? 2u : 4u)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileCols), static_cast<cuuint32_t>(kRowsPerBlock)};
  const cuuint32_t estride[2] = {1, 1};
  if (encode(&wmap, BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
             const_cast<void*>(a.W), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  a.C = p.C;
  a.tpc = p.tpc;
  a.nbuf = p.nbuf;
  auto kern = vr ? build_vr_kernel<BF16, HAS_IMP> : build_kernel<BF16, HAS_IMP, VAR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(p.smem));
  if (e != cudaSuccess) return e;
  if (p.C > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.C, static_cast<unsigned>(nrb), 1);
  cfg.blockDim = dim3(kBuildThreads, 1, 1);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, wmap);
}

cudaError_t launch_build(const void* W, bool bf16, int64_t M, int64_t K, int64_t ldw, const float* imp,
                         uint64_t seed, int8_t* codes, uint16_t* scales, uint32_t* status,
                         cudaStream_t stream, int cluster_override, int inject, int var, const RbMap& map,
                         int64_t nrb, int64_t g1, int64_t g2) {
  BuildArgs a;
  a.inject = inject;
  a.map = map;
  a.map.RB = M / kRowsPerBlock;
  a.g1 = g1;
  a.g2 = g2;
  if (map.order != nullptr) var = 0;  // the rate-map kernel covers every layout
  a.W = W; a.ldw = ldw; a.K = K; a.imp = imp; a.seed = seed;
  a.codes = codes; a.scales = scales; a.status = status;
  a.T = static_cast<int>(K / kTileCols);
  a.C = a.tpc = a.nbuf = 0;
  const int64_t RB = nrb;
  auto go = [&](auto V) {
    constexpr int kVar = decltype(V)::value;
    if (bf16)
      return imp ? launch_build_t<true, true, kVar>(a, RB, stream, cluster_override)
                 : launch_build_t<true, false, kVar>(a, RB, stream, cluster_override);
    return imp ? launch_build_t<false, true, kVar>(a, RB, stream, cluster_override)
               : launch_build_t<false, false, kVar>(a, RB, stream, cluster_override);
  };
  switch (var) {
    case 1: return go(std::integral_constant<int, 1>{});
    case 2: return go(std::integral_constant<int, 2>{});
    case 3: return go(std::integral_constant<int, 3>{});
    default: return go(std::integral_constant<int, 0>{});
  }
}

}  // namespace usk

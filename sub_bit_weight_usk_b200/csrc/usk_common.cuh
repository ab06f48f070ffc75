// usk_common.cuh -- device helpers shared by the libusk kernels (sm_100a).
//
// Format constants and the hash of the sketch format (version 1, declared in
// include/usk.h).  The hash key of a tile is a SplitMix64 output (Steele, Lea
// and Flood, OOPSLA 2014), written here from its published definition.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "usk.h"

#include <type_traits>
#include <utility>

namespace usk {

// Compile-time loop: f(std::integral_constant<int, I>{}) for I = 0 .. N-1.
template <typename F, int... I>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, I...>) {
  (f(std::integral_constant<int, I>{}), ...);
}
template <int N, typename F>
__device__ __forceinline__ void static_for(F&& f) {
  static_for_impl(f, std::make_integer_sequence<int, N>{});
}

constexpr int kRowsPerBlock = 64;                                 // scale block and tile height
constexpr int kTileCols = 256;                                    // hash tile width
constexpr int kBucketsPerTile = kRowsPerBlock * kTileCols / 16;   // 1024
constexpr int kOctetsPerRow = kTileCols / 8;                      // 32

// SplitMix64 output number n of the generator seeded with `seed`.
__host__ __device__ __forceinline__ uint64_t splitmix64(uint64_t seed, uint64_t n) {
  uint64_t z = seed + n * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Multiply-shift hash key (A odd, C) of tile `tile_id`.
__host__ __device__ __forceinline__ uint2 tile_key(uint64_t seed, uint64_t tile_id) {
  uint64_t z = splitmix64(seed, tile_id + 1);
  return make_uint2(static_cast<uint32_t>(z) | 1u, static_cast<uint32_t>(z >> 32));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void sts16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

// [addr + OFF] forms: the constant offset is folded into the instruction.
template <int OFF>
__device__ __forceinline__ uint32_t lds32_off(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(OFF));
  return v;
}

template <int OFF>
__device__ __forceinline__ void atoms_max_u32_off(uint32_t addr, uint32_t v) {
  asm volatile("red.shared.max.u32 [%0+%2], %1;" ::"r"(addr), "r"(v), "n"(OFF) : "memory");
}

template <int OFF>
__device__ __forceinline__ void atoms_min_u32_off(uint32_t addr, uint32_t v) {
  asm volatile("red.shared.min.u32 [%0+%2], %1;" ::"r"(addr), "r"(v), "n"(OFF) : "memory");
}

__device__ __forceinline__ void atoms_max_u32(uint32_t addr, uint32_t v) {
  asm volatile("red.shared.max.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void atoms_min_u32(uint32_t addr, uint32_t v) {
  asm volatile("red.shared.min.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ uint4 ldg_nc128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// bf16 pair (low half = element 0) -> two fp32 values, exact.
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }


// ---------------------------------------------------------------- mbarriers

constexpr uint64_t kWaitNs = 1000000000ull;  // bound of every device-side wait (1 s)

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(addr), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase; false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity) {
  if (mbar_try_wait(addr, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(addr, parity)) {
    if (globaltimer_ns() - t0 > kWaitNs) return false;
  }
  return true;
}

// Arrive once and add `bytes` to the transaction count of the current phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t addr, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(addr), "r"(bytes) : "memory");
}

// 1-D bulk copy global -> this block's shared memory, completion counted on an
// mbarrier (no multicast).  Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(mbar)
      : "memory");
}

// 2-D tiled tensor copy global -> this block's shared memory (no multicast):
// box origin (x = column, y = row) of the tensor map; x * element size must be a
// multiple of 16 bytes; dst 128-byte aligned.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar)
      : "memory");
}

// The driver's tensor-map encoder, looked up once through the runtime (no libcuda link).
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts64(uint32_t addr, uint2 v) {
  asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(addr), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

template <int OFF>
__device__ __forceinline__ uint4 lds128_off(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4+%5];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr), "n"(OFF));
  return v;
}

// Predicated forms: the reduction happens only when key == ref (no branch).
template <int OFF>
__device__ __forceinline__ void atoms_min_u32_off_if_eq(uint32_t addr, uint32_t v, uint32_t key, uint32_t ref) {
  asm volatile(
      "{\n .reg .pred p;\n setp.eq.u32 p, %2, %3;\n @p red.shared.min.u32 [%0+%4], %1;\n}" ::"r"(addr), "r"(v),
      "r"(key), "r"(ref), "n"(OFF)
      : "memory");
}

template <int OFF>
__device__ __forceinline__ void atoms_min_u64_off_if_eq(uint32_t addr, uint64_t v, uint32_t key, uint32_t ref) {
  asm volatile(
      "{\n .reg .pred p;\n setp.eq.u32 p, %2, %3;\n @p red.shared.min.u64 [%0+%4], %1;\n}" ::"r"(addr), "l"(v),
      "r"(key), "r"(ref), "n"(OFF)
      : "memory");
}

template <int OFF>
__device__ __forceinline__ void atoms_max_u64_off(uint32_t addr, uint64_t v) {
  asm volatile("red.shared.max.u64 [%0+%2], %1;" ::"r"(addr), "l"(v), "n"(OFF) : "memory");
}

template <int OFF>
__device__ __forceinline__ void atoms_min_u64_off(uint32_t addr, uint64_t v) {
  asm volatile("red.shared.min.u64 [%0+%2], %1;" ::"r"(addr), "l"(v), "n"(OFF) : "memory");
}

// Address of the same shared-memory offset in cluster rank `rank`'s block.
__device__ __forceinline__ uint32_t mapa_cluster(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// One-way 16-byte store into a peer block's shared memory; completes 16 bytes
// of the transaction count of the peer's mbarrier `remote_bar` (both cluster
// addresses from mapa_cluster).
__device__ __forceinline__ void st_async_v4(uint32_t remote_addr, float a, float b, float c, float d,
                                            uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   remote_addr),
               "r"(__float_as_uint(a)), "r"(__float_as_uint(b)), "r"(__float_as_uint(c)), "r"(__float_as_uint(d)),
               "r"(remote_bar)
               : "memory");
}

__device__ __forceinline__ void report(uint32_t* d_status, uint32_t flags) {
  if (flags && d_status) atomicOr(d_status, flags);
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate (legacy warp-level MMA).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Bytes 0, 1 (sel 0x4140) or 2, 3 (sel 0x4342) of w, int8 codes, -> one bf16
// pair, exact, in four integer/FMA-pipe instructions (no conversion unit): the
// permute puts each byte b under a 0x43 high byte; with bit 7 cleared that is
// the bf16 value 128 + (b & 127), with only bit 7 kept it is 128 or 256; their
// difference is b as a two's-complement integer, exactly representable.
template <uint32_t SEL>
__device__ __forceinline__ uint32_t i8pair_to_bf16x2(uint32_t w) {
  const uint32_t p = __byte_perm(w, 0x43434343u, SEL);
  const uint32_t mag = p & 0xFF7FFF7Fu;                 // 128 + (b & 127)
  const uint32_t off = (p & 0x00800080u) | 0x43004300u;  // 128, or 256 when b < 0
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(mag), "r"(off));
  return r;
}

// Code layouts of the single-row max-key sketch (formats 1 and 4), by variant:
//   0: 4 slots per class, 8-bit codes (format 1, 0.5 bit/weight)
//   1: 8 slots, 4-bit codes (format 4, 0.5 bit/weight)
//   2: 2 slots, 8-bit codes (format 1 at 0.25 bit/weight)
//   3: 8 slots, 8-bit codes (format 1 at 1 bit/weight)
// slot = h >> kShift; a tile owns 256 * kSlots buckets; codes of tile (rb, tc)
// start at byte (rb * K/256 + tc) * kTileBytes.
template <int VAR>
struct CodeFmt {
  static constexpr uint32_t kSlots = VAR == 0 ? 4u : (VAR == 2 ? 2u : 8u);
  static constexpr bool kNibble = VAR == 1;
  static constexpr uint32_t kShift = kSlots == 2 ? 31u : (kSlots == 4 ? 30u : 29u);
  static constexpr uint32_t kBuckets = 256u * kSlots;                        // per tile
  static constexpr uint32_t kTileBytes = kNibble ? kBuckets / 2 : kBuckets;  // stored per tile
  static constexpr uint32_t kTileBf = 2u * kBuckets;                         // widened to bf16
};

// Format 4: 8 signed 4-bit codes (storage byte k holds bucket 2k in its low
// nibble, bucket 2k + 1 in its high nibble) -> 4 bf16 pairs in bucket order,
// exact: each nibble biased to u = n + 8 sits under a 0x43 exponent byte (the
// bf16 value 128 + u); subtracting 136 leaves n.
__device__ __forceinline__ void i4x8_to_bf16x8(uint32_t w, uint32_t (&o)[4]) {
  const uint32_t lo = (w & 0x0F0F0F0Fu) ^ 0x08080808u;         // biased low nibbles, one per byte
  const uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;  // biased high nibbles
  static_for<4>([&](auto Kc) {
    constexpr uint32_t k = decltype(Kc)::value;
    const uint32_t p = __byte_perm(lo, hi, k | (k << 4) | ((4u + k) << 8) | ((4u + k) << 12));
    const uint32_t v = (p & 0x00FF00FFu) | 0x43004300u;
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(0x43084308u));
    o[k] = r;
  });
}

// Format 2 (multi-row AbsMaxMin) decode: per 16-bit half, the bf16 code of
// larger magnitude of a and b (integer codes, |code| <= 127); ties keep a, the
// lower hash row.  (a | 0x8000) - |b| per half never borrows across halves and
// keeps bit 15 exactly when |a| >= |b| (bf16 magnitude bits order like values).
__device__ __forceinline__ uint32_t absmax_sel_bf16x2(uint32_t a, uint32_t b) {
  const uint32_t d = (a | 0x80008000u) - (b & 0x7FFF7FFFu);
  // mask 0xFFFF per half where bit 15 of the half is set: a byte permute whose
  // selectors 9 and 11 replicate the sign bit of bytes 1 and 3 (PTX prmt, default mode)
  uint32_t m;
  asm("prmt.b32 %0, %1, 0, 0xBB99;" : "=r"(m) : "r"(d));
  return (a & m) | (b & ~m);
}

__device__ __forceinline__ uint4 absmax_sel(uint4 a, uint4 b) {
  return make_uint4(absmax_sel_bf16x2(a.x, b.x), absmax_sel_bf16x2(a.y, b.y), absmax_sel_bf16x2(a.z, b.z),
                    absmax_sel_bf16x2(a.w, b.w));
}

// Key of hash row rho of tile `tile_id` in a depth-D sketch (format 2): the
// SplitMix64 output tile_id * D + rho + 1; D = 1 gives the format-1 key.
__host__ __device__ __forceinline__ uint2 row_key(uint64_t seed, uint64_t tile_id, int depth, int rho) {
  return tile_key(seed, tile_id * static_cast<uint64_t>(depth) + static_cast<uint64_t>(rho));
}

// ---- integer tensor path helpers (mma.sync m16n8k32 s8)

__device__ __forceinline__ void imma_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint2 ldg_nc64(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// bf16 bits -> (effective biased exponent, significand as an integer), subnormals with exponent 1
__device__ __forceinline__ void bf16_parts(uint32_t b, int& e_eff, int& mant) {
  const int e = static_cast<int>((b >> 7) & 0xFFu);
  const int m = static_cast<int>(b & 0x7Fu);
  e_eff = e == 0 ? 1 : e;
  mant = e == 0 ? m : (128 + m);
}

// Row blocks of one launch.  Uniform sketches: grid row g is row block g, its
// codes at g * T * tile bytes.  Per-row-block rates: grid row g is row block
// order[g] of the launch's slot group, its codes at offset[rb]; an entry out of
// range (rb outside [0, RB), a block ending past code_bytes, an offset not
// 16-byte aligned, or a block whose extent offset[rb + 1] - offset[rb] (the
// end of the codes for the last block) is not its group's) is reported and
// skipped by the whole cluster (every block of a cluster shares the grid row).
struct RbMap {
  const int32_t* order;   // nullptr: identity
  const int64_t* offset;
  int64_t code_bytes;
  int64_t RB;
};

__device__ __forceinline__ bool rb_resolve(const RbMap& m, int64_t g, int64_t rb_bytes, int& rb, int64_t& off) {
  if (m.order == nullptr) {
    rb = static_cast<int>(g);
    off = g * rb_bytes;
    return true;
  }
  const int64_t r = m.order[g];
  if (r < 0 || r >= m.RB) return false;
  const int64_t o = m.offset[r];
  if (o < 0 || (o & 15) != 0 || o + rb_bytes > m.code_bytes) return false;
  // the block's extent in the table (blocks are back to back in matrix order)
  // must be its group's: a block listed in the wrong slot group is refused
  const int64_t end = r + 1 < m.RB ? m.offset[r + 1] : m.code_bytes;
  if (end - o != rb_bytes) return false;
  rb = static_cast<int>(r);
  off = o;
  return true;
}

}  // namespace usk

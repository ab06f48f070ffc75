// usk_gemm.cu -- y = W_hat x for batch 16..256 on the 5th-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory).
//
// "UltraSketchLLM" explainer, Metodologia §4: decompression as the matrix
// product W_hat = S . P^T; here W_hat is decoded tile by tile straight into the
// tensor-core operand layout and never reaches global memory.
//
// Design (B200, sm_100a), warp-specialised pipeline:
//  * A thread block owns 128 output rows (two 64-row scale blocks) and a range
//    of whole hash tiles along K; blocks that split K for the same rows form a
//    cluster and add their fp32 partials through distributed shared memory in
//    rank order (deterministic, no workspace).
//  * The block's int8 codes (2 row blocks x its tiles) stream through a ring
//    of 8 raw tile slots, one bulk copy per row block and tile completing on
//    the slot's mbarrier; the widen warp refills a slot as soon as it has
//    read it (staging all tiles would hold shared memory that pipeline
//    stages and a second block per SM use better).  The widen warp converts
//    each tile's 2 x 1024 codes to bf16 once (instead of once per use: 16
//    uses) with an exact integer/FMA-pipe bit trick (the conversion unit of
//    one sub-partition was measured as the bottleneck), into a ring of tile
//    buffers guarded by ready/free mbarriers.
//  * 16 decoder warps: per 64-column chunk each thread rebuilds 2 octets of one
//    row -- one multiply-add of the hash per octet, one 16-byte conflict-free
//    gather of the 8 bf16 codes (class = (octet + row) mod 32) -- and writes
//    the 16 weights straight into tensor memory (tcgen05.st, its row is its
//    TMEM lane): the A operand never touches shared memory, which leaves the
//    shared-memory bandwidth to the code gathers and the B (x) operand.
//    For a multi-row AbsMaxMin sketch (format 2, depth D) the thread gathers
//    the octet from each of the D hash rows (segments of 2048/D bytes of the
//    widened tile, class = (octet + row) mod 32/D) and keeps, per weight, the
//    code of largest magnitude (integer select on the bf16 pairs).
//  * 1 copy warp: per chunk, as soon as the stage is free, one tensor copy of
//    the x tile (B operand, 128-byte swizzle) onto the stage's "full" barrier.
//  * I = 1, 2 or 4 MMA warps: warp i takes the chunks c = i (mod I); once the
//    stage is full, four tcgen05.mma (M=128, N=batch, K=16, A from tensor
//    memory, B from shared memory, bf16 -> fp32) into its own accumulator and
//    a commit to the stage's "empty" mbarrier.  A tcgen05.mma keeps its issuing
//    warp busy for about 180 cycles whatever N is (measured on B200), so at
//    small batches one issuer leaves the tensor core mostly idle; I x N <= 256
//    issuers fill it.  The epilogue adds the I accumulators in a fixed order.
//    A ring of stages lets decode, copy and MMA overlap.
//  * Epilogue: tcgen05.ld of the accumulator, x row-block scale, y.
//  * Every mbarrier wait is bounded (about 1 s); a wait that gives up sets
//    USK_FLAG_TIMEOUT, the pipeline stops, one final commit drains the tensor
//    core before tensor memory is freed, and the kernel returns.
#include <cooperative_groups.h>

#include "usk_common.cuh"

namespace cg = cooperative_groups;

namespace usk {

constexpr int kDecWarps = 16;
constexpr int kDecGroups = kDecWarps / 4;  // groups of 128 threads (one per row); group g decodes chunk g of every tile
constexpr int kWidenWarp = kDecWarps;      // widens each tile's codes to bf16, up to kTileRing tiles ahead
constexpr int kCopyWarp = kDecWarps + 1;   // lane 0 copies the x tiles ahead of the MMAs
constexpr int kMmaWarp0 = kDecWarps + 2;   // first MMA warp; it also owns the TMEM allocation
constexpr int kMaxIssuers = 4;             // MMA warps: a tcgen05.mma holds its issuing warp ~180 cycles
constexpr int kGemmThreads = (kDecWarps + 2 + kMaxIssuers) * 32;
constexpr int kTileRing = 4;               // bf16 tile-code buffers
constexpr int kRawRingMin = 8;             // raw tile-code slots (fewer only when a block has fewer tiles)
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kMaxStages = 16;  // pipeline stages (A in tensor memory, B in shared memory)
constexpr int kMaxTiles = 32;  // hash tiles per block (keys of each kept in shared memory)

struct GemmArgs {
  const int8_t* codes;
  const uint16_t* scales;
  float* y;
  int64_t M, K;
  uint64_t seed;
  uint32_t* status;
  int T;       // tiles per row block
  int N;       // batch (multiple of 16, <= 256)
  int splits;  // blocks along K per row tile (cluster size)
  uint32_t tmem_cols;
  uint32_t a_col;  // first tensor-memory column of the A stages
  int S;           // pipeline stages
  int I;           // MMA issuer warps, each with its own accumulator (columns [i N, (i + 1) N))
  int R;           // raw tile-code slots: min(tiles per block, kRawRingMin)
  int inject;  // test hook: block (0, 0) skips the x copy of its first chunk
  int pdl;     // launched as a programmatic dependent: x, scales, y and status only after the wait
  int early;   // let dependents launch after set-up (else after the main loop)
  RbMap map;    // grid rows -> row blocks and code offsets
  int64_t nrb;  // row blocks of this launch (a tile takes grid rows 2 mt and 2 mt + 1)
  int64_t g1, g2;  // per-row-block rates: where the 4- and 8-slot groups start in the order list
};

struct GemmLayout {
  uint32_t b, cbf, codes, keys, bars, misc, total;
};

// tile_bytes / tile_bf: stored and widened bytes per row block and tile
__host__ __device__ inline GemmLayout gemm_layout(int N, int tcta, int S, int depth, uint32_t tile_bytes,
                                                  uint32_t tile_bf, int R) {
  GemmLayout L;
  L.b = 0;  // [S][N x 64] bf16, SW128; after the main loop the K-split partials [N][128] fp32
  const uint32_t ring = static_cast<uint32_t>(S) * N * kBK * 2, parts = static_cast<uint32_t>(N) * kBM * 4;
  L.cbf = L.b + (ring > parts ? ring : parts);                         // bf16 [kTileRing][2][1024 or 2048]
  L.codes = L.cbf + kTileRing * 2u * tile_bf;                          // raw codes [R][2][tile_bytes]
  L.keys = L.codes + static_cast<uint32_t>(R) * 2u * tile_bytes;       // uint2 [2][tcta][depth]
  // full[S], empty[S], done, ready[ring], free[ring], raw[R]
  L.bars = (L.keys + 2u * tcta * depth * 8u + 7u) & ~7u;
  L.misc = L.bars + (2 * S + 1 + 2 * kTileRing + R) * 8;               // tmem holder, abort, 2 scales
  L.total = L.misc + 16;
  return L;
}

// Tensor memory: the issuers' fp32 accumulators [0, I N), then the A stages,
// 32 columns (128 rows x 64 bf16) each, from column a_col(N).
__host__ __device__ inline int gemm_issuers(int N) { return N <= 64 ? 4 : (N <= 128 ? 2 : 1); }
__host__ __device__ inline uint32_t gemm_a_col(int N, int I) {
  return (static_cast<uint32_t>(I * N) + 31u) & ~31u;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint32_t addr) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(addr) : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (start address and offsets in 16-byte units).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;           // leading byte offset (unused for this layout) = 16 B
  d |= static_cast<uint64_t>(1024 >> 4) << 32;   // stride byte offset = 1024 B
  d |= static_cast<uint64_t>(1) << 46;           // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;           // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor: D fp32, A and B bf16, both K-major, M = 128, N.
__device__ __forceinline__ uint32_t idesc_bf16_f32(int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(kBM >> 4) << 24);
}

// D (tmem) += A (tmem) * B (smem descriptor); accumulate = 0 overwrites D.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
               : "memory");
}

// 4 columns of this thread's lane into r without waiting: r must not be read
// before tmem_ld_wait4 has been given it
__device__ __forceinline__ void tmem_ld4_async(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}

// Waits for this thread's tensor-memory loads; the registers are operands, so
// no use of them is scheduled before the wait
__device__ __forceinline__ void tmem_ld_wait4(uint32_t (&r)[4][4]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0][0]), "+r"(r[0][1]), "+r"(r[0][2]), "+r"(r[0][3]), "+r"(r[1][0]), "+r"(r[1][1]),
                 "+r"(r[1][2]), "+r"(r[1][3]), "+r"(r[2][0]), "+r"(r[2][1]), "+r"(r[2][2]), "+r"(r[2][3]),
                 "+r"(r[3][0]), "+r"(r[3][1]), "+r"(r[3][2]), "+r"(r[3][3])
               :
               : "memory");
}

// D = hash rows of the sketch (1: format 1 or format 2 at depth 1; 2, 4: the
// multi-row AbsMaxMin sketch: the decoders gather every row and keep the code
// of largest magnitude)
// VAR: code layout (CodeFmt; D == 1 unless VAR == 0): the widen warp expands
// each row block's stored tile (512 to 2048 bytes) into 256 x slots bf16.
// mt: the tile within its slot group; order0 / nrb: where the group starts in
// the order list and its row blocks (the whole matrix for a uniform sketch).
template <int D, int VAR>
__device__ __forceinline__ void gemm_body(const GemmArgs& a, const CUtensorMap* xmap, int mt, int64_t order0,
                                          int64_t nrb) {
  using F = CodeFmt<VAR>;
  constexpr bool Q4 = F::kNibble;
  constexpr uint32_t kNc = 32u / D;  // classes per slot in one hash row
  constexpr uint32_t kRbBf = F::kTileBf;         // widened bytes per row block and tile
  constexpr uint32_t kRbBytes = F::kTileBytes;   // stored bytes per row block and tile
  constexpr uint32_t kShift = F::kShift;
  extern __shared__ __align__(16) uint8_t sm_raw[];
  cg::cluster_group cluster = cg::this_cluster();
  const int ks = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const uint32_t raw_s = smem_u32(sm_raw);
  const uint32_t s0 = (raw_s + 1023u) & ~1023u;
  uint8_t* sm = sm_raw + (s0 - raw_s);

  const int t_begin = static_cast<int>((static_cast<int64_t>(a.T) * ks) / a.splits);
  const int t_end = static_cast<int>((static_cast<int64_t>(a.T) * (ks + 1)) / a.splits);
  const int tcta = t_end - t_begin;
  const int nk = tcta * (kTileCols / kBK);  // 64-column chunks
  const int S = a.S;
  const int R = a.R;
  const GemmLayout L = gemm_layout(a.N, tcta, S, D, kRbBytes, kRbBf, R);
  const uint32_t bstage = static_cast<uint32_t>(a.N) * kBK * 2;
  const uint32_t full_s = s0 + L.bars, empty_s = full_s + 8 * S, done_bar = empty_s + 8 * S;
  const uint32_t ready_s = done_bar + 8, free_s = ready_s + 8 * kTileRing, rawbar_s = free_s + 8 * kTileRing;
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(sm + L.misc);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sm + L.misc + 4);
  volatile float* scale_s = reinterpret_cast<volatile float*>(sm + L.misc + 8);  // the tile's two row-block scales
  uint2* keytab = reinterpret_cast<uint2*>(sm + L.keys);
  // the tile's two row blocks and where their codes start; with a rate map a
  // block whose entry is out of range is skipped on its own (its rows are
  // neither decoded nor written), the other one of the tile still computed
  bool okA = false, okB = false;
  int rbA = 0, rbB = 0;
  int64_t cbA = 0, cbB = 0;
  {
    const bool has_b = 2 * static_cast<int64_t>(mt) + 1 < nrb;
    const int64_t rb_bytes = static_cast<int64_t>(a.T) * kRbBytes;
    RbMap gm = a.map;
    if (gm.order != nullptr) gm.order += order0;
    okA = rb_resolve(gm, 2 * static_cast<int64_t>(mt), rb_bytes, rbA, cbA);
    if (has_b) okB = rb_resolve(gm, 2 * static_cast<int64_t>(mt) + 1, rb_bytes, rbB, cbB);
    if ((!okA || (has_b && !okB)) && tid == 0 && ks == 0) {
      if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
      report(a.status, USK_FLAG_RATE_MAP);
    }
    if (!okA && !okB) return;  // the whole cluster (same tile) leaves before any barrier or allocation
  }
  // raw ring slot r holds tile t = r (mod R) of both row blocks; one
  // expect-tx arrive and one bulk copy per valid row block fill it
  const uint32_t raw_tx = kRbBytes * ((okA ? 1u : 0u) + (okB ? 1u : 0u));
  auto issue_raw = [&](int t) {
    const uint32_t slot = s0 + L.codes + static_cast<uint32_t>(t % R) * (2u * kRbBytes);
    const uint32_t bar = rawbar_s + 8u * static_cast<uint32_t>(t % R);
    mbar_arrive_expect_tx(bar, raw_tx);
    const int64_t toff = static_cast<int64_t>(t_begin + t) * kRbBytes;
    if (okA) bulk_g2s(slot, a.codes + cbA + toff, kRbBytes, bar);
    if (okB) bulk_g2s(slot + kRbBytes, a.codes + cbB + toff, kRbBytes, bar);
  };

  if (warp == kMmaWarp0) {
    if (lane == 0) {
      for (int s = 0; s < S; ++s) {
        mbar_init(full_s + 8 * s, 128 + 1);  // one decoder group + the x copy
        mbar_init(empty_s + 8 * s, 1);
      }
      mbar_init(done_bar, a.I);
      for (int q = 0; q < kTileRing; ++q) {
        mbar_init(ready_s + 8 * q, 32);           // the widen warp
        mbar_init(free_s + 8 * q, kDecThreads);   // every decoder
      }
      for (int r = 0; r < R; ++r) mbar_init(rawbar_s + 8 * r, 1);
      *abort_flag = 0u;
      mbar_fence_init();
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(xmap)) : "memory");
      // the first R tiles' codes (the widen warp issues the rest)
      for (int t = 0; t < R && t < tcta; ++t) issue_raw(t);
    }
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(const_cast<uint32_t*>(tmem_holder))),
                 "r"(a.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  } else if (tid < 2 * tcta * D) {
    const int rbl = tid / (tcta * D), tl = (tid / D) % tcta;
    keytab[tid] = row_key(a.seed, static_cast<uint64_t>(rbl ? rbB : rbA) * a.T + t_begin + tl, D, tid % D);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_holder;
  bool aborted = false;
  // dependents may launch now (grids of more blocks than SMs): their set-up,
  // code copies and decoding into tensor memory overlap this block's main
  // loop and epilogue
  if (a.early) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp < kDecWarps) {
    // ---------------- decoders: group g = warp / 4 rebuilds chunk g (octets
    // 8g .. 8g + 7) of every tile, thread = row; the four groups work on
    // different chunks concurrently
    const int m = tid & 127;  // row in the 128-row tile
    const int g = tid >> 7;
    const int rbl = m >> 6;
    const uint32_t r = static_cast<uint32_t>(m & 63);
    const bool row_ok = m < kRowsPerBlock ? okA : okB;
    // this thread's tensor-memory lane (= its row) in the A stages
    const uint32_t a_taddr = tmem_d + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + a.a_col;
    // loop exits are warp-uniform: tcgen05.st is a whole-warp instruction
    for (int t = 0; t < tcta && !aborted; ++t) {
      const int c = 4 * t + g;
      const int q = t % kTileRing;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(ready_s + 8 * q, static_cast<uint32_t>(t / kTileRing) & 1u))) {
        aborted = true;
        break;
      }
      const int s = c % S;
      if (c >= S) {
        // the MMAs that read this A stage have completed (they need x: under a
        // programmatic launch the bounded wait starts after the previous kernel)
        if (c - 4 < S && a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(empty_s + 8 * s, static_cast<uint32_t>(c / S - 1) & 1u))) {
          aborted = true;
          break;
        }
        tc_fence_after();
      }
      const uint32_t ob = static_cast<uint32_t>(8 * g);
      uint2 hk[D];
      uint32_t h[D];
#pragma unroll
      for (int rho = 0; rho < D; ++rho) {
        hk[rho] = keytab[(rbl * tcta + t) * D + rho];
        h[rho] = hk[rho].x * (32u * r + ob) + hk[rho].y;
      }
      const uint32_t tile_codes = s0 + L.cbf + q * (2u * kRbBf) + rbl * kRbBf;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {  // octets 4hh .. 4hh + 3 -> columns 16hh .. 16hh + 15 of the stage
        uint32_t v[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 w = make_uint4(0u, 0u, 0u, 0u);
          if (row_ok) {
            const uint32_t cls = (ob + 4u * hh + j + r) & (kNc - 1u);
#pragma unroll
            for (int rho = 0; rho < D; ++rho) {
              const uint4 u = lds128(tile_codes + static_cast<uint32_t>(rho) * (2048u / D) +
                                     ((h[rho] >> kShift) * kNc + cls) * 16u);
              w = rho == 0 ? u : absmax_sel(w, u);
            }
          }
          v[4 * j + 0] = w.x;
          v[4 * j + 1] = w.y;
          v[4 * j + 2] = w.z;
          v[4 * j + 3] = w.w;
#pragma unroll
          for (int rho = 0; rho < D; ++rho) h[rho] += hk[rho].x;
        }
        tmem_st(a_taddr + s * 32u + 16u * hh, v);
      }
      mbar_arrive(free_s + 8 * q);  // this thread is done with the tile's codes
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(full_s + 8 * s);
    }
  } else if (warp == kWidenWarp) {
    // ---------------- tile codes int8 -> bf16 (exact), kTileRing tiles ahead;
    // the raw codes stream in R tiles ahead (this warp refills a raw slot once
    // it has read it)
    int consumed = 0;  // raw tiles read by this warp
    for (int t = 0; t < tcta && !aborted; ++t) {
      const int q = t % kTileRing;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(rawbar_s + 8 * (t % R), static_cast<uint32_t>(t / R) & 1u))) {
        aborted = true;
        break;
      }
      // the decoders free a tile buffer only as the MMAs advance (they need x):
      // under a programmatic launch the bounded wait starts after the previous kernel
      if (t == kTileRing && a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
      if (t >= kTileRing &&
          !__all_sync(0xFFFFFFFFu, mbar_wait(free_s + 8 * q, static_cast<uint32_t>(t / kTileRing - 1) & 1u))) {
        aborted = true;
        break;
      }
      // 2 x kRbBytes stored bytes, 16 per lane per step; all loads in flight first
      constexpr int kSteps = static_cast<int>(2u * kRbBytes / 512u);
      const uint32_t slot = s0 + L.codes + static_cast<uint32_t>(t % R) * (2u * kRbBytes);
      uint4 w[kSteps];
#pragma unroll
      for (int i = 0; i < kSteps; ++i) {
        const uint32_t idx = static_cast<uint32_t>(lane) * 16u + static_cast<uint32_t>(i) * 512u;
        w[i] = lds128(slot + idx);  // [row block][kRbBytes] within the slot
      }
#pragma unroll
      for (int i = 0; i < kSteps; ++i) {
        const uint32_t idx = static_cast<uint32_t>(lane) * 16u + static_cast<uint32_t>(i) * 512u;
        if constexpr (Q4) {
          const uint32_t dst = s0 + L.cbf + q * (2u * kRbBf) + (idx / kRbBytes) * kRbBf + 4u * (idx % kRbBytes);
          const uint32_t ws[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t o4[4];
            i4x8_to_bf16x8(ws[e], o4);
            sts128(dst + 16u * e, make_uint4(o4[0], o4[1], o4[2], o4[3]));
          }
        } else {
          const uint32_t dst = s0 + L.cbf + q * (2u * kRbBf) + (idx / kRbBytes) * kRbBf + 2u * (idx % kRbBytes);
          sts128(dst, make_uint4(i8pair_to_bf16x2<0x4140>(w[i].x), i8pair_to_bf16x2<0x4342>(w[i].x),
                                 i8pair_to_bf16x2<0x4140>(w[i].y), i8pair_to_bf16x2<0x4342>(w[i].y)));
          sts128(dst + 16u, make_uint4(i8pair_to_bf16x2<0x4140>(w[i].z), i8pair_to_bf16x2<0x4342>(w[i].z),
                                       i8pair_to_bf16x2<0x4140>(w[i].w), i8pair_to_bf16x2<0x4342>(w[i].w)));
        }
      }
      mbar_arrive(ready_s + 8 * q);
      // the raw slot has been read (its values used above): refill it with tile
      // t + R (generic reads ordered before the async-proxy copy)
      consumed = t + 1;
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0 && t + R < tcta) issue_raw(t + R);
      __syncwarp();
    }
    // after a wait gave up: wait (bounded) for the raw copies still in flight
    if (aborted && lane == 0) {
      const int issued = tcta < consumed + R ? tcta : consumed + R;
      for (int t = consumed; t < issued; ++t) mbar_wait(rawbar_s + 8 * (t % R), static_cast<uint32_t>(t / R) & 1u);
    }
    __syncwarp();
  } else if (warp == kCopyWarp) {
    // ---------------- x tiles, up to S chunks ahead of the MMAs.  The whole
    // warp runs the loop (a lane spinning elsewhere would steal the warp from
    // the issuing lane); lane 0 issues.
    // x may come from the previous kernel in the stream: it is read only after
    // that kernel has completed (the codes and the decoding did not wait)
    if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
    // the scales for the epilogue, read once here, off its path
    if (lane < 2) scale_s[lane] = __half2float(__ushort_as_half(a.scales[lane ? rbB : rbA]));
    int s = 0;
    uint32_t ph = 0;
    for (int c = 0; c < nk && !aborted; ++c, s = (s + 1 == S) ? 0 : s + 1, ph ^= (s == 0) ? 1u : 0u) {
      if (c >= S && !__all_sync(0xFFFFFFFFu, mbar_wait(empty_s + 8 * s, ph ^ 1u))) {
        aborted = true;
        break;
      }
      if (lane == 0 && !(a.inject && c == 0 && ks == 0 && mt == 0)) {
        mbar_arrive_expect_tx(full_s + 8 * s, bstage);
        tma_load_2d(s0 + L.b + s * bstage, xmap, t_begin * kTileCols + c * kBK, 0, full_s + 8 * s);
      }
      __syncwarp();
    }
  } else if (warp >= kMmaWarp0 && warp < kMmaWarp0 + a.I) {
    // ---------------- MMAs: warp i takes chunks i, i + I, ... into accumulator i
    // (whole warp in the loop, lane 0 issues)
    const int i = warp - kMmaWarp0;
    if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");  // the x stages follow the previous kernel
    const uint32_t idesc = idesc_bf16_f32(a.N);
    const uint32_t d_tm = tmem_d + static_cast<uint32_t>(i * a.N);
    for (int c = i; c < nk && !aborted; c += a.I) {
      const int s = c % S;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(full_s + 8 * s, static_cast<uint32_t>(c / S) & 1u))) {
        aborted = true;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a_tm = tmem_d + a.a_col + s * 32u;
        const uint32_t bst = s0 + L.b + s * bstage;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          mma_bf16_ts(d_tm, a_tm + 8u * kk, sw128_desc(bst + 32 * kk), idesc, (c > i || kk > 0) ? 1u : 0u);
        mma_commit(empty_s + 8 * s);
      }
      __syncwarp();
    }
    // one more commit per issuer: tracks every MMA it issued (also after a failed wait)
    if (lane == 0) mma_commit(done_bar);
    __syncwarp();
  }
  if (aborted) *abort_flag = 1u;
  // one thread waits (bounded) for the tensor core to drain; the others wait in
  // the block barrier, which does not poll shared memory
  if (warp == kMmaWarp0 && lane == 0 && !mbar_wait(done_bar, 0)) *abort_flag = 1u;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // otherwise dependents launch now, over the epilogue: launched earlier, they
  // would take second slots on busy SMs and leave the next call unbalanced
  if (!a.early) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const bool failed = *abort_flag != 0u;
  // scales, y and status after the previous kernel (the copy warp has already
  // waited, so this returns at once)
  if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
  if (failed && tid == 0) report(a.status, USK_FLAG_TIMEOUT);

  // ---------------- epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31; the
  // kDecGroups groups of four warps take the 8-column groups round robin
  if (warp < kDecWarps) {
    const int sub = warp & 3, grp = warp >> 2;
    const int m = sub * 32 + lane;
    const int rbm = m < kRowsPerBlock ? rbA : rbB;
    const int64_t row = static_cast<int64_t>(rbm) * kRowsPerBlock + (m & 63);
    const bool row_ok = m < kRowsPerBlock ? okA : okB;
    const float scale = row_ok ? scale_s[m < kRowsPerBlock ? 0 : 1] : 0.0f;
    const uint32_t lane_base = static_cast<uint32_t>(sub * 32) << 16;
    float* part = reinterpret_cast<float*>(sm + L.b);  // [N][128]: the x stage ring is free now
    for (int n0 = 8 * grp; n0 < a.N; n0 += 8 * kDecGroups) {
      // the issuers' accumulators, every issuer's load in flight per wait (4
      // columns at a time), summed in issuer order
      float v[8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t u[kMaxIssuers][4] = {};
#pragma unroll
        for (int i = 0; i < kMaxIssuers; ++i)
          if (i < a.I) tmem_ld4_async(tmem_d + lane_base + static_cast<uint32_t>(i * a.N) + n0 + 4u * h, u[i]);
        tmem_ld_wait4(u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float t = __uint_as_float(u[0][e]);
#pragma unroll
          for (int i = 1; i < kMaxIssuers; ++i)
            if (i < a.I) t += __uint_as_float(u[i][e]);
          v[4 * h + e] = t;
        }
      }
      if (a.splits == 1) {
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            a.y[static_cast<int64_t>(n0 + i) * a.M + row] = (nk > 0 && !failed) ? v[i] * scale : 0.0f;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) part[(n0 + i) * kBM + m] = (nk > 0 && !failed) ? v[i] : 0.0f;
      }
    }
  }
  if (a.splits > 1) {
    cluster.sync();
    // rank ks finishes a slice of the outputs, adding the blocks in rank order
    float* part = reinterpret_cast<float*>(sm + L.b);
    const int total = a.N * kBM;
    const int per = (total + a.splits - 1) / a.splits;
    const int q0 = ks * per, q1 = min(total, q0 + per);
    for (int q = q0 + tid; q < q1; q += kGemmThreads) {
      // all remote loads in flight at once, then the sum in rank order
      float v[16];
#pragma unroll
      for (int s = 0; s < 16; ++s) v[s] = s < a.splits ? *cluster.map_shared_rank(&part[q], s) : 0.0f;
      float acc = 0.0f;
#pragma unroll
      for (int s = 0; s < 16; ++s) acc += v[s];
      const int n = q / kBM, mm = q % kBM;
      if (mm < kRowsPerBlock ? okA : okB) {
        const int rbm = mm < kRowsPerBlock ? rbA : rbB;
        const int64_t orow = static_cast<int64_t>(rbm) * kRowsPerBlock + (mm & 63);
        a.y[static_cast<int64_t>(n) * a.M + orow] = acc * scale_s[mm < kRowsPerBlock ? 0 : 1];
      }
    }
    cluster.sync();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d), "r"(a.tmem_cols)
                 : "memory");
  }
}

template <int D, int VAR>
__global__ void __launch_bounds__(kGemmThreads, 2) gemm_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap xmap) {
  gemm_body<D, VAR>(a, &xmap, static_cast<int>(blockIdx.y), 0, a.nrb);
}

// Per-row-block rates in one launch: the tiles of the 2-, 4- and 8-slot groups
// follow one another in grid y (a tile never mixes groups; an odd group leaves
// a one-block tile), so grid row y gives the group, its layout and its tile.
__global__ void __launch_bounds__(kGemmThreads, 2) gemm_vr_kernel(const GemmArgs a,
                                                                  const __grid_constant__ CUtensorMap xmap) {
  const int64_t c0 = a.g1, c1 = a.g2 - a.g1, c2 = a.map.RB - a.g2;
  const int64_t t0 = (c0 + 1) / 2, t1 = (c1 + 1) / 2;
  const int64_t y = blockIdx.y;
  if (y < t0) gemm_body<1, 2>(a, &xmap, static_cast<int>(y), 0, c0);
  else if (y < t0 + t1) gemm_body<1, 0>(a, &xmap, static_cast<int>(y - t0), a.g1, c1);
  else gemm_body<1, 3>(a, &xmap, static_cast<int>(y - t0 - t1), a.g2, c2);
}

// ---------------------------------------------------------------- launch

constexpr uint32_t kSmemLimit = 227u * 1024u;

static uint32_t var_tile_bytes(int var) {
  return var == 1 ? CodeFmt<1>::kTileBytes : var == 2 ? CodeFmt<2>::kTileBytes : var == 3 ? CodeFmt<3>::kTileBytes
                                                                                         : CodeFmt<0>::kTileBytes;
}
static uint32_t var_tile_bf(int var) {
  return var == 1 ? CodeFmt<1>::kTileBf : var == 2 ? CodeFmt<2>::kTileBf : var == 3 ? CodeFmt<3>::kTileBf
                                                                                   : CodeFmt<0>::kTileBf;
}

// 256 columns (two blocks per SM) when four stages fit next to the accumulators, else 512
__host__ __device__ inline uint32_t gemm_tmem_cols(int N, int I) {
  return gemm_a_col(N, I) + 4u * 32u <= 256u ? 256u : 512u;
}

// Raw tile-code slots for tpb tiles per block: min(tpb, kRawRingMin).  A ring
// of 8 was measured no slower than one slot per tile on every shape (and
// 21% faster at 28672x8192 batch 64, where the smaller footprint lets two
// blocks share an SM), even where staging every tile would cost no stages.
static int gemm_raw_ring(int tpb) { return tpb < kRawRingMin ? tpb : kRawRingMin; }

// Pipeline stages for batch N and tpb tiles per block: as many as tensor
// memory and shared memory (the B stages next to the raw code ring and the
// keys; half of the SM's when two blocks share it) hold, at most kMaxStages;
// 0 if fewer than 4.
//
// S is a multiple of 4: stage s = c mod S is then always filled by decoder
// group s mod 4 and consumed by MMA warp s mod I (I divides 4), so every
// mbarrier has one in-order waiter per role.  Otherwise consecutive uses of a
// stage belong to different warps, and a warp running ahead can take a
// completed phase of use n - 2 for use n (a phase wait only tells parity).
static int gemm_stages(int N, int tpb, int depth, int var, int I) {
  const uint32_t cols = gemm_tmem_cols(N, I);
  const uint32_t smem_cap = cols == 256u ? 233472u / 2u - 1024u : kSmemLimit;
  int S = static_cast<int>((cols - gemm_a_col(N, I)) / 32u);
  if (S > kMaxStages) S = kMaxStages;
  S &= ~3;
  const uint32_t tb = var_tile_bytes(var), tbf = var_tile_bf(var);
  while (S >= 4 && gemm_layout(N, tpb, S, depth, tb, tbf, gemm_raw_ring(tpb)).total + 1024u > smem_cap) S -= 4;
  return S >= 4 ? S : 0;
}

// Largest number of tiles per block (the keys of every tile are kept) that
// still leaves a four-stage pipeline for batch N.
static int gemm_max_tiles(int N, int depth, int var, int I) {
  int t = kMaxTiles;
  while (t > 1 && gemm_stages(N, t, depth, var, I) == 0) --t;
  return t;
}

// Dynamic shared memory of a launch: the layout, padded so that no more blocks
// share an SM than its 512 tensor-memory columns hold (a block waiting in
// tcgen05.alloc for a co-resident block of its own cluster would never proceed).
static uint32_t gemm_smem_bytes(int N, int tpb, int S, int depth, int var, int I) {
  const uint32_t tb = var_tile_bytes(var), tbf = var_tile_bf(var);
  const uint32_t smem = gemm_layout(N, tpb, S, depth, tb, tbf, gemm_raw_ring(tpb)).total + 1024u;
  const uint32_t max_blocks = 512u / gemm_tmem_cols(N, I);
  const uint32_t floor_bytes = 233472u / (max_blocks + 1u) + 1u - 1024u;  // 228 KiB per SM, 1 KiB reserved per block
  return smem > floor_bytes ? smem : floor_bytes;
}

// Blocks along K per 128-row tile: minimise (waves of blocks) x (tiles per
// block + 6 + the cluster's launch penalty), in units of about one tile's
// time.  Fitted to split sweeps on B200 (4096 x 4096, 11008 x 4096, 4096 x
// 11008, 28672 x 8192 at batch 16 and 64): a block's fixed cost (prologue,
// pipeline fill, epilogue, cluster reduction) is about 6 tiles; clusters of
// 5 to 8 blocks cost about 5 tiles more, larger ones about 14 more.  Within the
// shared-memory bound on tiles per block and clusters of at most 16.
//
// The MMA issuer count I is chosen with it: the default (4 up to batch 64, 2 up
// to 128, 1 above) keeps one block per SM where the accumulators need 512
// tensor-memory columns (batch 48 and 64); half the issuers fit two blocks per
// SM, which pays when there are more blocks than SMs (28672 x 8192 at batch 64:
// one wave of 224 instead of 1.5).  Two co-resident blocks share the SM, so
// such a plan is charged 1.5x per wave.
struct GemmPlan {
  int splits, I;
};

static GemmPlan gemm_plan(int64_t m_tiles, int T, int N, int sms, int depth, int var, int issuers_override) {
  const int I0 = gemm_issuers(N);
  GemmPlan best{-1, I0};
  int64_t best_cost = -1;
  for (int I = I0; I >= 1; I /= 2) {
    if (issuers_override > 0 && I != issuers_override) continue;
    if (issuers_override <= 0 && I != I0 && !(gemm_tmem_cols(N, I0) == 512u && gemm_tmem_cols(N, I) == 256u))
      continue;  // fewer issuers only where that fits a second block per SM
    const int max_tiles = gemm_max_tiles(N, depth, var, I);
    const int per_sm = 512 / static_cast<int>(gemm_tmem_cols(N, I));
    const int64_t slots = static_cast<int64_t>(sms) * per_sm;
    for (int s = 1; s <= 16 && s <= T; ++s) {
      const int tpb = (T + s - 1) / s;
      if (tpb > max_tiles) continue;
      const int64_t blocks = m_tiles * s;
      const int64_t waves = (blocks + slots - 1) / slots;
      int64_t cost = 2 * waves * (tpb + 6 + (s > 4 ? 5 : 0) + (s > 8 ? 9 : 0));
      if (I != I0 && blocks > sms) cost = cost * 3 / 2;  // two blocks sharing an SM
      if (best_cost < 0 || cost < best_cost) {
        best_cost = cost;
        best = GemmPlan{s, I};
      }
    }
  }
  return best;
}

// Whether K fits: at most 16 blocks along K, each staging the codes of up to
// gemm_max_tiles(batch) tiles (32 for every batch: K <= 131072).
bool gemm_supported(int64_t K, int batch, int depth, int var) {
  return K / kTileCols <= 16 * static_cast<int64_t>(gemm_max_tiles(batch, depth, var, gemm_issuers(batch)));
}

cudaError_t launch_gemm(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                        const uint16_t* x, int batch, float* y, uint32_t* status, cudaStream_t stream, int inject,
                        int depth, int var, const RbMap& map, int64_t nrb, int64_t g1, int64_t g2,
                        int splits_override, int issuers_override, bool pdl) {
  // a rate map: one launch over the tiles of every slot group, planned for the
  // 8-slot layout (the largest staged and widened tiles)
  const bool vr = map.order != nullptr;
  if (vr) {
    depth = 1;
    var = 3;
  }
  if ((depth != 1 && depth != 2 && depth != 4) || (var != 0 && depth != 1) || var < 0 || var > 3)
    return cudaErrorInvalidValue;
  GemmArgs a;
  a.codes = codes; a.scales = scales; a.y = y;
  a.M = M; a.K = K; a.seed = seed; a.status = status; a.inject = inject; a.pdl = pdl ? 1 : 0;
  a.T = static_cast<int>(K / kTileCols);
  a.N = batch;
  a.map = map;
  a.map.RB = M / kRowsPerBlock;
  a.nrb = nrb;
  a.g1 = g1;
  a.g2 = g2;
  const int64_t m_tiles = vr ? (g1 + 1) / 2 + (g2 - g1 + 1) / 2 + (a.map.RB - g2 + 1) / 2 : (nrb + 1) / 2;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // test hook: a given issuer count (1, 2 or 4 dividing the default's work)
  const int io = (issuers_override == 1 || issuers_override == 2 || issuers_override == 4) &&
                         issuers_override <= gemm_issuers(batch)
                     ? issuers_override
                     : 0;
  const GemmPlan plan = gemm_plan(m_tiles, a.T, batch, sms, depth, var, io);
  a.splits = plan.splits;
  a.I = plan.I;
  if (splits_override > 0) {  // test hook: a given split, where its tiles fit
    const int s = splits_override < a.T ? splits_override : a.T;
    if (s <= 16 && (a.T + s - 1) / s <= gemm_max_tiles(batch, depth, var, a.I)) a.splits = s;
  }
  if (a.splits < 1) return cudaErrorInvalidValue;  // K beyond 16 blocks x the tiles one block can stage
  a.tmem_cols = gemm_tmem_cols(batch, a.I);
  a.a_col = gemm_a_col(batch, a.I);
  const int tcta_max = (a.T + a.splits - 1) / a.splits;
  a.R = gemm_raw_ring(tcta_max);
  // measured: the early trigger pays where the grid already doubles up on SMs
  // (28672x8192 batch 64: 65.3 -> 61.3 us), the late one where it does not
  // (4096x11008 batch 16: 22.2 -> 17.1 us; 4096x4096: 10.1 -> 9.3 us)
  a.early = static_cast<int64_t>(a.splits) * m_tiles > sms ? 1 : 0;
  a.S = gemm_stages(batch, tcta_max, depth, var, a.I);
  if (a.S < 4 || a.S % 4 != 0) return cudaErrorInvalidValue;
  const size_t smem = gemm_smem_bytes(batch, tcta_max, a.S, depth, var, a.I);
  // tensor map over x [batch, K] bf16: one 64-column x batch box per chunk, 128-byte swizzle
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap xmap;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(batch)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(K) * 2u};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(batch)};
  const cuuint32_t estride[2] = {1, 1};
  if (encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), gdim, gstride, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  auto kern = vr ? gemm_vr_kernel
             : var == 1 ? gemm_kernel<1, 1>
             : var == 2 ? gemm_kernel<1, 2>
             : var == 3 ? gemm_kernel<1, 3>
             : (depth == 4 ? gemm_kernel<4, 0> : (depth == 2 ? gemm_kernel<2, 0> : gemm_kernel<1, 0>));
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (a.splits > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.splits, static_cast<unsigned>(m_tiles), 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, a, xmap);
}

}  // namespace usk

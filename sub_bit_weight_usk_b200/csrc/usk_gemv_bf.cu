// usk_gemv_bf.cu -- y = W_hat x for bf16 x at batch 1..8 with the fewest
// serial steps: x goes straight from global memory into the tensor-core B
// fragment, and the blocks of a row block meet only through one-way
// asynchronous stores into the first block's shared memory.
//
// "UltraSketchLLM" explainer, Metodologia §4: decompression is the product
// W_hat = S . P^T with a one-hot P; every weight (i, j) reads the code of the
// bucket its index hashes to, rehashed in registers once per octet of 8 columns.
//
// Design (B200, sm_100a):
//  * One thread block per (64-row block, tpc hash tiles); the C blocks of a row
//    block form a cluster.  The first instructions issue every global load the
//    block needs: lane (g, t) of warp w loads, for every tile, the 8 bf16 x
//    values of octet o = (w & 1) + 8 (w >> 1) + 2t of batch row g -- already
//    the B fragment of two mma.sync m16n8k16 (the reduction index is permuted
//    the same way for A and B, which the sum does not see) -- and 16 codes per
//    thread per 16 tiles' worth of codes.  No x staging, no x preparation, no
//    barrier set-up or bulk-copy issue ahead of the loads (measured: those
//    cost about 1000 cycles before the first byte moved).
//  * The codes are widened to bf16 in registers on arrival (exact: |code| <=
//    127), stored once, and gathered per (row, octet) with one 16-byte shared
//    load; because class = (o + row) mod 32 and the lanes of a quarter warp
//    cover rows g, g+1 and octets o0 + 2t, the 8 lanes hit 8 distinct 16-byte
//    bank groups.  Two accumulator sets (even and odd tiles) double the
//    independent MMA chains.
//  * Multi-row AbsMaxMin sketches (format 2, depth D): each hash row is
//    gathered the same way from its own 2048/D-byte segment of the widened
//    tile (class = (o + row) mod 32/D keeps a quarter warp on 8 distinct bank
//    groups), and the D words reduce to the code of largest magnitude with four
//    integer instructions per bf16 pair before the MMA.
//  * 4-bit codes (format 4): the 16-byte loads hold 32 nibbles, widened to bf16
//    the same way (exact), 4 KiB per tile; 8 hash slots (slot = h >> 29).
//  * fp32 accumulation of exact bf16 products; the 8 warps' sums are added in
//    a fixed order, then every block but the first writes its 64 x batch
//    partials into the first block's shared memory with st.async, which counts
//    the bytes on the first block's mbarrier; the first block waits only for
//    those bytes, adds the partials in rank order (deterministic) and scales.
#include <cooperative_groups.h>

#include "usk_common.cuh"

namespace cg = cooperative_groups;

namespace usk {

struct GemvBfArgs {
  const int8_t* codes;
  const uint16_t* scales;
  const uint16_t* x;  // bf16 [batch, K]
  float* y;
  int64_t M, K;
  uint64_t seed;
  uint32_t* status;
  int T, C, tpc;
  int pdl;     // launched as a programmatic dependent: wait before reading x
  int inject;  // test hook: block 1 of row block 0 skips its partial-sum stores
  RbMap map;   // grid row -> row block and code offset
  int64_t g1, g2;  // per-row-block rates: first grid rows of the 4- and 8-slot groups
};

constexpr int kBfThreads = 256;
constexpr int kBfMaxTiles = 8;  // tiles per block (x fragments live in registers)

struct GemvBfLayout {
  uint32_t cbf, keys, red, push, bars, total;
};

// tile_bf: widened bytes per tile (2 x buckets per tile)
__host__ __device__ inline GemvBfLayout gemv_bf_layout(int tpc, int batch, int C, int depth, uint32_t tile_bf) {
  GemvBfLayout L;
  L.cbf = 0;                                                       // bf16 [tpc][buckets per tile]
  L.keys = L.cbf + static_cast<uint32_t>(tpc) * tile_bf;          // uint2 [tpc][depth]
  L.red = (L.keys + static_cast<uint32_t>(tpc * depth) * 8u + 15u) & ~15u;  // fp32 [8 warps][batch][64]
  L.push = L.red + 8u * batch * 64u * 4u;                          // fp32 [C][batch][64] (used in rank 0)
  L.bars = (L.push + static_cast<uint32_t>(C) * batch * 64u * 4u + 7u) & ~7u;  // push
  L.total = L.bars + 8u;
  return L;
}

__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// remote 4-byte store into a peer block's shared memory, completing `4` bytes
// of the transaction count of the peer's mbarrier
__device__ __forceinline__ void st_async_f32(uint32_t remote_addr, float v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(remote_addr),
               "r"(__float_as_uint(v)), "r"(remote_bar)
               : "memory");
}

// D = hash rows of the sketch (1: format 1, or format 2 at depth 1; 2, 4: the
// multi-row AbsMaxMin sketch, whose rows are gathered and reduced to the code
// of largest magnitude before the MMA)
// VAR: code layout (CodeFmt; D == 1 unless VAR == 0): 2, 4 or 8 slots per
// class, 8-bit codes, or 8 slots with 4-bit codes (32 codes per 16-byte load).
template <int B, int D, int VAR>
__device__ __forceinline__ void gemv_bf_body(const GemvBfArgs& a, int64_t grid_row) {
  using F = CodeFmt<VAR>;
  constexpr bool Q4 = F::kNibble;
  constexpr uint32_t kNc = 32u / D;  // classes per slot in one hash row
  constexpr uint32_t kTileBf = F::kTileBf;  // widened bytes per tile
  constexpr uint32_t kShift = F::kShift;
  constexpr int kChunks = static_cast<int>(F::kTileBytes / 16u);  // 16-byte code loads per tile
  extern __shared__ __align__(128) uint8_t sm[];
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
  const int nt = min(a.tpc, a.T - t0);
  const GemvBfLayout L = gemv_bf_layout(a.tpc, B, a.C, D, kTileBf);
  const uint32_t s0 = smem_u32(sm);
  const uint32_t push_bar = s0 + L.bars;
  uint2* keytab = reinterpret_cast<uint2*>(sm + L.keys);
  float* red = reinterpret_cast<float*>(sm + L.red);
  float* push = reinterpret_cast<float*>(sm + L.push);
  constexpr uint32_t kPartBytes = static_cast<uint32_t>(B) * 64u * 4u;
  constexpr int kCodeLoads = kBfMaxTiles * kChunks / kBfThreads;  // 16-byte code loads per thread (at most)

  // ---- every global load first.  The codes are never written by a neighbour
  // in a programmatic-dependent chain (the caller's contract), so they go
  // before the dependency wait and overlap the previous kernel's tail; x after.
  const int8_t* codes_blk = a.codes + code_base + static_cast<int64_t>(t0) * F::kTileBytes;
  uint4 cv[kCodeLoads];
#pragma unroll
  for (int u = 0; u < kCodeLoads; ++u) {
    const int q = tid + u * kBfThreads;  // 16-code chunk
    cv[u] = make_uint4(0u, 0u, 0u, 0u);
    if (q < nt * kChunks) cv[u] = ldg_nc128(codes_blk + 16 * q);
  }
  if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
  const int g = lane >> 2, t = lane & 3;
  const int o = (warp & 1) + 8 * (warp >> 1) + 2 * t;  // this lane's octet in every tile
  uint4 xv[kBfMaxTiles];
#pragma unroll
  for (int tt = 0; tt < kBfMaxTiles; ++tt) {
    xv[tt] = make_uint4(0u, 0u, 0u, 0u);
    if (tt < nt && g < B)
      xv[tt] = ldg_nc128(a.x + static_cast<int64_t>(g) * a.K + static_cast<int64_t>(t0 + tt) * kTileCols + 8 * o);
  }
  if (tid == 0 && a.C > 1) {
    mbar_init(push_bar, 1);
    mbar_fence_init();
    if (crank == 0) mbar_arrive_expect_tx(push_bar, static_cast<uint32_t>(a.C - 1) * kPartBytes);
  }
  // first half of a split cluster barrier; its wait, before the first remote
  // store, guarantees that the first block's push barrier is initialised and
  // armed (the init is published by its cluster-scope fence).  Relaxed: a
  // release arrive would first wait for this thread's loads in flight.
  if (a.C > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  if (tid < nt * D) keytab[tid] = row_key(a.seed, static_cast<uint64_t>(rb) * a.T + t0 + tid / D, D, tid % D);

  // ---- codes: widen to bf16 once
#pragma unroll
  for (int u = 0; u < kCodeLoads; ++u) {
    const int q = tid + u * kBfThreads;
    if (q < nt * kChunks) {
      const uint32_t ws[4] = {cv[u].x, cv[u].y, cv[u].z, cv[u].w};
      if constexpr (Q4) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t o4[4];
          i4x8_to_bf16x8(ws[e], o4);
          sts128(s0 + L.cbf + 64u * q + 16u * e, make_uint4(o4[0], o4[1], o4[2], o4[3]));
        }
      } else {
        uint32_t o8[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          o8[2 * e] = i8pair_to_bf16x2<0x4140>(ws[e]);
          o8[2 * e + 1] = i8pair_to_bf16x2<0x4342>(ws[e]);
        }
        sts128(s0 + L.cbf + 32u * q, make_uint4(o8[0], o8[1], o8[2], o8[3]));
        sts128(s0 + L.cbf + 32u * q + 16u, make_uint4(o8[4], o8[5], o8[6], o8[7]));
      }
    }
  }
  __syncthreads();
  // blocks other than the first: the first block's push barrier is ready (this
  // wait overlaps nothing on their own path but is far from their tail)
  if (a.C > 1 && crank != 0) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");

  // ---- main loop: per tile and 16-row group, two MMAs (columns 0-3, 4-7 of
  // the octet); even and odd tiles accumulate into separate sets
  float d[2][4][4];
#pragma unroll
  for (int st = 0; st < 2; ++st)
#pragma unroll
    for (int mb = 0; mb < 4; ++mb)
#pragma unroll
      for (int e = 0; e < 4; ++e) d[st][mb][e] = 0.0f;
#pragma unroll
  for (int tt = 0; tt < kBfMaxTiles; ++tt) {
    if (tt < nt) {
      const uint32_t tile_s = s0 + L.cbf + tt * kTileBf;
      uint2 hk[D];
      uint32_t h[D];
#pragma unroll
      for (int rho = 0; rho < D; ++rho) {
        hk[rho] = keytab[tt * D + rho];
        h[rho] = hk[rho].x * (32u * g + o) + hk[rho].y;
      }
#pragma unroll
      for (int mb = 0; mb < 4; ++mb) {
        const uint32_t c0 = (static_cast<uint32_t>(o + g) + 16u * mb) & (kNc - 1u);  // row 16 mb + g
        const uint32_t c1 = (c0 + 8u) & (kNc - 1u);                                  // row 16 mb + g + 8
        uint4 q0 = make_uint4(0u, 0u, 0u, 0u), q1 = q0;
#pragma unroll
        for (int rho = 0; rho < D; ++rho) {
          const uint32_t h0 = h[rho] + static_cast<uint32_t>(mb) * 512u * hk[rho].x;
          const uint32_t h1 = h0 + 256u * hk[rho].x;
          const uint32_t seg = tile_s + static_cast<uint32_t>(rho) * (2048u / D);
          const uint4 u0 = lds128(seg + ((h0 >> kShift) * kNc + c0) * 16u);
          const uint4 u1 = lds128(seg + ((h1 >> kShift) * kNc + c1) * 16u);
          q0 = rho == 0 ? u0 : absmax_sel(q0, u0);
          q1 = rho == 0 ? u1 : absmax_sel(q1, u1);
        }
        mma_bf16_16816(d[tt & 1][mb], q0.x, q1.x, q0.y, q1.y, xv[tt].x, xv[tt].y);
        mma_bf16_16816(d[tt & 1][mb], q0.z, q1.z, q0.w, q1.w, xv[tt].z, xv[tt].w);
      }
    }
  }
  // dependents may start launching now: their code prefetch overlaps this epilogue
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- block sums: lane (g, t) holds rows 16 mb + g (+8) of batch rows 2t, 2t + 1
#pragma unroll
  for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int bi = 2 * t + (e & 1);
      const int r = 16 * mb + g + 8 * (e >> 1);
      if (bi < B) red[(warp * B + bi) * 64 + r] = d[0][mb][e] + d[1][mb][e];
    }
  }
  __syncthreads();
  // (batch row, row) pairs q = bi * 64 + r, kQ per thread
  constexpr int kQ = (B * 64 + kBfThreads - 1) / kBfThreads;
  float part[kQ];
#pragma unroll
  for (int k = 0; k < kQ; ++k) {
    const int q = tid + k * kBfThreads;
    part[k] = 0.0f;
    if (q < B * 64) {
#pragma unroll
      for (int w = 0; w < 8; ++w) part[k] += red[w * B * 64 + q];
    }
  }
  const float s = __half2float(__ushort_as_half(a.scales[rb]));
  float* yrb = a.y + static_cast<int64_t>(rb) * 64;
  if (a.C == 1) {
#pragma unroll
    for (int k = 0; k < kQ; ++k) {
      const int q = tid + k * kBfThreads;
      if (q < B * 64) yrb[static_cast<int64_t>(q / 64) * a.M + q % 64] = part[k] * s;
    }
    return;
  }
  if (crank != 0) {
    if (a.inject && crank == 1 && rb == 0) return;  // test hook: the first block's wait gives up
    const uint32_t bar0 = mapa_shared(push_bar, 0);
#pragma unroll
    for (int k = 0; k < kQ; ++k) {
      const int q = tid + k * kBfThreads;
      if (q < B * 64)
        st_async_f32(mapa_shared(s0 + L.push + (static_cast<uint32_t>(crank) * B * 64u + q) * 4u, 0), part[k], bar0);
    }
    return;
  }
#pragma unroll
  for (int k = 0; k < kQ; ++k) {
    const int q = tid + k * kBfThreads;
    if (q < B * 64) push[q] = part[k];
  }
  if (!mbar_wait(push_bar, 0)) report(a.status, USK_FLAG_TIMEOUT);  // bounded (about 1 s)
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kQ; ++k) {
    const int q = tid + k * kBfThreads;
    if (q < B * 64) {
      float tot = 0.0f;
      for (int c = 0; c < a.C; ++c) tot += push[c * B * 64 + q];
      yrb[static_cast<int64_t>(q / 64) * a.M + q % 64] = tot * s;
    }
  }
}

template <int B, int D, int VAR>
__global__ void __launch_bounds__(kBfThreads) gemv_bf_kernel(const GemvBfArgs a) {
  gemv_bf_body<B, D, VAR>(a, blockIdx.y);
}

// Per-row-block rates in one launch: grid row g is entry g of the rate map's
// order list (grouped by slot count), so its code layout follows from g.
template <int B>
__global__ void __launch_bounds__(kBfThreads) gemv_bf_vr_kernel(const GemvBfArgs a) {
  const int64_t g = blockIdx.y;
  if (g < a.g1) gemv_bf_body<B, 1, 2>(a, g);
  else if (g < a.g2) gemv_bf_body<B, 1, 0>(a, g);
  else gemv_bf_body<B, 1, 3>(a, g);
}

template <int B, int D, int VAR>
static cudaError_t launch_bf_t(GemvBfArgs a, int64_t nrb, cudaStream_t stream) {
  // a rate map: one launch over every row block, shared memory for 8 slots
  const bool vr = a.map.order != nullptr;
  const size_t smem = gemv_bf_layout(a.tpc, B, a.C, D, vr ? CodeFmt<3>::kTileBf : CodeFmt<VAR>::kTileBf).total;
  auto kern = vr ? gemv_bf_vr_kernel<B> : gemv_bf_kernel<B, D, VAR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (a.C > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.C, static_cast<unsigned>(nrb), 1);
  cfg.blockDim = dim3(kBfThreads, 1, 1);
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
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int D, int VAR>
static cudaError_t launch_bf_batch(const GemvBfArgs& a, int batch, int64_t RB, cudaStream_t stream) {
  switch (batch) {
    case 1: return launch_bf_t<1, D, VAR>(a, RB, stream);
    case 2: return launch_bf_t<2, D, VAR>(a, RB, stream);
    case 3: return launch_bf_t<3, D, VAR>(a, RB, stream);
    case 4: return launch_bf_t<4, D, VAR>(a, RB, stream);
    case 5: return launch_bf_t<5, D, VAR>(a, RB, stream);
    case 6: return launch_bf_t<6, D, VAR>(a, RB, stream);
    case 7: return launch_bf_t<7, D, VAR>(a, RB, stream);
    default: return launch_bf_t<8, D, VAR>(a, RB, stream);
  }
}

// Tiles per block: tpc_override if given, else the fewest tiles per block
// (most blocks) that keeps the cluster within 16 blocks, at least 4.
bool gemv_bf_supported(int64_t K, int batch, int tpc_override) {
  const int T = static_cast<int>(K / kTileCols);
  int tpc = tpc_override > 0 ? tpc_override : 4;
  while ((T + tpc - 1) / tpc > 16) ++tpc;
  return batch >= 1 && batch <= 8 && T >= 1 && tpc <= kBfMaxTiles;
}

cudaError_t launch_gemv_bf(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                           const uint16_t* x, int batch, float* y, uint32_t* status, bool pdl, cudaStream_t stream,
                           int tpc_override, int inject, int depth, int var, const RbMap& map, int64_t nrb,
                           int64_t g1, int64_t g2) {
  GemvBfArgs a;
  a.map = map;
  a.map.RB = M / kRowsPerBlock;
  a.g1 = g1;
  a.g2 = g2;
  if (map.order != nullptr) {  // the rate-map kernel covers every layout (depth 1)
    var = 0;
    depth = 1;
  }
  a.codes = codes; a.scales = scales; a.x = x; a.y = y;
  a.M = M; a.K = K; a.seed = seed; a.status = status;
  a.T = static_cast<int>(K / kTileCols);
  a.tpc = tpc_override > 0 ? tpc_override : 4;
  if (a.tpc > a.T) a.tpc = a.T;
  while ((a.T + a.tpc - 1) / a.tpc > 16) ++a.tpc;
  a.C = (a.T + a.tpc - 1) / a.tpc;
  a.pdl = pdl ? 1 : 0;
  a.inject = inject;
  const int64_t RB = nrb;
  if (var == 1) return launch_bf_batch<1, 1>(a, batch, RB, stream);
  if (var == 2) return launch_bf_batch<1, 2>(a, batch, RB, stream);
  if (var == 3) return launch_bf_batch<1, 3>(a, batch, RB, stream);
  if (depth == 2) return launch_bf_batch<2, 0>(a, batch, RB, stream);
  if (depth == 4) return launch_bf_batch<4, 0>(a, batch, RB, stream);
  return launch_bf_batch<1, 0>(a, batch, RB, stream);
}

}  // namespace usk

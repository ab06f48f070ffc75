// usk_gemv_i8.cu -- y = W_hat x for bf16 x at batch 1..4 on the integer tensor
// path: int8 codes straight from shared memory, x as four signed-byte digit
// planes.
//
// "UltraSketchLLM" explainer, Metodologia §4 (decompression W_hat = S . P^T,
// fused into the product here).  The codes are integers in [-127, 127]; the
// product sum_j code_j x_j is formed exactly in integer arithmetic:
//  * per thread block, each batch row of its x slice is written as
//    v_j * 2^(E - 156) with E the largest (biased) exponent in the slice and v_j
//    an integer of at most 30 bits (exact for every bf16 element within 2^22
//    of the largest; any other element, and any Inf/NaN, is left out of the
//    planes and added back by an exact scalar correction);
//  * v_j is split into balanced base-256 digits d_p in [-128, 127]
//    ((v + 0x80808080) ^ 0x80808080 gives their bytes), plane p = digit p;
//  * mma.sync m16n8k32 s8 x s8 -> s32 multiplies the gathered codes (A
//    fragment: one 8-byte load per row and octet, conflict-free because
//    class = (octet + row) mod 32) with the digit planes (B fragment: one
//    8-byte load), accumulating each plane in int32 (no overflow: |sum| <
//    K_block * 127 * 128);
//  * the four plane sums are recombined in 64-bit integers and the 8 warps
//    added (exact), scaled to float64, and the blocks of a row block send
//    their float64 partials into the first block's shared memory with
//    st.async (counted on its mbarrier); the first block adds them in rank
//    order and writes y = float(sum * scale).
// Shared-memory traffic of the gathers is one byte per weight (the bucket
// code), half of the bf16 path's.  Start-up follows the measured costs: every
// global load is issued first (codes with plain 16-byte loads, no bulk copy or
// barrier set-up ahead of them), no integer division in the x indexing, and a
// relaxed cluster arrive (a release arrive waits for the loads in flight).
#include <cooperative_groups.h>

#include "usk_common.cuh"

namespace cg = cooperative_groups;

namespace usk {

struct GemvI8Args {
  const int8_t* codes;
  const uint16_t* scales;
  const uint16_t* x;  // bf16 [batch, K]
  float* y;
  int64_t M, K;
  uint64_t seed;
  uint32_t* status;
  int T, C, tpc, batch;
  int pdl;     // launched as a programmatic dependent: wait before reading x
  int inject;  // test hook: block 1 of row block 0 skips its partial sums
};

constexpr int kI8Threads = 256;
constexpr int kI8MaxTiles = 32;                                     // tiles per block
constexpr int kI8CodeLoads = kI8MaxTiles * 1024 / 16 / kI8Threads;  // 16-byte code loads per thread
constexpr int kI8MaxChunks = 2048;                                  // 4-element x chunks: batch * tpc * 64
constexpr int kI8XR = kI8MaxChunks / kI8Threads;                    // x chunks per thread

struct GemvI8Layout {
  uint32_t codes, keys, xs, pitch, mask, emax, acc, push, bar, total;
};

__host__ __device__ inline GemvI8Layout gemv_i8_layout(int tpc, int batch, int C) {
  GemvI8Layout L;
  L.codes = 0;                                                 // int8 [tpc][1024]
  L.keys = static_cast<uint32_t>(tpc) * 1024u;                 // uint2 [tpc]
  L.xs = (L.keys + static_cast<uint32_t>(tpc) * 8u + 15u) & ~15u;
  L.pitch = static_cast<uint32_t>(tpc) * 256u + 8u;            // int8 plane row (+8: conflict-free)
  L.mask = (L.xs + 4u * batch * L.pitch + 15u) & ~15u;         // u32 [batch][tpc * 8] residual bits
  L.emax = L.mask + static_cast<uint32_t>(batch) * tpc * 32u;  // u32 [8]: exponents, any-residual
  L.acc = (L.emax + 32u + 15u) & ~15u;                         // s64 [8 warps][64][batch]
  L.push = L.acc + 8u * 64u * batch * 8u;                      // f64 [C][batch][64] (used in rank 0)
  L.bar = L.push + static_cast<uint32_t>(C) * 64u * batch * 8u;  // mbarrier
  L.total = L.bar + 8u;
  return L;
}

__device__ __forceinline__ uint32_t mapa_shared_u32(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// remote 8-byte store into a peer block's shared memory, completing 8 bytes of
// the transaction count of the peer's mbarrier
__device__ __forceinline__ void st_async_f64(uint32_t remote_addr, double v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];" ::"r"(remote_addr),
               "l"(__double_as_longlong(v)), "r"(remote_bar)
               : "memory");
}

// batch row of x chunk c when a row has cpr chunks (batch <= 4, no division)
__device__ __forceinline__ int chunk_row(int c, int cpr) {
  return c >= cpr ? (c >= 2 * cpr ? (c >= 3 * cpr ? 3 : 2) : 1) : 0;
}

template <int B>
__global__ void __launch_bounds__(kI8Threads) gemv_i8_kernel(const GemvI8Args a) {
  constexpr int NB = (4 * B + 7) / 8;  // n tiles of 8 planes
  constexpr int kQ = (B * 64 + kI8Threads - 1) / kI8Threads;
  extern __shared__ __align__(16) uint8_t sm[];
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int rb = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = crank * a.tpc;
  const int nt = min(a.tpc, a.T - t0);
  const GemvI8Layout L = gemv_i8_layout(a.tpc, B, a.C);
  const uint32_t s0 = smem_u32(sm);
  const uint32_t push_bar = s0 + L.bar;
  uint2* keytab = reinterpret_cast<uint2*>(sm + L.keys);
  uint32_t* mask = reinterpret_cast<uint32_t*>(sm + L.mask);
  uint32_t* emax = reinterpret_cast<uint32_t*>(sm + L.emax);  // [0..3] exponent, [4] any residual
  long long* acc = reinterpret_cast<long long*>(sm + L.acc);
  constexpr uint32_t kPartBytes = static_cast<uint32_t>(B) * 64u * 8u;

  // ---- every global load first.  The codes are never written by a neighbour
  // in a programmatic-dependent chain (the caller's contract), so they go
  // before the dependency wait; x after it.
  const int8_t* codes_blk = a.codes + static_cast<int64_t>(rb) * 4 * a.K + 1024 * static_cast<int64_t>(t0);
  uint4 cv[kI8CodeLoads];
#pragma unroll
  for (int u = 0; u < kI8CodeLoads; ++u) {
    const int q = tid + u * kI8Threads;  // 16-code chunk
    cv[u] = make_uint4(0u, 0u, 0u, 0u);
    if (q < nt * 64) cv[u] = ldg_nc128(codes_blk + 16 * q);
  }
  if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
  const int cpr = nt * 64;  // 4-element chunks per batch row
  uint2 xv[kI8XR];
#pragma unroll
  for (int u = 0; u < kI8XR; ++u) {
    const int c = tid + u * kI8Threads;
    xv[u] = make_uint2(0u, 0u);
    if (c < B * cpr) {
      const int bi = chunk_row(c, cpr), cc = c - bi * cpr;
      xv[u] = ldg_nc64(a.x + static_cast<int64_t>(bi) * a.K + static_cast<int64_t>(t0) * kTileCols + 4 * cc);
    }
  }
  if (tid == 0 && a.C > 1) {
    mbar_init(push_bar, 1);
    mbar_fence_init();
    if (crank == 0) mbar_arrive_expect_tx(push_bar, static_cast<uint32_t>(a.C - 1) * kPartBytes);
  }
  // first half of a split cluster barrier; its wait, before the first remote
  // store, guarantees that the first block's push barrier is set up (relaxed:
  // a release arrive would wait for this thread's loads in flight)
  if (a.C > 1) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  if (tid < nt) keytab[tid] = tile_key(a.seed, static_cast<uint64_t>(rb) * a.T + t0 + tid);
  if (tid < 8) emax[tid] = 0u;
  for (int q = tid; q < B * a.tpc * 8; q += kI8Threads) mask[q] = 0u;
#pragma unroll
  for (int u = 0; u < kI8CodeLoads; ++u) {
    const int q = tid + u * kI8Threads;
    if (q < nt * 64) sts128(s0 + L.codes + 16u * q, cv[u]);
  }

  // ---- x pass 1: largest finite exponent per batch row
  {
    int em[B];
#pragma unroll
    for (int bi = 0; bi < B; ++bi) em[bi] = 0;
#pragma unroll
    for (int u = 0; u < kI8XR; ++u) {
      const int c = tid + u * kI8Threads;
      if (c < B * cpr) {
        const int bi = chunk_row(c, cpr);
        const uint32_t w[2] = {xv[u].x, xv[u].y};
        int m = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t b = (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu);
          const int ex = static_cast<int>((b >> 7) & 0xFFu);
          if ((b & 0x7FFFu) != 0u && ex != 0xFF) m = max(m, ex == 0 ? 1 : ex);
        }
#pragma unroll
        for (int q = 0; q < B; ++q)
          if (q == bi) em[q] = max(em[q], m);
      }
    }
#pragma unroll
    for (int bi = 0; bi < B; ++bi) {
      const int m = __reduce_max_sync(0xFFFFFFFFu, em[bi]);
      if (lane == 0 && m > 0) atomicMax(&emax[bi], static_cast<uint32_t>(m));
    }
  }
  __syncthreads();

  // ---- x pass 2: digit planes (one 4-byte word per plane per chunk) and residual bits
#pragma unroll
  for (int u = 0; u < kI8XR; ++u) {
    const int c = tid + u * kI8Threads;
    if (c < B * cpr) {
      const int bi = chunk_row(c, cpr), cc = c - bi * cpr;
      const int E = static_cast<int>(emax[bi]);
      const uint32_t w[2] = {xv[u].x, xv[u].y};
      uint32_t dw[4];
      uint32_t rbits = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t b = (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu);
        int ee, mm;
        bf16_parts(b, ee, mm);
        const int sh = ee - E + 22;
        int v = 0;
        if (mm != 0) {
          if (((b >> 7) & 0xFFu) == 0xFFu || sh < 0) rbits |= 1u << e;  // handled by the exact correction
          else v = mm << sh;
        }
        if (b & 0x8000u) v = -v;
        dw[e] = (static_cast<uint32_t>(v) + 0x80808080u) ^ 0x80808080u;  // balanced base-256 digits
      }
      // 4x4 byte transpose: plane p gets byte p of the four columns' digit words
      const uint32_t t_0 = __byte_perm(dw[0], dw[1], 0x5140);
      const uint32_t t_1 = __byte_perm(dw[0], dw[1], 0x7362);
      const uint32_t t_2 = __byte_perm(dw[2], dw[3], 0x5140);
      const uint32_t t_3 = __byte_perm(dw[2], dw[3], 0x7362);
      const uint32_t pl[4] = {__byte_perm(t_0, t_2, 0x5410), __byte_perm(t_0, t_2, 0x7632),
                              __byte_perm(t_1, t_3, 0x5410), __byte_perm(t_1, t_3, 0x7632)};
#pragma unroll
      for (int p = 0; p < 4; ++p) sts32(s0 + L.xs + (4 * bi + p) * L.pitch + 4 * cc, pl[p]);
      if (rbits) {
        atomicOr(&mask[bi * a.tpc * 8 + (cc >> 3)], rbits << (4 * (cc & 7)));
        emax[4] = 1u;
      }
    }
  }
  __syncthreads();
  // blocks other than the first: the first block's push barrier is set up
  if (a.C > 1 && crank != 0) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");

  // ---- main loop: warp = column phase, lane (g, t) gathers octet o of rows g, g + 8
  const int g = lane >> 2, t = lane & 3;
  const int o = (warp & 3) + 16 * (warp >> 2) + 4 * t;
  const uint32_t c0 = static_cast<uint32_t>(o + g) & 31u;
  uint32_t cls8[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) cls8[k] = ((c0 + 8u * k) & 31u) * 8u;
  int d[4][NB][4];
#pragma unroll
  for (int mb = 0; mb < 4; ++mb)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) d[mb][nb][e] = 0;

  for (int tt = 0; tt < nt; ++tt) {
    const uint2 hk = keytab[tt];
    uint2 bq[NB];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int n = nb * 8 + g;
      bq[nb] = make_uint2(0u, 0u);
      if (n < 4 * B) bq[nb] = lds64(s0 + L.xs + n * L.pitch + tt * 256 + 8 * o);
    }
    const uint32_t tile_s = s0 + L.codes + tt * 1024u;
    const uint32_t h = hk.x * (32u * g + o) + hk.y;
    const uint32_t d512 = hk.x * 512u, d256 = hk.x * 256u;
#pragma unroll
    for (int mb = 0; mb < 4; ++mb) {
      const uint32_t h0 = h + mb * d512;
      const uint32_t h1 = h0 + d256;
      const uint2 q0 = lds64(tile_s + (h0 >> 30) * 256u + cls8[(2 * mb) & 3]);
      const uint2 q1 = lds64(tile_s + (h1 >> 30) * 256u + cls8[(2 * mb + 1) & 3]);
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) imma_16832(d[mb][nb], q0.x, q1.x, q0.y, q1.y, bq[nb].x, bq[nb].y);
    }
  }

  // dependents may start launching now: their code prefetch overlaps this epilogue
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- recombine the planes in 64-bit integers (exact); each warp stores its
  // sums, then the block adds the 8 warps (integer addition: exact).
  // Lanes with even t hold planes 0, 1 of batch row nb*2 + t/2, the next lane 2, 3.
#pragma unroll
  for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      int hi[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) hi[e] = __shfl_down_sync(0xFFFFFFFFu, d[mb][nb][e], 1);
      const int bi = nb * 2 + (t >> 1);
      if ((t & 1) == 0 && bi < B) {
        const long long v0 = static_cast<long long>(d[mb][nb][0]) + 256ll * d[mb][nb][1] + 65536ll * hi[0] +
                             16777216ll * hi[1];
        const long long v1 = static_cast<long long>(d[mb][nb][2]) + 256ll * d[mb][nb][3] + 65536ll * hi[2] +
                             16777216ll * hi[3];
        acc[(warp * 64 + 16 * mb + g) * B + bi] = v0;
        acc[(warp * 64 + 16 * mb + g + 8) * B + bi] = v1;
      }
    }
  }
  __syncthreads();

  // ---- block partial: scale and the exact correction for residual columns
  const bool any_resid = emax[4] != 0u;
  double part[kQ];
#pragma unroll
  for (int k = 0; k < kQ; ++k) {
    const int q = tid + k * kI8Threads;  // q = bi * 64 + r
    part[k] = 0.0;
    if (q < B * 64) {
      const int bi = q >> 6, r = q & 63;
      long long tot = 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) tot += acc[(w * 64 + r) * B + bi];
      double v = ldexp(static_cast<double>(tot), static_cast<int>(emax[bi]) - 156);
      if (any_resid) {
        double corr = 0.0;
        for (int wd = 0; wd < nt * 8; ++wd) {
          uint32_t bits = mask[bi * a.tpc * 8 + wd];
          while (bits) {
            const int j = __ffs(bits) - 1;
            bits &= bits - 1;
            const int col = wd * 32 + j;  // column inside this block's slice
            const int tt = col >> 8, c = col & 255, oc = c >> 3;
            const uint2 hk = keytab[tt];
            const uint32_t hh = hk.x * (32u * r + oc) + hk.y;
            const uint32_t bkt = ((hh >> 30) * 32u + ((oc + r) & 31u)) * 8u + (c & 7);
            const int code = static_cast<int8_t>(sm[L.codes + tt * 1024 + bkt]);
            const uint16_t xb = a.x[static_cast<int64_t>(bi) * a.K + static_cast<int64_t>(t0) * kTileCols + col];
            corr += static_cast<double>(code) * static_cast<double>(__uint_as_float(static_cast<uint32_t>(xb) << 16));
          }
        }
        v += corr;
      }
      part[k] = v;
    }
  }

  // ---- partials of the row block: into the first block, added in rank order
  const double s = static_cast<double>(__half2float(__ushort_as_half(a.scales[rb])));
  float* yrb = a.y + static_cast<int64_t>(rb) * 64;
  if (a.C == 1) {
#pragma unroll
    for (int k = 0; k < kQ; ++k) {
      const int q = tid + k * kI8Threads;
      if (q < B * 64) yrb[static_cast<int64_t>(q >> 6) * a.M + (q & 63)] = static_cast<float>(part[k] * s);
    }
    return;
  }
  double* push = reinterpret_cast<double*>(sm + L.push);
  if (crank != 0) {
    if (a.inject && crank == 1 && rb == 0) return;  // test hook: the first block's wait gives up
    const uint32_t bar0 = mapa_shared_u32(push_bar, 0);
#pragma unroll
    for (int k = 0; k < kQ; ++k) {
      const int q = tid + k * kI8Threads;
      if (q < B * 64)
        st_async_f64(mapa_shared_u32(s0 + L.push + (static_cast<uint32_t>(crank) * B * 64u + q) * 8u, 0), part[k],
                     bar0);
    }
    return;
  }
#pragma unroll
  for (int k = 0; k < kQ; ++k) {
    const int q = tid + k * kI8Threads;
    if (q < B * 64) push[q] = part[k];
  }
  if (!mbar_wait(push_bar, 0)) report(a.status, USK_FLAG_TIMEOUT);  // bounded (about 1 s)
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kQ; ++k) {
    const int q = tid + k * kI8Threads;
    if (q < B * 64) {
      double tot = 0.0;
      for (int c = 0; c < a.C; ++c) tot += push[c * B * 64 + q];
      yrb[static_cast<int64_t>(q >> 6) * a.M + (q & 63)] = static_cast<float>(tot * s);
    }
  }
}

template <int B>
static cudaError_t launch_i8_t(GemvI8Args a, int64_t RB, cudaStream_t stream) {
  const size_t smem = gemv_i8_layout(a.tpc, B, a.C).total;
  auto kern = gemv_i8_kernel<B>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.C, static_cast<unsigned>(RB), 1);
  cfg.blockDim = dim3(kI8Threads, 1, 1);
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

// T, C, tpc: the same block geometry as the staged-x bf16 path (C <= 8);
// batch * tpc * 64 <= kI8MaxChunks.
cudaError_t launch_gemv_i8(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                           const uint16_t* x, int batch, float* y, uint32_t* status, int T, int C, int tpc, bool pdl,
                           cudaStream_t stream, int inject) {
  GemvI8Args a;
  a.inject = inject;
  a.codes = codes; a.scales = scales; a.x = x; a.y = y;
  a.M = M; a.K = K; a.seed = seed; a.status = status;
  a.T = T; a.C = C; a.tpc = tpc; a.batch = batch; a.pdl = pdl ? 1 : 0;
  const int64_t RB = M / kRowsPerBlock;
  switch (batch) {
    case 1: return launch_i8_t<1>(a, RB, stream);
    case 2: return launch_i8_t<2>(a, RB, stream);
    case 3: return launch_i8_t<3>(a, RB, stream);
    default: return launch_i8_t<4>(a, RB, stream);
  }
}

}  // namespace usk

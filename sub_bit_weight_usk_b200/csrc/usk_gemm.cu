// usk_gemm.cu -- y = W_hat x for batch 16..256 on the 5th-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory).
//
// "UltraSketchLLM" explainer, Metodologia §4: decompression as the matrix
// product W_hat = S . P^T; here W_hat is decoded tile by tile straight into the
// tensor-core operand layout and never reaches global memory.
//
// Design (B200, sm_100a):
//  * A thread block owns 128 output rows (two 64-row scale blocks) and a range
//    of the K dimension; blocks that split K for the same rows form a cluster
//    and add their fp32 partials through distributed shared memory in rank
//    order (deterministic, no workspace).
//  * K advances in chunks of 64 columns.  Per chunk, each of the 128 threads
//    decodes the 8 octets of its row: rehash (one multiply-add per octet),
//    gather the 8 bf16 bucket codes with one 16-byte shared load from the
//    staged tile codes (conflict-free because class = (octet + row) mod 32),
//    and store them as one 16-byte chunk of the 128-byte-swizzled K-major
//    operand tile.  x is copied into the B operand tile with cp.async.
//  * One thread issues four tcgen05.mma (M=128, N=batch, K=16, bf16 x bf16 ->
//    fp32) per chunk and commits them to the chunk's stage barrier; a ring of
//    4 stages lets decoding run ahead of the tensor core.  Codes are exact in
//    bf16 and so are the products; the row-block scale is applied in the
//    epilogue after tcgen05.ld.
//  * Every mbarrier wait is bounded (about 1 s of globaltimer); a wait that
//    gives up sets USK_FLAG_TIMEOUT, the block skips the remaining work, frees
//    its tensor memory and returns.
#include <cooperative_groups.h>

#include "usk_common.cuh"

namespace cg = cooperative_groups;

namespace usk {

constexpr int kGemmThreads = 128;
constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kStages = 4;

struct GemmArgs {
  const int8_t* codes;
  const uint16_t* scales;
  const uint16_t* x;
  float* y;
  int64_t M, K;
  uint64_t seed;
  uint32_t* status;
  int T;       // tiles per row block
  int N;       // batch (multiple of 16, <= 256)
  int splits;  // blocks along K per row tile (cluster size)
  uint32_t tmem_cols;
  int inject;  // test hook: block (0, 0) skips the commit of its last chunk
};

__host__ __device__ constexpr size_t gemm_stage_a_bytes() { return kBM * kBK * 2; }  // 16 KiB
__host__ __device__ constexpr size_t gemm_stage_b_bytes(int N) { return static_cast<size_t>(N) * kBK * 2; }
__host__ __device__ constexpr size_t gemm_smem_bytes(int N) {
  // 1 KiB alignment slack | A stages | B stages | 2 code buffers (2 row blocks x 1024 bf16) | barriers
  return 1024 + kStages * (gemm_stage_a_bytes() + gemm_stage_b_bytes(N)) + 2 * 4096 + 192;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

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

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  const uint32_t no_mask = 0u;  // no output lane disabled
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(no_mask)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t bf16x2_from_i8(int lo, int hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(static_cast<float>(lo), static_cast<float>(hi));
  return *reinterpret_cast<uint32_t*>(&v);
}

// Load 16 codes (one 16-byte chunk) of tile tc for the block's row block
// rb_local, or zeros for a row block past the end of the matrix.
__device__ __forceinline__ uint4 load_code_chunk(const GemmArgs& a, int64_t rb, int tc, int chunk) {
  if (rb >= a.M / kRowsPerBlock) return make_uint4(0u, 0u, 0u, 0u);
  return ldg_nc128(a.codes + rb * 4 * a.K + 1024 * static_cast<int64_t>(tc) + 16 * chunk);
}

__device__ __forceinline__ void store_code_chunk(uint32_t dst, uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    o[2 * e] = bf16x2_from_i8(static_cast<int8_t>(w[e] & 0xFF), static_cast<int8_t>((w[e] >> 8) & 0xFF));
    o[2 * e + 1] = bf16x2_from_i8(static_cast<int8_t>((w[e] >> 16) & 0xFF), static_cast<int8_t>(w[e] >> 24));
  }
  sts128(dst, make_uint4(o[0], o[1], o[2], o[3]));
  sts128(dst + 16, make_uint4(o[4], o[5], o[6], o[7]));
}

__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const GemmArgs a) {
  extern __shared__ __align__(16) uint8_t sm_raw[];
  cg::cluster_group cluster = cg::this_cluster();
  const int ks = static_cast<int>(cluster.block_rank());
  const int mt = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5;

  const uint32_t raw_s = smem_u32(sm_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* base_g = sm_raw + (base_s - raw_s);
  const uint32_t a_s = base_s;
  const uint32_t b_s = a_s + kStages * static_cast<uint32_t>(gemm_stage_a_bytes());
  const uint32_t bstage = static_cast<uint32_t>(gemm_stage_b_bytes(a.N));
  const uint32_t c_s = b_s + kStages * bstage;  // code buffers: [2][2 row blocks][2048 B]
  const uint32_t bar_s = c_s + 2 * 4096;        // kStages stage mbarriers + 1 drain mbarrier (8 B each)
  const uint32_t drain_s = bar_s + 8 * kStages;
  uint8_t* misc_g = base_g + (bar_s - base_s) + 64;
  volatile uint32_t* tmem_holder = reinterpret_cast<volatile uint32_t*>(misc_g);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(misc_g + 4);

  // K range of this block (whole tiles)
  const int t_begin = static_cast<int>((static_cast<int64_t>(a.T) * ks) / a.splits);
  const int t_end = static_cast<int>((static_cast<int64_t>(a.T) * (ks + 1)) / a.splits);
  const int nk = (t_end - t_begin) * (kTileCols / kBK);  // chunks

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(bar_s + 8 * s, 1);
    mbar_init(drain_s, 1);
    *abort_flag = 0u;
    mbar_fence_init();
  }
  __syncwarp();
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(const_cast<uint32_t*>(tmem_holder))),
                 "r"(a.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }

  // this thread's decode row
  const int m = tid;
  const int64_t row = static_cast<int64_t>(mt) * kBM + m;
  const bool row_ok = row < a.M;
  const int rbl = m >> 6;                                   // row block inside the 128-row tile
  const int64_t rb = static_cast<int64_t>(mt) * 2 + rbl;    // global row block
  const uint32_t r = static_cast<uint32_t>(m & 63);

  // stage the first tile's codes; prefetch the next one into registers
  const int crbl = tid >> 6, cchunk = tid & 63;  // staging role: row block, 16-code chunk
  const int64_t crb = static_cast<int64_t>(mt) * 2 + crbl;
  uint4 pre = make_uint4(0u, 0u, 0u, 0u);
  if (nk > 0) {
    store_code_chunk(c_s + crbl * 2048 + 32 * cchunk, load_code_chunk(a, crb, t_begin, cchunk));
    if (t_begin + 1 < t_end) pre = load_code_chunk(a, crb, t_begin + 1, cchunk);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_holder;
  const uint32_t idesc = idesc_bf16_f32(a.N);
  bool aborted = false;

  // B (x) copies of chunk c into stage c % kStages
  auto issue_x = [&](int c) {
    const uint32_t dst_stage = b_s + (c % kStages) * bstage;
    const int64_t k0 = static_cast<int64_t>(t_begin) * kTileCols + static_cast<int64_t>(c) * kBK;
    for (int p = tid; p < a.N * 8; p += kGemmThreads) {
      const int n = p >> 3, c8 = p & 7;
      const uint32_t dst = dst_stage + (n >> 3) * 1024 + (n & 7) * 128 + ((c8 ^ (n & 7)) << 4);
      cp_async16(dst, a.x + static_cast<int64_t>(n) * a.K + k0 + 8 * c8);
    }
    cp_async_commit();
  };

  if (nk > 0) issue_x(0);
  uint2 hk = tile_key(a.seed, static_cast<uint64_t>(rb) * a.T + t_begin);

  for (int c = 0; c < nk; ++c) {
    const int tl = c >> 2;  // tile index inside this block's range
    const int tc = t_begin + tl;
    if ((c & 3) == 0 && c > 0) hk = tile_key(a.seed, static_cast<uint64_t>(rb) * a.T + tc);

    // the stage of chunk c + 1 must have been consumed by the MMAs of chunk c + 1 - kStages
    if (c + 1 < nk) {
      const int prev = c + 1 - kStages;
      if (prev >= 0 && !aborted) {
        if (!mbar_wait(bar_s + 8 * (prev % kStages), (prev / kStages) & 1)) aborted = true;
      }
      issue_x(c + 1);
    } else {
      cp_async_commit();  // keep the group count uniform
    }

    // decode the 8 octets of row m in this chunk into stage c % kStages
    const uint32_t a_stage = a_s + (c % kStages) * static_cast<uint32_t>(gemm_stage_a_bytes());
    const uint32_t cbuf = c_s + (tl & 1) * 4096 + rbl * 2048;
    const uint32_t arow = a_stage + (m >> 3) * 1024 + (m & 7) * 128;
    const uint32_t ob = static_cast<uint32_t>((c & 3) * 8);
    uint32_t h = hk.x * (32u * r + ob) + hk.y;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (row_ok) {
        const uint32_t cls = (ob + j + r) & 31u;
        v = lds128(cbuf + ((h >> 30) * 32u + cls) * 16u);
      }
      sts128(arow + ((static_cast<uint32_t>(j) ^ static_cast<uint32_t>(m & 7)) << 4), v);
      h += hk.x;
    }

    // last chunk of a tile: stage the next tile's codes into the other buffer
    if ((c & 3) == 3 && tl + 1 < t_end - t_begin) {
      store_code_chunk(c_s + ((tl + 1) & 1) * 4096 + crbl * 2048 + 32 * cchunk, pre);
      if (tc + 2 < t_end) pre = load_code_chunk(a, crb, tc + 2, cchunk);
    }

    cp_async_wait<1>();  // this chunk's x copies have landed
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (aborted) *abort_flag = 1u;
    if (tid == 0 && !*abort_flag) {
      tc_fence_after();
      const uint32_t bst = b_s + (c % kStages) * bstage;
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk) {
        mma_bf16(tmem_d, sw128_desc(a_stage + 32 * kk), sw128_desc(bst + 32 * kk), idesc,
                 (c > 0 || kk > 0) ? 1u : 0u);
      }
      const bool skip = a.inject && c == nk - 1 && ks == 0 && mt == 0;
      if (!skip) mma_commit(bar_s + 8 * (c % kStages));
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  aborted = aborted || (*abort_flag != 0u);

  // Wait for the last chunk's MMAs (bounded).  If any wait gave up, thread 0
  // commits once more to a dedicated barrier -- a commit tracks every earlier
  // MMA of the issuing thread -- and the block waits for it (bounded again),
  // so that no MMA is in flight when tensor memory is freed.
  if (!aborted && nk > 0) {
    const int last = nk - 1;
    if (!mbar_wait(bar_s + 8 * (last % kStages), (last / kStages) & 1)) aborted = true;
  }
  aborted = __syncthreads_or(aborted ? 1 : 0) != 0;
  if (aborted) {
    if (tid == 0) mma_commit(drain_s);
    mbar_wait(drain_s, 0);
    report(a.status, USK_FLAG_TIMEOUT);
  }
  tc_fence_after();

  // ---- epilogue: TMEM -> registers (this warp's 32 lanes = rows 32 warp .. +31)
  const float scale = row_ok ? __half2float(__ushort_as_half(a.scales[rb])) : 0.0f;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  if (a.splits == 1) {
    for (int n0 = 0; n0 < a.N; n0 += 16) {
      float v[16];
      tmem_ld16(tmem_d + lane_base + n0, v);
      if (row_ok && nk > 0 && !aborted) {
#pragma unroll
        for (int i = 0; i < 16; ++i) a.y[static_cast<int64_t>(n0 + i) * a.M + row] = v[i] * scale;
      } else if (row_ok) {
#pragma unroll
        for (int i = 0; i < 16; ++i) a.y[static_cast<int64_t>(n0 + i) * a.M + row] = 0.0f;
      }
    }
  } else {
    // partials to this block's shared memory as [n][128] (the stage area is free now)
    float* part = reinterpret_cast<float*>(base_g);
    for (int n0 = 0; n0 < a.N; n0 += 16) {
      float v[16];
      tmem_ld16(tmem_d + lane_base + n0, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) part[(n0 + i) * kBM + m] = (nk > 0 && !aborted) ? v[i] : 0.0f;
    }
    cluster.sync();
    // rank ks reduces a slice of the outputs, adding the blocks in rank order
    const int total = a.N * kBM;
    const int per = (total + a.splits - 1) / a.splits;
    const int q0 = ks * per, q1 = min(total, q0 + per);
    for (int q = q0 + tid; q < q1; q += kGemmThreads) {
      float acc = 0.0f;
      for (int s = 0; s < a.splits; ++s) acc += *cluster.map_shared_rank(&part[q], s);
      const int n = q / kBM, mm = q % kBM;
      const int64_t orow = static_cast<int64_t>(mt) * kBM + mm;
      if (orow < a.M) {
        const float sc = __half2float(__ushort_as_half(a.scales[orow / kRowsPerBlock]));
        a.y[static_cast<int64_t>(n) * a.M + orow] = acc * sc;
      }
    }
    cluster.sync();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d), "r"(a.tmem_cols)
                 : "memory");
  }
}

// ---------------------------------------------------------------- launch

static int gemm_splits(int64_t m_tiles, int T) {
  int s = static_cast<int>(296 / (m_tiles > 0 ? m_tiles : 1));
  if (s < 1) s = 1;
  if (s > 8) s = 8;
  if (s > T) s = T;
  return s;
}

static uint32_t tmem_columns(int N) {
  uint32_t c = 32;
  while (c < static_cast<uint32_t>(N)) c <<= 1;
  return c;
}

cudaError_t launch_gemm(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                        const uint16_t* x, int batch, float* y, uint32_t* status, cudaStream_t stream, int inject) {
  GemmArgs a;
  a.inject = inject;
  a.codes = codes; a.scales = scales; a.x = x; a.y = y;
  a.M = M; a.K = K; a.seed = seed; a.status = status;
  a.T = static_cast<int>(K / kTileCols);
  a.N = batch;
  const int64_t m_tiles = (M + kBM - 1) / kBM;
  a.splits = gemm_splits(m_tiles, a.T);
  a.tmem_cols = tmem_columns(batch);
  const size_t smem = gemm_smem_bytes(batch);
  cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.splits, static_cast<unsigned>(m_tiles), 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_kernel, a);
}

}  // namespace usk

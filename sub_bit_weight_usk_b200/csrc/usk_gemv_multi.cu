// usk_gemv_multi.cu -- y_l = W_hat_l x_l for one or several sketches in one
// launch (batch 1..8, bf16 x): a persistent, software-pipelined kernel.
//
// "UltraSketchLLM" explainer, Metodologia §4: decompression is the product
// W_hat = S . P^T with a one-hot P -- every weight (i, j) reads back the code
// of the bucket its index hashes to.  The math of one 64 x 1024 chunk is the
// same as in the single-launch kernels (octet hash in registers, conflict-free
// 16-byte gathers of bf16-widened codes as the A fragment of mma.sync, x as
// the B fragment); what changes is how the chunks are fed and summed.
//
// Design (B200, sm_100a):
//  * Work item = (linear l, 64-row block rb, segment of its 1024-column
//    chunks).  A row is one segment unless the launch has too few row blocks
//    to fill the GPU; then rows split into a few segments (the host picks the
//    split that minimises waves x segment length).  The items of all the
//    launch's linears form one list; the grid is as many thread blocks as fit
//    on the GPU at once (never more than the items) and block b takes items
//    b, b + G, ... in order.
//  * 8 math warps stream the block's chunks through a ring of 3 shared-memory
//    stages: one thread issues, per chunk, a bulk copy of its codes
//    (contiguous in the format) and one per batch row of its x slice onto the
//    stage's mbarrier, 3 chunks ahead of the math.  Per chunk: codes widened
//    to bf16 once (exact) into one of two buffers, tile keys (SplitMix64),
//    x fragments, one barrier among the math warps, then 4 tiles x 4 16-row
//    groups x two m16n8k16 MMAs per warp, ACCUMULATED across the chunks of the
//    item in registers.  Consecutive products in a stream (programmatic
//    dependent launch): the first chunks' code copies go out before the
//    dependency wait, x after it.
//  * At the end of an item the 8 warps' sums go to one of two shared buffers
//    and a 9th warp finishes the item while the math warps go on: it adds the
//    8 warps in a fixed order and writes y -- or, for a split row, the
//    segment's partial sums to the caller's workspace followed by a
//    release/acquire count on the row's counter; the block whose segment
//    arrives last adds the partials in segment order (deterministic), writes
//    y and returns the counter to zero.  It reads its own count one item
//    later, so the atomic's round trip overlaps the next item.
//  * Every mbarrier wait is bounded (about 1 s): a wait that gives up sets
//    USK_FLAG_TIMEOUT, and the block waits (bounded) for its copies in flight
//    before it leaves; that call's outputs and workspace counters are then
//    undefined.
#include <cuda/atomic>
#include <mutex>

#include "usk_common.cuh"

namespace usk {

constexpr int kMlThreads = 288;  // 8 math warps + 1 epilogue warp
constexpr int kMlMath = 256;
constexpr int kMlMaxLinears = 16;
constexpr int kMlTiles = 4;   // hash tiles per chunk (1024 columns)
constexpr int kMlStages = 3;  // chunks in flight per block

struct MlLinear {
  const int8_t* codes;
  const uint16_t* scales;
  const uint16_t* x;  // bf16 [batch, K]
  float* y;           // [batch, M]
  int64_t M, K;
  uint64_t seed;
  int64_t item0;  // first work item of this linear in the launch's list
  int64_t part0;  // first partial slot (Bp x 64 floats each) when nseg > 1
  int64_t cnt0;   // first row-block counter when nseg > 1
  int T, nch;     // hash tiles per row, chunks per row
  int nseg, seglen;  // segments per row, chunks per segment
};

struct MlArgs {
  MlLinear lin[kMlMaxLinears];
  int n;
  int batch;
  int64_t items;
  float* part;    // workspace: partial sums of split rows
  uint32_t* cnt;  // workspace: one arrival counter per split row block
  uint32_t* status;
  int pdl;
  int inject;  // test hook: block 0 never issues the x copies of its first chunk
};

struct MlLayout {
  uint32_t stage, stage_bytes, cbf, keys, red, bars, misc, total;
};

template <int B, int D, int VAR>
__host__ __device__ constexpr MlLayout ml_layout() {
  using F = CodeFmt<VAR>;
  MlLayout L{};
  L.stage = 0;
  L.stage_bytes = ((kMlTiles * F::kTileBytes + B * kMlTiles * 512u) + 127u) & ~127u;  // codes | x [B][1024]
  L.cbf = L.stage + kMlStages * L.stage_bytes;                                      // bf16 [2][4][tile_bf]
  L.keys = L.cbf + 2u * kMlTiles * F::kTileBf;                                      // uint2 [2][4][D]
  L.red = (L.keys + 2u * kMlTiles * D * 8u + 15u) & ~15u;                           // fp32 [2][8][B][64]
  L.bars = L.red + 2u * 8u * B * 64u * 4u;                                          // full[S], rfull[2], rempty[2]
  L.misc = L.bars + 8u * (kMlStages + 4);                                           // flags, issue cursor
  L.total = L.misc + 64u;
  return L;
}

struct MlItem {
  int l;
  int64_t rb;
  int seg, c0, c1;  // segment and its chunks [c0, c1)
};

__device__ __forceinline__ MlItem ml_item(const MlArgs& a, int64_t it) {
  int l = 0;
  while (l + 1 < a.n && it >= a.lin[l + 1].item0) ++l;
  const MlLinear& L = a.lin[l];
  const uint32_t q = static_cast<uint32_t>(it - L.item0);  // items of one linear < 2^31
  const uint32_t ns = static_cast<uint32_t>(L.nseg);
  MlItem r;
  r.l = l;
  r.rb = static_cast<int64_t>(q / ns);
  r.seg = static_cast<int>(q - (q / ns) * ns);
  r.c0 = r.seg * L.seglen;
  r.c1 = min(L.nch, r.c0 + L.seglen);
  return r;
}

__device__ __forceinline__ int ml_nt(const MlLinear& L, int c) { return min(kMlTiles, L.T - c * kMlTiles); }

// bulk copies of chunk c of item m into stage buffer `dst`, completing on `bar`
template <int VAR>
__device__ __forceinline__ void ml_copy_codes(const MlArgs& a, const MlItem& m, int c, uint32_t dst, uint32_t bar) {
  using F = CodeFmt<VAR>;
  const MlLinear& L = a.lin[m.l];
  const int nt = ml_nt(L, c);
  mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nt) * (F::kTileBytes + 512u * static_cast<uint32_t>(a.batch)));
  bulk_g2s(dst, L.codes + (m.rb * L.T + c * kMlTiles) * static_cast<int64_t>(F::kTileBytes),
           static_cast<uint32_t>(nt) * F::kTileBytes, bar);
}

__device__ __forceinline__ void ml_copy_x(const MlArgs& a, const MlItem& m, int c, uint32_t dst, uint32_t bar) {
  const MlLinear& L = a.lin[m.l];
  const int nt = ml_nt(L, c);
  for (int g = 0; g < a.batch; ++g)
    bulk_g2s(dst + static_cast<uint32_t>(g) * (kMlTiles * 512u),
             L.x + g * L.K + static_cast<int64_t>(c) * (kMlTiles * kTileCols), static_cast<uint32_t>(nt) * 512u, bar);
}

// bar.sync / bar.red.or on a named barrier among the math warps only
__device__ __forceinline__ void math_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool math_bar_or(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
      : "memory");
  return r != 0u;
}

__device__ __forceinline__ void mbar_arrive_cta(uint32_t addr) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(addr) : "memory");
}

// Epilogue warp, a split row block whose segments have all arrived: sum the
// segments' partials in segment order (loads 8 at a time in flight), scale,
// write y, return the counter to zero.
template <int B>
__device__ __forceinline__ void ml_finish(const MlArgs& a, int l, int64_t rb, int lane) {
  const MlLinear& L = a.lin[l];
  // acquire side of the arrival counter: lane 0 read the last arrival (relaxed
  // part of its release RMW); its acquire fence, then the warp barrier, order
  // every lane's loads below after all segments' releases
  cuda::atomic_thread_fence(cuda::memory_order_acquire, cuda::thread_scope_device);
  __syncwarp();
  const float s = __half2float(__ushort_as_half(L.scales[rb]));
  const float* pbase = a.part + (L.part0 + rb * L.nseg) * static_cast<int64_t>(B * 64);
  for (int q = lane; q < a.batch * 64; q += 32) {
    float tot = 0.0f;
    for (int c0 = 0; c0 < L.nseg; c0 += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = c0 + u < L.nseg ? __ldcg(pbase + static_cast<int64_t>(c0 + u) * (B * 64) + q) : 0.0f;
#pragma unroll
      for (int u = 0; u < 8; ++u) tot += v[u];
    }
    L.y[static_cast<int64_t>(q / 64) * L.M + rb * 64 + q % 64] = tot * s;
  }
  if (lane == 0) a.cnt[L.cnt0 + rb] = 0u;
}

// The block's chunk sequence (items b, b + G, ..., each its chunks in order),
// walked by the issuing thread.
struct MlCursor {
  int k;  // item index within the block
  int c;  // chunk
  MlItem m;
};

__device__ __forceinline__ void ml_cursor_next(const MlArgs& a, MlCursor& cu, int64_t first, int64_t G, int my) {
  if (++cu.c < cu.m.c1) return;
  if (++cu.k < my) {
    cu.m = ml_item(a, first + cu.k * G);
    cu.c = cu.m.c0;
  }
}

template <int B, int D, int VAR>
__global__ void __launch_bounds__(kMlThreads, 2) gemv_multi_kernel(const __grid_constant__ MlArgs a) {
  using F = CodeFmt<VAR>;
  constexpr bool Q4 = F::kNibble;
  constexpr uint32_t kNc = 32u / D;
  constexpr uint32_t kTileBf = F::kTileBf;
  constexpr uint32_t kShift = F::kShift;
  constexpr int kChunks = static_cast<int>(F::kTileBytes / 16u);  // 16-byte code pieces per tile
  constexpr MlLayout Lo = ml_layout<B, D, VAR>();
  extern __shared__ __align__(128) uint8_t sm[];
  const uint32_t s0 = smem_u32(sm);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  volatile uint32_t* flags = reinterpret_cast<volatile uint32_t*>(sm + Lo.misc);  // [0] math gave up
  const uint32_t full0 = s0 + Lo.bars;             // full[S]: a stage's bytes landed
  const uint32_t rfull0 = full0 + 8u * kMlStages;  // red_full[2]: the math warps' sums are in red[buf]
  const uint32_t rempty0 = rfull0 + 16u;           // red_empty[2]: the epilogue warp has read red[buf]

  const int64_t G = gridDim.x, first = blockIdx.x;
  const int my = static_cast<int>((a.items - first + G - 1) / G);

  if (tid == 0) {
    for (int s = 0; s < kMlStages; ++s) mbar_init(full0 + 8 * s, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(rfull0 + 8 * b, kMlMath);
      mbar_init(rempty0 + 8 * b, 32);
    }
    mbar_fence_init();
    flags[0] = 0u;
  }
  __syncthreads();

  if (warp == kMlMath / 32) {
    // ================= epilogue warp: the 8 warps' sums of each item, y or
    // the workspace partial, the arrival count, and the finish of a row block
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
    uint32_t ticket = 0u;  // lane 0: the arrival of the previous split item, read one item later
    int pend_l = -1;
    int64_t pend_rb = 0;
    for (int k = 0; k < my; ++k) {
      const int buf = k & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(rfull0 + 8 * buf, static_cast<uint32_t>(k >> 1) & 1u))) {
        report(a.status, USK_FLAG_TIMEOUT);
        return;
      }
      if (flags[0] != 0u) return;  // the math warps gave up (they reported it)
      const MlItem m = ml_item(a, first + k * G);
      const MlLinear& L = a.lin[m.l];
      const float* red = reinterpret_cast<const float*>(sm + Lo.red + buf * (8u * B * 64u * 4u));
      constexpr int kQ = (B * 64 + 31) / 32;
      float part[kQ];
#pragma unroll
      for (int kq = 0; kq < kQ; ++kq) {
        const int q = lane + 32 * kq;
        part[kq] = 0.0f;
        if (q < B * 64) {
#pragma unroll
          for (int w = 0; w < 8; ++w) part[kq] += red[w * B * 64 + q];
        }
      }
      mbar_arrive_cta(rempty0 + 8 * buf);  // red[buf] may be refilled
      if (L.nseg == 1) {
        const float sc = __half2float(__ushort_as_half(L.scales[m.rb]));
#pragma unroll
        for (int kq = 0; kq < kQ; ++kq) {
          const int q = lane + 32 * kq;
          if (q < a.batch * 64) L.y[static_cast<int64_t>(q / 64) * L.M + m.rb * 64 + q % 64] = part[kq] * sc;
        }
      } else {
        float* pdst = a.part + (L.part0 + m.rb * L.nseg + m.seg) * static_cast<int64_t>(B * 64);
#pragma unroll
        for (int kq = 0; kq < kQ; ++kq) {
          const int q = lane + 32 * kq;
          if (q < a.batch * 64) __stcg(pdst + q, part[kq]);
        }
      }
      const int pl = pend_l >= 0 ? pend_l : 0;
      const bool last = __shfl_sync(0xFFFFFFFFu, pend_l >= 0 && ticket + 1u == static_cast<uint32_t>(a.lin[pl].nseg), 0);
      if (last) ml_finish<B>(a, pend_l, pend_rb, lane);
      pend_l = -1;
      if (L.nseg > 1) {
        __syncwarp();  // every lane's partial stores before lane 0's release
        uint32_t t = 0u;
        if (lane == 0) {
          cuda::atomic_ref<uint32_t, cuda::thread_scope_device> cnt(a.cnt[L.cnt0 + m.rb]);
          t = cnt.fetch_add(1u, cuda::memory_order_release);
        }
        ticket = t;
        pend_l = m.l;
        pend_rb = m.rb;
      }
    }
    const int pl = pend_l >= 0 ? pend_l : 0;
    const bool last = __shfl_sync(0xFFFFFFFFu, pend_l >= 0 && ticket + 1u == static_cast<uint32_t>(a.lin[pl].nseg), 0);
    if (last) ml_finish<B>(a, pend_l, pend_rb, lane);
    return;
  }

  // ================= math warps 0..7
  const int g = lane >> 2, t = lane & 3;
  const int o = (warp & 1) + 8 * (warp >> 1) + 2 * t;  // this lane's octet in every tile
  // the issuing thread's cursor (next chunk to copy) and count of chunks
  // issued live in shared memory: only thread 0 touches them
  MlCursor* cur = reinterpret_cast<MlCursor*>(sm + Lo.misc + 16);
  int* issued_p = reinterpret_cast<int*>(sm + Lo.misc + 8);
  if (tid == 0) {
    MlCursor pc;
    pc.k = 0;
    pc.m = ml_item(a, first);
    pc.c = pc.m.c0;
    *cur = pc;
    for (int n = 0; n < kMlStages && pc.k < my; ++n, ml_cursor_next(a, pc, first, G, my))
      ml_copy_codes<VAR>(a, pc.m, pc.c, s0 + Lo.stage + n * Lo.stage_bytes, full0 + 8 * n);
  }
  if (a.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) {
    MlCursor cu = *cur;
    int issued = 0;
    for (; issued < kMlStages && cu.k < my; ++issued, ml_cursor_next(a, cu, first, G, my)) {
      if (a.inject && blockIdx.x == 0 && issued == 0) continue;  // test hook: this stage never fills
      ml_copy_x(a, cu.m, cu.c, s0 + Lo.stage + issued * Lo.stage_bytes + kMlTiles * F::kTileBytes,
                full0 + 8 * issued);
    }
    *cur = cu;
    *issued_p = issued;
  }

  bool empty_failed = false;  // a wait for the epilogue warp gave up: stop at the next chunk
  int j = 0;                  // running chunk index of this block
  for (int k = 0; k < my; ++k) {
    const MlItem m = ml_item(a, first + k * G);
    const MlLinear& L = a.lin[m.l];
    const int buf = k & 1;
    float d[4][4];  // per 16-row group: rows g, g + 8 x batch columns 2t, 2t + 1
#pragma unroll
    for (int mb = 0; mb < 4; ++mb)
#pragma unroll
      for (int e = 0; e < 4; ++e) d[mb][e] = 0.0f;

    for (int c = m.c0; c < m.c1; ++c, ++j) {
      const int s = j % kMlStages;
      const int nt = ml_nt(L, c);
      const uint32_t stage = s0 + Lo.stage + s * Lo.stage_bytes;
      const uint32_t cbf = s0 + Lo.cbf + (j & 1) * (kMlTiles * kTileBf);
      uint2* keytab = reinterpret_cast<uint2*>(sm + Lo.keys + (j & 1) * (kMlTiles * D * 8u));
      const bool ok = mbar_wait(full0 + 8 * s, static_cast<uint32_t>(j / kMlStages) & 1u) && !empty_failed;
      if (math_bar_or(1, kMlMath, !ok)) {  // every math warp takes the same branch
        if (tid == 0) {
          flags[0] = 1u;
          report(a.status, USK_FLAG_TIMEOUT);
          // wait (bounded) for this block's copies still in flight before leaving
          for (int jj = j; jj < *issued_p; ++jj)
            mbar_wait(full0 + 8 * (jj % kMlStages), static_cast<uint32_t>(jj / kMlStages) & 1u);
        }
        math_bar(1, kMlMath);
        mbar_arrive_cta(rfull0 + 8 * buf);  // wakes the epilogue warp, which sees flags[0]
        return;
      }
      // ---- widen the chunk's codes to bf16 (exact), tile keys, x fragments
      for (int q = tid; q < nt * kChunks; q += kMlMath) {
        const uint4 w = lds128(stage + 16u * q);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        if constexpr (Q4) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t o4[4];
            i4x8_to_bf16x8(ws[e], o4);
            sts128(cbf + 64u * q + 16u * e, make_uint4(o4[0], o4[1], o4[2], o4[3]));
          }
        } else {
          uint32_t o8[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            o8[2 * e] = i8pair_to_bf16x2<0x4140>(ws[e]);
            o8[2 * e + 1] = i8pair_to_bf16x2<0x4342>(ws[e]);
          }
          sts128(cbf + 32u * q, make_uint4(o8[0], o8[1], o8[2], o8[3]));
          sts128(cbf + 32u * q + 16u, make_uint4(o8[4], o8[5], o8[6], o8[7]));
        }
      }
      if (tid < nt * D)
        keytab[tid] = row_key(L.seed, static_cast<uint64_t>(m.rb) * L.T + c * kMlTiles + tid / D, D, tid % D);
      uint4 xv[kMlTiles];
      const uint32_t xs = stage + kMlTiles * F::kTileBytes + static_cast<uint32_t>(g) * (kMlTiles * 512u) + 16u * o;
#pragma unroll
      for (int tt = 0; tt < kMlTiles; ++tt) {
        xv[tt] = make_uint4(0u, 0u, 0u, 0u);
        if (tt < nt && g < a.batch) xv[tt] = lds128(xs + 512u * tt);
      }
      // widened codes and keys ready; the stage's raw bytes are no longer read.
      // (cbf and keytab alternate between chunks: a warp past this barrier of
      // chunk j + 1 knows every warp has left chunk j - 1's math.)
      math_bar(1, kMlMath);
      if (tid == 0 && cur->k < my) {  // refill this stage with chunk j + S
        MlCursor cu = *cur;
        ml_copy_codes<VAR>(a, cu.m, cu.c, stage, full0 + 8 * s);
        ml_copy_x(a, cu.m, cu.c, stage + kMlTiles * F::kTileBytes, full0 + 8 * s);
        ++*issued_p;
        ml_cursor_next(a, cu, first, G, my);
        *cur = cu;
      }

      // ---- per tile and 16-row group two MMAs (columns 0-3 and 4-7 of the
      // lane's octet); the four 16-row groups are independent MMA chains
#pragma unroll
      for (int tt = 0; tt < kMlTiles; ++tt) {
        if (tt < nt) {
          const uint32_t tile_s = cbf + tt * kTileBf;
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
            mma_bf16_16816(d[mb], q0.x, q1.x, q0.y, q1.y, xv[tt].x, xv[tt].y);
            mma_bf16_16816(d[mb], q0.z, q1.z, q0.w, q1.w, xv[tt].z, xv[tt].w);
          }
        }
      }
    }
    if (k == my - 1) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---- the warp's sums into red[buf] once the epilogue warp has read it (two items ago)
    if (k >= 2 && !mbar_wait(rempty0 + 8 * buf, static_cast<uint32_t>((k - 2) >> 1) & 1u))
      empty_failed = true;  // the epilogue warp stopped (it reported the timeout)
    float* red = reinterpret_cast<float*>(sm + Lo.red + buf * (8u * B * 64u * 4u));
#pragma unroll
    for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int bi = 2 * t + (e & 1);
        const int r = 16 * mb + g + 8 * (e >> 1);
        if (bi < B) red[(warp * B + bi) * 64 + r] = d[mb][e];
      }
    }
    mbar_arrive_cta(rfull0 + 8 * buf);
  }
}

// ---------------------------------------------------------------- launch

static int ml_bucket(int batch) { return batch <= 1 ? 1 : batch <= 2 ? 2 : batch <= 4 ? 4 : 8; }

struct MlPlan {
  int64_t items, part_floats, counters;
};

// Segments per row for the launch: the split s minimising waves(s) x (chunks
// per segment + half a chunk of per-item flush), plus one chunk's worth for
// the cross-block sum when rows split; `slots` resident blocks.  Fills the per-linear item table when lin != null.
static MlPlan ml_plan(int n, const int64_t* Ms, const int64_t* Ks, int Bp, int64_t slots, MlLinear* lin) {
  int max_nch = 1;
  for (int l = 0; l < n; ++l) {
    const int nch = static_cast<int>((Ks[l] / kTileCols + kMlTiles - 1) / kMlTiles);
    max_nch = nch > max_nch ? nch : max_nch;
  }
  int best_s = 1;
  int64_t best_cost = -1;
  for (int sp = 1; sp <= max_nch && sp <= 64; ++sp) {
    int64_t items = 0, seglen_max = 1;
    for (int l = 0; l < n; ++l) {
      const int nch = static_cast<int>((Ks[l] / kTileCols + kMlTiles - 1) / kMlTiles);
      const int ns = sp < nch ? sp : nch;
      const int len = (nch + ns - 1) / ns;
      items += (Ms[l] / kRowsPerBlock) * ((nch + len - 1) / len);
      seglen_max = len > seglen_max ? len : seglen_max;
    }
    // in half-chunk units: an item costs its chunks plus about half a chunk of
    // flush (the 8 warps' sums, the epilogue); a split row one chunk more
    const int64_t waves = (items + slots - 1) / slots;
    const int64_t cost = waves * (2 * seglen_max + 1) + (sp > 1 ? 2 : 0);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_s = sp;
    }
  }
  MlPlan p{0, 0, 0};
  for (int l = 0; l < n; ++l) {
    const int T = static_cast<int>(Ks[l] / kTileCols);
    const int nch = (T + kMlTiles - 1) / kMlTiles;
    const int ns0 = best_s < nch ? best_s : nch;
    const int len = (nch + ns0 - 1) / ns0;
    const int nseg = (nch + len - 1) / len;
    const int64_t RB = Ms[l] / kRowsPerBlock;
    if (lin) {
      lin[l].T = T;
      lin[l].nch = nch;
      lin[l].nseg = nseg;
      lin[l].seglen = len;
      lin[l].item0 = p.items;
      lin[l].part0 = p.part_floats / (Bp * 64);
      lin[l].cnt0 = p.counters;
    }
    p.items += RB * nseg;
    if (nseg > 1) {
      p.part_floats += RB * nseg * Bp * 64;
      p.counters += RB;
    }
  }
  return p;
}

// Resident blocks of the kernel for batch bucket B, depth D, layout VAR on
// the current device (one occupancy query per instantiation and process).
template <int B, int D, int VAR>
static cudaError_t ml_slots(int64_t* slots) {
  constexpr MlLayout Lo = ml_layout<B, D, VAR>();
  auto kern = gemv_multi_kernel<B, D, VAR>;
  static int per_sm = 0;
  if (per_sm == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(Lo.total));
    if (e != cudaSuccess) return e;
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kMlThreads, Lo.total);
    if (e != cudaSuccess) return e;
    per_sm = nb > 0 ? nb : 1;
  }
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  *slots = static_cast<int64_t>(sms) * per_sm;
  return cudaSuccess;
}

template <int D, int VAR>
static cudaError_t ml_slots_b(int batch, int64_t* slots) {
  switch (ml_bucket(batch)) {
    case 1: return ml_slots<1, D, VAR>(slots);
    case 2: return ml_slots<2, D, VAR>(slots);
    case 4: return ml_slots<4, D, VAR>(slots);
    default: return ml_slots<8, D, VAR>(slots);
  }
}

static cudaError_t ml_slots_any(int batch, int depth, int var, int64_t* slots) {
  if (var == 1) return ml_slots_b<1, 1>(batch, slots);
  if (var == 2) return ml_slots_b<1, 2>(batch, slots);
  if (var == 3) return ml_slots_b<1, 3>(batch, slots);
  if (depth == 2) return ml_slots_b<2, 0>(batch, slots);
  if (depth == 4) return ml_slots_b<4, 0>(batch, slots);
  return ml_slots_b<1, 0>(batch, slots);
}

// Workspace of a list on the current device: counters first (256-byte
// aligned block), then the partials; 0 when no row is split.
size_t gemv_multi_ws_bytes(int n, const int64_t* Ms, const int64_t* Ks, int batch, int depth, int var) {
  int64_t slots = 0;
  if (ml_slots_any(batch, depth, var, &slots) != cudaSuccess) slots = 296;
  const MlPlan p = ml_plan(n, Ms, Ks, ml_bucket(batch), slots, nullptr);
  if (p.counters == 0) return 0;
  const size_t cnt_bytes = (static_cast<size_t>(p.counters) * 4u + 255u) & ~static_cast<size_t>(255u);
  return cnt_bytes + static_cast<size_t>(p.part_floats) * 4u;
}

template <int B, int D, int VAR>
static cudaError_t ml_launch_t(const MlArgs& a, int64_t slots, cudaStream_t stream) {
  constexpr MlLayout Lo = ml_layout<B, D, VAR>();
  auto kern = gemv_multi_kernel<B, D, VAR>;
  const unsigned grid = static_cast<unsigned>(a.items < slots ? a.items : slots);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kMlThreads, 1, 1);
  cfg.dynamicSmemBytes = Lo.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int D, int VAR>
static cudaError_t ml_launch_b(const MlArgs& a, int64_t slots, cudaStream_t stream) {
  switch (ml_bucket(a.batch)) {
    case 1: return ml_launch_t<1, D, VAR>(a, slots, stream);
    case 2: return ml_launch_t<2, D, VAR>(a, slots, stream);
    case 4: return ml_launch_t<4, D, VAR>(a, slots, stream);
    default: return ml_launch_t<8, D, VAR>(a, slots, stream);
  }
}

// All sketches of one launch share depth and code layout (checked by the caller).
cudaError_t launch_gemv_multi(int n, const int8_t* const* codes, const uint16_t* const* scales, const int64_t* Ms,
                              const int64_t* Ks, const uint64_t* seeds, const uint16_t* const* x, float* const* y,
                              int batch, void* ws, uint32_t* status, bool pdl, cudaStream_t stream, int inject,
                              int depth, int var) {
  if (n < 1 || n > kMlMaxLinears || batch < 1 || batch > 8) return cudaErrorInvalidValue;
  int64_t slots = 0;
  cudaError_t e = ml_slots_any(batch, depth, var, &slots);
  if (e != cudaSuccess) return e;
  MlArgs a;
  const int Bp = ml_bucket(batch);
  const MlPlan p = ml_plan(n, Ms, Ks, Bp, slots, a.lin);
  for (int l = 0; l < n; ++l) {
    a.lin[l].codes = codes[l];
    a.lin[l].scales = scales[l];
    a.lin[l].x = x[l];
    a.lin[l].y = y[l];
    a.lin[l].M = Ms[l];
    a.lin[l].K = Ks[l];
    a.lin[l].seed = seeds[l];
  }
  a.n = n;
  a.batch = batch;
  a.items = p.items;
  a.status = status;
  a.pdl = pdl ? 1 : 0;
  a.inject = inject;
  a.cnt = static_cast<uint32_t*>(ws);
  const size_t cnt_bytes = (static_cast<size_t>(p.counters) * 4u + 255u) & ~static_cast<size_t>(255u);
  a.part = p.counters ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + cnt_bytes) : nullptr;
  if (p.items == 0) return cudaSuccess;
  if (var == 1) return ml_launch_b<1, 1>(a, slots, stream);
  if (var == 2) return ml_launch_b<1, 2>(a, slots, stream);
  if (var == 3) return ml_launch_b<1, 3>(a, slots, stream);
  if (depth == 2) return ml_launch_b<2, 0>(a, slots, stream);
  if (depth == 4) return ml_launch_b<4, 0>(a, slots, stream);
  return ml_launch_b<1, 0>(a, slots, stream);
}

// ---------------------------------------------------------------- fixed scratch
//
// usk_gemv_multi_static: the same launch with the workspace in this array
// instead of caller memory, for callers that may not allocate device memory.
// The array lives in every device's copy of this module from the moment the
// library is loaded until the process exits.  Host code must not hand the
// array's name to a kernel (on the host it only stands for the symbol); the
// device address comes from cudaGetSymbolAddress, looked up once per device
// with that device current, the first time the entry point runs there.
static __device__ __align__(256) uint8_t g_ml_scratch[USK_GEMV_MULTI_STATIC_BYTES];

static cudaError_t ml_static_scratch(void** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_ml_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

// Bytes at the start of the workspace that must be zero when a launch starts
// (the arrival counters; 0 when no row is split).
static size_t ml_counter_bytes(int n, const int64_t* Ms, const int64_t* Ks, int batch, int depth, int var) {
  int64_t slots = 0;
  if (ml_slots_any(batch, depth, var, &slots) != cudaSuccess) slots = 296;
  const MlPlan p = ml_plan(n, Ms, Ks, ml_bucket(batch), slots, nullptr);
  return p.counters ? (static_cast<size_t>(p.counters) * 4u + 255u) & ~static_cast<size_t>(255u) : 0;
}

// The caller has checked that the list's workspace fits the array.  The
// counters are cleared on the stream first (a call that gave up could have
// left them non-zero), then the kernel runs on the array.
cudaError_t launch_gemv_multi_static(int n, const int8_t* const* codes, const uint16_t* const* scales,
                                     const int64_t* Ms, const int64_t* Ks, const uint64_t* seeds,
                                     const uint16_t* const* x, float* const* y, int batch, uint32_t* status, bool pdl,
                                     cudaStream_t stream, int depth, int var) {
  void* base = nullptr;
  cudaError_t e = ml_static_scratch(&base);
  if (e != cudaSuccess) return e;
  const size_t cnt = ml_counter_bytes(n, Ms, Ks, batch, depth, var);
  if (cnt > 0) {
    e = cudaMemsetAsync(base, 0, cnt, stream);
    if (e != cudaSuccess) return e;
  }
  return launch_gemv_multi(n, codes, scales, Ms, Ks, seeds, x, y, batch, base, status, pdl, stream, 0, depth, var);
}

}  // namespace usk

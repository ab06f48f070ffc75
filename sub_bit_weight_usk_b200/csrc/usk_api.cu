// usk_api.cu -- the C ABI of libusk (declared in include/usk.h): argument
// validation, then one kernel launch per call.  No allocation, no global state
// beyond CUDA's cached kernel attributes.
#include <algorithm>
#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "usk.h"
#include "usk_common.cuh"

namespace usk {
cudaError_t launch_build(const void* W, bool bf16, int64_t M, int64_t K, int64_t ldw, const float* imp,
                         uint64_t seed, int8_t* codes, uint16_t* scales, uint32_t* status,
                         cudaStream_t stream, int cluster_override, int inject, int var, const RbMap& map,
                         int64_t nrb, int64_t g1, int64_t g2);
cudaError_t launch_build_amm(const void* W, bool bf16, int64_t M, int64_t K, int64_t ldw, uint64_t seed, int depth,
                             int8_t* codes, uint16_t* scales, uint32_t* status, cudaStream_t stream,
                             int cluster_override, int inject);
cudaError_t launch_build_cs(const void* W, bool bf16, int64_t M, int64_t K, int64_t ldw, uint64_t seed,
                            int8_t* codes, uint16_t* scales, uint32_t* status, cudaStream_t stream,
                            int cluster_override, int inject);
cudaError_t launch_gemv_cs(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                           const void* x, bool xf32, int batch, float* y, uint32_t* status, bool pdl,
                           cudaStream_t stream, int tpb_override, int rows_override, int inject);
cudaError_t launch_gemv(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                        const void* x, bool xf32, int batch, float* y, uint32_t* status, bool pdl, int path,
                        cudaStream_t stream, int tpc_override, int rows_override, int inject, int depth, int var,
                        const RbMap& map, int64_t nrb, int64_t g1, int64_t g2);
cudaError_t launch_gemm(const int8_t* codes, const uint16_t* scales, int64_t M, int64_t K, uint64_t seed,
                        const uint16_t* x, int batch, float* y, uint32_t* status, cudaStream_t stream, int inject,
                        int depth, int var, const RbMap& map, int64_t nrb, int64_t g1, int64_t g2,
                        int splits_override, int issuers_override, bool pdl);
bool gemm_supported(int64_t K, int batch, int depth, int var);
size_t gemv_multi_ws_bytes(int n, const int64_t* Ms, const int64_t* Ks, int batch, int depth, int var);
cudaError_t launch_gemv_multi(int n, const int8_t* const* codes, const uint16_t* const* scales, const int64_t* Ms,
                              const int64_t* Ks, const uint64_t* seeds, const uint16_t* const* x, float* const* y,
                              int batch, void* ws, uint32_t* status, bool pdl, cudaStream_t stream, int inject,
                              int depth, int var);
cudaError_t launch_gemv_multi_static(int n, const int8_t* const* codes, const uint16_t* const* scales,
                                     const int64_t* Ms, const int64_t* Ks, const uint64_t* seeds,
                                     const uint16_t* const* x, float* const* y, int batch, uint32_t* status, bool pdl,
                                     cudaStream_t stream, int depth, int var);
}  // namespace usk

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

usk_status check_shape(int64_t M, int64_t K) {
  if (M < 0 || K < 0) return USK_ERR_SHAPE;
  if (M % USK_ROWS_PER_BLOCK != 0 || K % USK_TILE_COLS != 0) return USK_ERR_SHAPE;
  if (M > USK_MAX_M || K > USK_MAX_K) return USK_ERR_SHAPE;
  return USK_OK;
}

// Hash rows of a sketch or a build request; 0 if the (format, depth) pair is not valid.
int format_depth(uint32_t version, uint32_t depth) {
  if (version == 0 || version == USK_FORMAT_MAXKEY) return depth <= 1 ? 1 : 0;
  if (version == USK_FORMAT_ABSMAXMIN) return (depth == 1 || depth == 2 || depth == 4) ? static_cast<int>(depth) : 0;
  if (version == USK_FORMAT_COLSHARED || version == USK_FORMAT_Q4) return depth <= 1 ? 1 : 0;
  return 0;
}

// Code layout of a (format, slots) pair: 0 = 4 slots 8-bit (format 1 default,
// and formats 2 and 3), 1 = 8 slots 4-bit (format 4), 2 = 2 slots 8-bit,
// 3 = 8 slots 8-bit (format 1 at 0.25 / 1 bit per weight); -1 if not valid.
int layout_of(uint32_t version, uint32_t slots) {
  if (version == 0 || version == USK_FORMAT_MAXKEY) {
    if (slots == 0 || slots == 4) return 0;
    if (slots == 2) return 2;
    if (slots == 8) return 3;
    return -1;
  }
  if (version == USK_FORMAT_Q4) return (slots == 0 || slots == 8) ? 1 : -1;
  return (slots == 0 || slots == 4) ? 0 : -1;
}

// Code bytes of an M x K sketch in a layout.
size_t layout_code_bytes(int64_t M, int64_t K, int layout) {
  const size_t n = static_cast<size_t>(M) * static_cast<size_t>(K);
  return layout == 2 ? n / 32 : (layout == 3 ? n / 8 : n / 16);
}

// A rate map for an M x K format-1 sketch: counts that add up to the row
// blocks, code_bytes = K * (2 c0 + 4 c1 + 8 c2), aligned device arrays.
usk_status check_rate_map(const usk_rate_map* m, int64_t M, int64_t K) {
  const int64_t RB = M / USK_ROWS_PER_BLOCK;
  if (m->count[0] < 0 || m->count[1] < 0 || m->count[2] < 0) return USK_ERR_PARAMS;
  if (m->count[0] + m->count[1] + m->count[2] != RB) return USK_ERR_PARAMS;
  if (m->code_bytes != K * (2 * m->count[0] + 4 * m->count[1] + 8 * m->count[2])) return USK_ERR_PARAMS;
  if (RB > 0 && (!m->offset || !m->order)) return USK_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(m->offset) & 7u) != 0 || (reinterpret_cast<uintptr_t>(m->order) & 3u) != 0)
    return USK_ERR_ALIGN;
  return USK_OK;
}

// The row-block map of one launch: identity for a uniform sketch; with a rate
// map, its order and offsets, and where the 4- and 8-slot groups start in the
// order list (the kernels pick each block's code layout from that).
struct Launch {
  usk::RbMap map;
  int64_t nrb, g1, g2;
};

Launch launch_of(const usk_rate_map* rm, int64_t M) {
  const int64_t RB = M / USK_ROWS_PER_BLOCK;
  if (!rm) return Launch{usk::RbMap{nullptr, nullptr, 0, RB}, RB, 0, 0};
  return Launch{usk::RbMap{rm->order, rm->offset, rm->code_bytes, RB}, RB, rm->count[0],
                rm->count[0] + rm->count[1]};
}

usk_status check_sketch(const usk_sketch* s) {
  if (!s) return USK_ERR_NULL;
  if (format_depth(s->version, s->depth) == 0) return USK_ERR_PARAMS;
  if (layout_of(s->version, s->slots) < 0) return USK_ERR_PARAMS;
  usk_status st = check_shape(s->M, s->K);
  if (st != USK_OK) return st;
  if (s->rates) {
    if ((s->version != 0 && s->version != USK_FORMAT_MAXKEY) || s->slots != 0) return USK_ERR_PARAMS;
    st = check_rate_map(s->rates, s->M, s->K);
    if (st != USK_OK) return st;
  }
  if (s->M > 0 && s->K > 0) {
    if (!s->codes || !s->scales) return USK_ERR_NULL;
    if (!aligned16(s->codes)) return USK_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(s->scales) & 1u) != 0) return USK_ERR_ALIGN;
  }
  return USK_OK;
}

usk_status from_cuda(cudaError_t e) { return e == cudaSuccess ? USK_OK : USK_ERR_CUDA; }

// Optional launch-geometry overrides (used by the determinism tests to show the
// result does not depend on the geometry).  0 = library default.
int g_build_cluster = 0;
int g_gemv_tiles_per_block = 0;
int g_gemv_path = 0;
int g_gemv_rows = 0;
int g_gemm_splits = 0;
int g_gemm_issuers = 0;
int g_inject = 0;  // 1 build, 2 gemm, 3 gemv, 4 gemv_multi: skip one copy/commit in block (0, 0)

constexpr int64_t kMultiMax = 16;  // sketches per usk_gemv_multi launch

// Checks of a usk_gemv_multi list shared by the call and its workspace query:
// every sketch valid, one format / depth / slot count, no rate map, not format
// 3.  Fills the shapes of the sketches that have work (M > 0 and K > 0).
usk_status check_multi(int64_t n, const usk_sketch* sk, int64_t batch, int64_t* Ms, int64_t* Ks, int* idx,
                       int* nwork) {
  if (n < 0 || n > kMultiMax) return USK_ERR_SHAPE;
  if (batch < 0 || batch > 8) return USK_ERR_BATCH;
  *nwork = 0;
  if (n == 0) return USK_OK;
  if (!sk) return USK_ERR_NULL;
  for (int64_t l = 0; l < n; ++l) {
    usk_status st = check_sketch(&sk[l]);
    if (st != USK_OK) return st;
    if (sk[l].rates || sk[l].version == USK_FORMAT_COLSHARED) return USK_ERR_PARAMS;
    if (format_depth(sk[l].version, sk[l].depth) != format_depth(sk[0].version, sk[0].depth) ||
        layout_of(sk[l].version, sk[l].slots) != layout_of(sk[0].version, sk[0].slots))
      return USK_ERR_PARAMS;
    if (sk[l].M > 0 && sk[l].K > 0) {
      Ms[*nwork] = sk[l].M;
      Ks[*nwork] = sk[l].K;
      idx[*nwork] = static_cast<int>(l);
      ++*nwork;
    }
  }
  return USK_OK;
}

}  // namespace

extern "C" {

USK_API uint32_t usk_format_version(void) { return USK_FORMAT_VERSION; }

USK_API const char* usk_status_str(usk_status status) {
  switch (status) {
    case USK_OK: return "ok";
    case USK_ERR_NULL: return "a required pointer is NULL";
    case USK_ERR_SHAPE: return "shape: M must be a multiple of 64, K a multiple of 256, within the limits";
    case USK_ERR_DTYPE: return "unknown dtype";
    case USK_ERR_BATCH: return "batch outside the range of this call";
    case USK_ERR_WORKSPACE: return "workspace missing or too small";
    case USK_ERR_PARAMS:
      return "params NULL, unknown format, bad depth or slot count, non-zero flags, importance with format 2 or 3, "
             "a rate map that is not for format 1 or whose counts do not match, or usk_gemm on a format-3 sketch";
    case USK_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case USK_ERR_NONFINITE: return "non-finite weight";
    case USK_ERR_TIMEOUT: return "a bounded device wait gave up";
    case USK_ERR_ALIGN: return "pointer or row stride not 16-byte aligned";
    case USK_ERR_IMPORTANCE: return "importance must be finite with the sign bit clear";
    case USK_ERR_SCALE_OVERFLOW: return "block maximum / 127 exceeds the binary16 range";
  }
  return "unknown status";
}

USK_API usk_status usk_sizes(int64_t M, int64_t K, size_t* code_bytes, size_t* scale_bytes) {
  usk_status st = check_shape(M, K);
  if (st != USK_OK) return st;
  if (!code_bytes || !scale_bytes) return USK_ERR_NULL;
  *code_bytes = static_cast<size_t>(M) * static_cast<size_t>(K) / USK_WEIGHTS_PER_BUCKET;
  *scale_bytes = 2 * static_cast<size_t>(M / USK_ROWS_PER_BLOCK);
  return USK_OK;
}

USK_API usk_status usk_sizes_ex(int64_t M, int64_t K, uint32_t version, uint32_t slots, size_t* code_bytes,
                                size_t* scale_bytes) {
  usk_status st = check_shape(M, K);
  if (st != USK_OK) return st;
  if (!code_bytes || !scale_bytes) return USK_ERR_NULL;
  const int layout = layout_of(version, slots);
  if (layout < 0 || (version > USK_FORMAT_VERSION)) return USK_ERR_PARAMS;
  *code_bytes = layout_code_bytes(M, K, layout);
  *scale_bytes = 2 * static_cast<size_t>(M / USK_ROWS_PER_BLOCK);
  return USK_OK;
}

// Importance-aware space allocation: every unit starts at 2 slots; the upgrades
// 2 -> 4 (gain per bit = importance) and 4 -> 8 (importance / 4) of all units are
// visited in decreasing gain order (ties: the 2 -> 4 step first, then the lower
// index) and taken while the unit is at the step's starting level and the total
// stays within the budget.
USK_API usk_status usk_plan_slots(int64_t n, const int64_t* weights, const double* importance, double budget_bits,
                                  uint32_t* slots) {
  if (n < 0) return USK_ERR_SHAPE;
  if (n == 0) return USK_OK;
  if (!weights || !importance || !slots) return USK_ERR_NULL;
  if (!(budget_bits >= 0.25 && budget_bits <= 1.0)) return USK_ERR_PARAMS;
  double total = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    if (weights[i] <= 0 || !(importance[i] >= 0.0) || importance[i] > 1e300) return USK_ERR_PARAMS;
    total += static_cast<double>(weights[i]);
  }
  struct Step {
    double gain;
    int level;
    int64_t unit;
  };
  std::vector<Step> steps;
  steps.reserve(static_cast<size_t>(2 * n));
  for (int64_t i = 0; i < n; ++i) {
    steps.push_back({importance[i], 0, i});
    steps.push_back({importance[i] / 4.0, 1, i});
  }
  std::stable_sort(steps.begin(), steps.end(), [](const Step& x, const Step& y) {
    if (x.gain != y.gain) return x.gain > y.gain;
    if (x.level != y.level) return x.level < y.level;
    return x.unit < y.unit;
  });
  const double cap = budget_bits * total;
  double used = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    slots[i] = 2u;
    used += 0.25 * static_cast<double>(weights[i]);
  }
  for (const Step& st : steps) {
    const uint32_t from = st.level == 0 ? 2u : 4u;
    if (slots[st.unit] != from) continue;
    const double cost = (st.level == 0 ? 0.25 : 0.5) * static_cast<double>(weights[st.unit]);
    if (used + cost <= cap) {
      slots[st.unit] = 2u * from;
      used += cost;
    }
  }
  return USK_OK;
}

USK_API usk_status usk_rate_map_plan(int64_t M, int64_t K, const uint32_t* slots, int64_t* offset, int32_t* order,
                                     int64_t* count, int64_t* code_bytes) {
  usk_status st = check_shape(M, K);
  if (st != USK_OK) return st;
  if (!count || !code_bytes) return USK_ERR_NULL;
  const int64_t RB = M / USK_ROWS_PER_BLOCK;
  if (RB > 0 && (!slots || !offset || !order)) return USK_ERR_NULL;
  for (int64_t rb = 0; rb < RB; ++rb)
    if (slots[rb] != 2 && slots[rb] != 4 && slots[rb] != 8) return USK_ERR_PARAMS;
  int64_t acc = 0, n = 0;
  count[0] = count[1] = count[2] = 0;
  for (int64_t rb = 0; rb < RB; ++rb) {
    offset[rb] = acc;
    acc += K * static_cast<int64_t>(slots[rb]);
  }
  for (int g = 0; g < 3; ++g) {
    const uint32_t want = 2u << g;
    for (int64_t rb = 0; rb < RB; ++rb)
      if (slots[rb] == want) {
        order[n++] = static_cast<int32_t>(rb);
        ++count[g];
      }
  }
  *code_bytes = acc;
  return USK_OK;
}

USK_API usk_status usk_build(const void* W, usk_dtype wdtype, int64_t M, int64_t K, int64_t ldw,
                     const float* importance, const usk_params* params, int8_t* codes,
                     uint16_t* scales, uint32_t* d_status, void* stream) {
  usk_status st = check_shape(M, K);
  if (st != USK_OK) return st;
  if (wdtype != USK_F32 && wdtype != USK_BF16) return USK_ERR_DTYPE;
  if (!params) return USK_ERR_PARAMS;
  if (params->flags != 0) return USK_ERR_PARAMS;
  if (params->version != USK_FORMAT_MAXKEY && params->version != USK_FORMAT_ABSMAXMIN &&
      params->version != USK_FORMAT_COLSHARED && params->version != USK_FORMAT_Q4)
    return USK_ERR_PARAMS;
  const int depth = format_depth(params->version, params->depth);
  if (depth == 0) return USK_ERR_PARAMS;
  const int layout = layout_of(params->version, params->slots);
  if (layout < 0) return USK_ERR_PARAMS;
  const bool amm = params->version == USK_FORMAT_ABSMAXMIN, cs = params->version == USK_FORMAT_COLSHARED;
  if ((amm || cs) && importance) return USK_ERR_PARAMS;
  const usk_rate_map* rm = params->rates;
  if (rm) {
    if (params->version != USK_FORMAT_MAXKEY || params->slots != 0) return USK_ERR_PARAMS;
    st = check_rate_map(rm, M, K);
    if (st != USK_OK) return st;
  }
  if (M == 0) return USK_OK;
  if (!scales) return USK_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(scales) & 1u) != 0) return USK_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (K == 0) return from_cuda(cudaMemsetAsync(scales, 0, 2 * static_cast<size_t>(M / 64), s));
  if (!W || !codes) return USK_ERR_NULL;
  if (ldw < K) return USK_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(codes)) return USK_ERR_ALIGN;
  if (ldw % (wdtype == USK_BF16 ? 8 : 4) != 0) return USK_ERR_ALIGN;
  if (importance && !aligned16(importance)) return USK_ERR_ALIGN;
  cudaError_t e;
  if (cs)
    e = usk::launch_build_cs(W, wdtype == USK_BF16, M, K, ldw, params->seed, codes, scales, d_status, s,
                             g_build_cluster, g_inject == 1);
  else if (amm)
    e = usk::launch_build_amm(W, wdtype == USK_BF16, M, K, ldw, params->seed, depth, codes, scales, d_status, s,
                              g_build_cluster, g_inject == 1);
  else {
    const Launch l = launch_of(rm, M);
    e = usk::launch_build(W, wdtype == USK_BF16, M, K, ldw, importance, params->seed, codes, scales, d_status, s,
                          g_build_cluster, g_inject == 1, layout, l.map, l.nrb, l.g1, l.g2);
  }
  if (e != cudaSuccess) return USK_ERR_CUDA;
  return from_cuda(cudaGetLastError());
}

USK_API usk_status usk_gemv_ex(const usk_sketch* sketch, const void* x, usk_dtype xdtype, int64_t batch, float* y,
                               uint32_t flags, uint32_t* d_status, void* stream) {
  usk_status st = check_sketch(sketch);
  if (st != USK_OK) return st;
  if (xdtype != USK_F32 && xdtype != USK_BF16) return USK_ERR_DTYPE;
  if (batch < 0 || batch > USK_GEMV_MAX_BATCH) return USK_ERR_BATCH;
  if ((flags & ~static_cast<uint32_t>(USK_GEMV_PDL)) != 0) return USK_ERR_PARAMS;
  if (batch == 0 || sketch->M == 0) return USK_OK;
  if (!y) return USK_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (sketch->K == 0)
    return from_cuda(cudaMemsetAsync(y, 0, sizeof(float) * static_cast<size_t>(batch * sketch->M), s));
  if (!x) return USK_ERR_NULL;
  if (!aligned16(x)) return USK_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(y) & 3u) != 0) return USK_ERR_ALIGN;
  if (sketch->version == USK_FORMAT_COLSHARED) {
    cudaError_t e = usk::launch_gemv_cs(sketch->codes, sketch->scales, sketch->M, sketch->K, sketch->seed, x,
                                        xdtype == USK_F32, static_cast<int>(batch), y, d_status,
                                        (flags & USK_GEMV_PDL) != 0, s, g_gemv_tiles_per_block, g_gemv_rows,
                                        g_inject == 3);
    if (e != cudaSuccess) return USK_ERR_CUDA;
    return from_cuda(cudaGetLastError());
  }
  const Launch l = launch_of(sketch->rates, sketch->M);
  cudaError_t e = usk::launch_gemv(sketch->codes, sketch->scales, sketch->M, sketch->K, sketch->seed, x,
                                   xdtype == USK_F32, static_cast<int>(batch), y, d_status,
                                   (flags & USK_GEMV_PDL) != 0, g_gemv_path, s, g_gemv_tiles_per_block, g_gemv_rows,
                                   g_inject == 3, format_depth(sketch->version, sketch->depth),
                                   layout_of(sketch->version, sketch->slots), l.map, l.nrb, l.g1, l.g2);
  if (e != cudaSuccess) return USK_ERR_CUDA;
  return from_cuda(cudaGetLastError());
}

USK_API usk_status usk_gemv(const usk_sketch* sketch, const void* x, usk_dtype xdtype, int64_t batch, float* y,
                            uint32_t* d_status, void* stream) {
  return usk_gemv_ex(sketch, x, xdtype, batch, y, 0u, d_status, stream);
}

USK_API usk_status usk_gemm(const usk_sketch* sketch, const uint16_t* x_bf16, int64_t batch, float* y, void* ws,
                    size_t ws_bytes, uint32_t* d_status, void* stream) {
  (void)ws;
  (void)ws_bytes;
  return usk_gemm_ex(sketch, x_bf16, batch, y, 0u, d_status, stream);
}

USK_API usk_status usk_gemm_ex(const usk_sketch* sketch, const uint16_t* x_bf16, int64_t batch, float* y,
                               uint32_t flags, uint32_t* d_status, void* stream) {
  if ((flags & ~static_cast<uint32_t>(USK_GEMM_PDL)) != 0) return USK_ERR_PARAMS;
  usk_status st = check_sketch(sketch);
  if (st != USK_OK) return st;
  if (sketch->version == USK_FORMAT_COLSHARED) return USK_ERR_PARAMS;  // format 3: usk_gemv only
  if (batch < USK_GEMM_MIN_BATCH || batch > USK_GEMM_MAX_BATCH || batch % 16 != 0) return USK_ERR_BATCH;
  const int depth = format_depth(sketch->version, sketch->depth);
  const int layout = layout_of(sketch->version, sketch->slots);
  if (!usk::gemm_supported(sketch->K, static_cast<int>(batch), depth, layout)) return USK_ERR_SHAPE;
  if (sketch->rates && !usk::gemm_supported(sketch->K, static_cast<int>(batch), 1, 3))
    return USK_ERR_SHAPE;  // the 8-slot group stages the most codes
  if (sketch->M == 0) return USK_OK;
  if (!y) return USK_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (sketch->K == 0)
    return from_cuda(cudaMemsetAsync(y, 0, sizeof(float) * static_cast<size_t>(batch * sketch->M), s));
  if (!x_bf16) return USK_ERR_NULL;
  if (!aligned16(x_bf16) || !aligned16(y)) return USK_ERR_ALIGN;
  const Launch l = launch_of(sketch->rates, sketch->M);
  cudaError_t e = usk::launch_gemm(sketch->codes, sketch->scales, sketch->M, sketch->K, sketch->seed, x_bf16,
                                   static_cast<int>(batch), y, d_status, s, g_inject == 2, depth, layout, l.map,
                                   l.nrb, l.g1, l.g2, g_gemm_splits, g_gemm_issuers, (flags & USK_GEMM_PDL) != 0);
  if (e != cudaSuccess) return USK_ERR_CUDA;
  return from_cuda(cudaGetLastError());
}

USK_API usk_status usk_gemv_multi_ws_bytes(int64_t n, const usk_sketch* sketches, int64_t batch, size_t* ws_bytes) {
  int64_t Ms[kMultiMax], Ks[kMultiMax];
  int idx[kMultiMax], nw = 0;
  usk_status st = check_multi(n, sketches, batch, Ms, Ks, idx, &nw);
  if (st != USK_OK) return st;
  if (!ws_bytes) return USK_ERR_NULL;
  const usk_sketch* k0 = nw > 0 ? &sketches[idx[0]] : nullptr;
  *ws_bytes = (nw > 0 && batch > 0) ? usk::gemv_multi_ws_bytes(nw, Ms, Ks, static_cast<int>(batch),
                                                              format_depth(k0->version, k0->depth),
                                                              layout_of(k0->version, k0->slots))
                                    : 0;
  return USK_OK;
}

USK_API usk_status usk_gemv_multi(int64_t n, const usk_sketch* sketches, const void* const* x, usk_dtype xdtype,
                                  int64_t batch, float* const* y, void* ws, size_t ws_bytes, uint32_t flags,
                                  uint32_t* d_status, void* stream) {
  int64_t Ms[kMultiMax], Ks[kMultiMax];
  int idx[kMultiMax], nw = 0;
  usk_status st = check_multi(n, sketches, batch, Ms, Ks, idx, &nw);
  if (st != USK_OK) return st;
  if (xdtype != USK_BF16) return USK_ERR_DTYPE;  // fp32 x: usk_gemv
  if ((flags & ~static_cast<uint32_t>(USK_GEMV_PDL)) != 0) return USK_ERR_PARAMS;
  if (n == 0 || batch == 0) return USK_OK;
  if (!x || !y) return USK_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int64_t l = 0; l < n; ++l) {
    if (sketches[l].M == 0) continue;
    if (!y[l]) return USK_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(y[l]) & 3u) != 0) return USK_ERR_ALIGN;
    if (sketches[l].K == 0) continue;
    if (!x[l]) return USK_ERR_NULL;
    if (!aligned16(x[l])) return USK_ERR_ALIGN;
  }
  const usk_sketch* kw = nw > 0 ? &sketches[idx[0]] : nullptr;
  const size_t need = nw > 0 ? usk::gemv_multi_ws_bytes(nw, Ms, Ks, static_cast<int>(batch),
                                                        format_depth(kw->version, kw->depth),
                                                        layout_of(kw->version, kw->slots))
                             : 0;
  if (need > 0) {
    if (!ws || ws_bytes < need) return USK_ERR_WORKSPACE;
    if (!aligned16(ws)) return USK_ERR_ALIGN;
  }
  for (int64_t l = 0; l < n; ++l)  // K == 0: y = 0
    if (sketches[l].M > 0 && sketches[l].K == 0) {
      cudaError_t e = cudaMemsetAsync(y[l], 0, sizeof(float) * static_cast<size_t>(batch * sketches[l].M), s);
      if (e != cudaSuccess) return USK_ERR_CUDA;
    }
  if (nw == 0) return USK_OK;
  const int8_t* codes[kMultiMax];
  const uint16_t* scales[kMultiMax];
  const uint16_t* xs[kMultiMax];
  float* ys[kMultiMax];
  uint64_t seeds[kMultiMax];
  for (int w = 0; w < nw; ++w) {
    const usk_sketch& k = sketches[idx[w]];
    codes[w] = k.codes;
    scales[w] = k.scales;
    seeds[w] = k.seed;
    xs[w] = static_cast<const uint16_t*>(x[idx[w]]);
    ys[w] = y[idx[w]];
  }
  const usk_sketch& k0 = sketches[idx[0]];
  cudaError_t e = usk::launch_gemv_multi(nw, codes, scales, Ms, Ks, seeds, xs, ys, static_cast<int>(batch), ws,
                                         d_status, (flags & USK_GEMV_PDL) != 0, s, g_inject == 4,
                                         format_depth(k0.version, k0.depth), layout_of(k0.version, k0.slots));
  if (e != cudaSuccess) return USK_ERR_CUDA;
  return from_cuda(cudaGetLastError());
}

USK_API usk_status usk_gemv_multi_static(int64_t n, const usk_sketch* sketches, const void* const* x,
                                         usk_dtype xdtype, int64_t batch, float* const* y, uint32_t flags,
                                         uint32_t* d_status, void* stream) {
  int64_t Ms[kMultiMax], Ks[kMultiMax];
  int idx[kMultiMax], nw = 0;
  usk_status st = check_multi(n, sketches, batch, Ms, Ks, idx, &nw);
  if (st != USK_OK) return st;
  if (xdtype != USK_BF16) return USK_ERR_DTYPE;
  if ((flags & ~static_cast<uint32_t>(USK_GEMV_PDL)) != 0) return USK_ERR_PARAMS;
  if (n == 0 || batch == 0) return USK_OK;
  if (!x || !y) return USK_ERR_NULL;
  for (int64_t l = 0; l < n; ++l) {
    if (sketches[l].M == 0) continue;
    if (!y[l]) return USK_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(y[l]) & 3u) != 0) return USK_ERR_ALIGN;
    if (sketches[l].K == 0) continue;
    if (!x[l]) return USK_ERR_NULL;
    if (!aligned16(x[l])) return USK_ERR_ALIGN;
  }
  int depth = 1, layout = 0;
  if (nw > 0) {
    const usk_sketch& k0 = sketches[idx[0]];
    depth = format_depth(k0.version, k0.depth);
    layout = layout_of(k0.version, k0.slots);
    // the list's scratch must fit the library's fixed array
    if (usk::gemv_multi_ws_bytes(nw, Ms, Ks, static_cast<int>(batch), depth, layout) > USK_GEMV_MULTI_STATIC_BYTES)
      return USK_ERR_WORKSPACE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int64_t l = 0; l < n; ++l)  // K == 0: y = 0
    if (sketches[l].M > 0 && sketches[l].K == 0) {
      cudaError_t e = cudaMemsetAsync(y[l], 0, sizeof(float) * static_cast<size_t>(batch * sketches[l].M), s);
      if (e != cudaSuccess) return USK_ERR_CUDA;
    }
  if (nw == 0) return USK_OK;
  const int8_t* codes[kMultiMax];
  const uint16_t* scales[kMultiMax];
  const uint16_t* xs[kMultiMax];
  float* ys[kMultiMax];
  uint64_t seeds[kMultiMax];
  for (int w = 0; w < nw; ++w) {
    const usk_sketch& k = sketches[idx[w]];
    codes[w] = k.codes;
    scales[w] = k.scales;
    seeds[w] = k.seed;
    xs[w] = static_cast<const uint16_t*>(x[idx[w]]);
    ys[w] = y[idx[w]];
  }
  cudaError_t e = usk::launch_gemv_multi_static(nw, codes, scales, Ms, Ks, seeds, xs, ys, static_cast<int>(batch),
                                                d_status, (flags & USK_GEMV_PDL) != 0, s, depth, layout);
  if (e != cudaSuccess) return USK_ERR_CUDA;
  return from_cuda(cudaGetLastError());
}

// Test hooks: launch-geometry overrides// Test hooks: launch-geometry overrides (0 restores the defaults).  They change
// how work is split between thread blocks, never the result.
USK_API void usk_debug_set_geometry(int build_cluster, int gemv_tiles_per_block) {
  g_build_cluster = build_cluster;
  g_gemv_tiles_per_block = gemv_tiles_per_block;
}

USK_API void usk_debug_set_gemv_path(int path) { g_gemv_path = path; }

USK_API void usk_debug_set_gemv_rows(int rows) { g_gemv_rows = rows; }

USK_API void usk_debug_set_gemm_splits(int splits) { g_gemm_splits = splits; }

USK_API void usk_debug_set_gemm_issuers(int issuers) { g_gemm_issuers = issuers; }

USK_API void usk_debug_inject_timeout(int kernel) { g_inject = kernel; }

}  // extern "C"

// moe_api.cu -- the C ABI declared in include/moe.h: argument checks,
// workspace layout, TMA tensor maps and the launch sequence of the layer.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/moe.h"
#include "kernels.h"
#include "status.cuh"

namespace moe {
cudaError_t gemm_set_attributes();
cudaError_t gemm_pair_set_attributes();
cudaError_t gemm_pair_max_clusters(int *clusters);
cudaError_t gemm_fused_set_attributes();
}

namespace {

using namespace moe;

thread_local int32_t g_last_launches = 0;
#ifdef MOE_TRACE
unsigned long long *g_trace_gemm1 = nullptr;
unsigned long long *g_trace_gemm2 = nullptr;
#endif
thread_local void **g_prof_events = nullptr;
thread_local int32_t g_prof_n = 0;

// Records the next armed profiling event (if any) on stream s.  Takes over
// the armed event list, so only one call records into it.
struct EventMarker {
  cudaStream_t s;
  void **events;
  int n;
  int next = 0;
  explicit EventMarker(cudaStream_t st) : s(st), events(g_prof_events), n(g_prof_n) {
    g_prof_events = nullptr;
    g_prof_n = 0;
  }
  void mark() {
    if (events != nullptr && next < n && events[next] != nullptr)
      cudaEventRecord(static_cast<cudaEvent_t>(events[next]), s);
    ++next;
  }
};

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_sms[kMaxDevices] = {0};
int g_pair_clusters[kMaxDevices] = {0};
bool g_attrs[kMaxDevices] = {false};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Per-device one-time set-up: SM count, shared-memory limits of the GEMM kernels.
cudaError_t device_setup(int *sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
      return e != cudaSuccess ? e : cudaErrorNotSupported;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  if (!g_attrs[dev]) {
    e = cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = gemm_set_attributes();
    if (e != cudaSuccess) return e;
    e = gemm_pair_set_attributes();
    if (e != cudaSuccess) return e;
    e = gemm_pair_max_clusters(&g_pair_clusters[dev]);
    if (e != cudaSuccess) return e;
    e = gemm_fused_set_attributes();
    if (e != cudaSuccess) return e;
    g_attrs[dev] = true;
  }
  *sms = g_sms[dev];
  return cudaSuccess;
}

int pair_clusters() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev >= 0 && dev < kMaxDevices) ? g_pair_clusters[dev] : 0;
}

// 2-D tensor [rows, cols] (row-major), 128-byte swizzle, box of one 128-byte
// row segment (64 16-bit or 128 8-bit elements) x box_rows.
bool make_map(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  const uint64_t esize = dtype == CU_TENSOR_MAP_DATA_TYPE_UINT8 ? 1 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esize), box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, dtype, 2, const_cast<void *>(ptr), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Dims {
  int T, d, E, k, F, Fs, flags, norm;
  float scale;
};

struct WsLayout {
  size_t header, chunk_hist, tiles, tiles_pair, logits, inv, h, h_sh, o, s_out, yacc, down16,
      down16_sh;
  size_t xq, sx, hq, sh, hshq, shs;  // FP8 experts: e4m3 rows of x, h, h_shared and their scales
  size_t total;
  int max_tiles;
};

bool use_tensor_router(const Dims &D);

// K slices of the tensor-core router GEMM: with few 128-token tiles, up to 4
// slices of d (each slice's CTAs write partial logits, summed in slice order
// by the select kernel), so that about one CTA per SM streams its share of x
// once instead of a few CTAs streaming whole rows.  Four slices only up to 18
// tiles (T <= 2304): at T = 4096 two slices measured faster than four (router
// GEMM + select 28.0 against 30.4 us, ncu), the select kernel summing half as
// many planes.  A function of the dimensions only, since the workspace holds
// one logit plane per slice.
constexpr int kRouterSplitSms = 148;
int router_ksplit(const Dims &D) {
  if (!use_tensor_router(D)) return 1;
  const int tiles = (D.T + kBlockM - 1) / kBlockM;
  const int max_ks = tiles <= kRouterSplitSms / 8 ? 4 : 2;
  int ks = 1;
  while (ks < max_ks && tiles * ks * 2 <= kRouterSplitSms && (D.d / kBlockK) % (ks * 2) == 0)
    ks *= 2;
  return ks;
}

WsLayout ws_layout(const Dims &D) {
  WsLayout L;
  const size_t n = static_cast<size_t>(D.T) * D.k;
  const size_t nchunks = (n + index_chunk_entries(n) - 1) / index_chunk_entries(n);
  L.max_tiles = static_cast<int>((n + kBlockM - 1) / kBlockM + D.E + (D.T + kBlockM - 1) / kBlockM);
  size_t off = 0;
  L.header = off;
  off += align256(sizeof(WsHeader));
  L.chunk_hist = off;
  off += align256(std::max<size_t>(nchunks, 1) * D.E * 4);
  L.tiles = off;  // 128-row tiles (single-CTA GEMMs)
  off += align256(static_cast<size_t>(L.max_tiles) * sizeof(Tile));
  L.tiles_pair = off;  // 256-row tiles (CTA-pair GEMMs); fewer than the 128-row ones
  off += align256(static_cast<size_t>(L.max_tiles) * sizeof(Tile));
  L.logits = off;  // plane 0: the logits; planes 1..: partial logits of the router's K slices
  off += align256(static_cast<size_t>(router_ksplit(D)) * D.T * D.E * 4);
  L.inv = off;
  off += align256(n * 4);
  const bool fused = (D.flags & MOE_FLAG_FUSED_EXPERTS) != 0;
  L.h = L.h_sh = off;
  if (!fused) {  // the fused kernel keeps h in tensor memory
    L.h = off;
    off += align256(n * D.F * 2);
    L.h_sh = off;
    off += align256(static_cast<size_t>(D.T) * D.Fs * 2);
  }
  L.o = L.s_out = L.yacc = off;
  if (D.flags & (MOE_FLAG_COMBINE_REDUCE | MOE_FLAG_FUSED_EXPERTS)) {
    L.yacc = off;  // fp32 token rows the down GEMM reduces into
    off += align256(static_cast<size_t>(D.T) * D.d * 4);
  } else {
    L.o = off;  // routed contributions, expert-order rows
    off += align256(n * D.d * 2);
    L.s_out = off;  // shared-expert output, token rows
    off += align256(D.Fs > 0 ? static_cast<size_t>(D.T) * D.d * 2 : 0);
  }
  L.down16 = L.down16_sh = off;
  // per-call fp16 copy of the down projections (16-bit path without prepared copies)
  if (!(D.flags & (MOE_FLAG_DOWN_F16 | MOE_FLAG_FP8_EXPERTS))) {
    off += align256(static_cast<size_t>(D.E) * D.d * D.F * 2);
    L.down16_sh = off;
    off += align256(static_cast<size_t>(D.d) * D.Fs * 2);
  }
  L.xq = L.sx = L.hq = L.sh = L.hshq = L.shs = off;
  if (D.flags & MOE_FLAG_FP8_EXPERTS) {
    L.xq = off;
    off += align256(static_cast<size_t>(D.T) * D.d);
    L.sx = off;
    off += align256(static_cast<size_t>(D.T) * 4);
    L.hq = off;
    off += align256(n * D.F);
    L.sh = off;
    off += align256(n * 4);
    L.hshq = off;
    off += align256(static_cast<size_t>(D.T) * D.Fs);
    L.shs = off;
    off += align256(static_cast<size_t>(D.T) * 4);
  }
  L.total = off;
  return L;
}

// Width of one part of an FFN of width f in the fused kernel: f split into the
// fewest equal parts of at most 512 columns (and at least min_parts parts, as
// far as parts of whole 128-column chunks allow); 0 if no such split exists.
int fused_part(int f, int min_parts = 1) {
  if (f <= 0 || f % 128 != 0) return 0;
  int parts = (f + 511) / 512;
  while (parts <= f / 128 && (f % parts != 0 || (f / parts) % 128 != 0)) ++parts;
  if (parts > f / 128) return 0;
  int best = parts;
  for (int q = parts; q <= f / 128 && best < min_parts; ++q)
    if (f % q == 0 && (f / q) % 128 == 0) best = q;
  return f / best;
}

moe_status check_dims(const moe_dims_t *dims, Dims *D) {
  if (dims == nullptr || dims->struct_size != sizeof(moe_dims_t)) return MOE_ERR_INVALID_ARG;
  D->T = dims->T;
  D->d = dims->d_model;
  D->E = dims->num_experts;
  D->k = dims->num_experts_per_tok;
  D->F = dims->moe_intermediate_size;
  D->Fs = dims->shared_intermediate_size;
  D->scale = dims->routed_scaling_factor;
  D->norm = dims->norm_topk_prob ? 1 : 0;
  D->flags = dims->flags;
  if (D->T < 0) return MOE_ERR_INVALID_ARG;
  if (D->d < 64 || D->d % 64 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (D->E < 1 || D->E > 512) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (D->k < 1 || D->k > 16 || D->k > D->E) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (D->F < 64 || D->F % 64 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (D->Fs < 0 || D->Fs % 64 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(D->T) * D->k >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(D->E) * std::max(D->F, D->d) >= (int64_t(1) << 31))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((dims->flags & MOE_FLAG_ROUTER_TENSOR) && (D->E % 16 != 0 || D->E > 256))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  // FP8 experts: K stages of 128 e4m3 elements; 256-column down-projection tiles
  if ((dims->flags & MOE_FLAG_FP8_EXPERTS) &&
      (D->F % 128 != 0 || D->Fs % 128 != 0 || D->d % 256 != 0))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  // fused experts: 128-column chunks of each FFN part and 128-column d tiles
  if ((dims->flags & MOE_FLAG_FUSED_EXPERTS) &&
      (D->d % 128 != 0 || fused_part(D->F) == 0 || (D->Fs > 0 && fused_part(D->Fs) == 0)))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

// Shapes the router itself cannot take: a batch routed on CUDA cores stages
// 8 bf16 token rows per CTA in shared memory (227 KB at most; router_cc.cu),
// so d is capped on that path.
constexpr int kRouterCcMaxD = 232448 / (8 * 2);
moe_status check_router_dims(const Dims &D) {
  if (!use_tensor_router(D) && D.d > kRouterCcMaxD) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

moe_status check_ws(const Dims &D, const void *ws, size_t ws_bytes) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < ws_layout(D).total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return MOE_OK;
}

inline char *wsp(void *ws, size_t off) { return static_cast<char *>(ws) + off; }

bool use_tensor_router(const Dims &D) {
  if (D.flags & MOE_FLAG_ROUTER_CUDA_CORE) return false;
  const bool fits = D.E % 16 == 0 && D.E <= 256;
  if (D.flags & MOE_FLAG_ROUTER_TENSOR) return fits;
  return fits && D.T >= 1024;
}

// Router: fp32 logits (tcgen05 GEMM or CUDA-core FMA) into the workspace,
// then the warp-per-token selection kernel.
moe_status route_impl(const Dims &D, const void *x, const void *w_router, const float *bias,
                      const uint8_t *token_mask, int32_t *topk_idx, float *topk_w, void *ws,
                      cudaStream_t s, int sms, int *launches,
                      const SelectIndexOut *ix = nullptr, bool *indexed = nullptr) {
  if (indexed) *indexed = false;
  const WsLayout L = ws_layout(D);
  float *logits = reinterpret_cast<float *>(wsp(ws, L.logits));
  // A selection-only bias stays out of the logits and goes to the select kernel.
  const float *sel_bias = (D.flags & MOE_FLAG_BIAS_SELECTION_ONLY) ? bias : nullptr;
  if (sel_bias) bias = nullptr;
  if (use_tensor_router(D)) {
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.status = reinterpret_cast<int *>(wsp(ws, L.header));
    p.n_tiles_host = (D.T + kBlockM - 1) / kBlockM;
    p.ksplit = router_ksplit(D);
    // Still few items (small T): split the experts into column blocks too, so
    // that more SMs share the work; each block re-reads the token tile from L2.
    int nsplit = 1;
    while (nsplit < 8 && p.n_tiles_host * p.ksplit * nsplit * 2 <= sms &&
           D.E % (nsplit * 2 * 32) == 0)
      nsplit *= 2;
    p.n_ntiles = nsplit;
    p.T = D.T;
    p.d = D.d;
    p.E = D.E;
    p.k = D.k;
    p.F = D.F;
    p.Fs = D.Fs;
    p.n_tile = D.E / nsplit;
    p.bias = bias;
    p.logits_out = logits;

    const uint32_t a_rows = static_cast<uint32_t>(std::min(D.T, kBlockM));
    p.a_bytes = a_rows * kBlockK * 2;
    GemmMaps m;
    std::memset(&m, 0, sizeof(m));
    if (!make_map(&m.a, x, D.T, D.d, a_rows)) return MOE_ERR_CUDA;
    if (!make_map(&m.b0, w_router, D.E, D.d, p.n_tile)) return MOE_ERR_CUDA;
    m.b1 = m.b0;
    m.a_sh = m.a;
    m.b0_sh = m.b0;
    m.b1_sh = m.b0;
    const int grid = std::min(sms, p.n_tiles_host * p.n_ntiles * p.ksplit);
    if (launch_gemm(MODE_ROUTER, p, m, grid, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (launch_router_select(logits, p.ksplit, static_cast<const uint16_t *>(x),
                             static_cast<const uint16_t *>(w_router), bias, sel_bias, token_mask,
                             D.T, D.d, D.E, D.k, D.norm, topk_idx, topk_w, s, ix,
                             indexed) != cudaSuccess)
      return MOE_ERR_CUDA;
    *launches += 2;
    return MOE_OK;
  }
  if (launch_router_cc(static_cast<const uint16_t *>(x), static_cast<const uint16_t *>(w_router),
                       bias, logits, D.T, D.d, D.E, sms, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (launch_router_select(logits, 1, static_cast<const uint16_t *>(x),
                           static_cast<const uint16_t *>(w_router), bias, sel_bias, token_mask,
                           D.T, D.d, D.E, D.k, D.norm, topk_idx, topk_w, s, ix,
                           indexed) != cudaSuccess)
    return MOE_ERR_CUDA;
  *launches += 2;
  return MOE_OK;
}

moe_status clear_header(void *ws, cudaStream_t s) {
  return cudaMemsetAsync(ws, 0, sizeof(WsHeader), s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status check_routing_ptrs(const moe_routing_t *r) {
  const void *ptrs[] = {r->topk_idx, r->topk_w, r->counts, r->offsets, r->perm};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status check_fp8_ptrs(const Dims &D, const moe_fp8_weights_t *q) {
  const void *ptrs[] = {q->w_gate, q->w_up, q->w_down, q->s_gate, q->s_up, q->s_down};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (D.Fs > 0) {
    const void *sh[] = {q->ws_gate, q->ws_up, q->ws_down, q->ss_gate, q->ss_up, q->ss_down};
    for (const void *p : sh)
      if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

// The whole layer after argument checks; q != nullptr selects the FP8 experts.
moe_status forward_impl(const Dims &D, const moe_weights_t *w, const moe_fp8_weights_t *q,
                        const void *x, const uint8_t *token_mask, void *y,
                        const moe_routing_t *routing, void *ws, void *stream);

}  // namespace

namespace moe {
// Launch accounting of entry points implemented in other files.
void set_last_launch_count(int n) { g_last_launches = n; }
}  // namespace moe

extern "C" {

size_t moe_workspace_size(const moe_dims_t *dims) {
  Dims D;
  if (check_dims(dims, &D) != MOE_OK) return 0;
  return ws_layout(D).total;
}

moe_status moe_route(const moe_dims_t *dims, const void *x, const void *w_router,
                     const float *router_bias, int32_t *topk_idx, float *topk_w, void *ws,
                     size_t ws_bytes, void *stream) {
  return moe_route_masked(dims, x, w_router, router_bias, nullptr, topk_idx, topk_w, ws, ws_bytes,
                          stream);
}

moe_status moe_route_masked(const moe_dims_t *dims, const void *x, const void *w_router,
                            const float *router_bias, const uint8_t *token_mask,
                            int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes,
                            void *stream) {
  Dims D;
  moe_status st = check_dims(dims, &D);
  if (st != MOE_OK) return st;
  if ((st = check_router_dims(D)) != MOE_OK) return st;
  if (!x || !w_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(topk_idx) || !aligned16(topk_w) ||
      (router_bias && !aligned16(router_bias)))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(D, ws, ws_bytes)) != MOE_OK) return st;
  g_last_launches = 0;
  if (D.T == 0) return MOE_OK;
  int sms = 0;
  if (device_setup(&sms) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = clear_header(ws, s)) != MOE_OK) return st;
  int launches = 0;
  st = route_impl(D, x, w_router, router_bias, token_mask, topk_idx, topk_w, ws, s, sms,
                  &launches);
  g_last_launches = launches;
  return st;
}

moe_status moe_permute(const moe_dims_t *dims, const int32_t *topk_idx, int32_t *counts,
                       int32_t *offsets, int32_t *perm, const void *x, void *x_perm, void *ws,
                       size_t ws_bytes, void *stream) {
  Dims D;
  moe_status st = check_dims(dims, &D);
  if (st != MOE_OK) return st;
  if (!topk_idx || !counts || !offsets || !perm) return MOE_ERR_INVALID_ARG;
  if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(topk_idx) || !aligned16(counts) || !aligned16(offsets) || !aligned16(perm) ||
      (x && (!aligned16(x) || !aligned16(x_perm))))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(D, ws, ws_bytes)) != MOE_OK) return st;
  g_last_launches = 0;
  if (D.T == 0) return MOE_OK;
  int sms = 0;
  if (device_setup(&sms) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = clear_header(ws, s)) != MOE_OK) return st;
  const WsLayout L = ws_layout(D);
  int launches = 0;
  if (launch_index(topk_idx, D.T, D.k, D.E, D.Fs > 0, reinterpret_cast<int *>(wsp(ws, L.chunk_hist)),
                   reinterpret_cast<Tile *>(wsp(ws, L.tiles)),
                   reinterpret_cast<int *>(wsp(ws, L.header)), counts, offsets, perm, s,
                   &launches) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (x) {
    if (launch_gather_rows(static_cast<const uint16_t *>(x), perm, offsets + D.E, D.T * D.k, D.k,
                           D.d, static_cast<uint16_t *>(x_perm), s) != cudaSuccess)
      return MOE_ERR_CUDA;
    launches += 1;
  }
  g_last_launches = launches;
  return MOE_OK;
}

moe_status moe_forward(const moe_dims_t *dims, const moe_weights_t *w, const void *x, void *y,
                       const moe_routing_t *routing, void *ws, size_t ws_bytes, void *stream) {
  return moe_forward_masked(dims, w, x, nullptr, y, routing, ws, ws_bytes, stream);
}

moe_status moe_forward_masked(const moe_dims_t *dims, const moe_weights_t *w, const void *x,
                              const uint8_t *token_mask, void *y, const moe_routing_t *routing,
                              void *ws, size_t ws_bytes, void *stream) {
  Dims D;
  moe_status st = check_dims(dims, &D);
  if (st != MOE_OK) return st;
  if ((st = check_router_dims(D)) != MOE_OK) return st;
  if (!w || !x || !y || !routing) return MOE_ERR_INVALID_ARG;
  if (!w->w_router || !w->w_gate || !w->w_up || !w->w_down) return MOE_ERR_INVALID_ARG;
  if (D.Fs > 0 && (!w->ws_gate || !w->ws_up || !w->ws_down)) return MOE_ERR_INVALID_ARG;
  if ((st = check_routing_ptrs(routing)) != MOE_OK) return st;
  const void *ptrs[] = {x, y, w->w_router, w->w_gate, w->w_up, w->w_down};
  for (const void *p : ptrs)
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (w->router_bias && !aligned16(w->router_bias)) return MOE_ERR_INVALID_ARG;
  if (D.Fs > 0 && (!aligned16(w->ws_gate) || !aligned16(w->ws_up) || !aligned16(w->ws_down)))
    return MOE_ERR_INVALID_ARG;
  if (D.flags & MOE_FLAG_DOWN_F16) {
    if (!w->w_down_f16 || !aligned16(w->w_down_f16)) return MOE_ERR_INVALID_ARG;
    if (D.Fs > 0 && (!w->ws_down_f16 || !aligned16(w->ws_down_f16))) return MOE_ERR_INVALID_ARG;
  } else if (D.flags & MOE_FLAG_FP8_EXPERTS) {
    return MOE_ERR_INVALID_ARG;  // that workspace has no room for the per-call fp16 copy
  }
  if ((st = check_ws(D, ws, ws_bytes)) != MOE_OK) return st;
  return forward_impl(D, w, nullptr, x, token_mask, y, routing, ws, stream);
}

moe_status moe_forward_fp8(const moe_dims_t *dims, const moe_weights_t *w,
                           const moe_fp8_weights_t *q, const void *x, void *y,
                           const moe_routing_t *routing, void *ws, size_t ws_bytes, void *stream) {
  Dims D;
  moe_status st = check_dims(dims, &D);
  if (st != MOE_OK) return st;
  if ((st = check_router_dims(D)) != MOE_OK) return st;
  if (!(D.flags & MOE_FLAG_FP8_EXPERTS) ||
      (D.flags & (MOE_FLAG_COMBINE_REDUCE | MOE_FLAG_FUSED_EXPERTS)))
    return MOE_ERR_INVALID_ARG;
  if (!w || !q || !x || !y || !routing || !w->w_router) return MOE_ERR_INVALID_ARG;
  if ((st = check_fp8_ptrs(D, q)) != MOE_OK) return st;
  if ((st = check_routing_ptrs(routing)) != MOE_OK) return st;
  if (!aligned16(x) || !aligned16(y) || !aligned16(w->w_router) ||
      (w->router_bias && !aligned16(w->router_bias)))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(D, ws, ws_bytes)) != MOE_OK) return st;
  return forward_impl(D, w, q, x, nullptr, y, routing, ws, stream);
}

moe_status moe_prepare_fp8(const moe_dims_t *dims, const moe_weights_t *w,
                           const moe_fp8_weights_t *q, void *ws, size_t ws_bytes, void *stream) {
  Dims D;
  moe_status st = check_dims(dims, &D);
  if (st != MOE_OK) return st;
  if (!w || !q || !w->w_gate || !w->w_up || !w->w_down) return MOE_ERR_INVALID_ARG;
  if (D.Fs > 0 && (!w->ws_gate || !w->ws_up || !w->ws_down)) return MOE_ERR_INVALID_ARG;
  if ((st = check_fp8_ptrs(D, q)) != MOE_OK) return st;
  if (ws == nullptr || ws_bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(ws) & 255))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  if (device_setup(&sms) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = clear_header(ws, s)) != MOE_OK) return st;
  const int EF = D.E * D.F, Ed = D.E * D.d;
  struct Job { const void *src; int rows, K; void *codes; float *scales; };
  const Job jobs[] = {{w->w_gate, EF, D.d, q->w_gate, q->s_gate},
                      {w->w_up, EF, D.d, q->w_up, q->s_up},
                      {w->w_down, Ed, D.F, q->w_down, q->s_down},
                      {w->ws_gate, D.Fs, D.d, q->ws_gate, q->ss_gate},
                      {w->ws_up, D.Fs, D.d, q->ws_up, q->ss_up},
                      {w->ws_down, D.Fs > 0 ? D.d : 0, D.Fs, q->ws_down, q->ss_down}};
  int launches = 0;
  for (const Job &j : jobs) {
    if (j.rows == 0) continue;
    if (launch_quant_rows_e4m3(static_cast<const uint16_t *>(j.src), false, false, j.rows, nullptr,
                               j.K, static_cast<uint8_t *>(j.codes), j.scales, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    ++launches;
  }
  g_last_launches = launches;
  return MOE_OK;
}

}  // extern "C"

namespace {

moe_status forward_impl(const Dims &D, const moe_weights_t *w, const moe_fp8_weights_t *q,
                        const void *x, const uint8_t *token_mask, void *y,
                        const moe_routing_t *routing, void *ws, void *stream) {
  moe_status st = MOE_OK;
  const bool fp8 = q != nullptr;
  g_last_launches = 0;
  if (D.T == 0) return MOE_OK;
  int sms = 0;
  if (device_setup(&sms) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = clear_header(ws, s)) != MOE_OK) return st;
  const WsLayout L = ws_layout(D);
  int *header = reinterpret_cast<int *>(wsp(ws, L.header));
  Tile *tiles = reinterpret_cast<Tile *>(wsp(ws, L.tiles));
  uint16_t *h = reinterpret_cast<uint16_t *>(wsp(ws, L.h));
  uint16_t *h_sh = reinterpret_cast<uint16_t *>(wsp(ws, L.h_sh));
  const bool fused = (D.flags & MOE_FLAG_FUSED_EXPERTS) != 0 && !fp8;
  const bool reduce = ((D.flags & MOE_FLAG_COMBINE_REDUCE) != 0 || fused) && !fp8;
  uint16_t *o_out = reduce ? nullptr : reinterpret_cast<uint16_t *>(wsp(ws, L.o));
  uint16_t *s_out = (D.Fs > 0 && !reduce) ? reinterpret_cast<uint16_t *>(wsp(ws, L.s_out)) : nullptr;
  float *yacc = reduce ? reinterpret_cast<float *>(wsp(ws, L.yacc)) : nullptr;
  int32_t *inv = reinterpret_cast<int32_t *>(wsp(ws, L.inv));
  int launches = 0;
  EventMarker ev(s);

  // Engines, as measured on B200: the gate/up GEMM runs on single CTAs
  // (128-row tiles; with its A rows gathered by cp.async, the CTA-pair engine
  // lost 12-14% to it at the large prefill shapes); the down GEMM runs on CTA
  // pairs (256-row tiles, half of B per SM) when the average expert fills a
  // 256-row tile, below that single CTAs waste less of the tensor core.  The
  // flags force one engine for both.
  const int pair_grid = 2 * std::min(pair_clusters(), sms / 2);  // all pairs co-resident
  bool pair1 = false;
  bool pair2 = static_cast<int64_t>(D.T) * D.k >= static_cast<int64_t>(2 * kBlockM) * D.E;
  if (D.flags & MOE_FLAG_GEMM_PAIR) pair1 = pair2 = true;
  if (D.flags & MOE_FLAG_GEMM_SINGLE_CTA) pair1 = pair2 = false;
  if (pair_grid < 2 || fp8) pair1 = pair2 = false;
  Tile *tiles_pair = reinterpret_cast<Tile *>(wsp(ws, L.tiles_pair));
  SelectIndexOut ix;
  ix.with_shared = D.Fs > 0;
  ix.chunk_hist = reinterpret_cast<int *>(wsp(ws, L.chunk_hist));
  ix.counts = routing->counts;
  ix.offsets = routing->offsets;
  ix.perm = routing->perm;
  ix.inv = inv;
  ix.tiles = tiles;
  ix.tiles_pair = (pair1 || pair2) ? tiles_pair : nullptr;
  ix.header = header;

  // 1. router (for a decode-sized batch its selection kernel also builds the index); the
  // reduce combine's fp32 token rows are zeroed first (counted in the router stage)
  ev.mark();
  if (reduce &&
      cudaMemsetAsync(yacc, 0, static_cast<size_t>(D.T) * D.d * sizeof(float), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  bool indexed = false;
  st = route_impl(D, x, w->w_router, w->router_bias, token_mask, routing->topk_idx,
                  routing->topk_w, ws, s, sms, &launches, &ix, &indexed);
  if (st != MOE_OK) return st;
  // 2. expert order + tile lists
  ev.mark();
  if (!indexed &&
      launch_index(routing->topk_idx, D.T, D.k, D.E, D.Fs > 0, ix.chunk_hist, tiles, header,
                   routing->counts, routing->offsets, routing->perm, s, &launches, ix.tiles_pair,
                   inv) != cudaSuccess)
    return MOE_ERR_CUDA;

  // FP8 experts: e4m3 rows of x with their scales
  uint8_t *xq = reinterpret_cast<uint8_t *>(wsp(ws, L.xq));
  float *sx = reinterpret_cast<float *>(wsp(ws, L.sx));
  if (fp8) {
    if (launch_quant_rows_e4m3(static_cast<const uint16_t *>(x), false, false, D.T, nullptr, D.d,
                               xq, sx, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    launches += 1;
  }

  // fp16 down projections: caller-prepared, or converted here every call
  const void *wd16 = w->w_down_f16;
  const void *wsd16 = w->ws_down_f16;
  if (!fp8 && !(D.flags & MOE_FLAG_DOWN_F16)) {
    uint16_t *dst = reinterpret_cast<uint16_t *>(wsp(ws, L.down16));
    if (launch_bf16_to_f16(static_cast<const uint16_t *>(w->w_down),
                           static_cast<size_t>(D.E) * D.d * D.F, dst, header, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    wd16 = dst;
    launches += 1;
    if (D.Fs > 0) {
      uint16_t *dsh = reinterpret_cast<uint16_t *>(wsp(ws, L.down16_sh));
      if (launch_bf16_to_f16(static_cast<const uint16_t *>(w->ws_down),
                             static_cast<size_t>(D.d) * D.Fs, dsh, header, s) != cudaSuccess)
        return MOE_ERR_CUDA;
      wsd16 = dsh;
      launches += 1;
    }
  }

  const int n_rows = D.T * D.k;
  const int n_half = (D.F % 128 == 0 && D.Fs % 128 == 0) ? 128 : 64;
  // down-projection N tile: the widest of 256 / 128 / 64 columns that divides d
  const int n2 = (D.d % 256 == 0) ? 256 : (D.d % 128 == 0) ? 128 : 64;

  GemmParams base;
  std::memset(&base, 0, sizeof(base));
  base.status = header;
  int *n_tiles = header + offsetof(WsHeader, n_tiles) / sizeof(int);
  int *n_tiles_pair = header + offsetof(WsHeader, n_tiles_pair) / sizeof(int);
  base.T = D.T;
  base.d = D.d;
  base.E = D.E;
  base.k = D.k;
  base.F = D.F;
  base.Fs = D.Fs;
  base.routed_scale = D.scale;
  base.perm = routing->perm;
  base.topk_w = routing->topk_w;
  base.h = h;
  base.h_shared = h_sh;
  base.o_out = o_out;
  base.s_out = s_out;
  base.yacc = yacc;

  if (fused) {
    // 3+4. the fused expert kernel: gate/up GEMM, SwiGLU into tensor memory, down GEMM
    // with A from tensor memory, modulation and reduce combine into yacc
    GemmParams p = base;
    p.tiles = tiles;
    p.n_tiles_dev = n_tiles;
    // Items are (row tile, FFN part).  With few tiles (small batches: about one tile
    // per touched expert) the FFN is cut into more parts so that the persistent grid
    // has about three items per SM; each part adds its partial down projection into
    // the token rows, so more parts cost more reduce-adds (cheap at these sizes).
    const int64_t tiles_est = std::min<int64_t>(D.E, static_cast<int64_t>(D.T) * D.k) +
                              (static_cast<int64_t>(D.T) * D.k + kBlockM - 1) / kBlockM;
    const int want_parts = static_cast<int>(std::min<int64_t>(
        D.F / 128, (3 * static_cast<int64_t>(sms) + tiles_est - 1) / std::max<int64_t>(tiles_est, 1)));
    p.fp = fused_part(D.F, want_parts);
    p.n_parts = D.F / p.fp;
    // The shared expert's tiles come last in the tile list, so with few of them their
    // items are cut to single 128-column chunks and do not trail the routed ones.
    const int sh_tiles = (D.T + kBlockM - 1) / kBlockM;
    p.fp_sh = D.Fs > 0 ? fused_part(D.Fs, sh_tiles < sms ? D.Fs / 128 : want_parts) : 128;
    p.n_parts_sh = D.Fs > 0 ? D.Fs / p.fp_sh : 0;
    p.n_ntiles = std::max(p.n_parts, p.n_parts_sh);
    p.x = static_cast<const uint16_t *>(x);
    FusedMaps m;
    std::memset(&m, 0, sizeof(m));
    const CUtensorMapDataType f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (!make_map(&m.gate, w->w_gate, static_cast<uint64_t>(D.E) * D.F, D.d, 128) ||
        !make_map(&m.up, w->w_up, static_cast<uint64_t>(D.E) * D.F, D.d, 128) ||
        !make_map(&m.down, wd16, static_cast<uint64_t>(D.E) * D.d, D.F, 128, f16))
      return MOE_ERR_CUDA;
    if (D.Fs > 0) {
      if (!make_map(&m.gate_sh, w->ws_gate, D.Fs, D.d, 128) ||
          !make_map(&m.up_sh, w->ws_up, D.Fs, D.d, 128) ||
          !make_map(&m.down_sh, wsd16, D.d, D.Fs, 128, f16))
        return MOE_ERR_CUDA;
    } else {
      m.gate_sh = m.gate;
      m.up_sh = m.up;
      m.down_sh = m.down;
    }
    ev.mark();
    if (launch_gemm_fused(p, m, sms, s) != cudaSuccess) return MOE_ERR_CUDA;
    launches += 1;
    ev.mark();  // (no separate down GEMM)
    ev.mark();
    if (launch_finalize(yacc, static_cast<size_t>(D.T) * D.d, static_cast<uint16_t *>(y), s) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    launches += 1;
    ev.mark();
    g_last_launches = launches;
    return MOE_OK;
  }

  // 3. GEMM1: gathered x rows . [W_gate | W_up]^T -> SwiGLU -> h (bf16)
  {
    GemmParams p = base;
    p.tiles = pair1 ? tiles_pair : tiles;
    p.n_tiles_dev = pair1 ? n_tiles_pair : n_tiles;
    p.n_half = n_half;
    p.n_tile = 2 * n_half;
    p.n_ntiles = std::max(D.F, D.Fs) / n_half;
    p.x = static_cast<const uint16_t *>(x);
#ifdef MOE_TRACE
    p.trace = g_trace_gemm1;
#endif
    p.a_bytes = kBlockM * kBlockK * 2;
    p.a_sh_bytes = p.a_bytes;
    GemmMaps m;
    std::memset(&m, 0, sizeof(m));
    const CUtensorMapDataType bt = fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                       : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const void *wg = fp8 ? q->w_gate : w->w_gate;
    const void *wu = fp8 ? q->w_up : w->w_up;
    if (!make_map(&m.a, fp8 ? static_cast<const void *>(xq) : x, D.T, D.d, 1, bt))
      return MOE_ERR_CUDA;
    if (!make_map(&m.b0, wg, static_cast<uint64_t>(D.E) * D.F, D.d, n_half, bt)) return MOE_ERR_CUDA;
    if (!make_map(&m.b1, wu, static_cast<uint64_t>(D.E) * D.F, D.d, n_half, bt)) return MOE_ERR_CUDA;
    m.a_sh = m.a;
    if (fp8) {
      p.xq = xq;
      p.sx = sx;
      p.sb0 = q->s_gate;
      p.sb1 = q->s_up;
      p.sb0_sh = q->ss_gate;
      p.sb1_sh = q->ss_up;
    }
    const CUtensorMapDataType f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (!make_map(&m.out, h, n_rows, D.F, std::min(32, n_rows), f16)) return MOE_ERR_CUDA;
    if (D.Fs > 0) {
      if (!make_map(&m.b0_sh, fp8 ? q->ws_gate : w->ws_gate, D.Fs, D.d, n_half, bt))
        return MOE_ERR_CUDA;
      if (!make_map(&m.b1_sh, fp8 ? q->ws_up : w->ws_up, D.Fs, D.d, n_half, bt))
        return MOE_ERR_CUDA;
      if (!make_map(&m.out_sh, h_sh, D.T, D.Fs, std::min(32, D.T), f16)) return MOE_ERR_CUDA;
    } else {
      m.b0_sh = m.b0;
      m.b1_sh = m.b1;
      m.out_sh = m.out;
    }
    ev.mark();
    const cudaError_t e = pair1 ? launch_gemm_pair(MODE_GEMM1, p, m, pair_grid, s)
                               : launch_gemm(fp8 ? MODE_GEMM1_F8 : MODE_GEMM1, p, m, sms, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    launches += 1;
  }
  // FP8 experts: e4m3 rows of h (the routed rows up to offsets[E]) and h_shared
  uint8_t *hq = reinterpret_cast<uint8_t *>(wsp(ws, L.hq));
  float *shq = reinterpret_cast<float *>(wsp(ws, L.sh));
  uint8_t *hshq = reinterpret_cast<uint8_t *>(wsp(ws, L.hshq));
  float *shs = reinterpret_cast<float *>(wsp(ws, L.shs));
  if (fp8) {
    // h rows: power-of-two scales (see launch_quant_rows_e4m3)
    if (launch_quant_rows_e4m3(h, true, true, n_rows, routing->offsets + D.E, D.F, hq, shq, s) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    launches += 1;
    if (D.Fs > 0) {
      if (launch_quant_rows_e4m3(h_sh, true, true, D.T, nullptr, D.Fs, hshq, shs, s) != cudaSuccess)
        return MOE_ERR_CUDA;
      launches += 1;
    }
  }
  // 4. GEMM2: h . W_down^T -> x (routed_scaling_factor * w) -> expert-order rows
  {
    GemmParams p = base;
    p.tiles = pair2 ? tiles_pair : tiles;
    p.n_tiles_dev = pair2 ? n_tiles_pair : n_tiles;
    p.n_tile = n2;
    p.n_ntiles = D.d / n2;
#ifdef MOE_TRACE
    p.trace = g_trace_gemm2;
#endif
    const uint32_t a_rows = static_cast<uint32_t>(std::min(n_rows, kBlockM));
    const uint32_t a_sh_rows = static_cast<uint32_t>(std::min(D.T, kBlockM));
    p.a_bytes = a_rows * kBlockK * 2;
    p.a_sh_bytes = a_sh_rows * kBlockK * 2;
    GemmMaps m;
    std::memset(&m, 0, sizeof(m));
    const CUtensorMapDataType f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const CUtensorMapDataType at = fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : f16;
    if (!make_map(&m.a, fp8 ? static_cast<const void *>(hq) : h, n_rows, D.F, a_rows, at))
      return MOE_ERR_CUDA;
    const uint32_t b_rows = pair2 ? n2 / 2 : n2;  // a pair splits B along N
    if (!make_map(&m.b0, fp8 ? q->w_down : wd16, static_cast<uint64_t>(D.E) * D.d, D.F, b_rows, at))
      return MOE_ERR_CUDA;
    m.b1 = m.b0;
    if (fp8) {
      p.sa = shq;
      p.sa_sh = shs;
      p.sb0 = q->s_down;
      p.sb0_sh = q->ss_down;
    }
    // (the reduce combine stores no rows through tensor maps: out / out_sh stay unused)
    if (reduce) m.out = m.a;
    else if (!make_map(&m.out, o_out, n_rows, D.d, std::min(32, n_rows), f16)) return MOE_ERR_CUDA;
    m.out_sh = m.out;
    if (D.Fs > 0) {
      if (!make_map(&m.a_sh, fp8 ? static_cast<const void *>(hshq) : h_sh, D.T, D.Fs, a_sh_rows, at))
        return MOE_ERR_CUDA;
      if (!make_map(&m.b0_sh, fp8 ? q->ws_down : wsd16, D.d, D.Fs, b_rows, at)) return MOE_ERR_CUDA;
      if (!reduce && !make_map(&m.out_sh, s_out, D.T, D.d, std::min(32, D.T), f16))
        return MOE_ERR_CUDA;
    } else {
      m.a_sh = m.a;
      m.b0_sh = m.b0;
    }
    m.b1_sh = m.b0_sh;
    ev.mark();
    const int mode2 = reduce ? MODE_GEMM2_RED : MODE_GEMM2;
    const cudaError_t e = pair2 ? launch_gemm_pair(mode2, p, m, pair_grid, s)
                               : launch_gemm(fp8 ? MODE_GEMM2_F8 : mode2, p, m, sms, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    launches += 1;
  }
  // 5. combine: y = bf16(sum of the scaled routed rows + shared row); with the reduce
  // combine the down GEMM already summed them in fp32, and y is that sum rounded
  ev.mark();
  const cudaError_t ec =
      reduce ? launch_finalize(yacc, static_cast<size_t>(D.T) * D.d, static_cast<uint16_t *>(y), s)
             : launch_combine(o_out, s_out, inv, D.T, D.k, D.d, static_cast<uint16_t *>(y), s);
  if (ec != cudaSuccess) return MOE_ERR_CUDA;
  launches += 1;
  ev.mark();
  g_last_launches = launches;
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_prepare_down_f16(const moe_dims_t *dims, const void *w_down, const void *ws_down,
                                void *w_down_f16, void *ws_down_f16, void *ws, size_t ws_bytes,
                                void *stream) {
  Dims D;
  moe_status st = check_dims(dims, &D);
  if (st != MOE_OK) return st;
  if (!w_down || !w_down_f16 || !aligned16(w_down) || !aligned16(w_down_f16))
    return MOE_ERR_INVALID_ARG;
  if (D.Fs > 0 && (!ws_down || !ws_down_f16 || !aligned16(ws_down) || !aligned16(ws_down_f16)))
    return MOE_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(ws) & 255))
    return MOE_ERR_INVALID_ARG;
  int sms = 0;
  if (device_setup(&sms) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = clear_header(ws, s)) != MOE_OK) return st;
  int *status = static_cast<int *>(ws);
  int launches = 0;
  if (launch_bf16_to_f16(static_cast<const uint16_t *>(w_down), static_cast<size_t>(D.E) * D.d * D.F,
                         static_cast<uint16_t *>(w_down_f16), status, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  ++launches;
  if (D.Fs > 0) {
    if (launch_bf16_to_f16(static_cast<const uint16_t *>(ws_down), static_cast<size_t>(D.d) * D.Fs,
                           static_cast<uint16_t *>(ws_down_f16), status, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    ++launches;
  }
  g_last_launches = launches;
  return MOE_OK;
}

size_t moe_logits_offset(const moe_dims_t *dims) {
  Dims D;
  if (check_dims(dims, &D) != MOE_OK) return 0;
  return ws_layout(D).logits;
}

moe_status moe_read_device_status(const void *ws, void *stream, int32_t *site) {
  if (ws == nullptr) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int hdr[2] = {0, 0};
  if (cudaMemcpyAsync(hdr, ws, sizeof(hdr), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (site) *site = hdr[1];
  return static_cast<moe_status>(hdr[0]);
}

moe_status moe_selftest_bounded_wait(void *ws, size_t ws_bytes, uint32_t limit_us, void *stream) {
  if (ws == nullptr || ws_bytes < sizeof(WsHeader) || (reinterpret_cast<uintptr_t>(ws) & 255))
    return MOE_ERR_INVALID_ARG;
  int dev = 0, khz = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  moe_status st = clear_header(ws, s);
  if (st != MOE_OK) return st;
  const long long cycles = static_cast<long long>(limit_us) * (khz / 1000);
  if (launch_selftest_wait(static_cast<int *>(ws), cycles, s) != cudaSuccess) return MOE_ERR_CUDA;
  g_last_launches = 1;
  return MOE_OK;
}

const char *moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
    case MOE_ERR_DEVICE_BOUNDS: return "MOE_ERR_DEVICE_BOUNDS";
  }
  return "MOE_ERR_UNKNOWN";
}

int32_t moe_last_launch_count(void) { return g_last_launches; }

#ifdef MOE_TRACE
// Trace builds only: device buffers receiving the pipeline timestamps of the
// next forward calls' GEMMs (layout in kernels.h).
void moe_debug_set_trace(void *gemm1, void *gemm2) {
  g_trace_gemm1 = static_cast<unsigned long long *>(gemm1);
  g_trace_gemm2 = static_cast<unsigned long long *>(gemm2);
}
#endif

moe_status moe_profile_next_forward(void **events, int32_t n_events) {
  if (events != nullptr && n_events < 1) return MOE_ERR_INVALID_ARG;
  g_prof_events = events;
  g_prof_n = events ? n_events : 0;
  return MOE_OK;
}

}  // extern "C"

// C ABI of libbsa: argument validation, workspace sizing and dispatch to the kernels.
// No entry point allocates, synchronises or copies between host and device. Each entry
// point that enqueues work is an NVTX range named after it (a no-op unless a profiler is
// attached), so that profiles and ncu's NVTX filters can tell the calls apart.
#include <atomic>
#include <math.h>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "window.cuh"

namespace bsa {

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

namespace {

bool valid_geom(const bsa_geom* g) {
  if (!g) return false;
  if (g->B < 1 || g->H < 1 || g->T < 1 || g->Hs < 1 || g->Ws < 1) return false;
  if (g->d != 64 && g->d != 128) return false;
  if (g->Hs > 4096 || g->Ws > 4096 || g->T > 4096) return false;   // 10-bit tile coordinates
  // A grid of more than 64 * kMaxTiles tokens has more than kMaxTiles tiles; rejecting it
  // here keeps the token count in make_geom within int range.
  if ((long long)g->T * g->Hs * g->Ws > 64LL * kMaxTiles) return false;
  // The mask builder puts B, H and B*H on grid axes limited to 65535 blocks.
  if ((long long)g->B * g->H > 65535) return false;
  const Geom G = make_geom(*g);
  if (G.NT > kMaxTiles) return false;
  const long long rows = (long long)g->B * g->H * G.NT * 64;
  if (rows >= (1LL << 31)) return false;
  const long long tokens = (long long)g->B * G.N * g->H;
  if (tokens >= (1LL << 31)) return false;
  return true;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// NVTX range for the lifetime of one entry point call.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

// Window kinds 0 and 1 take a radius in tiles, kind 2 a radius in tokens (window.cuh).
bool valid_window(int kind, int radius) {
  if (kind != 0 && kind != 1 && kind != 2) return false;
  if (radius < 0) return false;
  return kind != 2 || radius <= kMaxTokenRadius;
}

bool valid_params(const bsa_geom* g, const bsa_mask_params* p) {
  if (!p) return false;
  if (!(p->dense_fraction >= 0.0f && p->dense_fraction <= 1.0f)) return false;
  if (p->budget_mode == 0) {
    if (!valid_window(p->window_kind, p->radius)) return false;
    if (p->topk < 0) return false;
  } else if (p->budget_mode == 1) {
    if (p->window_kind != 1) return false;
    if (!(p->budget_target > 0.0f && p->budget_target <= 1.0f)) return false;
  } else if (p->budget_mode == 2) {
    if (!valid_window(p->window_kind, p->radius)) return false;
    if (!(p->budget_target > 0.0f && p->budget_target <= 1.0f)) return false;
  } else {
    return false;
  }
  (void)g;
  return true;
}

int device_ok() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (major != 10 || minor != 0) return BSA_ERR_UNSUPPORTED_DEVICE;
  return BSA_OK;
}

int status_of(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

}  // namespace
}  // namespace bsa

using namespace bsa;

namespace bsa {
cudaError_t launch_wait_selftest(long long limit_cycles, uint32_t* err, cudaStream_t s);   // selftest.cu
}

extern "C" {

const char* bsa_status_string(int status) {
  switch (status) {
    case BSA_OK: return "BSA_OK";
    case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
    case BSA_ERR_WORKSPACE: return "BSA_ERR_WORKSPACE";
    case BSA_ERR_UNSUPPORTED_DEVICE: return "BSA_ERR_UNSUPPORTED_DEVICE";
    case BSA_ERR_CUDA: return "BSA_ERR_CUDA";
    default: return "BSA_ERR_UNKNOWN";
  }
}

int bsa_tile_grid(const bsa_geom* g, int* nT, int* nY, int* nX, int* NT) {
  if (!valid_geom(g)) return BSA_ERR_INVALID_ARG;
  const Geom G = make_geom(*g);
  if (nT) *nT = G.nT;
  if (nY) *nY = G.nY;
  if (nX) *nX = G.nX;
  if (NT) *NT = G.NT;
  return BSA_OK;
}

size_t bsa_workspace_bytes(const bsa_geom* g, const bsa_mask_params* p) {
  (void)p;
  if (!valid_geom(g)) return 0;
  return ws_layout(make_geom(*g)).total;
}

int bsa_clear_error(void* ws, void* stream) {
  const CallRange range("bsa_clear_error");
  if (!ws) return BSA_ERR_INVALID_ARG;
  const int dev = device_ok();
  if (dev != BSA_OK) return dev;
  return status_of(cudaMemsetAsync(ws, 0, 4, static_cast<cudaStream_t>(stream)));
}

int bsa_reorder(const bsa_geom* g, const void* x, void* xt, void* stream) {
  const CallRange range("bsa_reorder");
  if (!valid_geom(g) || !aligned16(x) || !aligned16(xt)) return BSA_ERR_INVALID_ARG;
  const int dev = device_ok();
  if (dev != BSA_OK) return dev;
  return status_of(launch_reorder(make_geom(*g), static_cast<const __nv_bfloat16*>(x),
                                  static_cast<__nv_bfloat16*>(xt), static_cast<cudaStream_t>(stream)));
}

int bsa_reorder_pool(const bsa_geom* g, const void* x, void* xt, float* xbar, void* stream) {
  const CallRange range("bsa_reorder_pool");
  if (!valid_geom(g) || !aligned16(x) || !aligned16(xt) || !aligned16(xbar)) return BSA_ERR_INVALID_ARG;
  const int dev = device_ok();
  if (dev != BSA_OK) return dev;
  return status_of(launch_reorder_pool(make_geom(*g), static_cast<const __nv_bfloat16*>(x),
                                       static_cast<__nv_bfloat16*>(xt), xbar, static_cast<cudaStream_t>(stream)));
}

int bsa_unreorder(const bsa_geom* g, const void* xt, void* x, void* stream) {
  const CallRange range("bsa_unreorder");
  if (!valid_geom(g) || !aligned16(x) || !aligned16(xt)) return BSA_ERR_INVALID_ARG;
  const int dev = device_ok();
  if (dev != BSA_OK) return dev;
  return status_of(launch_unreorder(make_geom(*g), static_cast<const __nv_bfloat16*>(xt),
                                    static_cast<__nv_bfloat16*>(x), static_cast<cudaStream_t>(stream)));
}

int bsa_build_mask(const bsa_geom* g, const bsa_mask_params* p, const void* qt, const void* kt,
                   const float* difficulty, uint32_t* mask, int32_t* kv_count, void* ws, size_t ws_bytes,
                   void* stream) {
  const CallRange range("bsa_build_mask");
  if (!valid_geom(g) || !valid_params(g, p)) return BSA_ERR_INVALID_ARG;
  if (!aligned16(qt) || !aligned16(kt) || !aligned16(difficulty) || !aligned16(mask) || !aligned16(kv_count))
    return BSA_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return BSA_ERR_WORKSPACE;
  if (ws_bytes < bsa_workspace_bytes(g, p)) return BSA_ERR_WORKSPACE;
  const int dev = device_ok();
  if (dev != BSA_OK) return dev;
  return status_of(launch_build_mask(make_geom(*g), *p, static_cast<const __nv_bfloat16*>(qt),
                                     static_cast<const __nv_bfloat16*>(kt), difficulty, mask, kv_count,
                                     static_cast<uint8_t*>(ws), static_cast<cudaStream_t>(stream)));
}

int bsa_build_mask_pooled(const bsa_geom* g, const bsa_mask_params* p, const float* qbar, const float* kbar,
                          const float* difficulty, uint32_t* mask, int32_t* kv_count, void* ws, size_t ws_bytes,
                          void* stream) {
  const CallRange range("bsa_build_mask_pooled");
  if (!valid_geom(g) || !valid_params(g, p)) return BSA_ERR_INVALID_ARG;
  if (!aligned16(qbar) || !aligned16(kbar) || !aligned16(difficulty) || !aligned16(mask) || !aligned16(kv_count))
    return BSA_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return BSA_ERR_WORKSPACE;
  if (ws_bytes < bsa_workspace_bytes(g, p)) return BSA_ERR_WORKSPACE;
  const int dev = device_ok();
  if (dev != BSA_OK) return dev;
  return status_of(launch_build_mask_pooled(make_geom(*g), *p, qbar, kbar, difficulty, mask, kv_count,
                                            static_cast<uint8_t*>(ws), static_cast<cudaStream_t>(stream)));
}

// The checks shared by both workspace attention entry points; BSA_OK when the call may run.
static int check_attn_args(const bsa_geom* g, const void* qt, const void* kt, const void* vt,
                           const uint32_t* mask, const int32_t* kv_count, float softmax_scale, const void* out,
                           const float* lse, const void* ws, size_t ws_bytes) {
  if (!valid_geom(g)) return BSA_ERR_INVALID_ARG;
  if (!aligned16(qt) || !aligned16(kt) || !aligned16(vt) || !aligned16(mask) || !aligned16(kv_count) ||
      !aligned16(out))
    return BSA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return BSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.0f) || isinf(softmax_scale)) return BSA_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return BSA_ERR_WORKSPACE;
  if (ws_bytes < bsa_workspace_bytes(g, nullptr)) return BSA_ERR_WORKSPACE;
  return device_ok();
}

int bsa_sparse_attn_fwd(const bsa_geom* g, const void* qt, const void* kt, const void* vt, const uint32_t* mask,
                        const int32_t* kv_count, float softmax_scale, void* out, float* lse, void* ws,
                        size_t ws_bytes, void* stream) {
  const CallRange range("bsa_sparse_attn_fwd");
  const int st = check_attn_args(g, qt, kt, vt, mask, kv_count, softmax_scale, out, lse, ws, ws_bytes);
  if (st != BSA_OK) return st;
  return status_of(launch_sparse_attn(make_geom(*g), static_cast<const __nv_bfloat16*>(qt),
                                      static_cast<const __nv_bfloat16*>(kt), static_cast<const __nv_bfloat16*>(vt),
                                      mask, kv_count, softmax_scale, static_cast<__nv_bfloat16*>(out), lse,
                                      static_cast<uint8_t*>(ws), static_cast<cudaStream_t>(stream)));
}

int bsa_sparse_attn_fwd_token(const bsa_geom* g, const void* qt, const void* kt, const void* vt,
                              const uint32_t* mask, const int32_t* kv_count, const uint8_t* dense,
                              int token_radius, float softmax_scale, void* out, float* lse, void* ws,
                              size_t ws_bytes, void* stream) {
  const CallRange range("bsa_sparse_attn_fwd_token");
  if (!dense || token_radius < 0 || token_radius > kMaxTokenRadius) return BSA_ERR_INVALID_ARG;
  const int st = check_attn_args(g, qt, kt, vt, mask, kv_count, softmax_scale, out, lse, ws, ws_bytes);
  if (st != BSA_OK) return st;
  return status_of(launch_sparse_attn(make_geom(*g), static_cast<const __nv_bfloat16*>(qt),
                                      static_cast<const __nv_bfloat16*>(kt), static_cast<const __nv_bfloat16*>(vt),
                                      mask, kv_count, softmax_scale, static_cast<__nv_bfloat16*>(out), lse,
                                      static_cast<uint8_t*>(ws), static_cast<cudaStream_t>(stream), dense,
                                      token_radius));
}

size_t bsa_route_flags_offset(const bsa_geom* g) {
  if (!valid_geom(g)) return 0;
  return ws_layout(make_geom(*g)).dense;
}

int bsa_sparse_attn_fwd_fixed_scratch(const bsa_geom* g, const void* qt, const void* kt, const void* vt,
                                      const uint32_t* mask, const int32_t* kv_count, float softmax_scale,
                                      void* out, float* lse, uint32_t* kernel_errors, void* stream) {
  const CallRange range("bsa_sparse_attn_fwd_fixed_scratch");
  if (!valid_geom(g)) return BSA_ERR_INVALID_ARG;
  if (!aligned16(qt) || !aligned16(kt) || !aligned16(vt) || !aligned16(mask) || !aligned16(kv_count) ||
      !aligned16(out))
    return BSA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return BSA_ERR_INVALID_ARG;
  if (kernel_errors && (reinterpret_cast<uintptr_t>(kernel_errors) & 3u) != 0) return BSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.0f) || isinf(softmax_scale)) return BSA_ERR_INVALID_ARG;
  const Geom G = make_geom(*g);
  if (fixed_scratch_need(G) > fixed_scratch_capacity()) return BSA_ERR_WORKSPACE;
  const int dev = device_ok();
  if (dev != BSA_OK) return dev;
  return status_of(launch_sparse_attn_fixed_scratch(G, static_cast<const __nv_bfloat16*>(qt),
                                                    static_cast<const __nv_bfloat16*>(kt),
                                                    static_cast<const __nv_bfloat16*>(vt), mask, kv_count,
                                                    softmax_scale, static_cast<__nv_bfloat16*>(out), lse,
                                                    kernel_errors, static_cast<cudaStream_t>(stream)));
}

uint64_t bsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int bsa_selftest_bounded_wait(long long limit_cycles, uint32_t* err, void* stream) {
  const CallRange range("bsa_selftest_bounded_wait");
  if (!err || (reinterpret_cast<uintptr_t>(err) & 3u) != 0) return BSA_ERR_INVALID_ARG;
  if (limit_cycles <= 0 || limit_cycles > 4000000000LL) return BSA_ERR_INVALID_ARG;
  const int dev = device_ok();
  if (dev != BSA_OK) return dev;
  return status_of(bsa::launch_wait_selftest(limit_cycles, err, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

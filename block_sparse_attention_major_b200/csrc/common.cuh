// Shared definitions of the libbsa kernels: geometry, workspace layout, error bits and
// the internal launch functions behind the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bsa.h"

namespace bsa {

constexpr int kTileEdge = 4;
constexpr int kTileTokens = 64;
constexpr int kMaxTiles = 4096;          // NT limit (work lists and smem tables)

// Geometry with the derived tile counts, passed by value to kernels.
struct Geom {
  int B, H, d, T, Hs, Ws;
  int nT, nY, nX, NT, N;
  int NW;                                 // 32-bit words per mask row
};

inline __host__ __device__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

inline Geom make_geom(const bsa_geom& g) {
  Geom o;
  o.B = g.B; o.H = g.H; o.d = g.d; o.T = g.T; o.Hs = g.Hs; o.Ws = g.Ws;
  o.nT = ceil_div(g.T, kTileEdge); o.nY = ceil_div(g.Hs, kTileEdge); o.nX = ceil_div(g.Ws, kTileEdge);
  o.NT = o.nT * o.nY * o.nX;
  o.N = g.T * g.Hs * g.Ws;
  o.NW = ceil_div(o.NT, 32);
  return o;
}

// Unsigned division by a runtime constant (Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994): l = ceil(log2 d),
// m = floor(2^32 (2^l - d) / d) + 1, q = (mulhi(n, m) + n) >> l. Valid for n < 2^31
// (the sum then fits in 32 bits) and 1 <= d < 2^31.
struct FastDiv {
  uint32_t div, mul, shr;
  FastDiv() : div(1), mul(0), shr(0) {}
  explicit FastDiv(uint32_t d) : div(d) {
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    shr = l;
    uint64_t m = ((1ull << 32) * ((1ull << l) - d)) / d + 1;
    mul = (uint32_t)m;
  }
  __device__ __forceinline__ uint32_t q(uint32_t n) const {
    uint32_t t = __umulhi(n, mul);
    return (t + n) >> shr;
  }
};

// ------------------------------------------------------------------ workspace layout
// [0, 256)        header: error word (u32 @0), attention unit count (i32 @4)
// then 256-aligned regions: qbar, kbar (fp32 [B,H,NT,d]), dense flags (u8 [B,NT]),
// row entropy (fp32 [B,H,NT]), per-(b,h) unit counts/offsets (int4 [B*H]),
// attention units (8 ints each, [B*H*(NT/4+2)]), pooled scores (fp32 [B,H,NT,NTP],
// NTP = NT rounded up to a multiple of 4).
// Upper bound on attention work units (four query tiles each): per (b, h),
// ceil(nd/4) + ceil(nl/4) <= NT/4 + 2.
inline __host__ __device__ int units_per_bh(int NT) { return NT / 4 + 2; }

struct WsLayout {
  size_t qbar, kbar, dense, entropy, plan, bhcnt, units, scores, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(const Geom& g) {
  WsLayout L;
  size_t off = 256;
  const size_t pooled = (size_t)g.B * g.H * g.NT * g.d * sizeof(float);
  L.qbar = off; off = align256(off + pooled);
  L.kbar = off; off = align256(off + pooled);
  L.dense = off; off = align256(off + (size_t)g.B * g.NT);
  L.entropy = off; off = align256(off + (size_t)g.B * g.H * g.NT * sizeof(float));
  L.plan = off; off = align256(off + (size_t)g.B * g.H * g.NT * 2 * sizeof(int));
  L.bhcnt = off; off = align256(off + (size_t)g.B * g.H * 4 * sizeof(int));
  L.units = off; off = align256(off + (size_t)g.B * g.H * units_per_bh(g.NT) * 8 * sizeof(int));
  L.scores = off; off = align256(off + (size_t)g.B * g.H * g.NT * (size_t)((g.NT + 3) & ~3) * sizeof(float));
  L.total = off;
  return L;
}

// --------------------------------------------------------------------- tile geometry
// Tile coordinates of tile j.
__device__ __forceinline__ void tile_xyz(const Geom& g, int j, int& tt, int& ty, int& tx) {
  const int nyx = g.nY * g.nX;
  tt = j / nyx;
  const int rem = j - tt * nyx;
  ty = rem / g.nX;
  tx = rem - ty * g.nX;
}

// 64-bit mask of the valid slots of tile (tt, ty, tx): bit r = (dt*4+dy)*4+dx.
__device__ __forceinline__ uint64_t tile_valid_mask(const Geom& g, int tt, int ty, int tx) {
  const int vt = min(kTileEdge, g.T - tt * kTileEdge);
  const int vy = min(kTileEdge, g.Hs - ty * kTileEdge);
  const int vx = min(kTileEdge, g.Ws - tx * kTileEdge);
  const uint64_t row = (1ull << vx) - 1ull;                 // one (dt, dy) row of 4 slots
  uint64_t plane = 0;
  for (int dy = 0; dy < vy; ++dy) plane |= row << (4 * dy);
  uint64_t m = 0;
  for (int dt = 0; dt < vt; ++dt) m |= plane << (16 * dt);
  return m;
}

__device__ __forceinline__ int tile_valid_count(const Geom& g, int tt, int ty, int tx) {
  return min(kTileEdge, g.T - tt * kTileEdge) * min(kTileEdge, g.Hs - ty * kTileEdge) *
         min(kTileEdge, g.Ws - tx * kTileEdge);
}

// ------------------------------------------------------------------ error reporting
__device__ __forceinline__ void report_error(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

}  // namespace bsa

// ------------------------------------------------------------------ host-side launch API
// Internal entry points implemented in the .cu files, called by the C ABI in abi.cu.
namespace bsa {
cudaError_t launch_reorder(const Geom& g, const __nv_bfloat16* x, __nv_bfloat16* xt, cudaStream_t s);
cudaError_t launch_unreorder(const Geom& g, const __nv_bfloat16* xt, __nv_bfloat16* x, cudaStream_t s);
cudaError_t launch_reorder_pool(const Geom& g, const __nv_bfloat16* x, __nv_bfloat16* xt, float* xbar,
                                cudaStream_t s);
cudaError_t launch_build_mask_pooled(const Geom& g, const bsa_mask_params& p, const float* qbar,
                                     const float* kbar, const float* difficulty, uint32_t* mask,
                                     int32_t* kv_count, uint8_t* ws, cudaStream_t s);
cudaError_t launch_build_mask(const Geom& g, const bsa_mask_params& p, const __nv_bfloat16* qt,
                              const __nv_bfloat16* kt, const float* difficulty, uint32_t* mask,
                              int32_t* kv_count, uint8_t* ws, cudaStream_t s);
cudaError_t launch_sparse_attn(const Geom& g, const __nv_bfloat16* qt, const __nv_bfloat16* kt,
                               const __nv_bfloat16* vt, const uint32_t* mask, const int32_t* kv_count,
                               float scale, __nv_bfloat16* out, float* lse, uint8_t* ws, cudaStream_t s,
                               const uint8_t* dense = nullptr, int token_rho = -1);
// Attention with its scratch in the library's fixed device array (no workspace argument).
size_t fixed_scratch_capacity();
size_t fixed_scratch_need(const Geom& g);
cudaError_t launch_sparse_attn_fixed_scratch(const Geom& g, const __nv_bfloat16* qt, const __nv_bfloat16* kt,
                                             const __nv_bfloat16* vt, const uint32_t* mask,
                                             const int32_t* kv_count, float scale, __nv_bfloat16* out,
                                             float* lse, uint32_t* errors, cudaStream_t s);
void count_launches(int n);
}  // namespace bsa

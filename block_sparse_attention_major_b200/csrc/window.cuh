// Local-support (window) predicate of the mask builder, on packed tile coordinates.
//
// Plain integer code, compiled for the device by the select kernel and for the host by
// whoever wants to enumerate a window (the tests do, against an independent enumeration).
//
//  kind 0  cube: max(|dt|, |dy|, |dx|) <= r, in tiles (sliding-tile local branch, VORTA
//          summary)
//  kind 1  temporal decay: |dt| <= r and max(|dy|, |dx|) <= r - |dt|, in tiles (Token
//          Radius Attention summary, "Radius construction": a base radius applied across
//          frames with temporal distance decay)
//  kind 2  token-level circular support, radius r in TOKENS (the same summary: query-centred
//          circular neighbourhoods). Key token m supports query token n when
//          |t_m - t_n| <= r and (y_m - y_n)^2 + (x_m - x_n)^2 <= (r - |t_m - t_n|)^2. Tile j
//          is a window tile of tile i when some valid token of j supports some valid token
//          of i. The valid tokens of a tile form a box, and the condition only gets easier
//          as any axis distance shrinks, so it holds for some pair exactly when it holds at
//          the smallest distance along each axis. Two tiles 0 < D tiles apart along an axis
//          are 4 D - 3 tokens apart at the closest: only the last tile of an axis can be
//          partial, and it is never the lower of two distinct tiles, so the lower tile
//          always spans its full 4 tokens. The same tile is 0 apart.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define BSA_HD __host__ __device__ __forceinline__
#else
#define BSA_HD inline
#endif

namespace bsa {

// Largest window radius accepted for kind 2: (r - gap)^2 stays within int range.
constexpr int kMaxTokenRadius = 32767;

// Tile coordinates packed 10 bits each (every axis has at most 1024 tiles).
BSA_HD uint32_t pack_coord(int tt, int ty, int tx) {
  return ((uint32_t)tt << 20) | ((uint32_t)ty << 10) | (uint32_t)tx;
}

BSA_HD int iabs_(int v) { return v < 0 ? -v : v; }
BSA_HD int imax_(int a, int b) { return a > b ? a : b; }

// Smallest token distance along one axis between two tiles D tiles apart.
BSA_HD int token_gap(int D) { return D == 0 ? 0 : 4 * D - 3; }

// Kinds 0 and 1 (tile radius).
BSA_HD bool in_tile_window(uint32_t ci, uint32_t cj, int kind, int r) {
  const int dt = iabs_((int)(ci >> 20) - (int)(cj >> 20));
  const int dy = iabs_((int)((ci >> 10) & 1023u) - (int)((cj >> 10) & 1023u));
  const int dx = iabs_((int)(ci & 1023u) - (int)(cj & 1023u));
  if (kind == 0) return imax_(dt, imax_(dy, dx)) <= r;
  return dt <= r && imax_(dy, dx) <= r - dt;
}

// Kind 2 (token radius).
BSA_HD bool in_token_window(uint32_t ci, uint32_t cj, int r) {
  const int gt = token_gap(iabs_((int)(ci >> 20) - (int)(cj >> 20)));
  const int gy = token_gap(iabs_((int)((ci >> 10) & 1023u) - (int)((cj >> 10) & 1023u)));
  const int gx = token_gap(iabs_((int)(ci & 1023u) - (int)(cj & 1023u)));
  return gt <= r && gy * gy + gx * gx <= (r - gt) * (r - gt);
}

BSA_HD bool in_window(uint32_t ci, uint32_t cj, int kind, int r) {
  return kind == 2 ? in_token_window(ci, cj, r) : in_tile_window(ci, cj, kind, r);
}

// ---- the token-level support inside window tiles (the attention side of kind 2)

// Slots of key tile (tt, ty, tx), bit (a * 4 + b) * 4 + c for the token
// (4 tt + a, 4 ty + b, 4 tx + c), whose token lies in the support of query token
// (qt, qy, qx). Slots beyond the grid are not excluded here.
BSA_HD uint64_t token_support_slots(int qt, int qy, int qx, int tt, int ty, int tx, int r) {
  uint64_t m = 0;
#ifdef __CUDA_ARCH__
#pragma unroll
#endif
  for (int a = 0; a < 4; ++a) {
    const int dt = iabs_(4 * tt + a - qt);
    const int rr = r - dt;
    const int R2 = dt <= r ? rr * rr : -1;
#ifdef __CUDA_ARCH__
#pragma unroll
#endif
    for (int b = 0; b < 4; ++b) {
      const int dy = 4 * ty + b - qy;
      const int lim = R2 - dy * dy;
#ifdef __CUDA_ARCH__
#pragma unroll
#endif
      for (int c = 0; c < 4; ++c) {
        const int dx = 4 * tx + c - qx;
        if (dx * dx <= lim) m |= 1ull << (16 * a + 4 * b + c);
      }
    }
  }
  return m;
}

// Largest token distance along an axis of n tokens between tiles a and b.
BSA_HD int max_token_dist(int a, int b, int n) {
  const int ahi = 4 * a + 3 < n - 1 ? 4 * a + 3 : n - 1;
  const int bhi = 4 * b + 3 < n - 1 ? 4 * b + 3 : n - 1;
  return imax_(ahi - 4 * b, bhi - 4 * a);
}

// Whether every valid token of key tile cj lies in the support of every valid token of
// query tile ci (grid T x Hs x Ws): the condition at the largest distance along each axis,
// since the valid tokens of a tile form a box and the condition only gets harder as any
// distance grows. Such a tile needs no per-token mask.
BSA_HD bool token_tiles_all_inside(uint32_t ci, uint32_t cj, int T, int Hs, int Ws, int r) {
  const int mt = max_token_dist((int)(ci >> 20), (int)(cj >> 20), T);
  const int my = max_token_dist((int)((ci >> 10) & 1023u), (int)((cj >> 10) & 1023u), Hs);
  const int mx = max_token_dist((int)(ci & 1023u), (int)(cj & 1023u), Ws);
  return mt <= r && my * my + mx * mx <= (r - mt) * (r - mt);
}

}  // namespace bsa

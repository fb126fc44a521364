// Block-mask construction.
//
//  pool      mean of the valid tokens of every tile, for Q and K (VORTA summary, "average
//            pooling" of tiles) -> qbar, kbar fp32 [B, H, NT, d]
//  route     HetA-DiT routing (Abstract): the floor(rho*NQT + 1/2) query tiles of highest
//            difficulty of each batch item take dense attention, ties to the lower index
//  select    per (b, h, query tile): pooled scores against every key tile, then the local
//            support - a cube window or a window whose spatial radius decays with the
//            frame-tile distance (Token Radius Attention summary, "Radius construction") -
//            plus the best tiles outside it by pooled score: a fixed top-k, or the
//            remainder of a budget derived from the entropy of the pooled-score softmax
//            (Token Radius Attention summary, "Entropy-guided budgeting").
//
// The pooled-score contraction is an fp32 SIMT GEMM of [ROWS x d] query means against
// 64-key chunks staged in shared memory (float4 operands, padded rows, no bank
// conflicts). Selection works per row and per warp on order-preserving integer keys of
// the fp32 scores: a few extra tiles by repeated warp argmax (largest key, then lowest
// tile index), many by a bitwise binary search for the threshold key followed by an
// index-ordered pass over tied keys. Both reproduce "highest score, ties to the lower
// index" exactly and use no atomics.
#include "common.cuh"

#include <math.h>

namespace bsa {
namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kKeyChunk = 64;

// ------------------------------------------------------------------------ pooling
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(Geom g, const __nv_bfloat16* __restrict__ qt,
                                                   const __nv_bfloat16* __restrict__ kt,
                                                   float* __restrict__ qbar, float* __restrict__ kbar) {
  constexpr int kLanesPerRow = D / 8;              // 16-byte chunks per token row
  constexpr int kRowsPerIter = 32 / kLanesPerRow;
  const long long per_tensor = (long long)g.B * g.H * g.NT;
  const long long wid = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (wid >= 2 * per_tensor) return;
  const int which = wid >= per_tensor;
  const long long row = wid - which * per_tensor;  // (b*H + h)*NT + j
  const int j = (int)(row % g.NT);
  int tt, ty, tx;
  tile_xyz(g, j, tt, ty, tx);
  const uint64_t valid = tile_valid_mask(g, tt, ty, tx);
  const int nvalid = tile_valid_count(g, tt, ty, tx);
  const uint4* src = reinterpret_cast<const uint4*>((which ? kt : qt) + row * 64 * D);
  const int lane = threadIdx.x & 31;
  const int c = lane % kLanesPerRow, r0 = lane / kLanesPerRow;
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.f;
#pragma unroll 8
  for (int r = r0; r < 64; r += kRowsPerIter) {
    if ((valid >> r) & 1ull) {
      const uint4 v = __ldg(&src[r * kLanesPerRow + c]);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(p[k]);
        acc[2 * k] += f.x;
        acc[2 * k + 1] += f.y;
      }
    }
  }
#pragma unroll
  for (int off = kLanesPerRow; off < 32; off <<= 1)
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], off);
  if (r0 == 0) {
    const float inv = 1.0f / (float)nvalid;
    float* dst = (which ? kbar : qbar) + row * D + c * 8;
    float4 a = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    float4 b = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
    reinterpret_cast<float4*>(dst)[0] = a;
    reinterpret_cast<float4*>(dst)[1] = b;
  }
}

// ------------------------------------------------------------------------ routing
__global__ void __launch_bounds__(256) route_kernel(Geom g, const float* __restrict__ difficulty,
                                                    int n_dense, uint8_t* __restrict__ dense) {
  extern __shared__ float sdiff[];
  const int b = blockIdx.y;
  const int NQT = g.NT;
  for (int i = threadIdx.x; i < NQT; i += blockDim.x) sdiff[i] = difficulty[(long long)b * NQT + i];
  __syncthreads();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= NQT) return;
  const float di = sdiff[i];
  int rank = 0;
  for (int j = 0; j < NQT; ++j) {
    const float dj = sdiff[j];
    rank += (dj > di) || (dj == di && j < i);
  }
  dense[(long long)b * NQT + i] = rank < n_dense ? 1 : 0;
}

// ------------------------------------------------------------------------ selection
enum SelMode { kSelectFixed = 0, kEntropy = 1, kSelectBudget = 2 };

struct SelArgs {
  Geom g;
  int window_kind, radius, topk;
  float scale;                 // 1/sqrt(d), used by the entropy only
  double tau;
  const float* qbar;
  const float* kbar;
  const uint8_t* dense;
  float* entropy;              // [B, H, NQT]
  uint32_t* mask;              // [B, H, NQT, NW]
  int32_t* kv_count;           // [B, H, NQT]
};

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);      // +0 and -0 tie
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t pack_coord(int tt, int ty, int tx) {
  return ((uint32_t)tt << 20) | ((uint32_t)ty << 10) | (uint32_t)tx;
}

__device__ __forceinline__ bool in_window(uint32_t ci, uint32_t cj, int kind, int r) {
  const int dt = abs((int)(ci >> 20) - (int)(cj >> 20));
  const int dy = abs((int)((ci >> 10) & 1023u) - (int)((cj >> 10) & 1023u));
  const int dx = abs((int)(ci & 1023u) - (int)(cj & 1023u));
  if (kind == 0) return max(dt, max(dy, dx)) <= r;
  return dt <= r && max(dy, dx) <= r - dt;
}

// Number of tiles in [c - s, c + s] clipped to [0, n).
__device__ __forceinline__ int clip_count(int c, int s, int n) {
  return s < 0 ? 0 : min(c + s, n - 1) - max(c - s, 0) + 1;
}

// Closed-form size of the decayed window of radius r at tile (tt, ty, tx).
__device__ int decayed_window_size(const Geom& g, int tt, int ty, int tx, int r) {
  int s = 0;
  for (int dt = -r; dt <= r; ++dt) {
    if (tt + dt < 0 || tt + dt >= g.nT) continue;
    const int sr = r - abs(dt);
    s += clip_count(ty, sr, g.nY) * clip_count(tx, sr, g.nX);
  }
  return s;
}

template <int D, int ROWS, int MODE>
__global__ void __launch_bounds__(kSelThreads) select_kernel(SelArgs a) {
  extern __shared__ __align__(16) float smem[];
  constexpr int DP = D + 4;                         // padded row stride (floats)
  constexpr int TPR = kSelThreads / ROWS;           // threads per query row in the GEMM
  constexpr int KPT = kKeyChunk / TPR;              // keys per thread per chunk
  const Geom& g = a.g;
  const int NKT = g.NT, NQT = g.NT;
  const int NKTP = (NKT + 3) & ~3;
  const int b = blockIdx.z, h = blockIdx.y, i0 = blockIdx.x * ROWS;
  const long long bh = (long long)b * g.H + h;

  float* qs = smem;                                               // ROWS * DP
  float* ks = qs + ROWS * DP;                                     // kKeyChunk * DP
  float* sc = ks + kKeyChunk * DP;                                // ROWS * NKTP
  uint32_t* coord = reinterpret_cast<uint32_t*>(sc + ROWS * NKTP); // NKTP
  double* dsum = reinterpret_cast<double*>(coord + NKTP);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // query means of this row block, tile coordinate table
  const float4* qbar4 = reinterpret_cast<const float4*>(a.qbar);
  for (int e = tid; e < ROWS * (D / 4); e += kSelThreads) {
    const int r = e / (D / 4), c4 = e % (D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i0 + r < NQT) v = qbar4[(bh * g.NT + i0 + r) * (D / 4) + c4];
    reinterpret_cast<float4*>(qs + r * DP)[c4] = v;
  }
  for (int j = tid; j < NKT; j += kSelThreads) {
    int tt, ty, tx;
    tile_xyz(g, j, tt, ty, tx);
    coord[j] = pack_coord(tt, ty, tx);
  }
  if (MODE == kSelectBudget && warp == 0) {
    // sum_i exp(H_i) over every query tile of this (b, h), fixed order: lane-strided
    // partial sums, then a fixed butterfly; every block computes the same value.
    double s = 0.0;
    for (int i = lane; i < NQT; i += 32) s += exp((double)a.entropy[bh * NQT + i]);
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) *dsum = s;
  }

  // pooled scores qbar . kbar (unscaled) for ROWS x NKT
  const float4* kbar4 = reinterpret_cast<const float4*>(a.kbar);
  const int grow = tid / TPR, gk = tid % TPR;
  for (int c0 = 0; c0 < NKT; c0 += kKeyChunk) {
    __syncthreads();
    for (int e = tid; e < kKeyChunk * (D / 4); e += kSelThreads) {
      const int kr = e / (D / 4), c4 = e % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + kr < NKT) v = kbar4[(bh * g.NT + c0 + kr) * (D / 4) + c4];
      reinterpret_cast<float4*>(ks + kr * DP)[c4] = v;
    }
    __syncthreads();
    float acc[KPT];
#pragma unroll
    for (int u = 0; u < KPT; ++u) acc[u] = 0.f;
    const float4* qrow = reinterpret_cast<const float4*>(qs + grow * DP);
#pragma unroll 4
    for (int c4 = 0; c4 < D / 4; ++c4) {
      const float4 q = qrow[c4];
#pragma unroll
      for (int u = 0; u < KPT; ++u) {
        const float4 k = reinterpret_cast<const float4*>(ks + (gk + u * TPR) * DP)[c4];
        acc[u] = fmaf(q.x, k.x, acc[u]);
        acc[u] = fmaf(q.y, k.y, acc[u]);
        acc[u] = fmaf(q.z, k.z, acc[u]);
        acc[u] = fmaf(q.w, k.w, acc[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < KPT; ++u) {
      const int j = c0 + gk + u * TPR;
      if (j < NKT) sc[grow * NKTP + j] = acc[u];
    }
  }
  __syncthreads();

  // one warp per query row
  for (int rr = warp; rr < ROWS; rr += kSelWarps) {
    const int i = i0 + rr;
    if (i >= NQT) break;
    const float* srow = sc + rr * NKTP;
    const long long rowid = bh * NQT + i;

    if (MODE == kEntropy) {
      // H = log Z - sum(e (s - m)) / Z with s = scale * qbar.kbar, e = exp(s - m)
      float m = -INFINITY;
      for (int j = lane; j < NKT; j += 32) m = fmaxf(m, srow[j] * a.scale);
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      float z = 0.f, t = 0.f;
      for (int j = lane; j < NKT; j += 32) {
        const float x = srow[j] * a.scale - m;
        const float e = expf(x);
        z += e;
        t = fmaf(e, x, t);
      }
      for (int off = 16; off > 0; off >>= 1) {
        z += __shfl_xor_sync(0xffffffffu, z, off);
        t += __shfl_xor_sync(0xffffffffu, t, off);
      }
      if (lane == 0) a.entropy[rowid] = logf(z) - t / z;
      continue;
    }

    uint32_t* mrow = a.mask + rowid * g.NW;
    if (a.dense[(long long)b * NQT + i]) {
      for (int w = lane; w < g.NW; w += 32) {
        const int rem = NKT - 32 * w;
        mrow[w] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
      }
      if (lane == 0) a.kv_count[rowid] = NKT;
      continue;
    }

    const uint32_t ci = coord[i];
    int kind = a.window_kind, rad = a.radius, extra;
    if (MODE == kSelectFixed) {
      int wsize = 0;
      for (int w = 0; w < g.NW; ++w) {
        const int j = 32 * w + lane;
        wsize += __popc(__ballot_sync(0xffffffffu, j < NKT && in_window(ci, coord[j], kind, rad)));
      }
      extra = min(a.topk, NKT - wsize);
    } else {
      const double x = a.tau * (double)NKT * (double)NQT * exp((double)a.entropy[rowid]) / *dsum;
      int budget = (int)floor(x + 0.5);
      budget = max(1, min(budget, NKT));
      const int tt = (int)(ci >> 20), ty = (int)((ci >> 10) & 1023u), tx = (int)(ci & 1023u);
      kind = 1;
      rad = 0;
      int wsize = 1;
      const int rmax = g.nT + g.nY + g.nX;
      while (rad < rmax && wsize < NKT) {
        const int next = decayed_window_size(g, tt, ty, tx, rad + 1);
        if (next > budget) break;
        ++rad;
        wsize = next;
      }
      extra = budget - wsize;
    }

    // Order-preserving integer keys of the candidates (tiles outside the window), written
    // over the row's scores; 0 marks a window tile or a slot beyond NKT (no real score maps
    // to 0 or 1).
    uint32_t* krow = reinterpret_cast<uint32_t*>(sc + rr * NKTP);
    int ncand = 0;
    for (int w = 0; w < g.NW; ++w) {
      const int j = 32 * w + lane;
      const bool cand = j < NKT && !in_window(ci, coord[j], kind, rad);
      if (j < NKTP) krow[j] = cand ? order_key(srow[j]) : 0u;
      ncand += __popc(__ballot_sync(0xffffffffu, cand));
    }
    __syncwarp();
    extra = max(0, min(extra, ncand));

    int count = 0;
    if (extra == ncand || extra <= 32) {
      // Few extra tiles (or all of them): repeated warp argmax, the largest key first and
      // the lowest tile index among equal keys; a chosen tile's key becomes 1.
      for (int round = 0; round < extra && extra < ncand; ++round) {
        uint64_t best = 0;
        for (int w = 0; w < g.NW; ++w) {
          const int j = 32 * w + lane;
          const uint32_t k = j < NKTP ? krow[j] : 0u;
          const uint64_t v = ((uint64_t)k << 32) | (uint32_t)(0xffffffffu - (uint32_t)j);
          best = (k > 1u && v > best) ? v : best;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
          best = o > best ? o : best;
        }
        const int jbest = (int)(0xffffffffu - (uint32_t)best);
        if (lane == 0) krow[jbest] = 1u;
        __syncwarp();
      }
      for (int w = 0; w < g.NW; ++w) {
        const int j = 32 * w + lane;
        bool sel = false;
        if (j < NKT) {
          const uint32_t k = krow[j];
          sel = k <= 1u || extra == ncand;        // window (0), chosen (1), or every candidate
        }
        const uint32_t bits = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) mrow[w] = bits;
        count += __popc(bits);
      }
    } else {
      // Many extra tiles: bitwise binary search for the extra-th largest key T, counting
      // with warp reductions (no atomics); then every key above T and, among keys equal to
      // T, the lowest tile indices.
      uint32_t thr = 0u;
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand_t = thr | (1u << bit);
        int c = 0;
        for (int w = 0; w < g.NW; ++w) {
          const int j = 32 * w + lane;
          c += (j < NKTP && krow[j] >= cand_t) ? 1 : 0;
        }
        c = __reduce_add_sync(0xffffffffu, c);
        if (c >= extra) thr = cand_t;
      }
      int gt = 0;
      for (int w = 0; w < g.NW; ++w) {
        const int j = 32 * w + lane;
        gt += (j < NKTP && krow[j] > thr) ? 1 : 0;
      }
      const int need_eq = extra - __reduce_add_sync(0xffffffffu, gt);
      int eq_before = 0;
      for (int w = 0; w < g.NW; ++w) {
        const int j = 32 * w + lane;
        bool sel = false, eq = false;
        if (j < NKT) {
          const uint32_t k = krow[j];
          sel = k == 0u || k > thr;
          eq = k == thr;
        }
        const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
        const int rank = eq_before + __popc(eqb & ((1u << lane) - 1u));
        sel = sel || (eq && rank < need_eq);
        eq_before += __popc(eqb);
        const uint32_t bits = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) mrow[w] = bits;
        count += __popc(bits);
      }
    }
    if (lane == 0) a.kv_count[rowid] = count;
  }
}

template <int D, int ROWS, int MODE>
cudaError_t run_select(const SelArgs& a, cudaStream_t s) {
  const Geom& g = a.g;
  const int NKTP = (g.NT + 3) & ~3;
  const size_t smem = sizeof(float) * ((size_t)(ROWS + kKeyChunk) * (D + 4) + (size_t)ROWS * NKTP) +
                      sizeof(uint32_t) * (size_t)NKTP + sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(select_kernel<D, ROWS, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(ceil_div(g.NT, ROWS), g.H, g.B);
  select_kernel<D, ROWS, MODE><<<grid, kSelThreads, smem, s>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

template <int D, int MODE>
cudaError_t run_select_rows(const SelArgs& a, cudaStream_t s) {
  // 16 query rows per block while the score rows fit in shared memory, else 8.
  const size_t rows16 = sizeof(float) * ((size_t)(16 + kKeyChunk) * (D + 4) + 16ull * ((a.g.NT + 3) & ~3)) +
                        sizeof(uint32_t) * (size_t)((a.g.NT + 3) & ~3) + 8;
  if (rows16 <= 200 * 1024) return run_select<D, 16, MODE>(a, s);
  return run_select<D, 8, MODE>(a, s);
}

template <int D>
cudaError_t build_mask_d(const Geom& g, const bsa_mask_params& p, const __nv_bfloat16* qt,
                         const __nv_bfloat16* kt, const float* difficulty, uint32_t* mask,
                         int32_t* kv_count, uint8_t* ws, cudaStream_t s) {
  const WsLayout L = ws_layout(g);
  float* qbar = reinterpret_cast<float*>(ws + L.qbar);
  float* kbar = reinterpret_cast<float*>(ws + L.kbar);
  uint8_t* dense = ws + L.dense;
  float* entropy = reinterpret_cast<float*>(ws + L.entropy);

  const long long warps = 2LL * g.B * g.H * g.NT;
  pool_kernel<D><<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(g, qt, kt, qbar, kbar);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const int nd = (int)floor((double)p.dense_fraction * (double)g.NT + 0.5);
  route_kernel<<<dim3(ceil_div(g.NT, 256), g.B), 256, g.NT * sizeof(float), s>>>(g, difficulty, nd, dense);
  count_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  SelArgs a;
  a.g = g;
  a.window_kind = p.window_kind;
  a.radius = p.radius;
  a.topk = p.topk;
  a.scale = 1.0f / sqrtf((float)g.d);
  a.tau = (double)p.budget_target;
  a.qbar = qbar;
  a.kbar = kbar;
  a.dense = dense;
  a.entropy = entropy;
  a.mask = mask;
  a.kv_count = kv_count;
  if (p.budget_mode == 0) return run_select_rows<D, kSelectFixed>(a, s);
  e = run_select_rows<D, kEntropy>(a, s);
  if (e != cudaSuccess) return e;
  return run_select_rows<D, kSelectBudget>(a, s);
}

}  // namespace

cudaError_t launch_build_mask(const Geom& g, const bsa_mask_params& p, const __nv_bfloat16* qt,
                              const __nv_bfloat16* kt, const float* difficulty, uint32_t* mask,
                              int32_t* kv_count, uint8_t* ws, cudaStream_t s) {
  if (g.d == 128) return build_mask_d<128>(g, p, qt, kt, difficulty, mask, kv_count, ws, s);
  return build_mask_d<64>(g, p, qt, kt, difficulty, mask, kv_count, ws, s);
}

}  // namespace bsa

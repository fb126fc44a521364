// Block-mask construction.
//
//  pool      mean of the valid tokens of every tile, for Q and K (VORTA summary, "average
//            pooling" of tiles) -> qbar, kbar fp32 [B, H, NT, d]
//  route     HetA-DiT routing (Abstract): the floor(rho*NQT + 1/2) query tiles of highest
//            difficulty of each batch item take dense attention, ties to the lower index
//  score     pooled scores qbar_i . kbar_j of every (b, h, query tile, key tile), fp32-level
//            accuracy on the tensor cores (3xTF32, score_tc.cu), into the workspace
//  entropy   (budget mode) entropy of each row's softmax of the scaled scores
//  budget    (budget mode) per row: the tile budget, the window radius it affords and the
//            number of extra tiles
//  select    per (b, h, query tile): the local support - a cube window, a window whose
//            spatial radius decays with the frame-tile distance (Token Radius Attention
//            summary, "Radius construction"), or the tiles touched by a token-level
//            circular support (window.cuh) - plus the best tiles outside it by pooled
//            score: a fixed top-k, the remainder of a budget derived from the entropy
//            (Token Radius Attention summary, "Entropy-guided budgeting"), or as many as
//            it takes for the row's pooled probability to reach a target mass (the same
//            summary: keys needed to capture a target attention mass).
//
// Selection works per row (one to four warps) on order-preserving integer keys: the fp32
// bits of the scores mapped to unsigned order, or, in cumulative-mass mode, the bits of the
// row's positive pooled probabilities. A few extra tiles are found by repeated argmax
// (largest key, then lowest tile index), many by a bitwise binary search for the threshold
// key (on counts, or on mass) followed by an index-ordered pass over tied keys. Both
// reproduce "highest score, ties to the lower index" exactly and use no atomics.
#include "common.cuh"
#include "window.cuh"

#include <math.h>

namespace bsa {

// score_tc.cu
cudaError_t launch_score_tc(const Geom& g, const float* qbar, const float* kbar, float* S, int NKTP,
                            uint32_t* err, cudaStream_t s);

namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

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
enum SelMode { kSelectFixed = 0, kSelectMass = 1, kSelectBudget = 2 };

struct SelArgs {
  Geom g;
  int window_kind, radius, topk;
  float scale;                 // 1/sqrt(d), for the entropy and the pooled probabilities
  float theta;                 // cumulative-mass mode: target pooled probability of a row
  const float* qbar;
  const float* kbar;
  const uint8_t* dense;
  float* entropy;              // [B, H, NQT]
  const int2* plan;            // budget mode: [B, H, NQT] (window radius, extra tiles)
  uint32_t* mask;              // [B, H, NQT, NW]
  int32_t* kv_count;           // [B, H, NQT]
};

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);      // +0 and -0 tie
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
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

// ---- pooled scores: S = qbar kbar^T (unscaled) per (b, h), on the tensor cores in
// score_tc.cu (3xTF32 products, fp32-level accuracy).

// ---- row entropy (budget mode): H = log Z - sum(e (s - m)) / Z with s = scale * score,
// e = exp(s - m); one warp per row.
__global__ void __launch_bounds__(256) entropy_kernel(Geom g, const float* __restrict__ S, int NKTP,
                                                      float scale, float* __restrict__ entropy) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);   // (b*H + h)*NT + i
  const int lane = threadIdx.x & 31;
  if (row >= (long long)g.B * g.H * g.NT) return;
  const float* srow = S + row * NKTP;
  float m = -INFINITY;
  for (int j = lane; j < g.NT; j += 32) m = fmaxf(m, srow[j] * scale);
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float z = 0.f, t = 0.f;
  for (int j = lane; j < g.NT; j += 32) {
    const float x = srow[j] * scale - m;
    const float e = expf(x);
    z += e;
    t = fmaf(e, x, t);
  }
  for (int off = 16; off > 0; off >>= 1) {
    z += __shfl_xor_sync(0xffffffffu, z, off);
    t += __shfl_xor_sync(0xffffffffu, t, off);
  }
  if (lane == 0) entropy[row] = logf(z) - t / z;
}

// ---- budgets (budget mode): one block per (b, h). Z = sum_i exp(H_i) over the query tiles
// of the head in a fixed order (thread-strided partial sums, then a fixed tree), so every
// row sees the same value; then, per row, budget = round(tau * NKT * NQT * exp(H_i) / Z)
// clipped to [1, NKT], the largest decayed-window radius whose window fits in it, and the
// number of tiles left for the score ranking.
constexpr int kBudgetThreads = 256;

__global__ void __launch_bounds__(kBudgetThreads) budget_kernel(Geom g, const float* __restrict__ entropy,
                                                                const uint8_t* __restrict__ dense,
                                                                double tau, int2* __restrict__ plan) {
  __shared__ double part[kBudgetThreads];
  const int NKT = g.NT, NQT = g.NT;
  const long long bh = blockIdx.x;
  const int b = (int)(bh / g.H);
  const int tid = threadIdx.x;
  double z = 0.0;
  for (int i = tid; i < NQT; i += kBudgetThreads) z += exp((double)entropy[bh * NQT + i]);
  part[tid] = z;
  __syncthreads();
  for (int n = kBudgetThreads / 2; n > 0; n >>= 1) {
    if (tid < n) part[tid] += part[tid + n];
    __syncthreads();
  }
  const double zsum = part[0];
  const int rmax = g.nT + g.nY + g.nX;
  for (int i = tid; i < NQT; i += kBudgetThreads) {
    const long long rowid = bh * NQT + i;
    if (dense[(long long)b * NQT + i]) {
      plan[rowid] = make_int2(0, 0);
      continue;
    }
    const double x = tau * (double)NKT * (double)NQT * exp((double)entropy[rowid]) / zsum;
    const int budget = (int)fmin(fmax(floor(x + 0.5), 1.0), (double)NKT);
    int tt, ty, tx;
    tile_xyz(g, i, tt, ty, tx);
    int rad = 0, wsize = 1;
    while (rad < rmax && wsize < NKT) {
      const int next = decayed_window_size(g, tt, ty, tx, rad + 1);
      if (next > budget) break;
      ++rad;
      wsize = next;
    }
    plan[rowid] = make_int2(rad, budget - wsize);
  }
}

// ---- selection: one (b, h, query tile) row per WPR warps (1, 2 or 4), 8 / WPR rows per
// block. Warp q of a row holds the keys of mask words [q KW, (q + 1) KW) in registers,
// lane l the key of tile 32 w + l of each word w. Counts, maxima and tie prefixes of a row
// are combined across its warps through a double-buffered shared exchange and a named
// barrier per row (ids 1-8), so large rows need no more than 32 words per lane.

// Row-wide combination of one 64-bit value per warp (sum or max), warp-uniform result.
template <int WPR, bool kMax>
__device__ __forceinline__ uint64_t row_combine(uint64_t v, volatile uint64_t* xb, int& par, int q, int rw) {
  if (WPR == 1) return v;
  if ((threadIdx.x & 31) == 0) xb[par * WPR + q] = v;
  asm volatile("bar.sync %0, %1;" ::"r"(1 + rw), "r"(WPR * 32) : "memory");
  uint64_t r = 0ull;
#pragma unroll
  for (int k = 0; k < WPR; ++k) {
    const uint64_t x = xb[par * WPR + k];
    r = kMax ? (x > r ? x : r) : r + x;
  }
  par ^= 1;
  return r;
}

// Row-wide float sum. The butterfly leaves each lane with its own rounding of the total, so
// lane 0's value is broadcast first: every warp of the row then branches identically.
template <int WPR>
__device__ __forceinline__ float row_sum_f(float v, volatile uint64_t* xb, int& par, int q, int rw) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  v = __shfl_sync(0xffffffffu, v, 0);
  if (WPR == 1) return v;
  if ((threadIdx.x & 31) == 0) xb[par * WPR + q] = __float_as_uint(v);
  asm volatile("bar.sync %0, %1;" ::"r"(1 + rw), "r"(WPR * 32) : "memory");
  float r = 0.0f;
#pragma unroll
  for (int k = 0; k < WPR; ++k) r += __uint_as_float((uint32_t)xb[par * WPR + k]);
  par ^= 1;
  return r;
}

__device__ __forceinline__ float order_key_inverse(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// TOK: the window is the token-level support (kind 2), a separate instantiation so that the
// tile-window kinds keep their own register allocation.
template <bool TOK>
__device__ __forceinline__ bool sel_in_window(uint32_t ci, uint32_t cj, int kind, int r) {
  return TOK ? in_token_window(ci, cj, r) : in_tile_window(ci, cj, kind, r);
}

template <int MODE, int KW, int WPR, bool TOK>
__global__ void __launch_bounds__(kSelThreads) select_kernel(SelArgs a, const float* __restrict__ S, int NKTP) {
  extern __shared__ __align__(16) uint32_t sm_u32[];
  constexpr int kRows = kSelWarps / WPR;
  const Geom& g = a.g;
  const int NKT = g.NT, NQT = g.NT;
  const int b = blockIdx.z, h = blockIdx.y;
  const long long bh = (long long)b * g.H + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rw = warp / WPR, q = warp % WPR;                 // row in block, warp in row
  uint32_t* coord = sm_u32;                                   // NKTP tile coordinates
  volatile uint64_t* xb = reinterpret_cast<volatile uint64_t*>(sm_u32 + ((NKTP + 1) & ~1)) + rw * 2 * WPR;
  int par = 0;

  for (int j = tid; j < NKT; j += kSelThreads) {
    int tt, ty, tx;
    tile_xyz(g, j, tt, ty, tx);
    coord[j] = pack_coord(tt, ty, tx);
  }
  __syncthreads();

  const int i = blockIdx.x * kRows + rw;
  if (i >= NQT) return;                                       // whole row: its warps leave together
  const long long rowid = bh * NQT + i;
  const float* srow = S + rowid * NKTP;
  uint32_t* mrow = a.mask + rowid * g.NW;
  if (a.dense[(long long)b * NQT + i]) {
    for (int w = q * 32 + lane; w < g.NW; w += 32 * WPR) {
      const int rem = NKT - 32 * w;
      mrow[w] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
    }
    if (q == 0 && lane == 0) a.kv_count[rowid] = NKT;
    return;
  }

  const uint32_t ci = coord[i];
  int kind = a.window_kind, rad = a.radius, extra;
  if (MODE == kSelectFixed) {
    extra = a.topk;
  } else if (MODE == kSelectMass) {
    extra = 0;                 // set by the mass search below
  } else {
    const int2 pl = a.plan[rowid];
    kind = 1;
    rad = pl.x;
    extra = pl.y;
  }

  // Order-preserving integer keys of the candidates (tiles outside the window), held in
  // registers: element j = 32 (q KW + w) + lane is kr[w]. 0 marks a window tile or a slot
  // beyond NKT (no real score maps to 0 or 1).
  uint32_t kr[KW];
  int ncand = 0;
  float mass_need = 0.0f;     // cumulative-mass mode: pooled mass still to collect (unnormalised)
  if (MODE == kSelectMass) {
    // Pooled probabilities e_j / Z with e_j = 2^((s_j - max) * scale * log2 e). The keys are
    // the fp32 bits of e_j: positive floats, so their order is the order of the scores.
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < KW; ++w) {
      const int j = 32 * (q * KW + w) + lane;
      if (j < NKT) mx = fmaxf(mx, srow[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    mx = order_key_inverse((uint32_t)row_combine<WPR, true>((uint64_t)order_key(mx), xb, par, q, rw));
    const float c = a.scale * 1.4426950408889634f;
    float z = 0.0f, zw = 0.0f;
#pragma unroll
    for (int w = 0; w < KW; ++w) {
      const int j = 32 * (q * KW + w) + lane;
      const bool inrow = j < NKT;
      const bool inw = inrow && sel_in_window<TOK>(ci, coord[j], kind, rad);
      const float e = inrow ? exp2f((srow[j] - mx) * c) : 0.0f;
      z += e;
      zw += inw ? e : 0.0f;
      const bool cand = inrow && !inw;
      kr[w] = cand ? max(__float_as_uint(e), 1u) : 0u;
      ncand += __popc(__ballot_sync(0xffffffffu, cand));
    }
    z = row_sum_f<WPR>(z, xb, par, q, rw);
    zw = row_sum_f<WPR>(zw, xb, par, q, rw);
    mass_need = a.theta * z - zw;
  } else {
#pragma unroll
    for (int w = 0; w < KW; ++w) {
      const int j = 32 * (q * KW + w) + lane;
      const bool cand = j < NKT && !sel_in_window<TOK>(ci, coord[j], kind, rad);
      kr[w] = cand ? order_key(srow[j]) : 0u;
      ncand += __popc(__ballot_sync(0xffffffffu, cand));
    }
  }
  ncand = (int)row_combine<WPR, false>((uint64_t)ncand, xb, par, q, rw);
  if (MODE == kSelectMass) extra = mass_need > 0.0f ? ncand : 0;   // refined by the mass search
  extra = max(0, min(extra, ncand));
  // extra and ncand are row-uniform by construction, yet a build of this kernel without the
  // broadcast from lane 0 below, run in budget mode, selected wrong rows (most rows of a
  // ragged budget case; nvcc 12.9, -O3), and converging the warp before the named
  // barriers of row_combine did not change that; with the broadcast every mode is
  // bit-exact. The cause is not identified. The budget and fixed modes now run on
  // select_radix_kernel; this kernel serves the cumulative-mass mode, which passes with or
  // without the broadcast, and keeps it.
  extra = __shfl_sync(0xffffffffu, extra, 0);
  ncand = __shfl_sync(0xffffffffu, ncand, 0);

  // Threshold key thr and how many keys equal to it to take (need_eq, lowest index first):
  // every key > thr is selected. extra == ncand selects every candidate.
  uint32_t thr;
  int need_eq;
  if (MODE == kSelectMass) {
    // Smallest set of best candidates whose mass reaches mass_need: the largest key t with
    // mass(keys >= t) >= mass_need, every key above t, then the keys equal to t (equal
    // masses) in index order until the need is met. All candidates if it cannot be met.
    float total = 0.0f;
#pragma unroll
    for (int w = 0; w < KW; ++w) total += kr[w] != 0u ? __uint_as_float(kr[w]) : 0.0f;
    total = row_sum_f<WPR>(total, xb, par, q, rw);
    if (extra == 0) {
      thr = 0xffffffffu;
      need_eq = 0;
    } else if (total < mass_need) {
      thr = 0u;
      need_eq = 0;
    } else {
      uint32_t t = 0u;
      for (int bit = 30; bit >= 0; --bit) {
        const uint32_t cand_t = t | (1u << bit);
        float m = 0.0f;
#pragma unroll
        for (int w = 0; w < KW; ++w) m += kr[w] >= cand_t ? __uint_as_float(kr[w]) : 0.0f;
        if (row_sum_f<WPR>(m, xb, par, q, rw) >= mass_need) t = cand_t;
      }
      float above = 0.0f;
      int eqc = 0;
#pragma unroll
      for (int w = 0; w < KW; ++w) {
        above += kr[w] > t ? __uint_as_float(kr[w]) : 0.0f;
        eqc += kr[w] == t ? 1 : 0;
      }
      above = row_sum_f<WPR>(above, xb, par, q, rw);
      eqc = (int)row_combine<WPR, false>((uint64_t)__reduce_add_sync(0xffffffffu, eqc), xb, par, q, rw);
      const int need = (int)ceilf((mass_need - above) / __uint_as_float(t));
      thr = t;
      need_eq = __shfl_sync(0xffffffffu, max(1, min(need, eqc)), 0);
    }
  } else if (extra == 0) {
    thr = 0xffffffffu;
    need_eq = 0;
  } else if (extra == ncand) {
    thr = 1u;
    need_eq = 0;
  } else if (extra <= 32) {
    // Few extra tiles: repeated argmax over the row, the largest key first and the lowest
    // tile index among equal keys; a chosen key becomes 0xffffffff (above any score's key)
    // and thr = 0xfffffffe then selects exactly the chosen.
    for (int round = 0; round < extra; ++round) {
      uint64_t best = 0;
#pragma unroll
      for (int w = 0; w < KW; ++w) {
        const uint32_t j = 32u * (q * KW + w) + lane;
        const uint64_t v = ((uint64_t)kr[w] << 32) | (0xffffffffu - j);
        best = (kr[w] > 1u && kr[w] != 0xffffffffu && v > best) ? v : best;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
        best = o > best ? o : best;
      }
      best = row_combine<WPR, true>(best, xb, par, q, rw);
      const uint32_t jbest = 0xffffffffu - (uint32_t)best;
#pragma unroll
      for (int w = 0; w < KW; ++w)
        if (32u * (q * KW + w) + lane == jbest) kr[w] = 0xffffffffu;      // chosen: above any score
    }
    thr = 0xfffffffeu;
    need_eq = 0;
  } else {
    // Many extra tiles: bitwise binary search for the largest thr with at least `extra`
    // keys >= thr; it stops early once exactly `extra` keys are >= the candidate, which
    // then needs no tie pass.
    uint32_t t = 0u;
    bool exact = false;
    for (int bit = 31; bit >= 0 && !exact; --bit) {
      const uint32_t cand_t = t | (1u << bit);
      int c = 0;
#pragma unroll
      for (int w = 0; w < KW; ++w) c += kr[w] >= cand_t ? 1 : 0;
      c = (int)row_combine<WPR, false>((uint64_t)__reduce_add_sync(0xffffffffu, c), xb, par, q, rw);
      if (c >= extra) t = cand_t;
      exact = c == extra;
    }
    if (exact) {
      thr = t - 1u;           // every key >= t, i.e. > t - 1
      need_eq = 0;
    } else {
      int gt = 0;
#pragma unroll
      for (int w = 0; w < KW; ++w) gt += kr[w] > t ? 1 : 0;
      gt = (int)row_combine<WPR, false>((uint64_t)__reduce_add_sync(0xffffffffu, gt), xb, par, q, rw);
      thr = t;
      need_eq = extra - gt;
    }
  }

  // Keys equal to thr in the warps before this one (index order runs warp by warp).
  int eq_before = 0;
  if (WPR > 1 && need_eq > 0) {
    int eqc = 0;
#pragma unroll
    for (int w = 0; w < KW; ++w) {
      const int j = 32 * (q * KW + w) + lane;
      eqc += (j < NKT && kr[w] != 0u && kr[w] == thr) ? 1 : 0;
    }
    eqc = __reduce_add_sync(0xffffffffu, eqc);
    // exclusive prefix over the row's warps: combine (count << 8 * q) sums, then unpack
    const uint64_t packed = row_combine<WPR, false>((uint64_t)eqc << (16 * q), xb, par, q, rw);
    for (int k = 0; k < q; ++k) eq_before += (int)((packed >> (16 * k)) & 0xffffu);
  }

  // The row: window | key > thr | (key == thr, among the first need_eq in index order).
  int count = 0;
#pragma unroll
  for (int w = 0; w < KW; ++w) {
    const int wg = q * KW + w;
    if (wg < g.NW) {
      const int j = 32 * wg + lane;
      const uint32_t k = kr[w];
      const bool inrow = j < NKT;
      bool sel = inrow && (k == 0u || k > thr);
      const bool eq = inrow && k != 0u && k == thr;
      const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
      const int rank = eq_before + __popc(eqb & ((1u << lane) - 1u));
      sel = sel || (eq && rank < need_eq);
      eq_before += __popc(eqb);
      const uint32_t bits = __ballot_sync(0xffffffffu, sel);
      if (lane == 0) mrow[wg] = bits;
      count += __popc(bits);
    }
  }
  count = (int)row_combine<WPR, false>((uint64_t)count, xb, par, q, rw);
  if (q == 0 && lane == 0) a.kv_count[rowid] = count;
}

// ---- selection by radix (fixed top-k and budget modes): one block of 128 threads per
// row at a time, each block taking rows of one (b, h) in turn. A thread holds its KPT keys
// of the row in registers (key j at thread j mod 128, slot j / 128); 0 marks window tiles
// and slots past NKT. The key of the extra-th best candidate is found by narrowing a key
// range, starting from the candidates' [min, max]: each pass splits the range into at most
// 256 buckets of 2^shift keys (the bucket is (key - lo) >> shift, so the split follows the
// keys' spread, not fixed digit boundaries, and lanes seldom collide on a counter), counts
// them in per-warp shared histograms, and one warp finds the largest bucket at or above
// which at least the still-needed number of keys lie. A bucket holding exactly that number
// ends the search (every key from its low end up is taken); otherwise the range shrinks to
// that bucket, by at least eight bits of width per pass, down to one key value, of which
// the first in tile order are taken. The result is "highest score, ties to the lower
// index", as the argmax and threshold search of select_kernel give it.
constexpr int kRsThreads = 128;
constexpr int kRsBlocksPerSm = 8;

// Sum over the block's four warps; `red` holds four ints. Every thread gets the sum.
__device__ __forceinline__ int rs_block_sum(int v, int* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const int s = red[0] + red[1] + red[2] + red[3];
  __syncthreads();
  return s;
}

template <int MODE, bool TOK, int KPT>
__global__ void __launch_bounds__(kRsThreads, kRsBlocksPerSm) select_radix_kernel(SelArgs a, const float* __restrict__ S,
                                                                  int NKTP) {
  extern __shared__ __align__(16) uint32_t sm_u32[];
  const Geom& g = a.g;
  const int NKT = g.NT, NQT = g.NT;
  const int b = blockIdx.z, h = blockIdx.y;
  const long long bh = (long long)b * g.H + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* srows = reinterpret_cast<float*>(sm_u32);            // two score rows (NKTP each)
  uint32_t* coord = sm_u32 + 2 * NKTP;                         // NKT tile coordinates
  uint32_t* hist = coord + ((NKT + 3) & ~3);                   // 4 warps x 256 bucket counts
  uint32_t* eqw = hist + 1024;                                 // per mask word: keys equal to thr
  int* red = reinterpret_cast<int*>(eqw + ((g.NW + 3) & ~3));  // sums, broadcast values, key range

  for (int j = tid; j < NKT; j += kRsThreads) {
    int tt, ty, tx;
    tile_xyz(g, j, tt, ty, tx);
    coord[j] = pack_coord(tt, ty, tx);
  }
  __syncthreads();

  // The next row's scores are copied into shared memory (cp.async, 16 bytes per copy)
  // while this row is selected; one commit group per row, empty for dense rows.
  auto fetch_row = [&](int ii, int buf) {
    if (ii < NQT && !a.dense[(long long)b * NQT + ii]) {
      const float* src = S + (bh * NQT + ii) * NKTP;
      const uint32_t dst = (uint32_t)__cvta_generic_to_shared(srows + buf * NKTP);
      for (int c = tid; c < NKTP / 4; c += kRsThreads)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + 16u * c), "l"(src + 4 * c) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  fetch_row(blockIdx.x, 0);
  int buf = 0;
  for (int i = blockIdx.x; i < NQT; i += gridDim.x, buf ^= 1) {
    // Buffer buf ^ 1 was last read in the previous row, before its closing block sums.
    fetch_row(i + gridDim.x, buf ^ 1);
    asm volatile("cp.async.wait_group 1;" ::: "memory");      // this row's copy has landed
    __syncthreads();
    const long long rowid = bh * NQT + i;
    const float* srow = srows + buf * NKTP;
    uint32_t* mrow = a.mask + rowid * g.NW;
    if (a.dense[(long long)b * NQT + i]) {                     // the same branch for the whole block
      for (int w = tid; w < g.NW; w += kRsThreads) {
        const int rem = NKT - 32 * w;
        mrow[w] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
      }
      if (tid == 0) a.kv_count[rowid] = NKT;
      continue;
    }
    const uint32_t ci = coord[i];
    int kind = a.window_kind, rad = a.radius, extra;
    if (MODE == kSelectFixed) {
      extra = a.topk;
    } else {
      const int2 pl = a.plan[rowid];
      kind = 1;
      rad = pl.x;
      extra = pl.y;
    }
    uint32_t key[KPT];
    int ncand = 0;
#pragma unroll
    for (int m = 0; m < KPT; ++m) {
      const int j = tid + kRsThreads * m;
      const bool cand = j < NKT && !sel_in_window<TOK>(ci, coord[j], kind, rad);
      key[m] = cand ? order_key(srow[j]) : 0u;
      ncand += cand ? 1 : 0;
    }
    ncand = rs_block_sum(ncand, red);
    extra = max(0, min(extra, ncand));

    // keys >= t_ge are taken; of the keys equal to thr, the first need_eq in tile order
    uint32_t t_ge, thr = 0xffffffffu;
    int need_eq = 0;
    if (extra == 0) {
      t_ge = 0xffffffffu;                                       // no score maps to this key
    } else if (extra == ncand) {
      t_ge = 1u;                                                // every candidate
    } else {
      // key range [lo, hi] of the candidates
      uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
      for (int m = 0; m < KPT; ++m) {
        if (key[m] != 0u) {
          lo = min(lo, key[m]);
          hi = max(hi, key[m]);
        }
      }
      lo = __reduce_min_sync(0xffffffffu, lo);
      hi = __reduce_max_sync(0xffffffffu, hi);
      if (lane == 0) {
        red[8 + warp] = (int)lo;
        red[12 + warp] = (int)hi;
      }
      __syncthreads();
      lo = min(min((uint32_t)red[8], (uint32_t)red[9]), min((uint32_t)red[10], (uint32_t)red[11]));
      hi = max(max((uint32_t)red[12], (uint32_t)red[13]), max((uint32_t)red[14], (uint32_t)red[15]));
      int remaining = extra;
      bool done = false;
      while (!done) {
        // buckets of 2^shift keys over [lo, hi]: at most 256
        const uint32_t span = hi - lo;
        const int shift = span < 256u ? 0 : (32 - __clz(span)) - 8;
        uint32_t* wh = hist + warp * 256;                       // this warp's histogram
#pragma unroll
        for (int e = 0; e < 8; ++e) hist[tid + kRsThreads * e] = 0u;
        __syncthreads();
#pragma unroll
        for (int m = 0; m < KPT; ++m) {
          const uint32_t k = key[m];
          if (k >= lo && k <= hi) atomicAdd(&wh[(k - lo) >> shift], 1u);
        }
        __syncthreads();
        if (warp == 0) {
          // lane l holds buckets 8l .. 8l+7; find the largest bucket at or above which at
          // least `remaining` keys lie
          uint32_t c[8];
          int lt = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int d = 8 * lane + e;
            c[e] = hist[d] + hist[256 + d] + hist[512 + d] + hist[768 + d];
            lt += (int)c[e];
          }
          int incl = lt;                                        // keys in lanes >= this one
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_down_sync(0xffffffffu, incl, off);
            if (lane + off < 32) incl += v;
          }
          int sfx = incl - lt, best = -1, best_above = 0, best_at = 0;
#pragma unroll
          for (int e = 7; e >= 0; --e) {
            const int above = sfx;
            sfx += (int)c[e];
            if (best < 0 && sfx >= remaining) {
              best = 8 * lane + e;
              best_above = above;
              best_at = (int)c[e];
            }
          }
          const uint32_t okl = __ballot_sync(0xffffffffu, best >= 0);
          if (lane == 31 - __clz(okl)) {                       // the lane of the largest such bucket
            red[4] = best;
            red[5] = best_above;
            red[6] = best_at;
          }
        }
        __syncthreads();
        const int dsel = red[4], above = red[5], at = red[6];
        remaining -= above;
        const uint32_t blo = lo + ((uint32_t)dsel << shift);
        const uint32_t bhi = (uint32_t)min((unsigned long long)hi, (unsigned long long)blo + (1ull << shift) - 1ull);
        if (at == remaining) {                                  // the whole bucket is taken
          t_ge = blo;
          done = true;
        } else if (shift == 0) {                                // one key value: ties
          thr = blo;
          t_ge = blo + 1u;
          need_eq = remaining;
          done = true;
        }
        lo = blo;
        hi = bhi;
      }
      if (t_ge == 0u) t_ge = 1u;                                // a band from key 0: every candidate
    }

    if (need_eq > 0) {                                          // ties at the boundary key
#pragma unroll
      for (int m = 0; m < KPT; ++m) {
        const int w = warp + 4 * m;
        const int j = tid + kRsThreads * m;
        const uint32_t eqb = __ballot_sync(0xffffffffu, j < NKT && key[m] != 0u && key[m] == thr);
        if (lane == 0 && w < g.NW) eqw[w] = eqb;
      }
      __syncthreads();
    }
    int count = 0;
#pragma unroll
    for (int m = 0; m < KPT; ++m) {
      const int w = warp + 4 * m;                              // mask word of this slot (warp-uniform)
      if (w < g.NW) {
        const int j = tid + kRsThreads * m;
        const uint32_t k = key[m];
        const bool inrow = j < NKT;
        bool sel = inrow && (k == 0u || k >= t_ge);
        if (need_eq > 0 && inrow && k != 0u && k == thr) {
          int rank = __popc(eqw[w] & ((1u << lane) - 1u));
          for (int ww = 0; ww < w; ++ww) rank += __popc(eqw[ww]);
          sel = rank < need_eq;
        }
        const uint32_t bits = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) {
          mrow[w] = bits;
          count += __popc(bits);
        }
      }
    }
    count = rs_block_sum(count, red);
    if (tid == 0) a.kv_count[rowid] = count;
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
}

template <int MODE, bool TOK, int KPT>
cudaError_t launch_select_radix_kpt(const Geom& g, const SelArgs& a, const float* S, int NKTP, cudaStream_t s) {
  const size_t smem = sizeof(uint32_t) * (2 * (size_t)NKTP + (size_t)((g.NT + 3) & ~3) + 1024 +
                                          (size_t)((g.NW + 3) & ~3) + 16);
  cudaError_t e = cudaFuncSetAttribute(select_radix_kernel<MODE, TOK, KPT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_radix_kernel<MODE, TOK, KPT>, kRsThreads, smem);
  if (e != cudaSuccess) return e;
  // one wave: every block resident at once, each (b, h) with the same number of blocks
  const int per_bh = max(1, min(g.NT, (sms * max(per_sm, 1)) / (g.B * g.H)));
  const dim3 grid(per_bh, g.H, g.B);
  select_radix_kernel<MODE, TOK, KPT><<<grid, kRsThreads, smem, s>>>(a, S, NKTP);
  return cudaGetLastError();
}

// KPT = key slots per thread: the row's NW * 32 slots over 128 threads, rounded up to 8.
template <int MODE, bool TOK>
cudaError_t launch_select_radix(const Geom& g, const SelArgs& a, const float* S, int NKTP, cudaStream_t s) {
  const int kpt = ceil_div(g.NW * 32, kRsThreads);
  if (kpt <= 8) return launch_select_radix_kpt<MODE, TOK, 8>(g, a, S, NKTP, s);
  if (kpt <= 16) return launch_select_radix_kpt<MODE, TOK, 16>(g, a, S, NKTP, s);
  if (kpt <= 24) return launch_select_radix_kpt<MODE, TOK, 24>(g, a, S, NKTP, s);
  return launch_select_radix_kpt<MODE, TOK, 32>(g, a, S, NKTP, s);
}

template <int MODE, int KW, int WPR, bool TOK>
cudaError_t launch_select_kw(const Geom& g, size_t smem, const SelArgs& a, const float* S, int NKTP, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(select_kernel<MODE, KW, WPR, TOK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(ceil_div(g.NT, kSelWarps / WPR), g.H, g.B);
  select_kernel<MODE, KW, WPR, TOK><<<grid, kSelThreads, smem, s>>>(a, S, NKTP);
  return cudaGetLastError();
}

// Words of a mask row per lane at most 32: rows of more than 32 words span 2 or 4 warps.
template <int MODE, bool TOK>
cudaError_t launch_select(const Geom& g, size_t smem, const SelArgs& a, const float* S, int NKTP, cudaStream_t s) {
  if (g.NW <= 8) return launch_select_kw<MODE, 8, 1, TOK>(g, smem, a, S, NKTP, s);
  if (g.NW <= 16) return launch_select_kw<MODE, 16, 1, TOK>(g, smem, a, S, NKTP, s);
  if (g.NW <= 32) return launch_select_kw<MODE, 32, 1, TOK>(g, smem, a, S, NKTP, s);
  if (g.NW <= 64) return launch_select_kw<MODE, 32, 2, TOK>(g, smem, a, S, NKTP, s);
  return launch_select_kw<MODE, 32, 4, TOK>(g, smem, a, S, NKTP, s);
}

// The mask from tile-major Q and K (qt, kt: pooled here, into the workspace) or from
// pooled means computed by the fused reorder (qt, kt null; qbar_in, kbar_in given).
template <int D>
cudaError_t build_mask_d(const Geom& g, const bsa_mask_params& p, const __nv_bfloat16* qt,
                         const __nv_bfloat16* kt, const float* qbar_in, const float* kbar_in,
                         const float* difficulty, uint32_t* mask, int32_t* kv_count, uint8_t* ws,
                         cudaStream_t s) {
  const WsLayout L = ws_layout(g);
  const float* qbar = qbar_in;
  const float* kbar = kbar_in;
  uint8_t* dense = ws + L.dense;
  float* entropy = reinterpret_cast<float*>(ws + L.entropy);
  int2* plan = reinterpret_cast<int2*>(ws + L.plan);

  cudaError_t e;
  if (qt) {
    float* qb = reinterpret_cast<float*>(ws + L.qbar);
    float* kb = reinterpret_cast<float*>(ws + L.kbar);
    const long long warps = 2LL * g.B * g.H * g.NT;
    pool_kernel<D><<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(g, qt, kt, qb, kb);
    count_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    qbar = qb;
    kbar = kb;
  }

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
  a.qbar = qbar;
  a.kbar = kbar;
  a.dense = dense;
  a.entropy = entropy;
  a.plan = plan;
  a.mask = mask;
  a.kv_count = kv_count;

  float* S = reinterpret_cast<float*>(ws + L.scores);
  const int NKTP = (g.NT + 3) & ~3;
  e = launch_score_tc(g, qbar, kbar, S, NKTP, reinterpret_cast<uint32_t*>(ws), s);
  if (e != cudaSuccess) return e;

  a.theta = p.budget_target;
  const long long rows = (long long)g.B * g.H * g.NT;
  if (p.budget_mode == 1) {
    entropy_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(g, S, NKTP, a.scale, entropy);
    count_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    budget_kernel<<<(unsigned)(g.B * g.H), kBudgetThreads, 0, s>>>(g, entropy, dense,
                                                                  (double)p.budget_target, plan);
    count_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // coordinate table, then per row of the block a double-buffered exchange of one 64-bit
  // value per warp
  const size_t sel_smem = sizeof(uint32_t) * (size_t)((NKTP + 1) & ~1) + (size_t)kSelWarps * 2 * sizeof(uint64_t);
  // the budget mode always uses the decayed tile window (kind 1)
  const bool tok = p.window_kind == 2;
  if (p.budget_mode == 0)
    e = tok ? launch_select_radix<kSelectFixed, true>(g, a, S, NKTP, s)
            : launch_select_radix<kSelectFixed, false>(g, a, S, NKTP, s);
  else if (p.budget_mode == 2)
    e = tok ? launch_select<kSelectMass, true>(g, sel_smem, a, S, NKTP, s)
            : launch_select<kSelectMass, false>(g, sel_smem, a, S, NKTP, s);
  else
    e = launch_select_radix<kSelectBudget, false>(g, a, S, NKTP, s);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_build_mask(const Geom& g, const bsa_mask_params& p, const __nv_bfloat16* qt,
                              const __nv_bfloat16* kt, const float* difficulty, uint32_t* mask,
                              int32_t* kv_count, uint8_t* ws, cudaStream_t s) {
  if (g.d == 128) return build_mask_d<128>(g, p, qt, kt, nullptr, nullptr, difficulty, mask, kv_count, ws, s);
  return build_mask_d<64>(g, p, qt, kt, nullptr, nullptr, difficulty, mask, kv_count, ws, s);
}

cudaError_t launch_build_mask_pooled(const Geom& g, const bsa_mask_params& p, const float* qbar,
                                     const float* kbar, const float* difficulty, uint32_t* mask,
                                     int32_t* kv_count, uint8_t* ws, cudaStream_t s) {
  if (g.d == 128) return build_mask_d<128>(g, p, nullptr, nullptr, qbar, kbar, difficulty, mask, kv_count, ws, s);
  return build_mask_d<64>(g, p, nullptr, nullptr, qbar, kbar, difficulty, mask, kv_count, ws, s);
}

}  // namespace bsa

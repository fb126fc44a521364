// Block-sparse attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Execution of a block-sparse tile mask (Token Radius Attention summary, "Efficient
// execution"), FlashAttention-style: for every query row, an online softmax over the
// valid tokens of its retained key tiles, fp32 statistics, bf16 probabilities in the P.V
// product, fp32 accumulation, output and natural-log LSE written in raster order.
//
// Work unit: up to four query tiles of one (b, h) and of the same route class (all
// dense, or all local), consecutive in tile order. They form two sub-units of two tiles,
// A and B, each one M=128 tcgen05 tile. The CTA streams the union of the four rows'
// retained key tiles through one shared K/V ring, two key tiles (128 keys) per block.
// Each sub-unit issues its MMAs only for the blocks it needs, with N=128, or N=64 on the
// one tile it needs (descriptor offset), so no tensor work is spent on tiles that neither
// of its two query tiles retains; a tile retained by only one of its two query tiles is
// masked to -inf for the other half of the rows.
//
// The two sub-units ping-pong on the tensor core: while softmax warpgroup A turns S_A
// into P_A, the MMA warp runs P_B V and the next S_B = Q_B K^T, and the other way round.
//
// Schedule (one launch each, on the caller's stream):
//   sched_count  per (b, h): number of dense rows (kv_count == NKT) and local rows
//   sched_scan   offsets: every dense unit of every (b, h) first, then the local units
//   sched_write  per (b, h): the units, four consecutive rows of a class each
//   attn         one CTA per unit, in list order: heavy (dense) units first, and units of
//                the same head next to each other so that their K/V tiles stay in L2.
//
// CTA roles (320 threads):
//   warps 0-3  softmax of sub-unit A: thread t owns query row t = TMEM lane t
//   warps 4-7  softmax of sub-unit B
//              (each reads S from TMEM, writes P as bf16 pairs over S, rescales its O in
//              TMEM when the running max grows, and runs the epilogue)
//   warp 8     builds the key-tile lists in shared memory, then lane 0 issues the TMA
//              loads of Q and of the K/V ring
//   warp 9     allocates TMEM; lane 0 issues S = Q K^T (SS) and O += P V (TS)
// TMEM columns: S_A 0-127, S_B 128-255, O_A 256-383, O_B 384-511.
// Shared memory (1024-byte aligned): Q_A, Q_B, 2 K stages, 2 V stages, each
// [D/64][128 rows][128 B] with the 128-byte swizzle that TMA and tcgen05 share; the
// key-tile list; the per-sub-unit block lists; barriers.
#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tmem_ops.cuh"

#include <math.h>

namespace bsa {
namespace {

constexpr int kAttnThreads = 320;
constexpr int kNSK = 2;                            // K ring stages
constexpr int kNSV = 2;                            // V ring stages
constexpr int kMaxBlocks = kMaxTiles / 2 + 1;
constexpr long long kWaitLimit = 4000000000LL;     // SM cycles, about 2 s
constexpr int kTmemCols = 512;
constexpr int kUnitInts = 8;                       // {bh, q0, q1, q2, q3, 0, 0, 0}

template <int D>
struct Cfg {
  static constexpr int kTileBytes = 64 * D * 2;         // one 64-token tile
  static constexpr int kBufBytes = 2 * kTileBytes;      // two tiles (128 rows)
  static constexpr int kDBlockStride = 128 * 128;       // bytes between 64-column blocks
  static constexpr int kQOff = 0;                       // Q_A, then Q_B
  static constexpr int kKOff = 2 * kBufBytes;
  static constexpr int kVOff = kKOff + kNSK * kBufBytes;
  static constexpr int kBarOff = kVOff + kNSV * kBufBytes;
  // barriers: q, kfull[2], kempty[2], vfull[2], vempty[2], sfull[2], pfull[2], odone[2], drain
  static constexpr int kNumBars = 1 + 2 * kNSK + 2 * kNSV + 2 + 2 + 2 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;         // tmem base, counts, abort
  static constexpr int kListOff = kMiscOff + 64;
  static constexpr int kBlkOff = kListOff + kMaxTiles * 4;        // uint16 block lists A, B
  static constexpr int kSmemBytes = 1024 + kBlkOff + 2 * kMaxBlocks * 2;
};

struct AttnArgs {
  Geom g;
  const uint32_t* mask;
  const int* units;          // kUnitInts per unit
  const int* header;         // header[1] = number of units
  __nv_bfloat16* out;
  float* lse;
  uint32_t* err;
  float scale_log2;          // softmax scale * log2(e)
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

// All lanes take the same decision after a per-thread bounded wait.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          uint32_t* err) {
  const bool ok = ptx::mbar_wait(bar, parity, abort, err, kWaitLimit);
  return __all_sync(0xffffffffu, ok);
}

// Mask 64 score columns of key tile `e` (a list entry) for this thread's query row: all
// -inf when the row's query tile does not retain the tile, the tile's padding slots -inf
// otherwise. Both conditions are warp-uniform, so full retained tiles cost one test.
__device__ __forceinline__ void mask_tile(uint32_t (&r)[64], uint32_t e, int mshift, const Geom& g) {
  constexpr uint32_t kNegInf = 0xff800000u;
  if (!((e >> mshift) & 1u)) {
#pragma unroll
    for (int c = 0; c < 64; ++c) r[c] = kNegInf;
  } else if (!((e >> 20) & 1u)) {
    int tt, ty, tx;
    tile_xyz(g, (int)(e & 0xffffu), tt, ty, tx);
    const uint64_t valid = tile_valid_mask(g, tt, ty, tx);
    const uint32_t lo = (uint32_t)valid, hi = (uint32_t)(valid >> 32);
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      r[c] = ((lo >> c) & 1u) ? r[c] : kNegInf;
      r[32 + c] = ((hi >> c) & 1u) ? r[32 + c] : kNegInf;
    }
  }
}

// Row maximum with four independent chains (short dependency chains for the scheduler).
__device__ __forceinline__ float row_max64(const uint32_t (&r)[64], float m) {
  float a0 = m, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
  for (int c = 0; c < 64; c += 8) {
    a0 = max3(a0, __uint_as_float(r[c + 0]), __uint_as_float(r[c + 1]));
    a1 = max3(a1, __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
    a2 = max3(a2, __uint_as_float(r[c + 4]), __uint_as_float(r[c + 5]));
    a3 = max3(a3, __uint_as_float(r[c + 6]), __uint_as_float(r[c + 7]));
  }
  return fmaxf(max3(a0, a1, a2), a3);
}

// p = 2^(s*c - m) for 64 columns; accumulates the fp32 sum and packs the bf16 pairs into
// pk (column 2i in the low half of pk[i]).
__device__ __forceinline__ void exp_pack64(const uint32_t (&r)[64], float c, float m, float& sum,
                                           uint32_t (&pk)[32]) {
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;       // four short chains
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float p0 = ex2(fmaf(__uint_as_float(r[2 * i]), c, -m));
    const float p1 = ex2(fmaf(__uint_as_float(r[2 * i + 1]), c, -m));
    const float p2 = ex2(fmaf(__uint_as_float(r[2 * i + 2]), c, -m));
    const float p3 = ex2(fmaf(__uint_as_float(r[2 * i + 3]), c, -m));
    pk[i] = pack_bf16x2(p0, p1);
    pk[i + 1] = pack_bf16x2(p2, p3);
    s0 += p0;
    s1 += p1;
    s2 += p2;
    s3 += p3;
  }
  sum += (s0 + s1) + (s2 + s3);
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, AttnArgs a) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = ptx::smem_u32(smem);

  const Geom& g = a.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if ((int)blockIdx.x >= a.header[1]) return;
  const int* up = a.units + (size_t)blockIdx.x * kUnitInts;
  const int bh = up[0];
  int q[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) q[t] = up[1 + t];
  bool bad = bh < 0 || bh >= g.B * g.H || q[0] < 0;
#pragma unroll
  for (int t = 0; t < 4; ++t) bad = bad || q[t] >= g.NT || q[t] < -1;
  if (bad) {
    if (threadIdx.x == 0) report_error(a.err, BSA_KERR_BAD_UNIT);
    return;
  }
  const bool hasB = q[2] >= 0;

  const uint32_t bar_q = sbase + C::kBarOff;
  auto kfull = [&](int s) { return sbase + C::kBarOff + 8 * (1 + s); };
  auto kempty = [&](int s) { return sbase + C::kBarOff + 8 * (1 + kNSK + s); };
  auto vfull = [&](int s) { return sbase + C::kBarOff + 8 * (1 + 2 * kNSK + s); };
  auto vempty = [&](int s) { return sbase + C::kBarOff + 8 * (1 + 2 * kNSK + kNSV + s); };
  auto sfull = [&](int u) { return sbase + C::kBarOff + 8 * (1 + 2 * kNSK + 2 * kNSV + u); };
  auto pfull = [&](int u) { return sbase + C::kBarOff + 8 * (3 + 2 * kNSK + 2 * kNSV + u); };
  auto odone = [&](int u) { return sbase + C::kBarOff + 8 * (5 + 2 * kNSK + 2 * kNSV + u); };
  const uint32_t bar_drain = sbase + C::kBarOff + 8 * (7 + 2 * kNSK + 2 * kNSV);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  int* counts = reinterpret_cast<int*>(smem + C::kMiscOff + 4);        // L, cntA, cntB
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 16);
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + C::kListOff);
  uint16_t* blk = reinterpret_cast<uint16_t*>(smem + C::kBlkOff);      // [2][kMaxBlocks]

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_q, 1);
    for (int s = 0; s < kNSK; ++s) { ptx::mbar_init(kfull(s), 1); ptx::mbar_init(kempty(s), 1); }
    for (int s = 0; s < kNSV; ++s) { ptx::mbar_init(vfull(s), 1); ptx::mbar_init(vempty(s), 1); }
    for (int u = 0; u < 2; ++u) {
      ptx::mbar_init(sfull(u), 1);
      ptx::mbar_init(pfull(u), 128);
      ptx::mbar_init(odone(u), 1);
    }
    ptx::mbar_init(bar_drain, 1);
    *abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 8) {
    // Union of the four rows' key tiles, ascending; bit 16+t: retained by query tile q[t];
    // bit 20: the tile has no padding slot.
    if (lane == 0) {
      ptx::prefetch_tensormap(&tmQ);
      ptx::prefetch_tensormap(&tmK);
      ptx::prefetch_tensormap(&tmV);
    }
    const uint32_t* mrow[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) mrow[t] = a.mask + ((long long)bh * g.NT + (q[t] >= 0 ? q[t] : q[0])) * g.NW;
    int running = 0;
    for (int w0 = 0; w0 < g.NW; w0 += 32) {
      const int w = w0 + lane;
      uint32_t b[4] = {0u, 0u, 0u, 0u};
      if (w < g.NW) {
        const int rem = g.NT - 32 * w;
        const uint32_t keep = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
#pragma unroll
        for (int t = 0; t < 4; ++t) b[t] = q[t] >= 0 ? (__ldg(&mrow[t][w]) & keep) : 0u;
      }
      uint32_t u = b[0] | b[1] | b[2] | b[3];
      const int cnt = __popc(u);
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      int pos = running + incl - cnt;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        const int j = 32 * w + bit;
        int tt, ty, tx;
        tile_xyz(g, j, tt, ty, tx);
        const uint32_t full = tile_valid_count(g, tt, ty, tx) == 64 ? 1u : 0u;
        list[pos++] = (uint32_t)j | (((b[0] >> bit) & 1u) << 16) | (((b[1] >> bit) & 1u) << 17) |
                      (((b[2] >> bit) & 1u) << 18) | (((b[3] >> bit) & 1u) << 19) | (full << 20);
      }
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    // Per-sub-unit block lists: entry = block | need << 12, need bit t = tile slot t used.
    const int L = running, nblk = (L + 1) >> 1;
    int ca = 0, cb = 0;
    for (int j0 = 0; j0 < nblk; j0 += 32) {
      const int j = j0 + lane;
      uint32_t na = 0, nb = 0;
      if (j < nblk) {
        const uint32_t e0 = list[2 * j];
        const uint32_t e1 = (2 * j + 1 < L) ? list[2 * j + 1] : 0u;
        na = (((e0 >> 16) & 3u) ? 1u : 0u) | (((e1 >> 16) & 3u) ? 2u : 0u);
        nb = (((e0 >> 18) & 3u) ? 1u : 0u) | (((e1 >> 18) & 3u) ? 2u : 0u);
      }
      const uint32_t ba = __ballot_sync(0xffffffffu, na != 0), bb = __ballot_sync(0xffffffffu, nb != 0);
      const uint32_t lt = (1u << lane) - 1u;
      if (na) blk[ca + __popc(ba & lt)] = (uint16_t)(j | (na << 12));
      if (nb) blk[kMaxBlocks + cb + __popc(bb & lt)] = (uint16_t)(j | (nb << 12));
      ca += __popc(ba);
      cb += __popc(bb);
    }
    if (lane == 0) {
      counts[0] = L;
      counts[1] = ca;
      counts[2] = cb;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int L = counts[0];
  const int nblk = (L + 1) >> 1;
  if (nblk == 0 && threadIdx.x == 0) report_error(a.err, BSA_KERR_BAD_MASK);
  const long long tile_row0 = (long long)bh * g.NT;   // tile index base of this (b, h)

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && nblk > 0) {
      int last_k[kNSK], last_v[kNSV];
      for (int s = 0; s < kNSK; ++s) last_k[s] = -1;
      for (int s = 0; s < kNSV; ++s) last_v[s] = -1;
      const int nsub = hasB ? 2 : 1;
      ptx::mbar_arrive_expect_tx(bar_q, nsub * C::kBufBytes);
      for (int u = 0; u < nsub; ++u)
        for (int half = 0; half < 2; ++half) {
          const int tile = q[2 * u + half] >= 0 ? q[2 * u + half] : q[2 * u];
          const int row = (int)((tile_row0 + tile) * 64);
          for (int db = 0; db < D / 64; ++db)
            ptx::tma_load_2d(sbase + C::kQOff + u * C::kBufBytes + db * C::kDBlockStride + half * 8192, &tmQ,
                             bar_q, db * 64, row);
        }
      for (int j = 0; j < nblk; ++j) {
        const int nt = (2 * j + 1 < L) ? 2 : 1;
        const int sk = j % kNSK;
        if (!ptx::mbar_wait(kempty(sk), ((j / kNSK) & 1) ^ 1, abort, a.err, kWaitLimit)) break;
        ptx::mbar_arrive_expect_tx(kfull(sk), nt * C::kTileBytes);
        for (int t = 0; t < nt; ++t) {
          const int row = (int)((tile_row0 + (int)(list[2 * j + t] & 0xffffu)) * 64);
          for (int db = 0; db < D / 64; ++db)
            ptx::tma_load_2d(sbase + C::kKOff + sk * C::kBufBytes + db * C::kDBlockStride + t * 8192, &tmK,
                             kfull(sk), db * 64, row);
        }
        last_k[sk] = j;
        const int sv = j % kNSV;
        if (!ptx::mbar_wait(vempty(sv), ((j / kNSV) & 1) ^ 1, abort, a.err, kWaitLimit)) break;
        ptx::mbar_arrive_expect_tx(vfull(sv), nt * C::kTileBytes);
        for (int t = 0; t < nt; ++t) {
          const int row = (int)((tile_row0 + (int)(list[2 * j + t] & 0xffffu)) * 64);
          for (int db = 0; db < D / 64; ++db)
            ptx::tma_load_2d(sbase + C::kVOff + sv * C::kBufBytes + db * C::kDBlockStride + t * 8192, &tmV,
                             vfull(sv), db * 64, row);
        }
        last_v[sv] = j;
      }
      // Never leave with copies in flight: wait for the last load issued into each stage.
      int zero = 0;
      for (int s = 0; s < kNSK; ++s)
        if (last_k[s] >= 0) ptx::mbar_wait(kfull(s), (last_k[s] / kNSK) & 1, &zero, a.err, kWaitLimit);
      for (int s = 0; s < kNSV; ++s)
        if (last_v[s] >= 0) ptx::mbar_wait(vfull(s), (last_v[s] / kNSV) & 1, &zero, a.err, kWaitLimit);
      ptx::mbar_wait(bar_q, 0, &zero, a.err, kWaitLimit);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && nblk > 0) {
      constexpr uint32_t kIdQK128 = ptx::idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t kIdQK64 = ptx::idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t kIdPV = ptx::idesc_bf16_f32(128, D, 0, 1);
      int pend[2] = {-1, -1};       // block whose P.V is still to be issued, per sub-unit
      uint32_t pneed[2] = {0u, 0u};
      int npv[2] = {0, 0};          // P.V products issued, per sub-unit
      int vref[kNSV] = {0, 0};      // P.V products still to read each V stage
      bool ok = ptx::mbar_wait(bar_q, 0, abort, a.err, kWaitLimit);

      auto need_of = [&](int j, int u) -> uint32_t {
        const uint32_t e0 = list[2 * j];
        const uint32_t e1 = (2 * j + 1 < L) ? list[2 * j + 1] : 0u;
        const int sh = 16 + 2 * u;
        return (((e0 >> sh) & 3u) ? 1u : 0u) | (((e1 >> sh) & 3u) ? 2u : 0u);
      };
      auto issue_pv = [&](int u) -> bool {
        const int j = pend[u];
        const uint32_t n = pneed[u];
        const int sv = j % kNSV;
        if (!ptx::mbar_wait(pfull(u), npv[u] & 1, abort, a.err, kWaitLimit)) return false;
        if (!ptx::mbar_wait(vfull(sv), (j / kNSV) & 1, abort, a.err, kWaitLimit)) return false;
        ptx::tc_fence_after();
        const uint32_t p_tmem = tmem + 128 * u;
        const uint32_t o_tmem = tmem + 256 + 128 * u;
        const uint32_t vaddr = sbase + C::kVOff + sv * C::kBufBytes + (n == 2u ? 8192u : 0u);
        const int nk = (n == 3u) ? 8 : 4;
        for (int kk = 0; kk < nk; ++kk) {
          const uint64_t bd = ptx::smem_desc_sw128(vaddr + kk * 2048, C::kDBlockStride, 1024);
          ptx::mma_ts(o_tmem, p_tmem + kk * 8, bd, kIdPV, (npv[u] > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(odone(u));
        ++npv[u];
        if (--vref[sv] == 0) ptx::mma_commit(vempty(sv));
        pend[u] = -1;
        return true;
      };

      for (int j = 0; j < nblk && ok; ++j) {
        const int sk = j % kNSK;
        const uint32_t nA = need_of(j, 0), nB = need_of(j, 1);
        if (!ptx::mbar_wait(kfull(sk), (j / kNSK) & 1, abort, a.err, kWaitLimit)) break;
        ptx::tc_fence_after();
        vref[j % kNSV] = (nA != 0u) + (nB != 0u);
        for (int u = 0; u < 2 && ok; ++u) {
          const uint32_t n = u ? nB : nA;
          if (n == 0u) continue;
          if (pend[u] >= 0 && !issue_pv(u)) { ok = false; break; }
          const uint32_t s_tmem = tmem + 128 * u;
          const uint32_t qaddr = sbase + C::kQOff + u * C::kBufBytes;
          const uint32_t kaddr = sbase + C::kKOff + sk * C::kBufBytes + (n == 2u ? 8192u : 0u);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kDBlockStride + (kk & 3) * 32;
            const uint64_t ad = ptx::smem_desc_sw128(qaddr + off, 16, 1024);
            const uint64_t bd = ptx::smem_desc_sw128(kaddr + off, 16, 1024);
            ptx::mma_ss(s_tmem, ad, bd, n == 3u ? kIdQK128 : kIdQK64, kk > 0 ? 1u : 0u);
          }
          ptx::mma_commit(sfull(u));
          pend[u] = j;
          pneed[u] = n;
        }
        if (!ok) break;
        ptx::mma_commit(kempty(sk));
        // P.V of a sub-unit that has no work in the next block goes out now, so that every
        // V stage is released within one block of its use.
        for (int u = 0; u < 2; ++u)
          if (pend[u] >= 0 && (j + 1 >= nblk || need_of(j + 1, u) == 0u) && !issue_pv(u)) { ok = false; break; }
      }
      // Never free TMEM under a running MMA: wait until everything issued has completed.
      int zero = 0;
      ptx::mma_commit(bar_drain);
      ptx::mbar_wait(bar_drain, 0, &zero, a.err, kWaitLimit);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int u = warp >> 2;                 // sub-unit of this warpgroup
    const int row = threadIdx.x & 127;       // TMEM lane
    const int half = row >> 6;
    const int qt = q[2 * u + half];          // this row's query tile (-1: none)
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_tmem = tmem + 128 * u + lane_base;
    const uint32_t o_tmem = tmem + 256 + 128 * u + lane_base;
    const int cnt = counts[1 + u];
    const uint16_t* my_blk = blk + u * kMaxBlocks;
    const int mshift = 16 + 2 * u + half;
    const float c = a.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = cnt > 0;
    for (int it = 0; it < cnt; ++it) {
      if (!warp_wait(sfull(u), it & 1, abort, a.err)) { ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t bj = my_blk[it];
      const int j = bj & 4095;
      const uint32_t n = bj >> 12;
      const uint32_t e0 = list[2 * j];
      const uint32_t e1 = (2 * j + 1 < L) ? list[2 * j + 1] : 0u;
      const uint32_t ea = (n & 1u) ? e0 : e1;      // tile in S columns 0-63
      const bool two = n == 3u;                    // e1 in columns 64-127
      // Tile b's scores are read twice (max, then exponentials) instead of being kept
      // live next to tile a's, which keeps the warpgroup within its register budget.
      float mx;
      {
        uint32_t rb[64];
        if (two) {
          tmem_ld_x64(s_tmem + 64, rb);
          ptx::tmem_wait_ld();
          mask_tile(rb, e1, mshift, g);
          mx = row_max64(rb, -INFINITY);
        } else {
          mx = -INFINITY;
        }
      }
      uint32_t ra[64];
      tmem_ld_x64(s_tmem, ra);
      ptx::tmem_wait_ld();
      mask_tile(ra, ea, mshift, g);
      mx = row_max64(ra, mx);
      // The reference follows the running max exactly, so the row's largest probability
      // is 2^0 = 1, which bf16 holds exactly: rows dominated by one key lose nothing to
      // the bf16 rounding of P. O is rescaled in TMEM whenever the max grows.
      const float m_new = fmaxf(m_run, mx * c);
      const bool grow = m_new > m_run;
      const float m_ref = m_new;
      const float alpha = grow ? ex2(m_run - m_new) : 1.0f;
      const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
      float sum = 0.f;
      uint32_t pk[32];
      exp_pack64(ra, c, m_use, sum, pk);
      tmem_st_x32(s_tmem, pk);
      if (two) {
        uint32_t rb[64];
        tmem_ld_x64(s_tmem + 64, rb);
        ptx::tmem_wait_ld();
        mask_tile(rb, e1, mshift, g);
        exp_pack64(rb, c, m_use, sum, pk);
        tmem_st_x32(s_tmem + 32, pk);
      }
      l_run = l_run * alpha + sum;
      if (it > 0) {
        // O must hold exactly the previous blocks before it is rescaled.
        if (!warp_wait(odone(u), (it - 1) & 1, abort, a.err)) { ok = false; break; }
        ptx::tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t ov[32];
            tmem_ld_x32(o_tmem + ch * 32, ov);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
            tmem_st_x32(o_tmem + ch * 32, ov);
          }
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(pfull(u));
      m_run = m_ref;
    }
    if (ok && warp_wait(odone(u), (cnt - 1) & 1, abort, a.err)) {
      ptx::tc_fence_after();
      const int r = row & 63;
      int n_tok = -1;
      if (qt >= 0) {
        int tt, ty, tx;
        tile_xyz(g, qt, tt, ty, tx);
        const int t = tt * 4 + (r >> 4), y = ty * 4 + ((r >> 2) & 3), xx = tx * 4 + (r & 3);
        if (t < g.T && y < g.Hs && xx < g.Ws) n_tok = (t * g.Hs + y) * g.Ws + xx;
      }
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      const int b = bh / g.H, h = bh - b * g.H;
      uint4* dst = n_tok >= 0 ? reinterpret_cast<uint4*>(a.out + (((long long)b * g.N + n_tok) * g.H + h) * D) : nullptr;
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t ov[32];
        tmem_ld_x32(o_tmem + ch * 32, ov);
        ptx::tmem_wait_ld();
        if (dst) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(ov[8 * k + 0]) * inv_l, __uint_as_float(ov[8 * k + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(ov[8 * k + 2]) * inv_l, __uint_as_float(ov[8 * k + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(ov[8 * k + 4]) * inv_l, __uint_as_float(ov[8 * k + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(ov[8 * k + 6]) * inv_l, __uint_as_float(ov[8 * k + 7]) * inv_l);
            dst[ch * 4 + k] = v;
          }
        }
      }
      if (n_tok >= 0) {
        if (!(l_run > 0.f)) report_error(a.err, BSA_KERR_BAD_MASK);
        if (a.lse) {
          const float m_fin = (m_run == -INFINITY) ? 0.0f : m_run;
          a.lse[(long long)bh * g.N + n_tok] =
              l_run > 0.f ? (m_fin + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
        }
      }
    }
  }

  // ---------------------------------------------------------------------- teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------------ scheduler
__global__ void __launch_bounds__(256) sched_count_kernel(Geom g, const int32_t* __restrict__ kv_count,
                                                          int4* __restrict__ bhcnt) {
  __shared__ int s_nd;
  if (threadIdx.x == 0) s_nd = 0;
  __syncthreads();
  const long long base = (long long)blockIdx.x * g.NT;
  int nd = 0;
  for (int i = threadIdx.x; i < g.NT; i += blockDim.x) nd += kv_count[base + i] == g.NT;
  for (int off = 16; off > 0; off >>= 1) nd += __shfl_xor_sync(0xffffffffu, nd, off);
  if ((threadIdx.x & 31) == 0) atomicAdd(&s_nd, nd);
  __syncthreads();
  if (threadIdx.x == 0) {
    const int nl = g.NT - s_nd;
    bhcnt[blockIdx.x] = make_int4(s_nd, nl, (s_nd + 3) / 4, (nl + 3) / 4);
  }
}

// Single thread: exclusive offsets, dense units of every (b, h) before any local unit.
// bhcnt[i] = (nd, nl, ud, ul) on entry, (dense offset, local offset, ud, ul) on exit.
__global__ void sched_scan_kernel(int BH, int4* __restrict__ bhcnt, int* __restrict__ header) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int td = 0;
  for (int i = 0; i < BH; ++i) td += bhcnt[i].z;
  int od = 0, ol = td;
  for (int i = 0; i < BH; ++i) {
    const int4 c = bhcnt[i];
    bhcnt[i] = make_int4(od, ol, c.z, c.w);
    od += c.z;
    ol += c.w;
  }
  header[1] = ol;
}

// One warp per (b, h): ordered compaction of each class with ballots. The k-th row of a
// class becomes query tile k % 4 of unit k / 4 of that class; the last unit of a class
// may be short (missing tiles -1).
__global__ void __launch_bounds__(32) sched_write_kernel(Geom g, const int32_t* __restrict__ kv_count,
                                                         const int4* __restrict__ bhcnt,
                                                         int* __restrict__ units) {
  const int bh = blockIdx.x, lane = threadIdx.x;
  const long long base = (long long)bh * g.NT;
  const int od = bhcnt[bh].x, ol = bhcnt[bh].y;
  int cd = 0, cl = 0;
  for (int i0 = 0; i0 < g.NT; i0 += 32) {
    const int i = i0 + lane;
    const bool valid = i < g.NT;
    const bool isd = valid && kv_count[base + i] == g.NT;
    const bool isl = valid && !isd;
    const uint32_t bd = __ballot_sync(0xffffffffu, isd), bl = __ballot_sync(0xffffffffu, isl);
    const uint32_t lt = (1u << lane) - 1u;
    if (isd || isl) {
      const int k = (isd ? cd : cl) + __popc((isd ? bd : bl) & lt);
      int* up = units + (size_t)((isd ? od : ol) + (k >> 2)) * kUnitInts;
      up[1 + (k & 3)] = i;
      if ((k & 3) == 0) {
        up[0] = bh;
        up[5] = up[6] = up[7] = 0;
      }
    }
    cd += __popc(bd);
    cl += __popc(bl);
  }
  if (lane == 0) {
    for (int t = cd & 3; t != 0 && t < 4; ++t) units[(size_t)(od + (cd >> 2)) * kUnitInts + 1 + t] = -1;
    for (int t = cl & 3; t != 0 && t < 4; ++t) units[(size_t)(ol + (cl >> 2)) * kUnitInts + 1 + t] = -1;
  }
}

template <int D>
cudaError_t run_attn(const Geom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const AttnArgs& a, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = g.B * g.H * units_per_bh(g.NT);
  attn_kernel<D><<<grid, kAttnThreads, Cfg<D>::kSmemBytes, s>>>(mq, mk, mv, a);
  count_launches(1);
  return cudaGetLastError();
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D map over a tile-major tensor viewed as [rows = B*H*NT*64, D] bf16; box = 64 rows x
// 64 columns (128 bytes, the 128-byte swizzle span).
bool make_map(CUtensorMap* m, const void* base, long long rows, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_sparse_attn(const Geom& g, const __nv_bfloat16* qt, const __nv_bfloat16* kt,
                               const __nv_bfloat16* vt, const uint32_t* mask, const int32_t* kv_count,
                               float scale, __nv_bfloat16* out, float* lse, uint8_t* ws, cudaStream_t s) {
  const WsLayout L = ws_layout(g);
  int* header = reinterpret_cast<int*>(ws);
  int4* bhcnt = reinterpret_cast<int4*>(ws + L.bhcnt);
  int* units = reinterpret_cast<int*>(ws + L.units);
  const int BH = g.B * g.H;

  sched_count_kernel<<<BH, 256, 0, s>>>(g, kv_count, bhcnt);
  sched_scan_kernel<<<1, 32, 0, s>>>(BH, bhcnt, header);
  sched_write_kernel<<<BH, 32, 0, s>>>(g, kv_count, bhcnt, units);
  count_launches(3);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const long long rows = (long long)g.B * g.H * g.NT * 64;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, qt, rows, g.d) || !make_map(&mk, kt, rows, g.d) || !make_map(&mv, vt, rows, g.d))
    return cudaErrorInvalidValue;
  AttnArgs a;
  a.g = g;
  a.mask = mask;
  a.units = units;
  a.header = header;
  a.out = out;
  a.lse = lse;
  a.err = reinterpret_cast<uint32_t*>(ws);
  a.scale_log2 = scale * 1.4426950408889634f;
  if (g.d == 128) return run_attn<128>(g, mq, mk, mv, a, s);
  return run_attn<64>(g, mq, mk, mv, a, s);
}

}  // namespace bsa

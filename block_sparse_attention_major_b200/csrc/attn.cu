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
// retained key tiles, in ascending order, through a K ring and a V ring of one key tile
// (64 keys) per stage. A sub-unit's blocks are the union tiles one of its two query tiles
// retains; for each it computes S = Q K^T (N=64) and O += P V, so no tensor work is spent
// on tiles that neither of its query tiles retains; a tile retained by only one of them
// gets zero probabilities in the other half of the rows.
//
// Each sub-unit has two S buffers in TMEM. S of block c+1 is computed while the softmax
// warpgroup turns S of block c into P (written as bf16 over S), so the softmax warpgroups
// run back to back while the tensor pipe runs the other products. Each sub-unit has its
// own issuing thread, which sends each product out as soon as its inputs and buffers are
// ready; the two issuers cover each other's barrier tests, during which a single issuer
// would leave the tensor pipe idle.
//
// Schedule (one launch each, on the caller's stream):
//   sched_count  per (b, h): number of dense rows (kv_count == NKT) and local rows
//   sched_scan   offsets: every dense unit of every (b, h) first, then the local units
//   sched_write  per (b, h): the units, four consecutive rows of a class each
//   attn         one CTA per unit, in list order: heavy (dense) units first, and units of
//                the same head next to each other so that their K/V tiles stay in L2.
//
// CTA roles (352 threads):
//   warps 0-3  softmax of sub-unit A: thread t owns query row t = TMEM lane t
//   warps 4-7  softmax of sub-unit B
//              (each reads S from TMEM, writes P as bf16 pairs over S, rescales its O in
//              TMEM when the running max grows, and runs the epilogue)
//   warp 8     builds the key-tile lists in shared memory, then lane 0 issues the TMA
//              loads of Q and of the K/V rings
//   warp 9     allocates TMEM; lane 0 issues S_A = Q_A K^T (SS) and O_A += P_A V (TS)
//   warp 10    lane 0 issues the products of sub-unit B
// TMEM columns: S buffers A0, A1, B0, B1 at 0, 64, 128, 192 (64 each); O_A at 256, O_B at
// 256 + D. Shared memory (1024-byte aligned): Q_A, Q_B as [D/64][128 rows][128 B], four
// K and four V stages as [D/64][64 rows][128 B], each with the 128-byte swizzle that TMA
// and tcgen05 share; barriers; the key-tile list; the per-sub-unit block lists.
#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tmem_ops.cuh"

#include <math.h>

namespace bsa {
namespace {

constexpr int kAttnThreads = 352;
constexpr int kNS = 4;                             // K and V ring stages, one key tile each
constexpr long long kWaitLimit = 4000000000LL;     // SM cycles, about 2 s
constexpr int kTmemCols = 512;
constexpr int kUnitInts = 8;                       // {bh, q0, q1, q2, q3, 0, 0, 0}

template <int D>
struct Cfg {
  static constexpr int kTileBytes = 64 * D * 2;         // one 64-token tile
  static constexpr int kQBytes = 2 * kTileBytes;        // one sub-unit's Q (128 rows)
  static constexpr int kQDB = 128 * 128;                // Q: bytes between 64-column blocks
  static constexpr int kKDB = 64 * 128;                 // K/V stage: bytes between 64-column blocks
  static constexpr int kQOff = 0;                       // Q_A, then Q_B
  static constexpr int kKOff = 2 * kQBytes;
  static constexpr int kVOff = kKOff + kNS * kTileBytes;
  static constexpr int kBarOff = kVOff + kNS * kTileBytes;
  // barriers: q, kfull[NS], kempty[NS], vfull[NS], vempty[NS], sfull[4] (sub-unit u,
  // S buffer b at 2u + b), pfull[2], odone[2], drain[2] (one per issuer)
  static constexpr int kNumBars = 1 + 4 * kNS + 4 + 2 + 2 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;   // tmem base, counts, abort, stage counters
  static constexpr int kListOff = kMiscOff + 128;
  static constexpr int kBlkOff = kListOff + kMaxTiles * 4;  // uint16 block lists of A and B
  static constexpr int kSmemBytes = 1024 + kBlkOff + 2 * kMaxTiles * 2;
  // TMEM columns: S buffer b of sub-unit u at 64 (2u + b); O of sub-unit u at 256 + u D.
  static constexpr uint32_t s_col(int u, int b) { return 64u * (2u * u + b); }
  static constexpr uint32_t o_col(int u) { return 256u + (uint32_t)(u * D); }
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

// How one key tile's 64 score columns enter this thread's row (warp-uniform): all of them
// (the row's query tile retains the tile and the tile has no padding), only the valid
// slots (a retained edge tile), or none (the tile is not retained by this row's query
// tile: its probabilities are zero). The scores themselves are never rewritten, so the
// three paths share the registers the TMEM load filled.
enum TileUse { kUseFull = 0, kUsePartial = 1, kUseSkip = 2 };

// 64 score columns as two 32-column TMEM loads (32-register destination ranges are easier
// for the register allocator to place than one 64-register range).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  tmem_ld_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_ld_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}

__device__ __forceinline__ int tile_use(uint32_t e, int mshift) {
  if (!((e >> mshift) & 1u)) return kUseSkip;
  return ((e >> 20) & 1u) ? kUseFull : kUsePartial;
}

__device__ __forceinline__ uint64_t entry_valid_mask(uint32_t e, const Geom& g) {
  int tt, ty, tx;
  tile_xyz(g, (int)(e & 0xffffu), tt, ty, tx);
  return tile_valid_mask(g, tt, ty, tx);
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

// Same over the valid slots only (bit c of `valid` set).
__device__ __forceinline__ float row_max64_valid(const uint32_t (&r)[64], uint64_t valid, float m) {
  const uint32_t lo = (uint32_t)valid, hi = (uint32_t)(valid >> 32);
  float a0 = m, a1 = -INFINITY;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    a0 = fmaxf(a0, ((lo >> c) & 1u) ? __uint_as_float(r[c]) : -INFINITY);
    a1 = fmaxf(a1, ((hi >> c) & 1u) ? __uint_as_float(r[32 + c]) : -INFINITY);
  }
  return fmaxf(a0, a1);
}

// p = 2^(s*c - m) for 64 columns (zero on slots whose bit in `valid` is clear), added to
// the fp32 row sum and stored to TMEM as bf16 pairs (column 2i in the low half of 32-bit
// column i), 16 columns per store.
template <bool kMasked>
__device__ __forceinline__ void exp_store64(const uint32_t (&r)[64], uint64_t valid, float c, float m,
                                            float& sum, uint32_t taddr) {
  const uint32_t lo = (uint32_t)valid, hi = (uint32_t)(valid >> 32);
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;       // four short chains
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const int b = 16 * k + 2 * i;
      float p0 = ex2(fmaf(__uint_as_float(r[b + 0]), c, -m));
      float p1 = ex2(fmaf(__uint_as_float(r[b + 1]), c, -m));
      float p2 = ex2(fmaf(__uint_as_float(r[b + 2]), c, -m));
      float p3 = ex2(fmaf(__uint_as_float(r[b + 3]), c, -m));
      if (kMasked) {
        const uint32_t w = b < 32 ? lo : hi;
        const int sh = b & 31;
        p0 = ((w >> sh) & 1u) ? p0 : 0.f;
        p1 = ((w >> (sh + 1)) & 1u) ? p1 : 0.f;
        p2 = ((w >> (sh + 2)) & 1u) ? p2 : 0.f;
        p3 = ((w >> (sh + 3)) & 1u) ? p3 : 0.f;
      }
      pk[i] = pack_bf16x2(p0, p1);
      pk[i + 1] = pack_bf16x2(p2, p3);
      s0 += p0;
      s1 += p1;
      s2 += p2;
      s3 += p3;
    }
    tmem_st_x8(taddr + 8 * k, pk);
  }
  sum += (s0 + s1) + (s2 + s3);
}

// Zero probabilities for a tile the row does not retain (32 TMEM columns of bf16 pairs).
__device__ __forceinline__ void store_zero_p(uint32_t taddr) {
  uint32_t z[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) z[i] = 0u;
#pragma unroll
  for (int k = 0; k < 4; ++k) tmem_st_x8(taddr + 8 * k, z);
}

// Max over one key tile's columns for this row, by its use.
__device__ __forceinline__ float tile_max(const uint32_t (&r)[64], int use, uint64_t valid, float m) {
  if (use == kUseFull) return row_max64(r, m);
  if (use == kUsePartial) return row_max64_valid(r, valid, m);
  return m;
}

// Probabilities of one key tile into TMEM, by its use.
__device__ __forceinline__ void tile_exp(const uint32_t (&r)[64], int use, uint64_t valid, float c, float m,
                                         float& sum, uint32_t taddr) {
  if (use == kUseFull) exp_store64<false>(r, 0ull, c, m, sum, taddr);
  else if (use == kUsePartial) exp_store64<true>(r, valid, c, m, sum, taddr);
  else store_zero_p(taddr);
}

// O *= alpha for this thread's row of the D accumulator columns, 32 columns per TMEM
// round trip.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t o_tmem, float alpha) {
#pragma unroll
  for (int h = 0; h < D / 32; ++h) {
    uint32_t o[32];
    tmem_ld_x32(o_tmem + 32 * h, o);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
    tmem_st_x32(o_tmem + 32 * h, o);
  }
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
  const int q0 = up[1], q1 = up[2], q2 = up[3], q3 = up[4];
  const bool bad = bh < 0 || bh >= g.B * g.H || q0 < 0 || q0 >= g.NT || q1 >= g.NT || q2 >= g.NT ||
                   q3 >= g.NT || q1 < -1 || q2 < -1 || q3 < -1;
  if (bad) {
    if (threadIdx.x == 0) report_error(a.err, BSA_KERR_BAD_UNIT);
    return;
  }
  const bool hasB = q2 >= 0;

  const uint32_t bar0 = sbase + C::kBarOff;
  const uint32_t bar_q = bar0;
  const uint32_t kfull0 = bar0 + 8, kempty0 = kfull0 + 8 * kNS, vfull0 = kempty0 + 8 * kNS,
                 vempty0 = vfull0 + 8 * kNS;
  const uint32_t sfull0 = vempty0 + 8 * kNS, pfull0 = sfull0 + 32, odone0 = pfull0 + 16,
                 bar_drain = odone0 + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  int* counts = reinterpret_cast<int*>(smem + C::kMiscOff + 4);        // L, nA, nB
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 16);
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + C::kListOff);
  uint16_t* blk = reinterpret_cast<uint16_t*>(smem + C::kBlkOff);      // [2][kMaxTiles]

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_q, 1);
    for (int s = 0; s < kNS; ++s) {
      ptx::mbar_init(kfull0 + 8 * s, 1);
      ptx::mbar_init(kempty0 + 8 * s, hasB ? 2 : 1);     // one arrival per issuer
      ptx::mbar_init(vfull0 + 8 * s, 1);
      ptx::mbar_init(vempty0 + 8 * s, hasB ? 2 : 1);
    }
    for (int s = 0; s < 4; ++s) ptx::mbar_init(sfull0 + 8 * s, 1);
    for (int u = 0; u < 2; ++u) {
      ptx::mbar_init(pfull0 + 8 * u, 128);
      ptx::mbar_init(odone0 + 8 * u, 1);
    }
    ptx::mbar_init(bar_drain, 1);
    ptx::mbar_init(bar_drain + 8, 1);
    *abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 8) {
    // Union of the four rows' key tiles, ascending; bit 16+t: retained by query tile q_t;
    // bit 20: the tile has no padding slot.
    if (lane == 0) {
      ptx::prefetch_tensormap(&tmQ);
      ptx::prefetch_tensormap(&tmK);
      ptx::prefetch_tensormap(&tmV);
    }
    const long long rbase = (long long)bh * g.NT;
    const uint32_t* m0 = a.mask + (rbase + q0) * g.NW;
    const uint32_t* m1 = a.mask + (rbase + (q1 >= 0 ? q1 : q0)) * g.NW;
    const uint32_t* m2 = a.mask + (rbase + (q2 >= 0 ? q2 : q0)) * g.NW;
    const uint32_t* m3 = a.mask + (rbase + (q3 >= 0 ? q3 : q0)) * g.NW;
    int running = 0;
    for (int w0 = 0; w0 < g.NW; w0 += 32) {
      const int w = w0 + lane;
      uint32_t b0 = 0u, b1 = 0u, b2 = 0u, b3 = 0u;
      if (w < g.NW) {
        const int rem = g.NT - 32 * w;
        const uint32_t keep = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
        b0 = __ldg(&m0[w]) & keep;
        b1 = q1 >= 0 ? (__ldg(&m1[w]) & keep) : 0u;
        b2 = q2 >= 0 ? (__ldg(&m2[w]) & keep) : 0u;
        b3 = q3 >= 0 ? (__ldg(&m3[w]) & keep) : 0u;
      }
      uint32_t u = b0 | b1 | b2 | b3;
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
        list[pos++] = (uint32_t)j | (((b0 >> bit) & 1u) << 16) | (((b1 >> bit) & 1u) << 17) |
                      (((b2 >> bit) & 1u) << 18) | (((b3 >> bit) & 1u) << 19) | (full << 20);
      }
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    // Per-sub-unit block lists: the union entries one of the sub-unit's two query tiles
    // retains, in union order (one key tile per block), each with the number of sub-units
    // that use it (bits 13-14).
    const int L = running;
    int ca = 0, cb = 0;
    for (int i0 = 0; i0 < L; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t e = i < L ? list[i] : 0u;
      const bool na = ((e >> 16) & 3u) != 0u, nb = ((e >> 18) & 3u) != 0u;
      const uint32_t ba = __ballot_sync(0xffffffffu, na), bb = __ballot_sync(0xffffffffu, nb);
      const uint32_t lt = (1u << lane) - 1u;
      const uint16_t ent = (uint16_t)(i | ((na && nb ? 2 : 1) << 13));   // entry | users << 13
      if (na) blk[ca + __popc(ba & lt)] = ent;
      if (nb) blk[kMaxTiles + cb + __popc(bb & lt)] = ent;
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
  if (L == 0 && threadIdx.x == 0) report_error(a.err, BSA_KERR_BAD_MASK);
  const long long tile_row0 = (long long)bh * g.NT;   // tile index base of this (b, h)

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && L > 0) {
      const int nsub = hasB ? 2 : 1;
      ptx::mbar_arrive_expect_tx(bar_q, nsub * C::kQBytes);
      for (int t = 0; t < 2 * nsub; ++t) {
        const int qt = t == 0 ? q0 : t == 1 ? q1 : t == 2 ? q2 : q3;
        const int tile = qt >= 0 ? qt : (t < 2 ? q0 : q2);
        const int row = (int)((tile_row0 + tile) * 64);
        const uint32_t dst = sbase + C::kQOff + (t >> 1) * C::kQBytes + (t & 1) * 8192;
#pragma unroll
        for (int db = 0; db < D / 64; ++db) ptx::tma_load_2d(dst + db * C::kQDB, &tmQ, bar_q, db * 64, row);
      }
      int nk = 0, nv = 0;       // tiles whose K / V load was issued
      for (int i = 0; i < L; ++i) {
        const int s = i % kNS;
        const uint32_t ph = ((i / kNS) & 1) ^ 1;
        const int row = (int)((tile_row0 + (int)(list[i] & 0xffffu)) * 64);
        if (!ptx::mbar_wait(kempty0 + 8 * s, ph, abort, a.err, kWaitLimit)) break;
        ptx::mbar_arrive_expect_tx(kfull0 + 8 * s, C::kTileBytes);
#pragma unroll
        for (int db = 0; db < D / 64; ++db)
          ptx::tma_load_2d(sbase + C::kKOff + s * C::kTileBytes + db * C::kKDB, &tmK, kfull0 + 8 * s, db * 64, row);
        ++nk;
        if (!ptx::mbar_wait(vempty0 + 8 * s, ph, abort, a.err, kWaitLimit)) break;
        ptx::mbar_arrive_expect_tx(vfull0 + 8 * s, C::kTileBytes);
#pragma unroll
        for (int db = 0; db < D / 64; ++db)
          ptx::tma_load_2d(sbase + C::kVOff + s * C::kTileBytes + db * C::kKDB, &tmV, vfull0 + 8 * s, db * 64, row);
        ++nv;
      }
      // Never leave with copies in flight: wait for the last load issued into each stage.
      int zero = 0;
      for (int s = 0; s < kNS; ++s) {
        if (nk > s) {
          const int last = s + kNS * ((nk - 1 - s) / kNS);
          ptx::mbar_wait(kfull0 + 8 * s, (last / kNS) & 1, &zero, a.err, kWaitLimit);
        }
        if (nv > s) {
          const int last = s + kNS * ((nv - 1 - s) / kNS);
          ptx::mbar_wait(vfull0 + 8 * s, (last / kNS) & 1, &zero, a.err, kWaitLimit);
        }
      }
      ptx::mbar_wait(bar_q, 0, &zero, a.err, kWaitLimit);
    }
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------------ MMA issuers
    // One issuing thread per sub-unit (lane 0 of warp 9 for A, of warp 10 for B). Issue is
    // throttled to the tensor pipe's pace, so a single thread leaves the pipe idle while it
    // tests barriers between products; two threads cover each other's tests.
    //
    // Each issuer walks the whole union list in order with two cursors. K cursor: for an
    // entry its sub-unit uses, S = Q K^T into the next S buffer once the K tile is in and
    // the buffer is free (the P.V two blocks back has been issued: the tensor pipe runs a
    // thread's products in issue order, so S of block c can overwrite the P of block c - 2
    // issued before it), then a commit on the stage's empty barrier; for any other entry, a
    // plain arrive there once the entry's K tile was seen loaded. V cursor: for an entry it
    // uses, O += P V once its softmax has written P and the V tile is in, then a commit on
    // the stage's empty barrier; for any other entry, a plain arrive once its V tile was
    // seen loaded. The empty barriers count one arrival per issuer, so a stage is reloaded
    // only after both issuers' products on it have completed (a commit tracks its own
    // thread's products). Because each cursor sees every load of its ring in order, the
    // full barrier is never more than one phase behind the entry tested and the parity
    // tests are exact. Nothing blocks: a wait on one cursor could hold up the other.
    static_assert(kNS == 4, "stage arithmetic below assumes four stages");
    const int u = warp - 9;
    if (lane == 0 && L > 0 && (u == 0 || hasB)) {
      constexpr uint32_t kIdQK = ptx::idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t kIdPV = ptx::idesc_bf16_f32(128, D, 0, 1);
      constexpr int kNoEntry = 1 << 20;
      const uint64_t qd = ptx::smem_desc_sw128(sbase + C::kQOff + u * C::kQBytes, 16, 1024);
      const uint64_t dK0 = ptx::smem_desc_sw128(sbase + C::kKOff, 16, 1024);
      const uint64_t dV0 = ptx::smem_desc_sw128(sbase + C::kVOff, C::kKDB, 1024);
      const uint32_t o_tmem = tmem + C::o_col(u);
      const uint32_t pfull_u = pfull0 + 8 * u, odone_u = odone0 + 8 * u;
      const int n = counts[1 + u];
      const uint16_t* my_blk = blk + u * kMaxTiles;
      int qc = 0, pc = 0, ki = 0, vi = 0;
      int qnext = n > 0 ? (int)(my_blk[0] & 0x1fffu) : kNoEntry;   // union index of the next QK block
      int pnext = qnext;                                            // and of the next P.V block
      bool ok = ptx::mbar_wait(bar_q, 0, abort, a.err, kWaitLimit);
      long long idle_since = clock64();
      while (ok && vi < L) {
        bool progress = false;
        if (ki < L) {
          const uint32_t s = ki & 3;
          if (ki == qnext) {
            if (qc - pc < 2 && ptx::mbar_test_wait(kfull0 + 8 * s, (ki >> 2) & 1)) {
              // No tcgen05 fence: K arrived through the TMA barrier, and the S buffer is
              // reused behind this thread's own P.V (ordered by the fence on that path).
              const uint32_t s_tmem = tmem + C::s_col(u, qc & 1);
              const uint64_t kd = dK0 + s * (C::kTileBytes >> 4);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk)
                ptx::mma_ss(s_tmem, qd + (((kk >> 2) * C::kQDB + (kk & 3) * 32) >> 4),
                            kd + (((kk >> 2) * C::kKDB + (kk & 3) * 32) >> 4), kIdQK, kk > 0 ? 1u : 0u);
              ptx::mma_commit(sfull0 + 8 * (2 * u + (qc & 1)));
              ptx::mma_commit(kempty0 + 8 * s);
              ++qc;
              qnext = qc < n ? (int)(my_blk[qc] & 0x1fffu) : kNoEntry;
              ++ki;
              progress = true;
            }
          } else if (ptx::mbar_test_wait(kfull0 + 8 * s, (ki >> 2) & 1)) {
            ptx::mbar_arrive(kempty0 + 8 * s);
            ++ki;
            progress = true;
          }
        }
        if (vi < ki) {
          const uint32_t s = vi & 3;
          if (vi == pnext) {
            if (ptx::mbar_test_wait(pfull_u, pc & 1) && ptx::mbar_test_wait(vfull0 + 8 * s, (vi >> 2) & 1)) {
              ptx::tc_fence_after();
              const uint32_t p_tmem = tmem + C::s_col(u, pc & 1);
              const uint64_t vd = dV0 + s * (C::kTileBytes >> 4);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                ptx::mma_ts(o_tmem, p_tmem + kk * 8, vd + kk * (2048 >> 4), kIdPV, (pc > 0 || kk > 0) ? 1u : 0u);
              ptx::mma_commit(odone_u);
              ptx::mma_commit(vempty0 + 8 * s);
              ++pc;
              pnext = pc < n ? (int)(my_blk[pc] & 0x1fffu) : kNoEntry;
              ++vi;
              progress = true;
            }
          } else if (ptx::mbar_test_wait(vfull0 + 8 * s, (vi >> 2) & 1)) {
            ptx::mbar_arrive(vempty0 + 8 * s);
            ++vi;
            progress = true;
          }
        }
        if (progress) {
          idle_since = clock64();
        } else if (*abort) {
          ok = false;
        } else if (clock64() - idle_since > kWaitLimit) {
          *abort = 1;
          report_error(a.err, BSA_KERR_WAIT_TIMEOUT);
          ok = false;
        }
      }
      // Never free TMEM under a running MMA: wait until everything issued has completed.
      int zero = 0;
      ptx::mma_commit(bar_drain + 8 * u);
      ptx::mbar_wait(bar_drain + 8 * u, 0, &zero, a.err, kWaitLimit);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int u = warp >> 2;                 // sub-unit of this warpgroup
    const int row = threadIdx.x & 127;       // TMEM lane
    const int half = row >> 6;
    const int qt = u ? (half ? q3 : q2) : (half ? q1 : q0);   // this row's query tile (-1: none)
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t o_tmem = tmem + C::o_col(u) + lane_base;
    const uint32_t pfull_u = pfull0 + 8 * u, odone_u = odone0 + 8 * u;
    const int n = counts[1 + u];
    const uint16_t* my_blk = blk + u * kMaxTiles;
    const int mshift = 16 + 2 * u + half;
    const float c = a.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = n > 0;
    for (int it = 0; it < n; ++it) {
      const int b = it & 1;
      if (!warp_wait(sfull0 + 8 * (2 * u + b), (it >> 1) & 1, abort, a.err)) { ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t e = list[my_blk[it] & 0x1fffu];
      const uint32_t s_tmem = tmem + C::s_col(u, b) + lane_base;
      const int use = tile_use(e, mshift);
      const uint64_t valid = use == kUsePartial ? entry_valid_mask(e, g) : ~0ull;
      uint32_t r[64];
      float mx = -INFINITY;
      if (use != kUseSkip) {
        tmem_ld64(s_tmem, r);
        ptx::tmem_wait_ld();
        mx = tile_max(r, use, valid, mx);
      }
      // The reference follows the running max exactly, so the row's largest probability
      // is 2^0 = 1, which bf16 holds exactly: rows dominated by one key lose nothing to
      // the bf16 rounding of P. O is rescaled in TMEM whenever the max grows.
      const float m_new = fmaxf(m_run, mx * c);
      const bool grow = m_new > m_run;
      const float alpha = grow ? ex2(m_run - m_new) : 1.0f;
      const float m_use = (m_new == -INFINITY) ? 0.0f : m_new;
      float sum = 0.f;
      tile_exp(r, use, valid, c, m_use, sum, s_tmem);
      l_run = l_run * alpha + sum;
      if (it > 0) {
        // The previous block's P.V must be complete: O is rescaled only over exactly the
        // previous blocks, and P of this block is released only after it, so that the
        // issuing thread never sees P phases two ahead of the products it has issued.
        if (!warp_wait(odone_u, (it - 1) & 1, abort, a.err)) { ok = false; break; }
        ptx::tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) rescale_o<D>(o_tmem, alpha);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(pfull_u);
      m_run = m_new;
    }
    if (ok && warp_wait(odone_u, (n - 1) & 1, abort, a.err)) {
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
      const int bb = bh / g.H, h = bh - bb * g.H;
      uint4* dst = n_tok >= 0 ? reinterpret_cast<uint4*>(a.out + (((long long)bb * g.N + n_tok) * g.H + h) * D) : nullptr;
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

// ---------------------------------------------------------------------------------------
// Fixed-scratch variant of the attention call.
//
// Some callers cannot allocate device memory at all: a plug-in loaded into a host
// application whose device memory belongs to the host's own allocator (the plug-in gets
// tensors, never an allocator), or a serving loop that forbids cudaMalloc after start-up
// because it can block and synchronise the whole device. For them the attention call's
// scratch (work-list header, per-(b, h) counts, work units) lives in the library's own
// file-scope device array below, fixed in size and held by every GPU that loads the
// library until the process exits. The caller passes only inputs and outputs.
// ---------------------------------------------------------------------------------------
#include <mutex>

namespace bsa {
namespace {

constexpr size_t kFixedScratchBytes = size_t(1) << 20;   // 1 MiB
static __device__ __align__(256) uint8_t g_fixed_scratch[kFixedScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_fixed_mu;
uint8_t* g_fixed_addr[kMaxDevices] = {};   // device address of g_fixed_scratch, per device

// The array's device address on the current device. In host code the array's name is a
// host-side stand-in, not a device address, so the first call on each device looks the
// address up (with that device current) and keeps it.
cudaError_t fixed_scratch_addr(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_fixed_mu);
  if (!g_fixed_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fixed_scratch);
    if (e != cudaSuccess) return e;
    g_fixed_addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_fixed_addr[dev];
  return cudaSuccess;
}

}  // namespace

size_t fixed_scratch_capacity() { return kFixedScratchBytes; }

// Scratch of one call: 256-byte header (error word, unit count), per-(b, h) counts, units.
size_t fixed_scratch_need(const Geom& g) {
  const size_t bh = (size_t)g.B * g.H;
  return 256 + align256(bh * sizeof(int4)) + bh * units_per_bh(g.NT) * kUnitInts * sizeof(int);
}

cudaError_t launch_sparse_attn_fixed_scratch(const Geom& g, const __nv_bfloat16* qt, const __nv_bfloat16* kt,
                                             const __nv_bfloat16* vt, const uint32_t* mask,
                                             const int32_t* kv_count, float scale, __nv_bfloat16* out,
                                             float* lse, uint32_t* errors, cudaStream_t s) {
  if (fixed_scratch_need(g) > kFixedScratchBytes) return cudaErrorInvalidValue;
  uint8_t* base = nullptr;
  cudaError_t e = fixed_scratch_addr(&base);
  if (e != cudaSuccess) return e;
  const int BH = g.B * g.H;
  int* header = reinterpret_cast<int*>(base);
  int4* bhcnt = reinterpret_cast<int4*>(base + 256);
  int* units = reinterpret_cast<int*>(base + 256 + align256((size_t)BH * sizeof(int4)));

  // The array keeps the previous call's contents: the error word and the unit count must
  // start at zero; counts and units are fully rewritten by the scheduler before use.
  e = cudaMemsetAsync(base, 0, 256, s);
  if (e != cudaSuccess) return e;
  sched_count_kernel<<<BH, 256, 0, s>>>(g, kv_count, bhcnt);
  sched_scan_kernel<<<1, 32, 0, s>>>(BH, bhcnt, header);
  sched_write_kernel<<<BH, 32, 0, s>>>(g, kv_count, bhcnt, units);
  count_launches(3);
  e = cudaGetLastError();
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
  a.err = reinterpret_cast<uint32_t*>(base);
  a.scale_log2 = scale * 1.4426950408889634f;
  e = (g.d == 128) ? run_attn<128>(g, mq, mk, mv, a, s) : run_attn<64>(g, mq, mk, mv, a, s);
  if (e != cudaSuccess) return e;
  if (errors) e = cudaMemcpyAsync(errors, base, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s);
  return e;
}

}  // namespace bsa

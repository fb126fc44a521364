// Block-sparse attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Execution of a block-sparse tile mask (Token Radius Attention summary, "Efficient
// execution"), FlashAttention-style: for every query row, an online softmax over the
// valid tokens of its retained key tiles, fp32 statistics, bf16 probabilities in the P.V
// product, fp32 accumulation, output and natural-log LSE written in raster order.
//
// Work unit: two query tiles of one (b, h) of the same route class (both dense, or both
// local), i.e. 128 query rows = one M=128 tcgen05 tile. The unit iterates over the union
// of the two rows' retained key tiles, two key tiles (128 keys) per block; a key tile
// that only one of the two query tiles retains is masked to -inf for the other one.
//
// Schedule (one launch each, on the caller's stream):
//   sched_count  per (b, h): number of dense rows (kv_count == NKT) and local rows
//   sched_scan   offsets: every dense unit of every (b, h) first, then the local units
//   sched_write  per (b, h): the units, pairing consecutive rows of each class in index
//                order (neighbouring tiles share most of their key tiles)
//   attn         one CTA per unit, in list order: heavy (dense) units first, and units of
//                the same head next to each other so that their K/V tiles stay in L2.
//
// CTA roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t = TMEM lane t; reads S from TMEM,
//              writes P (bf16 pairs) back over S, rescales O in TMEM when the running
//              max grows by more than 2^8, and runs the epilogue
//   warp 4     builds the key-tile list in shared memory, then (lane 0) issues the TMA
//              loads of Q and of the K/V ring
//   warp 5     allocates TMEM; lane 0 issues S = Q K^T (SS) and O += P V (TS) and
//              commits to the barriers
// TMEM columns: S/P buffer 0 at 0, buffer 1 at 128, O at 256 (D columns); 512 allocated.
// Shared memory (1024-byte aligned): Q [D/64][128 rows][128 B], 3 K stages and 2 V
// stages of the same shape, the key-tile list, barriers. Every buffer uses the 128-byte
// swizzle that both TMA and the tcgen05 descriptors understand.
#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tmem_ops.cuh"

#include <math.h>

namespace bsa {
namespace {

constexpr int kAttnThreads = 192;
constexpr int kNSK = 3;                   // K ring stages
constexpr int kNSV = 2;                   // V ring stages
constexpr long long kWaitLimit = 4000000000LL;   // SM cycles, about 2 s
constexpr int kTmemCols = 512;

template <int D>
struct Cfg {
  static constexpr int kTileBytes = 64 * D * 2;         // one 64-token tile
  static constexpr int kBufBytes = 2 * kTileBytes;      // two tiles (128 rows)
  static constexpr int kDBlockStride = 128 * 128;       // bytes between 64-column blocks
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kBufBytes;
  static constexpr int kVOff = kKOff + kNSK * kBufBytes;
  static constexpr int kBarOff = kVOff + kNSV * kBufBytes;
  // barriers: q, kfull[3], kempty[3], vfull[2], vempty[2], sfull[2], pfull[2], odone, drain
  static constexpr int kNumBars = 1 + 2 * kNSK + 2 * kNSV + 2 + 2 + 1 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;         // tmem base, list len, abort
  static constexpr int kListOff = kMiscOff + 64;
  static constexpr int kSmemBytes = 1024 + kListOff + kMaxTiles * 4;
};

struct AttnArgs {
  Geom g;
  const uint32_t* mask;
  const int4* units;
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

// All lanes take the same decision after a per-thread bounded wait.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          uint32_t* err) {
  const bool ok = ptx::mbar_wait(bar, parity, abort, err, kWaitLimit);
  return __all_sync(0xffffffffu, ok);
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
  const int4 unit = a.units[blockIdx.x];
  const int bh = unit.x, i0 = unit.y, i1 = unit.z;
  if (bh < 0 || bh >= g.B * g.H || i0 < 0 || i0 >= g.NT || i1 >= g.NT) {
    if (threadIdx.x == 0) report_error(a.err, BSA_KERR_BAD_UNIT);
    return;
  }

  const uint32_t bar_q = sbase + C::kBarOff;
  auto kfull = [&](int s) { return sbase + C::kBarOff + 8 * (1 + s); };
  auto kempty = [&](int s) { return sbase + C::kBarOff + 8 * (1 + kNSK + s); };
  auto vfull = [&](int s) { return sbase + C::kBarOff + 8 * (1 + 2 * kNSK + s); };
  auto vempty = [&](int s) { return sbase + C::kBarOff + 8 * (1 + 2 * kNSK + kNSV + s); };
  auto sfull = [&](int s) { return sbase + C::kBarOff + 8 * (1 + 2 * kNSK + 2 * kNSV + s); };
  auto pfull = [&](int s) { return sbase + C::kBarOff + 8 * (3 + 2 * kNSK + 2 * kNSV + s); };
  const uint32_t bar_odone = sbase + C::kBarOff + 8 * (5 + 2 * kNSK + 2 * kNSV);
  const uint32_t bar_drain = bar_odone + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  int* list_len = reinterpret_cast<int*>(smem + C::kMiscOff + 4);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 8);
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + C::kListOff);

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_q, 1);
    for (int s = 0; s < kNSK; ++s) { ptx::mbar_init(kfull(s), 1); ptx::mbar_init(kempty(s), 1); }
    for (int s = 0; s < kNSV; ++s) { ptx::mbar_init(vfull(s), 1); ptx::mbar_init(vempty(s), 1); }
    for (int s = 0; s < 2; ++s) { ptx::mbar_init(sfull(s), 1); ptx::mbar_init(pfull(s), 128); }
    ptx::mbar_init(bar_odone, 1);
    ptx::mbar_init(bar_drain, 1);
    *abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 5) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 4) {
    // Union of the two rows' key tiles, ascending; bit 16 / 17: retained by row i0 / i1.
    if (lane == 0) ptx::prefetch_tensormap(&tmQ);
    const uint32_t* m0 = a.mask + ((long long)bh * g.NT + i0) * g.NW;
    const uint32_t* m1 = a.mask + ((long long)bh * g.NT + (i1 >= 0 ? i1 : i0)) * g.NW;
    int running = 0;
    for (int w0 = 0; w0 < g.NW; w0 += 32) {
      const int w = w0 + lane;
      uint32_t b0 = 0, b1 = 0;
      if (w < g.NW) {
        const int rem = g.NT - 32 * w;
        const uint32_t keep = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
        b0 = __ldg(&m0[w]) & keep;
        b1 = (i1 >= 0) ? (__ldg(&m1[w]) & keep) : 0u;
      }
      uint32_t u = b0 | b1;
      const int cnt = __popc(u);
      int incl = cnt;
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      int pos = running + incl - cnt;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        list[pos++] = (uint32_t)(32 * w + bit) | (((b0 >> bit) & 1u) << 16) | (((b1 >> bit) & 1u) << 17);
      }
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *list_len = running;
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int L = *list_len;
  const int nblk = (L + 1) >> 1;
  if (nblk == 0 && threadIdx.x == 0) report_error(a.err, BSA_KERR_BAD_MASK);

  const long long tile_row0 = (long long)bh * g.NT;   // tile index base of this (b, h)

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && nblk > 0) {
      int last_k[kNSK], last_v[kNSV];
      for (int s = 0; s < kNSK; ++s) last_k[s] = -1;
      for (int s = 0; s < kNSV; ++s) last_v[s] = -1;
      ptx::mbar_arrive_expect_tx(bar_q, C::kBufBytes);
      for (int half = 0; half < 2; ++half) {
        const int tile = (half == 1 && i1 >= 0) ? i1 : i0;
        const int row = (int)((tile_row0 + tile) * 64);
        for (int db = 0; db < D / 64; ++db)
          ptx::tma_load_2d(sbase + C::kQOff + db * C::kDBlockStride + half * 8192, &tmQ, bar_q, db * 64, row);
      }
      for (int blk = 0; blk < nblk; ++blk) {
        const int nt = (2 * blk + 1 < L) ? 2 : 1;
        const int sk = blk % kNSK;
        if (!ptx::mbar_wait(kempty(sk), ((blk / kNSK) & 1) ^ 1, abort, a.err, kWaitLimit)) break;
        ptx::mbar_arrive_expect_tx(kfull(sk), nt * C::kTileBytes);
        for (int t = 0; t < nt; ++t) {
          const int j = (int)(list[2 * blk + t] & 0xffffu);
          const int row = (int)((tile_row0 + j) * 64);
          for (int db = 0; db < D / 64; ++db)
            ptx::tma_load_2d(sbase + C::kKOff + sk * C::kBufBytes + db * C::kDBlockStride + t * 8192, &tmK,
                             kfull(sk), db * 64, row);
        }
        last_k[sk] = blk;
        const int sv = blk % kNSV;
        if (!ptx::mbar_wait(vempty(sv), ((blk / kNSV) & 1) ^ 1, abort, a.err, kWaitLimit)) break;
        ptx::mbar_arrive_expect_tx(vfull(sv), nt * C::kTileBytes);
        for (int t = 0; t < nt; ++t) {
          const int j = (int)(list[2 * blk + t] & 0xffffu);
          const int row = (int)((tile_row0 + j) * 64);
          for (int db = 0; db < D / 64; ++db)
            ptx::tma_load_2d(sbase + C::kVOff + sv * C::kBufBytes + db * C::kDBlockStride + t * 8192, &tmV,
                             vfull(sv), db * 64, row);
        }
        last_v[sv] = blk;
      }
      // Never leave with copies in flight: wait for the last load issued into each stage.
      int zero = 0;
      for (int s = 0; s < kNSK; ++s)
        if (last_k[s] >= 0) ptx::mbar_wait(kfull(s), (last_k[s] / kNSK) & 1, &zero, a.err, kWaitLimit);
      for (int s = 0; s < kNSV; ++s)
        if (last_v[s] >= 0) ptx::mbar_wait(vfull(s), (last_v[s] / kNSV) & 1, &zero, a.err, kWaitLimit);
      ptx::mbar_wait(bar_q, 0, &zero, a.err, kWaitLimit);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && nblk > 0) {
      constexpr uint32_t kIdQK2 = ptx::idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t kIdQK1 = ptx::idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t kIdPV = ptx::idesc_bf16_f32(128, D, 0, 1);
      const uint32_t o_tmem = tmem + 256;
      if (ptx::mbar_wait(bar_q, 0, abort, a.err, kWaitLimit)) {
        for (int blk = 0; blk <= nblk; ++blk) {
          if (blk < nblk) {
            const int sk = blk % kNSK;
            const int nt = (2 * blk + 1 < L) ? 2 : 1;
            if (!ptx::mbar_wait(kfull(sk), (blk / kNSK) & 1, abort, a.err, kWaitLimit)) break;
            ptx::tc_fence_after();
            const uint32_t s_tmem = tmem + (blk & 1) * 128;
            const uint32_t kaddr = sbase + C::kKOff + sk * C::kBufBytes;
            const uint32_t qaddr = sbase + C::kQOff;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::kDBlockStride + (kk & 3) * 32;
              const uint64_t ad = ptx::smem_desc_sw128(qaddr + off, 16, 1024);
              const uint64_t bd = ptx::smem_desc_sw128(kaddr + off, 16, 1024);
              ptx::mma_ss(s_tmem, ad, bd, nt == 2 ? kIdQK2 : kIdQK1, kk > 0 ? 1u : 0u);
            }
            ptx::mma_commit(kempty(sk));
            ptx::mma_commit(sfull(blk & 1));
          }
          if (blk > 0) {
            const int j = blk - 1;
            const int sv = j % kNSV;
            const int nt = (2 * j + 1 < L) ? 2 : 1;
            if (!ptx::mbar_wait(pfull(j & 1), (j >> 1) & 1, abort, a.err, kWaitLimit)) break;
            if (!ptx::mbar_wait(vfull(sv), (j / kNSV) & 1, abort, a.err, kWaitLimit)) break;
            ptx::tc_fence_after();
            const uint32_t p_tmem = tmem + (j & 1) * 128;
            const uint32_t vaddr = sbase + C::kVOff + sv * C::kBufBytes;
            for (int kk = 0; kk < nt * 4; ++kk) {
              const uint64_t bd = ptx::smem_desc_sw128(vaddr + kk * 2048, C::kDBlockStride, 1024);
              ptx::mma_ts(o_tmem, p_tmem + kk * 8, bd, kIdPV, (j > 0 || kk > 0) ? 1u : 0u);
            }
            ptx::mma_commit(vempty(sv));
            ptx::mma_commit(bar_odone);
          }
        }
      }
      // Never free TMEM under a running MMA: wait until everything issued has completed.
      int zero = 0;
      ptx::mma_commit(bar_drain);
      ptx::mbar_wait(bar_drain, 0, &zero, a.err, kWaitLimit);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int row = threadIdx.x;            // 0..127 = TMEM lane
    const int half = row >> 6;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t o_tmem = tmem + 256 + lane_base;
    float m_run = -INFINITY, l_run = 0.f, lr_run = 0.f;
    bool ok = nblk > 0;
    for (int blk = 0; blk < nblk && ok; ++blk) {
      if (!warp_wait(sfull(blk & 1), (blk >> 1) & 1, abort, a.err)) { ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t s_tmem = tmem + (blk & 1) * 128 + lane_base;
      uint32_t sraw[128];
      tmem_ld_x64(s_tmem, *reinterpret_cast<uint32_t(*)[64]>(&sraw[0]));
      tmem_ld_x64(s_tmem + 64, *reinterpret_cast<uint32_t(*)[64]>(&sraw[64]));
      ptx::tmem_wait_ld();

      const bool has1 = 2 * blk + 1 < L;
      const uint32_t e0 = list[2 * blk];
      const uint32_t e1 = has1 ? list[2 * blk + 1] : 0u;
      uint64_t vm0 = 0, vm1 = 0;
      if ((e0 >> (16 + half)) & 1u) {
        int tt, ty, tx;
        tile_xyz(g, (int)(e0 & 0xffffu), tt, ty, tx);
        vm0 = tile_valid_mask(g, tt, ty, tx);
      }
      if (has1 && ((e1 >> (16 + half)) & 1u)) {
        int tt, ty, tx;
        tile_xyz(g, (int)(e1 & 0xffffu), tt, ty, tx);
        vm1 = tile_valid_mask(g, tt, ty, tx);
      }
      float x[128];
      float bmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        x[c] = ((vm0 >> c) & 1ull) ? __uint_as_float(sraw[c]) * a.scale_log2 : -INFINITY;
        x[64 + c] = ((vm1 >> c) & 1ull) ? __uint_as_float(sraw[64 + c]) * a.scale_log2 : -INFINITY;
        bmax = fmaxf(bmax, fmaxf(x[c], x[64 + c]));
      }
      const float m_new = fmaxf(m_run, bmax);
      const bool grow = m_new > m_run + 8.0f;          // rescale only on a large jump
      const float m_ref = grow ? m_new : m_run;
      const float alpha = grow ? exp2f(m_run - m_new) : 1.0f;
      const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
      // l_run sums the fp32 probabilities (for the LSE); lr_run sums the bf16-rounded
      // ones that enter P.V, so that O is normalised by exactly the weights it used.
      float sum = 0.f, sum_r = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = exp2f(x[2 * c] - m_use);
        const float p1 = exp2f(x[2 * c + 1] - m_use);
        sum += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
        sum_r += __uint_as_float(pk[c] << 16) + __uint_as_float(pk[c] & 0xffff0000u);
      }
      l_run = l_run * alpha + sum;
      lr_run = lr_run * alpha + sum_r;
      if (has1) {
        tmem_st_x64(s_tmem, pk);
      } else {
        tmem_st_x32(s_tmem, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      }
      if (blk > 0) {
        // O must hold exactly blocks 0..blk-1 before it is rescaled.
        if (!warp_wait(bar_odone, (blk - 1) & 1, abort, a.err)) { ok = false; break; }
        ptx::tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t ov[32];
            tmem_ld_x32(o_tmem + ch * 32, ov);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
            tmem_st_x32(o_tmem + ch * 32, ov);
          }
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(pfull(blk & 1));
      m_run = m_ref;
    }
    if (ok) {
      if (warp_wait(bar_odone, (nblk - 1) & 1, abort, a.err)) {
        ptx::tc_fence_after();
        const int tile = half ? i1 : i0;
        const int r = row & 63;
        int n = -1;
        if (tile >= 0) {
          int tt, ty, tx;
          tile_xyz(g, tile, tt, ty, tx);
          const int t = tt * 4 + (r >> 4), y = ty * 4 + ((r >> 2) & 3), xx = tx * 4 + (r & 3);
          if (t < g.T && y < g.Hs && xx < g.Ws) n = (t * g.Hs + y) * g.Ws + xx;
        }
        const float inv_l = lr_run > 0.f ? 1.0f / lr_run : 0.f;
        const int b = bh / g.H, h = bh - (bh / g.H) * g.H;
        uint4* dst = n >= 0 ? reinterpret_cast<uint4*>(a.out + (((long long)b * g.N + n) * g.H + h) * D) : nullptr;
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t ov[32];
          tmem_ld_x32(o_tmem + ch * 32, ov);
          ptx::tmem_wait_ld();
          if (dst) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(ov[8 * q + 0]) * inv_l, __uint_as_float(ov[8 * q + 1]) * inv_l);
              v.y = pack_bf16x2(__uint_as_float(ov[8 * q + 2]) * inv_l, __uint_as_float(ov[8 * q + 3]) * inv_l);
              v.z = pack_bf16x2(__uint_as_float(ov[8 * q + 4]) * inv_l, __uint_as_float(ov[8 * q + 5]) * inv_l);
              v.w = pack_bf16x2(__uint_as_float(ov[8 * q + 6]) * inv_l, __uint_as_float(ov[8 * q + 7]) * inv_l);
              dst[ch * 4 + q] = v;
            }
          }
        }
        if (n >= 0) {
          if (!(l_run > 0.f)) report_error(a.err, BSA_KERR_BAD_MASK);
          if (a.lse) {
            const float m_use = (m_run == -INFINITY) ? 0.0f : m_run;
            a.lse[(long long)bh * g.N + n] = l_run > 0.f ? (m_use + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
          }
        }
      }
    }
  }

  // ---------------------------------------------------------------------- teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
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
    bhcnt[blockIdx.x] = make_int4(s_nd, nl, (s_nd + 1) / 2, (nl + 1) / 2);
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
// class becomes the first tile (k even) or the second tile (k odd) of unit k/2 of that
// class; a class with an odd count ends with a single-tile unit (second tile -1).
__global__ void __launch_bounds__(32) sched_write_kernel(Geom g, const int32_t* __restrict__ kv_count,
                                                         const int4* __restrict__ bhcnt,
                                                         int4* __restrict__ units) {
  const int bh = blockIdx.x, lane = threadIdx.x;
  const long long base = (long long)bh * g.NT;
  const int od = bhcnt[bh].x, ol = bhcnt[bh].y;
  int* u = reinterpret_cast<int*>(units);
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
      const int slot = (isd ? od : ol) + (k >> 1);
      if (k & 1) {
        u[4 * slot + 2] = i;
      } else {
        u[4 * slot + 0] = bh;
        u[4 * slot + 1] = i;
        u[4 * slot + 3] = 0;
      }
    }
    cd += __popc(bd);
    cl += __popc(bl);
  }
  if (lane == 0) {
    if (cd & 1) u[4 * (od + (cd >> 1)) + 2] = -1;
    if (cl & 1) u[4 * (ol + (cl >> 1)) + 2] = -1;
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
  int4* units = reinterpret_cast<int4*>(ws + L.units);
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

// Block-sparse attention forward for sm_100a (tcgen05 + TMEM + TMA), persistent.
//
// Execution of a block-sparse tile mask (Token Radius Attention summary, "Efficient
// execution"), FlashAttention-style: for every query row, an online softmax over the
// valid tokens of its retained key tiles, fp32 statistics, bf16 probabilities in the P.V
// product, fp32 accumulation, output and natural-log LSE written in raster order.
//
// Work unit: up to four query tiles of one (b, h) and of the same route class (all
// dense, or all local), consecutive in tile order. They form two query blocks of two
// tiles, A and B, each one M=128 tcgen05 tile. The unit's key stream is the union of the
// four rows' retained key tiles, ascending, one tile (64 keys) per stream block, through a
// K ring and a V ring of four stages. For each tile a query block uses (either of its two
// query tiles retains it) it computes S = Q K^T (N = 64) and O += P V; a tile retained by
// only one of the block's two query tiles gets zero probabilities in the other query
// tile's rows. Each query block has two S buffers, so the Q K^T of its next tile runs
// while its softmax works on the current one.
//
// Persistent grid: one CTA per SM takes units from a device work list through an atomic
// counter. The list (built by the scheduler kernels below) is ordered head by head, and
// within a head by decreasing cost (longest processing time first), so that the heads'
// K/V tiles stay in L2 while their units run and the last units of the launch are the
// cheapest. Units flow through the CTA without a barrier between them: the K/V ring, the
// Q buffers and the TMEM accumulators pass from one unit to the next through the same
// mbarriers that order the work inside a unit.
//
// CTA roles (384 threads, three warpgroups):
//   warps 0-3  softmax of query block A: thread t owns query row t = TMEM lane t
//   warps 4-7  softmax of query block B
//              (each reads S from TMEM, writes P as bf16 pairs over S, rescales its O in
//              TMEM when a row maximum grows by more than 2^8, and runs the epilogue)
//   warp 8     lane 0 issues the TMA loads of Q and of the K ring, lane 1 those of the V
//              ring (neither ring waits behind the other)
//   warp 9     allocates TMEM; lane 0 issues every tcgen05.mma of query block A
//   warp 10    takes the next unit from the work list and builds its key stream in shared
//              memory (double buffered, one unit ahead)
//   warp 11    lane 0 issues every tcgen05.mma of query block B
// The softmax warpgroups raise their register budget to 184 and the third lowers its own to
// 136 (setmaxnreg).
// TMEM columns: S buffer b of query block x at 64 (2x + b) (64 each; P is written over S as
// bf16 pairs, key k of the tile at column k/2), O_A at 256, O_B at 256 + D. Shared memory
// (1024-byte aligned): Q_A, Q_B as [D/64 column blocks][128 rows][128 B], four K and four V
// stages as [D/64][64 rows][128 B], each with the 128-byte swizzle that TMA and tcgen05
// share; two key-stream buffers; barriers.
//
// Softmax numerics. Scores are scaled by softmax_scale * log2(e) with one FFMA and
// exponentiated with ex2.approx. A row keeps a reference maximum m and is rescaled only
// when a block's maximum exceeds m by more than 8 (then, after the previous block's P.V has
// completed, O and the row sums are multiplied by 2^(m - m_new)); otherwise probabilities up to
// 2^8 enter P. O is normalised by the sum of the bf16-rounded probabilities that entered
// P.V (so a row dominated by one key returns that key's value exactly); the LSE uses the
// fp32 sum of the unrounded probabilities.
//
// Token-level support (window kind 2, Token Radius Attention summary: query-centred
// circular neighbourhoods): when a radius in tokens is given, the key-stream builder marks,
// per query tile of a local row, the window tiles that the support of some of the tile's
// tokens does not cover whole; the softmax masks those tiles' slots token by token (the
// support of this row's token), and treats every other retained tile as a whole tile.
#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tmem_ops.cuh"
#include "window.cuh"

#include <math.h>

namespace bsa {
namespace {

constexpr int kAttnThreads = 384;
constexpr int kRegsLaunch = 168;                   // 65536 / (3 warps per SM sub-partition x 32 x 4), rounded to 8
constexpr int kRegsSoftmax = 184;
constexpr int kRegsControl = 136;
static_assert(128 * (2 * kRegsSoftmax + kRegsControl) <= kAttnThreads * kRegsLaunch,
              "register split above the launch's pool");
constexpr int kNS = 4;                             // K and V ring stages, one key tile each
constexpr long long kWaitLimit = 4000000000LL;     // SM cycles, about 2 s
constexpr int kTmemCols = 512;
constexpr int kUnitInts = 8;                       // {bh, q0, q1, q2, q3, cost, 0, 0}
constexpr float kRescaleLog2 = 8.0f;               // O is rescaled only past 2^8 of growth
constexpr unsigned kIssuerSleepNs = 2000;          // longest suspension of an idle issuer

template <int D>
struct Cfg {
  static constexpr int kTileBytes = 64 * D * 2;         // one 64-token tile (a K or V stage)
  static constexpr int kQBytes = 2 * kTileBytes;        // one query block (128 rows)
  static constexpr int kQCB = 128 * 128;                // Q: bytes between 64-column blocks
  static constexpr int kKCB = 64 * 128;                 // K/V stage: bytes between 64-column blocks
  static constexpr int kHalf = 64 * 128;                // rows 64-127 of a query block start here
  static constexpr int kQOff = 0;                       // Q_A, then Q_B
  static constexpr int kKOff = 2 * kQBytes;
  static constexpr int kVOff = kKOff + kNS * kTileBytes;
  static constexpr int kListOff = kVOff + kNS * kTileBytes;
  // key-stream buffer: meta (8 ints: bh or -1, q0..q3, L), tile ids (u16), flags (u16:
  // bit t = query tile t retains the tile, bit 4 = the tile has no padding slot, bit 5 + t
  // = query tile t sees the tile through its tokens' support)
  static constexpr int kListMeta = 32;
  static constexpr int kListBytes = kListMeta + kMaxTiles * 2 + kMaxTiles * 2;
  static constexpr int kBarOff = kListOff + 2 * kListBytes;
  // kfull, kempty, vfull, vempty [kNS each]; qfull, qempty [2 each]; sfull, pfull, odone
  // [query block][S buffer]; lfull, lempty [2 each]; drain [one per issuer]
  static constexpr int kNumBars = 4 * kNS + 2 * 2 + 3 * 4 + 2 * 2 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;   // tmem base, abort
  static constexpr int kSmemBytes = 1024 + kMiscOff + 64;
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct AttnArgs {
  Geom g;
  const uint32_t* mask;
  const int* units;          // kUnitInts per unit
  int* header;               // header[1] = number of units, header[2] = next unit counter
  __nv_bfloat16* out;
  float* lse;
  uint32_t* err;
  float scale_log2;          // softmax scale * log2(e)
  // Token-level support: radius in tokens, or -1 for none; local rows (dense[b * NT + i]
  // == 0) see the tiles of their token window token by token.
  const uint8_t* dense;
  int token_rho;
};

struct Bars {
  uint32_t b0;
  __device__ uint32_t kfull(int s) const { return b0 + 8 * s; }
  __device__ uint32_t kempty(int s) const { return b0 + 8 * (kNS + s); }
  __device__ uint32_t vfull(int s) const { return b0 + 8 * (2 * kNS + s); }
  __device__ uint32_t vempty(int s) const { return b0 + 8 * (3 * kNS + s); }
  __device__ uint32_t qfull(int x) const { return b0 + 8 * (4 * kNS + x); }
  __device__ uint32_t qempty(int x) const { return b0 + 8 * (4 * kNS + 2 + x); }
  __device__ uint32_t sfull(int x, int b) const { return b0 + 8 * (4 * kNS + 4 + 2 * x + b); }
  __device__ uint32_t pfull(int x, int b) const { return b0 + 8 * (4 * kNS + 8 + 2 * x + b); }
  __device__ uint32_t odone(int x, int b) const { return b0 + 8 * (4 * kNS + 12 + 2 * x + b); }
  __device__ uint32_t lfull(int b) const { return b0 + 8 * (4 * kNS + 16 + b); }
  __device__ uint32_t lempty(int b) const { return b0 + 8 * (4 * kNS + 18 + b); }
  __device__ uint32_t drain(int x) const { return b0 + 8 * (4 * kNS + 20 + x); }
};

// lempty arrivals per key-stream buffer: the two TMA producers, the two issuers and
// the eight softmax warps.
constexpr int kListConsumers = 2 + 2 + 8;

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
// (the row's query tile retains the tile and the tile has no padding), only some slots (a
// retained edge tile: its valid slots; a tile seen through the token support: its valid
// slots in this row's support), or none (this row's query tile does not retain the tile:
// its probabilities are zero).
enum TileUse { kUseFull = 0, kUsePartial = 1, kUseSkip = 2 };

__device__ __forceinline__ int tile_use(uint32_t flags, int t) {
  if (!((flags >> t) & 1u)) return kUseSkip;
  return (((flags >> 4) & 1u) && !((flags >> (5 + t)) & 1u)) ? kUseFull : kUsePartial;
}

// Slots of key tile j that this row's scores may use: the valid slots, and under the token
// support (flag bit 5 + t) only those in the support of the row's token (tq, yq, xq).
__device__ __forceinline__ uint64_t tile_slots(int j, uint32_t flags, int t, const Geom& g, int tq, int yq,
                                               int xq, int rho) {
  int tt, ty, tx;
  tile_xyz(g, j, tt, ty, tx);
  uint64_t m = tile_valid_mask(g, tt, ty, tx);
  if ((flags >> (5 + t)) & 1u) m &= token_support_slots(tq, yq, xq, tt, ty, tx, rho);
  return m;
}

// Row maximum over 64 score columns (four short chains).
__device__ __forceinline__ float half_max_full(const uint32_t (&r)[64], float m) {
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

// Same over the slots whose bit in `valid` is set.
__device__ __forceinline__ float half_max_valid(const uint32_t (&r)[64], uint64_t valid, float m) {
  const uint32_t lo = (uint32_t)valid, hi = (uint32_t)(valid >> 32);
  float a0 = m, a1 = -INFINITY;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    a0 = fmaxf(a0, ((lo >> c) & 1u) ? __uint_as_float(r[c]) : -INFINITY);
    a1 = fmaxf(a1, ((hi >> c) & 1u) ? __uint_as_float(r[32 + c]) : -INFINITY);
  }
  return fmaxf(a0, a1);
}

__device__ __forceinline__ float half_max(const uint32_t (&r)[64], int use, uint64_t valid, float m) {
  if (use == kUseFull) return half_max_full(r, m);
  if (use == kUsePartial) return half_max_valid(r, valid, m);
  return m;
}

// Packed pairs of fp32 (sm_100a f32x2 instructions: one instruction, two lanes of work).
__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void uf2(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// p = 2^(s*c - m) for 64 score columns (zero on slots whose bit in `valid` is clear),
// stored to TMEM as bf16 pairs (column 2i in the low half of 32-bit column i), 16 columns
// per store. `sum` gets the fp32 probabilities, `sum_bf` the bf16-rounded ones that P.V
// uses (widened from the packed pairs). The scaling and the sums run as packed f32x2
// instructions: the softmax is bound by instruction issue, not by the exponentials.
template <bool kMasked>
__device__ __forceinline__ void exp_half(const uint32_t (&r)[64], uint64_t valid, float c, float m,
                                         float& sum, float& sum_bf, uint32_t taddr) {
  const uint32_t lo = (uint32_t)valid, hi = (uint32_t)(valid >> 32);
  const uint64_t cc = f2(c, c), mm = f2(-m, -m);
  uint64_t ex0 = f2(0.f, 0.f), ex1 = ex0, bf0 = ex0, bf1 = ex0;   // two chains each
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int b = 16 * k + 2 * i;
      float x0, x1;
      uf2(ffma2(f2(__uint_as_float(r[b]), __uint_as_float(r[b + 1])), cc, mm), x0, x1);
      float p0 = ex2(x0), p1 = ex2(x1);
      if (kMasked) {
        const uint32_t w = b < 32 ? lo : hi;
        const int sh = b & 31;
        p0 = ((w >> sh) & 1u) ? p0 : 0.f;
        p1 = ((w >> (sh + 1)) & 1u) ? p1 : 0.f;
      }
      pk[i] = pack_bf16x2(p0, p1);
      const uint64_t pe = f2(p0, p1);
      const uint64_t pb = f2(__uint_as_float(pk[i] << 16), __uint_as_float(pk[i] & 0xffff0000u));
      if (i & 1) {
        ex1 = fadd2(ex1, pe);
        bf1 = fadd2(bf1, pb);
      } else {
        ex0 = fadd2(ex0, pe);
        bf0 = fadd2(bf0, pb);
      }
    }
    tmem_st_x8(taddr + 8 * k, pk);
  }
  float a0, a1, a2, a3;
  uf2(fadd2(ex0, ex1), a0, a1);
  sum += a0 + a1;
  uf2(fadd2(bf0, bf1), a2, a3);
  sum_bf += a2 + a3;
}

// Zero probabilities for a tile the row does not retain (32 TMEM columns of bf16 pairs).
__device__ __forceinline__ void store_zero_p(uint32_t taddr) {
  uint32_t z[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) z[i] = 0u;
#pragma unroll
  for (int k = 0; k < 4; ++k) tmem_st_x8(taddr + 8 * k, z);
}

__device__ __forceinline__ void half_exp(const uint32_t (&r)[64], int use, uint64_t valid, float c, float m,
                                         float& sum, float& sum_bf, uint32_t taddr) {
  if (use == kUseFull) exp_half<false>(r, 0ull, c, m, sum, sum_bf, taddr);
  else if (use == kUsePartial) exp_half<true>(r, valid, c, m, sum, sum_bf, taddr);
  else store_zero_p(taddr);
}

// 64 score columns from TMEM (two 32-column loads) and the wait for them.
__device__ __forceinline__ void load_half(uint32_t taddr, uint32_t (&r)[64]) {
  tmem_ld_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_ld_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
  ptx::tmem_wait_ld();
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
  const Bars bar{sbase + C::kBarOff};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS; ++s) {
      ptx::mbar_init(bar.kfull(s), 1);
      ptx::mbar_init(bar.kempty(s), 2);   // one release per issuer
      ptx::mbar_init(bar.vfull(s), 1);
      ptx::mbar_init(bar.vempty(s), 2);
    }
    for (int x = 0; x < 2; ++x) {
      ptx::mbar_init(bar.qfull(x), 1);
      ptx::mbar_init(bar.qempty(x), 1);
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(bar.sfull(x, b), 1);
        ptx::mbar_init(bar.pfull(x, b), 4);   // one arrival per softmax warp
        ptx::mbar_init(bar.odone(x, b), 1);
      }
      ptx::mbar_init(bar.lfull(x), 1);
      ptx::mbar_init(bar.lempty(x), kListConsumers);
    }
    ptx::mbar_init(bar.drain(0), 1);
    ptx::mbar_init(bar.drain(1), 1);
    *abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
  ptx::setmaxnreg_dec<kRegsControl>();
  if (warp == 10) {
    // ------------------------------------------------------------ key-stream builder
    const int nunits = a.header[1];
    for (int it = 0;; ++it) {
      const int buf = it & 1;
      uint8_t* lb = smem + C::kListOff + buf * C::kListBytes;
      int* meta = reinterpret_cast<int*>(lb);
      uint16_t* tiles = reinterpret_cast<uint16_t*>(lb + C::kListMeta);
      uint16_t* flags = reinterpret_cast<uint16_t*>(lb + C::kListMeta + kMaxTiles * 2);
      if (it >= 2 && !warp_wait(bar.lempty(buf), ((it >> 1) - 1) & 1, abort, a.err)) break;
      int bh = -1, q0 = -1, q1 = -1, q2 = -1, q3 = -1;
      while (true) {
        int idx = 0;
        if (lane == 0) idx = atomicAdd(&a.header[2], 1);
        idx = __shfl_sync(0xffffffffu, idx, 0);
        if (idx >= nunits) {
          bh = -1;
          break;
        }
        const int* up = a.units + (size_t)idx * kUnitInts;
        bh = up[0];
        q0 = up[1], q1 = up[2], q2 = up[3], q3 = up[4];
        const bool bad = bh < 0 || bh >= g.B * g.H || q0 < 0 || q0 >= g.NT || q1 >= g.NT || q2 >= g.NT ||
                         q3 >= g.NT || q1 < -1 || q2 < -1 || q3 < -1;
        if (!bad) break;
        if (lane == 0) report_error(a.err, BSA_KERR_BAD_UNIT);
      }
      if (bh < 0) {
        if (lane == 0) {
          meta[0] = -1;
          ptx::mbar_arrive(bar.lfull(buf));
        }
        break;
      }
      // Union of the four rows' key tiles, ascending, with the retaining query tiles.
      const long long rbase = (long long)bh * g.NT;
      const uint32_t* m0 = a.mask + (rbase + q0) * g.NW;
      const uint32_t* m1 = a.mask + (rbase + (q1 >= 0 ? q1 : q0)) * g.NW;
      const uint32_t* m2 = a.mask + (rbase + (q2 >= 0 ? q2 : q0)) * g.NW;
      const uint32_t* m3 = a.mask + (rbase + (q3 >= 0 ? q3 : q0)) * g.NW;
      // token support: coordinates of the query tiles, and which of them are local rows
      const int rho = a.token_rho;
      uint32_t cq[4];
      bool loc[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int qtile = t == 0 ? q0 : t == 1 ? q1 : t == 2 ? q2 : q3;
        int tt, ty, tx;
        tile_xyz(g, qtile >= 0 ? qtile : q0, tt, ty, tx);
        cq[t] = pack_coord(tt, ty, tx);
        loc[t] = rho >= 0 && qtile >= 0 && a.dense[(long long)(bh / g.H) * g.NT + qtile] == 0;
      }
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
          const uint32_t kept = ((b0 >> bit) & 1u) | (((b1 >> bit) & 1u) << 1) | (((b2 >> bit) & 1u) << 2) |
                                (((b3 >> bit) & 1u) << 3);
          uint32_t tok = 0u;
          if (rho >= 0) {
            const uint32_t cj = pack_coord(tt, ty, tx);
#pragma unroll
            for (int t = 0; t < 4; ++t)
              if (loc[t] && ((kept >> t) & 1u) && in_token_window(cq[t], cj, rho) &&
                  !token_tiles_all_inside(cq[t], cj, g.T, g.Hs, g.Ws, rho))
                tok |= 1u << t;
          }
          tiles[pos] = (uint16_t)j;
          flags[pos] = (uint16_t)(kept | (full << 4) | (tok << 5));
          ++pos;
        }
        running += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) {
        meta[0] = bh;
        meta[1] = q0;
        meta[2] = q1;
        meta[3] = q2;
        meta[4] = q3;
        meta[5] = running;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar.lfull(buf));
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------------ TMA producers
    // Lane 0 of warp 8 loads Q and the K ring, lane 1 the V ring, so that a K stage never
    // waits behind a V stage (or the reverse).
    const bool vprod = lane == 1;
    if (lane <= 1) {
      ptx::prefetch_tensormap(&tmQ);
      ptx::prefetch_tensormap(&tmK);
      ptx::prefetch_tensormap(&tmV);
      int qn[2] = {0, 0};       // Q loads issued per query block
      uint32_t nk = 0, nv = 0;  // stream blocks whose K / V load was issued (only the low bits matter)
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int buf = it & 1;
        const uint8_t* lb = smem + C::kListOff + buf * C::kListBytes;
        const int* meta = reinterpret_cast<const int*>(lb);
        const uint16_t* tiles = reinterpret_cast<const uint16_t*>(lb + C::kListMeta);
        if (!ptx::mbar_wait(bar.lfull(buf), (it >> 1) & 1, abort, a.err, kWaitLimit)) break;
        const int bh = meta[0];
        if (bh < 0) break;
        const int q[4] = {meta[1], meta[2], meta[3], meta[4]};
        const int L = meta[5];
        const long long tile_row0 = (long long)bh * g.NT;
        for (int x = 0; x < 2 && ok && !vprod; ++x) {
          if (q[2 * x] < 0) continue;
          if (qn[x] > 0 && !ptx::mbar_wait(bar.qempty(x), (qn[x] - 1) & 1, abort, a.err, kWaitLimit)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(bar.qfull(x), C::kQBytes);
          for (int rh = 0; rh < 2; ++rh) {
            const int tile = q[2 * x + rh] >= 0 ? q[2 * x + rh] : q[2 * x];   // a missing tile repeats the first
            const int row = (int)((tile_row0 + tile) * 64);
            const uint32_t dst = sbase + C::kQOff + x * C::kQBytes + rh * C::kHalf;
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) ptx::tma_load_2d(dst + cb * C::kQCB, &tmQ, bar.qfull(x), cb * 64, row);
          }
          ++qn[x];
        }
        for (int c = 0; c < L && ok; ++c) {
          const int row = (int)((tile_row0 + tiles[c]) * 64);
          uint32_t& n = vprod ? nv : nk;
          const int s = (int)(n % kNS);
          const uint32_t ph = ((n / kNS) & 1) ^ 1;
          const uint32_t empty = vprod ? bar.vempty(s) : bar.kempty(s);
          const uint32_t full = vprod ? bar.vfull(s) : bar.kfull(s);
          if (!ptx::mbar_wait(empty, ph, abort, a.err, kWaitLimit)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(full, C::kTileBytes);
          const uint32_t dst = sbase + (vprod ? C::kVOff : C::kKOff) + s * C::kTileBytes;
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) ptx::tma_load_2d(dst + cb * C::kKCB, vprod ? &tmV : &tmK, full, cb * 64, row);
          ++n;
        }
        if (ok) ptx::mbar_arrive(bar.lempty(buf));
      }
      // Never leave with copies in flight: wait for the last load issued into each buffer.
      int zero = 0;
      for (int s = 0; s < kNS; ++s) {
        if (nk > s) {
          const uint32_t last = s + kNS * ((nk - 1 - s) / kNS);
          ptx::mbar_wait(bar.kfull(s), (uint32_t)((last / kNS) & 1), &zero, a.err, kWaitLimit);
        }
        if (nv > s) {
          const uint32_t last = s + kNS * ((nv - 1 - s) / kNS);
          ptx::mbar_wait(bar.vfull(s), (uint32_t)((last / kNS) & 1), &zero, a.err, kWaitLimit);
        }
      }
      for (int x = 0; x < 2; ++x)
        if (qn[x] > 0) ptx::mbar_wait(bar.qfull(x), (qn[x] - 1) & 1, &zero, a.err, kWaitLimit);
    }
  } else if (warp == 9 || warp == 11) {
    // ------------------------------------------------------------------ MMA issuers
    // Lane 0 of warp 9 issues every product of query block A, lane 0 of warp 11 those of
    // B: each MMA issue waits for the tensor pipe to take it, so one thread for both query
    // blocks could not keep the pipe fed. Each issuer's cursor walks the units' key streams
    // in order with a K position and a V position; each query block has two S buffers in
    // TMEM. At its K position a cursor issues S = Q K^T (N = 64) for a tile its query
    // block uses into the next S buffer, once the K stage is in and that buffer is free:
    // the P.V of the block two back has been issued (the tensor pipe runs one thread's
    // products in issue order, so S may overwrite that P). At its V position it issues
    // O += P V for the oldest block whose P.V is pending, once its softmax has released P
    // and the V stage is in. A tile the query block does not use is passed once its stage
    // is seen loaded. Each issuer releases each stage once (a commit after its product on
    // it, or an arrive when it passed the tile); a stage is reloaded after both releases,
    // and a commit tracks its own thread's products. Each cursor sees every load of the
    // ring in order, so a full barrier is never more than one phase behind the tile tested
    // and the parity tests are exact. The cursor takes its V position before its K
    // position, so that a query block's P.V and its next Q K^T go to the pipe back to back.
    const int x = warp == 9 ? 0 : 1;           // query block of this issuer
    if (lane == 0) {
      constexpr uint32_t kIdQK = ptx::idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t kIdPV = ptx::idesc_bf16_f32(128, D, 0, 1);
      struct Cursor {
        int it;            // key-stream buffer iteration
        bool have, done;
        int L, kc, vc;     // unit's stream length; next K and V positions
        bool hasq, qready, qreleased, first_pv;
        uint32_t gbase;    // index of the unit's first stream tile in this CTA's stream
        int qn;            // Q loads consumed (units with this query block)
        uint32_t qk, pv;   // Q K^T and P.V products issued (all units)
        int ent0, ent1;    // stream positions of the blocks whose P.V is pending, by S buffer
        const uint16_t* flags;
      };
      Cursor cu;
      cu.it = 0;
      cu.have = cu.done = false;
      cu.L = cu.kc = cu.vc = 0;
      cu.hasq = cu.qready = cu.qreleased = cu.first_pv = false;
      cu.gbase = 0;
      cu.qn = 0;
      cu.qk = cu.pv = 0;
      cu.ent0 = cu.ent1 = -1;
      cu.flags = nullptr;
      bool ok = true;
      long long idle_since = clock64();
      while (ok && !cu.done) {
        bool progress = false;
        do {
          if (!cu.have) {
            const int buf = cu.it & 1;
            if (!ptx::mbar_test_wait(bar.lfull(buf), (cu.it >> 1) & 1)) break;
            const uint8_t* lb = smem + C::kListOff + buf * C::kListBytes;
            const int* meta = reinterpret_cast<const int*>(lb);
            progress = true;
            if (meta[0] < 0) {
              cu.done = true;
              break;
            }
            cu.have = true;
            cu.L = meta[5];
            cu.kc = cu.vc = 0;
            cu.hasq = meta[1 + 2 * x] >= 0;
            cu.qready = false;
            cu.qreleased = false;
            cu.first_pv = true;
            cu.flags = reinterpret_cast<const uint16_t*>(lb + C::kListMeta + kMaxTiles * 2);
          }
          // ---- V position
          if (cu.vc < cu.kc) {
            const uint32_t gi = cu.gbase + (uint32_t)cu.vc;
            const int s = (int)(gi % kNS);
            const uint32_t fph = (uint32_t)((gi / kNS) & 1);
            bool passed = false, issued_pv = false;
            if (cu.pv != cu.qk && cu.vc == ((cu.pv & 1) ? cu.ent1 : cu.ent0)) {
              const int b = (int)(cu.pv & 1);
              if (ptx::mbar_test_wait(bar.pfull(x, b), (cu.pv >> 1) & 1) && ptx::mbar_test_wait(bar.vfull(s), fph)) {
                ptx::tc_fence_after();
                const uint32_t o_tmem = tmem + 256u + (uint32_t)(x * D);
                const uint32_t p_tmem = tmem + (uint32_t)(64 * (2 * x + b));
                const uint64_t vd = ptx::smem_desc_sw128(sbase + C::kVOff + s * C::kTileBytes, C::kKCB, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  ptx::mma_ts(o_tmem, p_tmem + kk * 8, vd + (uint64_t)(kk * (2048 >> 4)), kIdPV,
                              (cu.first_pv && kk == 0) ? 0u : 1u);
                ptx::mma_commit(bar.odone(x, b));
                cu.first_pv = false;
                ++cu.pv;
                passed = true;
                issued_pv = true;
              }
            } else {
              passed = ptx::mbar_test_wait(bar.vfull(s), fph);
            }
            if (passed) {
              if (issued_pv) ptx::mma_commit(bar.vempty(s));
              else ptx::mbar_arrive(bar.vempty(s));
              ++cu.vc;
              progress = true;
            }
          }
          // ---- K position
          if (cu.kc < cu.L) {
            const bool used = cu.hasq && ((cu.flags[cu.kc] >> (2 * x)) & 3u) != 0u;
            const uint32_t gi = cu.gbase + (uint32_t)cu.kc;
            const int s = (int)(gi % kNS);
            const uint32_t fph = (uint32_t)((gi / kNS) & 1);
            bool passed = false;
            if (!used) {
              passed = ptx::mbar_test_wait(bar.kfull(s), fph);
            } else if (cu.qk - cu.pv < 2u) {
              if (!cu.qready) cu.qready = ptx::mbar_test_wait(bar.qfull(x), cu.qn & 1);
              if (cu.qready && ptx::mbar_test_wait(bar.kfull(s), fph)) {
                const int b = (int)(cu.qk & 1);
                const uint32_t s_tmem = tmem + (uint32_t)(64 * (2 * x + b));
                const uint64_t qd = ptx::smem_desc_sw128(sbase + C::kQOff + x * C::kQBytes, 16, 1024);
                const uint64_t kd = ptx::smem_desc_sw128(sbase + C::kKOff + s * C::kTileBytes, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                  ptx::mma_ss(s_tmem, qd + (uint64_t)(((kk >> 2) * C::kQCB + (kk & 3) * 32) >> 4),
                              kd + (uint64_t)(((kk >> 2) * C::kKCB + (kk & 3) * 32) >> 4), kIdQK, kk > 0 ? 1u : 0u);
                ptx::mma_commit(bar.sfull(x, b));
                if (b) cu.ent1 = cu.kc;
                else cu.ent0 = cu.kc;
                ++cu.qk;
                passed = true;
              }
            }
            if (passed) {
              if (used) ptx::mma_commit(bar.kempty(s));
              else ptx::mbar_arrive(bar.kempty(s));
              ++cu.kc;
              progress = true;
              if (cu.kc == cu.L && cu.hasq && cu.qready && !cu.qreleased) {
                ptx::mma_commit(bar.qempty(x));      // the unit's last Q K^T has been issued
                cu.qreleased = true;
              }
            }
          }
          // ---- end of the unit
          if (cu.kc == cu.L && cu.vc == cu.L) {
            if (cu.hasq && !cu.qreleased) {
              // No product used Q (its rows retain nothing here): release it once loaded.
              if (!cu.qready) cu.qready = ptx::mbar_test_wait(bar.qfull(x), cu.qn & 1);
              if (!cu.qready) break;
              ptx::mma_commit(bar.qempty(x));
              cu.qreleased = true;
            }
            if (cu.hasq) ++cu.qn;
            ptx::mbar_arrive(bar.lempty(cu.it & 1));
            ++cu.it;
            cu.have = false;
            cu.gbase += (uint32_t)cu.L;
            progress = true;
          }
        } while (false);
        if (progress) {
          idle_since = clock64();
        } else if (*abort) {
          ok = false;
        } else if (clock64() - idle_since > kWaitLimit) {
          *abort = 1;
          report_error(a.err, BSA_KERR_WAIT_TIMEOUT);
          ok = false;
        } else {
          // Nothing to issue: suspend until the barrier this issuer most likely needs next
          // completes (at most kIssuerSleepNs), so that the two softmax warps sharing the
          // sub-partition get its issue slots. Then every position is tested again.
          uint32_t wb, wp;
          if (!cu.have) {
            wb = bar.lfull(cu.it & 1);
            wp = (uint32_t)(cu.it >> 1) & 1u;
          } else if (cu.vc < cu.kc) {
            const uint32_t gi = cu.gbase + (uint32_t)cu.vc;
            wb = bar.vfull((int)(gi % kNS));
            wp = (gi / kNS) & 1u;
            if (cu.pv != cu.qk && cu.vc == ((cu.pv & 1) ? cu.ent1 : cu.ent0) &&
                !ptx::mbar_test_wait(bar.pfull(x, (int)(cu.pv & 1)), (cu.pv >> 1) & 1)) {
              wb = bar.pfull(x, (int)(cu.pv & 1));
              wp = (cu.pv >> 1) & 1;
            }
          } else if (cu.kc < cu.L && (!cu.hasq || cu.qready || ((cu.flags[cu.kc] >> (2 * x)) & 3u) == 0u)) {
            const uint32_t gi = cu.gbase + (uint32_t)cu.kc;
            wb = bar.kfull((int)(gi % kNS));
            wp = (gi / kNS) & 1u;
          } else {
            wb = bar.qfull(x);
            wp = (uint32_t)cu.qn & 1u;
          }
          ptx::mbar_try_wait_ns(wb, wp, kIssuerSleepNs);
        }
      }
      // Never free TMEM under a running MMA: wait until everything issued has completed.
      int zero = 0;
      ptx::mma_commit(bar.drain(x));
      ptx::mbar_wait(bar.drain(x), 0, &zero, a.err, kWaitLimit);
    }
  }
  } else {
    ptx::setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax + epilogue
    const int x = warp >> 2;                 // query block of this warpgroup
    const int row = threadIdx.x & 127;       // TMEM lane
    const int rh = row >> 6;                 // which of the block's two query tiles
    const int t = 2 * x + rh;                // query tile slot in the unit
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_tmem0 = tmem + (uint32_t)(128 * x) + lane_base;   // S buffer b at + 64 b
    const uint32_t o_tmem = tmem + 256u + (uint32_t)(x * D) + lane_base;
    const float c = a.scale_log2;
    uint32_t sidx = 0;                       // blocks processed (sfull / pfull phases)
    for (int it = 0;; ++it) {
      const int buf = it & 1;
      const uint8_t* lb = smem + C::kListOff + buf * C::kListBytes;
      const int* meta = reinterpret_cast<const int*>(lb);
      const uint16_t* tiles = reinterpret_cast<const uint16_t*>(lb + C::kListMeta);
      const uint16_t* flags = reinterpret_cast<const uint16_t*>(lb + C::kListMeta + kMaxTiles * 2);
      if (!warp_wait(bar.lfull(buf), (it >> 1) & 1, abort, a.err)) break;
      const int bh = meta[0];
      if (bh < 0) break;
      const int qt = meta[1 + t];
      const int L = meta[5];
      int tq = 0, yq = 0, xq = 0;            // this row's token (the token support's centre)
      {
        int tt, ty, tx;
        tile_xyz(g, qt >= 0 ? qt : 0, tt, ty, tx);
        const int rr = row & 63;
        tq = 4 * tt + (rr >> 4);
        yq = 4 * ty + ((rr >> 2) & 3);
        xq = 4 * tx + (rr & 3);
      }
      float m_run = -INFINITY, l_ex = 0.f, l_bf = 0.f;
      int nused = 0;
      bool ok = true;
      for (int cb = 0; cb < L; ++cb) {
        const uint32_t f = flags[cb];
        if (meta[1 + 2 * x] < 0 || ((f >> (2 * x)) & 3u) == 0u) continue;   // not used by this query block
        const int use = tile_use(f, t);
        const uint64_t valid = use == kUsePartial ? tile_slots(tiles[cb], f, t, g, tq, yq, xq, a.token_rho) : ~0ull;
        const int b = (int)(sidx & 1);
        const uint32_t s_tmem = s_tmem0 + 64u * (uint32_t)b;
        if (!warp_wait(bar.sfull(x, b), (sidx >> 1) & 1, abort, a.err)) { ok = false; break; }
        ptx::tc_fence_after();
        uint32_t r[64];
        float mx = -INFINITY;
        if (use != kUseSkip) {
          load_half(s_tmem, r);
          mx = half_max(r, use, valid, mx);
        }
        const float mb = mx * c;                       // block maximum, log2 domain
        bool resc = false;
        if (m_run == -INFINITY) m_run = mb;            // O of this row is still zero
        else if (mb > m_run + kRescaleLog2) resc = true;
        if (__any_sync(0xffffffffu, resc)) {
          // O must hold exactly the unit's earlier blocks: wait for the previous block's
          // P.V (the block two back has completed: this block's Q K^T followed its P.V).
          if (!warp_wait(bar.odone(x, (int)((sidx - 1) & 1)), ((sidx - 1) >> 1) & 1, abort, a.err)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const float alpha = resc ? ex2(m_run - mb) : 1.0f;
          rescale_o<D>(o_tmem, alpha);
          l_ex *= alpha;
          l_bf *= alpha;
          if (resc) m_run = mb;
        }
        const float m_use = m_run == -INFINITY ? 0.0f : m_run;
        half_exp(r, use, valid, c, m_use, l_ex, l_bf, s_tmem);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar.pfull(x, b));
        ++sidx;
        ++nused;
      }
      const int bq = bh / g.H, hq = bh - (bh / g.H) * g.H;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar.lempty(buf));
      if (!ok) break;
      // ---- epilogue: O / l (bf16) and the LSE, in raster order
      const int rr = row & 63;
      int n_tok = -1;
      if (qt >= 0) {
        int tt, ty, tx;
        tile_xyz(g, qt, tt, ty, tx);
        const int tk = tt * 4 + (rr >> 4), y = ty * 4 + ((rr >> 2) & 3), xx = tx * 4 + (rr & 3);
        if (tk < g.T && y < g.Hs && xx < g.Ws) n_tok = (tk * g.Hs + y) * g.Ws + xx;
      }
      if (nused > 0) {
        if (!warp_wait(bar.odone(x, (int)((sidx - 1) & 1)), ((sidx - 1) >> 1) & 1, abort, a.err)) break;
        ptx::tc_fence_after();
      }
      const float inv_l = l_bf > 0.f ? 1.0f / l_bf : 0.f;
      uint4* dst = n_tok >= 0 ? reinterpret_cast<uint4*>(a.out + (((long long)bq * g.N + n_tok) * g.H + hq) * D)
                              : nullptr;
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t ov[32];
        if (nused > 0) {
          tmem_ld_x32(o_tmem + ch * 32, ov);
          ptx::tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) ov[k] = 0u;
        }
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
        if (!(l_ex > 0.f)) report_error(a.err, BSA_KERR_BAD_MASK);
        if (a.lse) {
          const float m_fin = m_run == -INFINITY ? 0.0f : m_run;
          a.lse[(long long)bh * g.N + n_tok] =
              l_ex > 0.f ? (m_fin + __log2f(l_ex)) * 0.69314718055994531f : -INFINITY;
        }
      }
      // The next unit's first P.V overwrites O: every TMEM read above must be complete
      // before this warp releases that unit's first P (ordered by the fence before it).
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
// Units of a (b, h): the dense rows (kv_count == NKT) four at a time in tile order, then
// the local rows four at a time. Unit cost = the key tiles query block A uses plus those B
// uses (popcounts of the OR of each block's two mask rows), the tensor work of the unit.

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

// Single thread: exclusive offsets of each (b, h)'s units, head by head; the unit count
// and a zeroed unit counter for the persistent attention kernel.
// bhcnt[i] = (nd, nl, ud, ul) on entry, (offset, nd, ud, ul) on exit.
__global__ void sched_scan_kernel(int BH, int4* __restrict__ bhcnt, int* __restrict__ header) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int off = 0;
  for (int i = 0; i < BH; ++i) {
    const int4 c = bhcnt[i];
    bhcnt[i] = make_int4(off, c.x, c.z, c.w);
    off += c.z + c.w;
  }
  header[1] = off;
  header[2] = 0;
}

constexpr int kSchedThreads = 512;
constexpr int kSortCap = 2048;      // power of two >= NT/4 + 2 for NT <= 4096

// One block per (b, h): form the units, cost them, sort by decreasing cost (ties by
// position), write them at the (b, h)'s offset.
__global__ void __launch_bounds__(kSchedThreads) sched_write_kernel(Geom g, const uint32_t* __restrict__ mask,
                                                                    const int32_t* __restrict__ kv_count,
                                                                    const int4* __restrict__ bhcnt,
                                                                    int* __restrict__ units) {
  __shared__ int rows[kMaxTiles];            // dense rows, then local rows, each in tile order
  __shared__ uint32_t key[kSortCap];
  const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long base = (long long)bh * g.NT;
  const int4 bc = bhcnt[bh];
  const int off = bc.x, nd = bc.y, ud = bc.z, ul = bc.w, nu = ud + ul;
  if (warp == 0) {
    int cd = 0, cl = 0;
    for (int i0 = 0; i0 < g.NT; i0 += 32) {
      const int i = i0 + lane;
      const bool valid = i < g.NT;
      const bool isd = valid && kv_count[base + i] == g.NT;
      const bool isl = valid && !isd;
      const uint32_t bd = __ballot_sync(0xffffffffu, isd), bl = __ballot_sync(0xffffffffu, isl);
      const uint32_t lt = (1u << lane) - 1u;
      if (isd) rows[cd + __popc(bd & lt)] = i;
      if (isl) rows[nd + cl + __popc(bl & lt)] = i;
      cd += __popc(bd);
      cl += __popc(bl);
    }
  }
  __syncthreads();
  // unit k: rows of its class, four at a time; q_t = -1 past the end of the class
  auto unit_row = [&](int k, int t) -> int {
    if (k < ud) {
      const int r = 4 * k + t;
      return r < nd ? rows[r] : -1;
    }
    const int r = 4 * (k - ud) + t;
    return r < g.NT - nd ? rows[nd + r] : -1;
  };
  const int nwarps = kSchedThreads / 32;
  for (int k = warp; k < kSortCap; k += nwarps) {
    if (k >= nu) {
      if (lane == 0) key[k] = 0xffffffffu;
      continue;
    }
    const int q0 = unit_row(k, 0), q1 = unit_row(k, 1), q2 = unit_row(k, 2), q3 = unit_row(k, 3);
    int cnt = 0;
    for (int w = lane; w < g.NW; w += 32) {
      const uint32_t a0 = mask[(base + q0) * g.NW + w] | (q1 >= 0 ? mask[(base + q1) * g.NW + w] : 0u);
      const uint32_t b0 = q2 >= 0 ? (mask[(base + q2) * g.NW + w] | (q3 >= 0 ? mask[(base + q3) * g.NW + w] : 0u)) : 0u;
      cnt += __popc(a0) + __popc(b0);
    }
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) key[k] = ((uint32_t)(16383 - min(cnt, 16383)) << 11) | (uint32_t)k;
  }
  __syncthreads();
  // bitonic sort of key[0, kSortCap) ascending: decreasing cost, then position
  for (int size = 2; size <= kSortCap; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < kSortCap / 2; i += kSchedThreads) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint32_t a = key[lo], b = key[hi];
        if ((a > b) == up) {
          key[lo] = b;
          key[hi] = a;
        }
      }
      __syncthreads();
    }
  }
  for (int p = tid; p < nu; p += kSchedThreads) {
    const int k = (int)(key[p] & 2047u);
    int* up = units + (size_t)(off + p) * kUnitInts;
    up[0] = bh;
    up[1] = unit_row(k, 0);
    up[2] = unit_row(k, 1);
    up[3] = unit_row(k, 2);
    up[4] = unit_row(k, 3);
    up[5] = 16383 - (int)(key[p] >> 11);
    up[6] = up[7] = 0;
  }
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

cudaError_t run_sched(const Geom& g, const uint32_t* mask, const int32_t* kv_count, int* header, int4* bhcnt,
                      int* units, cudaStream_t s) {
  const int BH = g.B * g.H;
  sched_count_kernel<<<BH, 256, 0, s>>>(g, kv_count, bhcnt);
  sched_scan_kernel<<<1, 32, 0, s>>>(BH, bhcnt, header);
  sched_write_kernel<<<BH, kSchedThreads, 0, s>>>(g, mask, kv_count, bhcnt, units);
  count_launches(3);
  return cudaGetLastError();
}

template <int D>
cudaError_t run_attn(const Geom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const AttnArgs& a, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  // The register split must not ask for more than the launch provides (a larger split
  // would wait forever in setmaxnreg): refuse a build that was allocated fewer registers.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_kernel<D>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs * kAttnThreads < 128 * (2 * kRegsSoftmax + kRegsControl)) return cudaErrorInvalidConfiguration;
  const long long max_units = (long long)g.B * g.H * units_per_bh(g.NT);
  const int grid = (int)(max_units < sm_count() ? max_units : sm_count());
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

cudaError_t attn_after_sched(const Geom& g, const __nv_bfloat16* qt, const __nv_bfloat16* kt,
                             const __nv_bfloat16* vt, const uint32_t* mask, float scale, __nv_bfloat16* out,
                             float* lse, int* header, const int* units, uint32_t* err, const uint8_t* dense,
                             int token_rho, cudaStream_t s) {
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
  a.err = err;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.dense = dense;
  a.token_rho = token_rho;
  if (g.d == 128) return run_attn<128>(g, mq, mk, mv, a, s);
  return run_attn<64>(g, mq, mk, mv, a, s);
}

}  // namespace

cudaError_t launch_sparse_attn(const Geom& g, const __nv_bfloat16* qt, const __nv_bfloat16* kt,
                               const __nv_bfloat16* vt, const uint32_t* mask, const int32_t* kv_count,
                               float scale, __nv_bfloat16* out, float* lse, uint8_t* ws, cudaStream_t s,
                               const uint8_t* dense, int token_rho) {
  const WsLayout L = ws_layout(g);
  int* header = reinterpret_cast<int*>(ws);
  int4* bhcnt = reinterpret_cast<int4*>(ws + L.bhcnt);
  int* units = reinterpret_cast<int*>(ws + L.units);
  cudaError_t e = run_sched(g, mask, kv_count, header, bhcnt, units, s);
  if (e != cudaSuccess) return e;
  return attn_after_sched(g, qt, kt, vt, mask, scale, out, lse, header, units,
                          reinterpret_cast<uint32_t*>(ws), dense, token_rho, s);
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
// host-side stand-in, not a device address, so the address is looked up with the device
// current. It is looked up again on every call made outside a stream capture, so that a
// context torn down and created again (cudaDeviceReset) never leaves a stale address; a
// call under capture uses the address its device had at its last call outside capture.
cudaError_t fixed_scratch_addr(cudaStream_t s, uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(s, &cap);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_fixed_mu);
  if (cap == cudaStreamCaptureStatusNone || !g_fixed_addr[dev]) {
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

// Scratch of one call: 256-byte header (error word, unit count, unit counter), per-(b, h)
// counts, units.
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
  cudaError_t e = fixed_scratch_addr(s, &base);
  if (e != cudaSuccess) return e;
  const int BH = g.B * g.H;
  int* header = reinterpret_cast<int*>(base);
  int4* bhcnt = reinterpret_cast<int4*>(base + 256);
  int* units = reinterpret_cast<int*>(base + 256 + align256((size_t)BH * sizeof(int4)));

  // The array keeps the previous call's contents: the error word and the unit count must
  // start at zero; counts and units are fully rewritten by the scheduler before use.
  e = cudaMemsetAsync(base, 0, 256, s);
  if (e != cudaSuccess) return e;
  e = run_sched(g, mask, kv_count, header, bhcnt, units, s);
  if (e != cudaSuccess) return e;
  e = attn_after_sched(g, qt, kt, vt, mask, scale, out, lse, header, units, reinterpret_cast<uint32_t*>(base),
                       nullptr, -1, s);
  if (e != cudaSuccess) return e;
  if (errors) e = cudaMemcpyAsync(errors, base, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s);
  return e;
}

}  // namespace bsa

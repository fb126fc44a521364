// Pooled scores on the tensor cores: S = qbar kbar^T for every (b, h), fp32 inputs, with
// tcgen05.mma kind::tf32 in three products per step (the 3xTF32 split): each operand is
// split into hi, its value with the low 13 mantissa bits cleared (exactly a tf32 value),
// and lo = x - hi (exact in fp32), and S accumulates hi*hi + hi*lo + lo*hi in fp32. The
// dropped lo*lo term is below 2^-22 of |x||y|, so the scores keep fp32-level accuracy, as
// the selection's near-tie band of 1e-4 of the row's score scale requires; one tf32
// product alone (about 2^-11 relative) would not.
//
// One CTA of 128 threads per (b*h, 128 query tiles, 128 key tiles); the 128 x 128 fp32
// accumulator lives in 128 TMEM columns. d is staged 32 columns (128 bytes of fp32) at a
// time: TMA loads the two 128-row slices with the 128-byte swizzle, the threads split them
// in place (elementwise, so the swizzled layout carries over to the hi and lo copies),
// and one thread issues the products. The epilogue reads the accumulator row by row (TMEM
// lane = query tile) and writes the score rows. Every wait is bounded.
#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tmem_ops.cuh"

namespace bsa {
namespace {

constexpr int kTcTile = 128;                        // query tiles x key tiles per CTA
constexpr int kTcChunk = 32;                        // d columns per stage
constexpr int kTcThreads = 128;
constexpr int kTcChunkBytes = kTcTile * kTcChunk * 4;   // 16 KB per operand slice
constexpr long long kTcWaitLimit = 4000000000LL;    // SM cycles, about 2 s

// Shared memory (1024-byte aligned): A (hi in place), A lo, B (hi in place), B lo, then the
// load and product barriers, the abort flag and the TMEM base.
constexpr int kTcA = 0, kTcALo = kTcChunkBytes, kTcB = 2 * kTcChunkBytes, kTcBLo = 3 * kTcChunkBytes;
constexpr int kTcBar = 4 * kTcChunkBytes;
constexpr int kTcMisc = kTcBar + 16;
constexpr int kTcSmemBytes = 1024 + kTcMisc + 16;

// Instruction descriptor of kind::tf32: fp32 accumulator (bits 4-5 = 1), A and B tf32
// (bits 7-9 = 2, 10-12 = 2), both K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kIdescTf32 = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(kTcTile >> 3) << 17) |
                                ((uint32_t)(kTcTile >> 4) << 24);

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(kIdescTf32), "r"(accumulate)
      : "memory");
}

// Generic-proxy writes to shared memory become visible to the tensor cores' reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// In place: x -> hi (low 13 mantissa bits cleared); lo[k] = x - hi (exact).
__device__ __forceinline__ void split_slice(uint8_t* hi_inplace, uint8_t* lo, int tid) {
  uint4* h = reinterpret_cast<uint4*>(hi_inplace);
  uint4* l = reinterpret_cast<uint4*>(lo);
#pragma unroll
  for (int k = tid; k < kTcChunkBytes / 16; k += kTcThreads) {
    const uint4 w = h[k];
    const uint4 hv = make_uint4(w.x & 0xffffe000u, w.y & 0xffffe000u, w.z & 0xffffe000u, w.w & 0xffffe000u);
    l[k] = make_uint4(__float_as_uint(__uint_as_float(w.x) - __uint_as_float(hv.x)),
                      __float_as_uint(__uint_as_float(w.y) - __uint_as_float(hv.y)),
                      __float_as_uint(__uint_as_float(w.z) - __uint_as_float(hv.z)),
                      __float_as_uint(__uint_as_float(w.w) - __uint_as_float(hv.w)));
    h[k] = hv;
  }
}

template <int D>
__global__ void __launch_bounds__(kTcThreads) score_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                              const __grid_constant__ CUtensorMap tmK, Geom g,
                                                              float* __restrict__ S, int NKTP, uint32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (ptx::smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sbase = ptx::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.z;
  const int i0 = blockIdx.x * kTcTile, j0 = blockIdx.y * kTcTile;
  const uint32_t bar_ld = sbase + kTcBar, bar_mma = bar_ld + 8;
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kTcMisc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTcMisc + 4);

  if (tid == 0) {
    ptx::prefetch_tensormap(&tmQ);
    ptx::prefetch_tensormap(&tmK);
    ptx::mbar_init(bar_ld, 1);
    ptx::mbar_init(bar_mma, 1);
    *abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), kTcTile);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int rowA = bh * g.NT + i0, rowB = bh * g.NT + j0;

  bool ok = true;
#pragma unroll 1
  for (int c = 0; c < D / kTcChunk; ++c) {
    if (tid == 0) {
      ptx::mbar_arrive_expect_tx(bar_ld, 2 * kTcChunkBytes);
      ptx::tma_load_2d(sbase + kTcA, &tmQ, bar_ld, c * kTcChunk, rowA);
      ptx::tma_load_2d(sbase + kTcB, &tmK, bar_ld, c * kTcChunk, rowB);
    }
    ok = ptx::mbar_wait(bar_ld, c & 1, abort, err, kTcWaitLimit);
    if (!__syncthreads_and(ok)) break;
    split_slice(smem + kTcA, smem + kTcALo, tid);
    split_slice(smem + kTcB, smem + kTcBLo, tid);
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      ptx::tc_fence_after();
      const uint64_t dA = ptx::smem_desc_sw128(sbase + kTcA, 16, 1024);
      const uint64_t dALo = ptx::smem_desc_sw128(sbase + kTcALo, 16, 1024);
      const uint64_t dB = ptx::smem_desc_sw128(sbase + kTcB, 16, 1024);
      const uint64_t dBLo = ptx::smem_desc_sw128(sbase + kTcBLo, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < kTcChunk / 8; ++kk) {       // 8 tf32 = 32 bytes per product
        const uint64_t off = (uint64_t)((kk * 32) >> 4);
        mma_tf32(tmem, dA + off, dB + off, (c > 0 || kk > 0) ? 1u : 0u);
        mma_tf32(tmem, dA + off, dBLo + off, 1u);
        mma_tf32(tmem, dALo + off, dB + off, 1u);
      }
      ptx::mma_commit(bar_mma);
    }
    // The products must have read this stage before the next one overwrites it.
    ok = ptx::mbar_wait(bar_mma, c & 1, abort, err, kTcWaitLimit);
    ptx::tc_fence_after();
    if (!__syncthreads_and(ok)) break;
  }

  if (ok) {
    // 32 accumulator columns at a time: each thread stages its row in shared memory (the
    // operand slices are free: every product has completed), then its warp writes its 32
    // rows with each instruction covering four rows of 128 contiguous bytes.
    constexpr int kStageRow = 36;                         // floats; 144-byte rows keep float4 accesses conflict-free
    float* stage = reinterpret_cast<float*>(smem + kTcA);
    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
    for (int q = 0; q < kTcTile / 32; ++q) {
      uint32_t v[32];
      tmem_ld_x32(taddr + 32 * q, v);
      ptx::tmem_wait_ld();
      float4* mine = reinterpret_cast<float4*>(stage + tid * kStageRow);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        mine[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                              __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
      __syncwarp();
      const int jj = j0 + 32 * q + 4 * (lane & 7);
#pragma unroll
      for (int rr = 0; rr < 32; rr += 4) {
        const int rloc = warp * 32 + rr + (lane >> 3);
        const int i = i0 + rloc;
        if (i < g.NT && jj < NKTP)
          *reinterpret_cast<float4*>(S + ((long long)bh * g.NT + i) * NKTP + jj) =
              *reinterpret_cast<const float4*>(stage + rloc * kStageRow + 4 * (lane & 7));
      }
      __syncwarp();
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTcTile);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once; a function-local static is initialised once even under concurrent calls.
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

// 2D map over pooled means viewed as [rows = B*H*NT, d] fp32; box = 128 rows x 32 columns
// (128 bytes, the 128-byte swizzle span). Rows past the end read as zero.
bool make_map_f32(CUtensorMap* m, const float* base, long long rows, int d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 4};
  cuuint32_t box[2] = {kTcChunk, kTcTile};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t run_score_tc(const Geom& g, const CUtensorMap& mq, const CUtensorMap& mk, float* S, int NKTP,
                         uint32_t* err, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kTcSmemBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid(ceil_div(g.NT, kTcTile), ceil_div(g.NT, kTcTile), g.B * g.H);
  score_tc_kernel<D><<<grid, kTcThreads, kTcSmemBytes, s>>>(mq, mk, g, S, NKTP, err);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_tc(const Geom& g, const float* qbar, const float* kbar, float* S, int NKTP,
                            uint32_t* err, cudaStream_t s) {
  const long long rows = (long long)g.B * g.H * g.NT;
  CUtensorMap mq, mk;
  if (!make_map_f32(&mq, qbar, rows, g.d) || !make_map_f32(&mk, kbar, rows, g.d)) return cudaErrorInvalidValue;
  return g.d == 128 ? run_score_tc<128>(g, mq, mk, S, NKTP, err, s) : run_score_tc<64>(g, mq, mk, S, NKTP, err, s);
}

}  // namespace bsa

// Tile-major reorder and its inverse (Token Radius Attention summary, "Efficient
// execution": tokens regrouped so that each 4x4x4 tile is contiguous, turning a tile
// mask into a block-sparse mask).
//
// Both kernels move 16-byte vectors (8 bf16) and are bound by HBM bandwidth. A flat
// grid-stride loop walks the vectors in an order that keeps both sides coalesced:
//  - reorder walks (b, tile, slot, head, chunk) with chunk fastest: the 32 lanes of a warp
//    read 512 contiguous bytes of one token's [H, d] row and write 256-byte runs of the
//    tile-major output;
//  - unreorder walks the raster output (b, n, head, chunk): contiguous writes, 256-byte
//    runs of reads.
// Each thread keeps 4 independent vectors in flight.
//
// reorder_pool does the reorder of Q or K and, in the same pass, the per-tile mean of the
// valid tokens (VORTA summary, "average pooling" of tiles) that the mask builder scores:
// one block per (b, tile, 128 (head, 16-byte chunk) vectors of the token rows) walks the
// tile's 64 slots, so each thread keeps the fp32 sums of its chunk in registers while the
// vectors move. The mask builder then starts from the means instead of reading the
// tile-major tensors a second time.
#include "common.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct ReorderArgs {
  Geom g;
  FastDiv div_H, div_NT, div_nYX, div_nX, div_Ws, div_HsWs, div_T;
  int d8_log2;             // log2(d / 8)
  long long total;         // vectors to move
};

// Raster token of slot r of tile j, or -1 for a padding slot.
__device__ __forceinline__ int slot_token(const ReorderArgs& a, int j, int r) {
  const uint32_t tt = a.div_nYX.q(j);
  const uint32_t rem = j - tt * a.div_nYX.div;
  const uint32_t ty = a.div_nX.q(rem);
  const uint32_t tx = rem - ty * a.div_nX.div;
  const int t = tt * 4 + (r >> 4), y = ty * 4 + ((r >> 2) & 3), x = tx * 4 + (r & 3);
  if (t >= a.g.T || y >= a.g.Hs || x >= a.g.Ws) return -1;
  return (t * a.g.Hs + y) * a.g.Ws + x;
}

__global__ void __launch_bounds__(kThreads) reorder_kernel(ReorderArgs a, const uint4* __restrict__ x,
                                                           uint4* __restrict__ xt) {
  const int d8 = 1 << a.d8_log2;
  const long long stride = (long long)gridDim.x * kThreads * kUnroll;
  for (long long base = (long long)blockIdx.x * kThreads * kUnroll + threadIdx.x; base < a.total;
       base += stride) {
    uint4 v[kUnroll];
    long long dst[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long e = base + (long long)u * kThreads;
      dst[u] = -1;
      if (e < a.total) {
        // e = (((b*NT + j)*64 + r)*H + h)*d8 + c
        const int c = (int)(e & (d8 - 1));
        const uint32_t rest = (uint32_t)(e >> a.d8_log2);      // ((b*NT + j)*64 + r)*H + h
        const uint32_t tok = a.div_H.q(rest);
        const int h = rest - tok * a.g.H;
        const int r = tok & 63;
        const uint32_t bj = tok >> 6;
        const uint32_t b = a.div_NT.q(bj);
        const int j = bj - b * a.g.NT;
        const int n = slot_token(a, j, r);
        dst[u] = ((((long long)b * a.g.H + h) * a.g.NT + j) * 64 + r) * d8 + c;
        v[u] = make_uint4(0, 0, 0, 0);
        if (n >= 0) v[u] = __ldg(&x[(((long long)b * a.g.N + n) * a.g.H + h) * d8 + c]);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (dst[u] >= 0) xt[dst[u]] = v[u];
  }
}

__global__ void __launch_bounds__(kThreads) unreorder_kernel(ReorderArgs a, const uint4* __restrict__ xt,
                                                             uint4* __restrict__ x) {
  const int d8 = 1 << a.d8_log2;
  const long long stride = (long long)gridDim.x * kThreads * kUnroll;
  for (long long base = (long long)blockIdx.x * kThreads * kUnroll + threadIdx.x; base < a.total;
       base += stride) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long e = base + (long long)u * kThreads;
      if (e < a.total) {
        // e = ((b*N + n)*H + h)*d8 + c
        const int c = (int)(e & (d8 - 1));
        const uint32_t rest = (uint32_t)(e >> a.d8_log2);
        const uint32_t bn = a.div_H.q(rest);
        const int h = rest - bn * a.g.H;
        const uint32_t b = a.div_T.q(a.div_HsWs.q(bn));
        const uint32_t n = bn - b * (uint32_t)a.g.N;
        const uint32_t t = a.div_HsWs.q(n);
        const uint32_t yx = n - t * a.div_HsWs.div;
        const uint32_t y = a.div_Ws.q(yx);
        const uint32_t xx = yx - y * a.g.Ws;
        const int j = ((t >> 2) * a.g.nY + (y >> 2)) * a.g.nX + (xx >> 2);
        const int r = ((t & 3) * 4 + (y & 3)) * 4 + (xx & 3);
        v[u] = __ldg(&xt[((((long long)b * a.g.H + h) * a.g.NT + j) * 64 + r) * d8 + c]);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long e = base + (long long)u * kThreads;
      if (e < a.total) x[e] = v[u];
    }
  }
}

constexpr int kPoolThreads = 128;
constexpr int kPoolUnroll = 16;

// One block per (b, tile j, 128 of the token row's vectors): each thread moves one
// (head, 16-byte chunk) vector of the tile's 64 slots and keeps its fp32 sums.
__global__ void __launch_bounds__(kPoolThreads) reorder_pool_kernel(ReorderArgs a, const uint4* __restrict__ x,
                                                                    uint4* __restrict__ xt, float* __restrict__ xbar) {
  __shared__ int tok[64];
  __shared__ int s_nvalid;
  const int d8 = 1 << a.d8_log2;
  const int b = blockIdx.x / a.g.NT, j = blockIdx.x - b * a.g.NT;
  if (threadIdx.x < 64) tok[threadIdx.x] = slot_token(a, j, threadIdx.x);
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = 0;
    for (int r = 0; r < 64; ++r) n += tok[r] >= 0;
    s_nvalid = n;
  }
  __syncthreads();
  const float inv = 1.0f / (float)s_nvalid;
  const int nv = a.g.H * d8;                       // vectors per token row
  const int v = blockIdx.y * kPoolThreads + threadIdx.x;
  if (v < nv) {
    const int h = v >> a.d8_log2, c = v & (d8 - 1);
    const uint4* src = x + (long long)b * a.g.N * nv + v;
    uint4* dst = xt + ((((long long)b * a.g.H + h) * a.g.NT + j) * 64) * d8 + c;
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
#pragma unroll 1
    for (int r0 = 0; r0 < 64; r0 += kPoolUnroll) {
      uint4 w[kPoolUnroll];
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u) {
        const int n = tok[r0 + u];
        w[u] = n >= 0 ? __ldg(&src[(long long)n * nv]) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u) {
        dst[(r0 + u) * d8] = w[u];
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&w[u]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(p[k]);
          acc[2 * k] += f.x;
          acc[2 * k + 1] += f.y;
        }
      }
    }
    float4* m = reinterpret_cast<float4*>(xbar + ((((long long)b * a.g.H + h) * a.g.NT + j) * d8 + c) * 8);
    m[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    m[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
}

ReorderArgs make_args(const Geom& g, long long total) {
  ReorderArgs a;
  a.g = g;
  a.div_H = FastDiv(g.H);
  a.div_NT = FastDiv(g.NT);
  a.div_nYX = FastDiv(g.nY * g.nX);
  a.div_nX = FastDiv(g.nX);
  a.div_Ws = FastDiv(g.Ws);
  a.div_HsWs = FastDiv(g.Hs * g.Ws);
  a.div_T = FastDiv(g.T);
  a.d8_log2 = (g.d == 128) ? 4 : 3;
  a.total = total;
  return a;
}

int grid_for(long long total) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long per_block = (long long)kThreads * kUnroll;
  long long blocks = (total + per_block - 1) / per_block;
  const long long cap = (long long)sms * 8;              // 8 resident blocks of 256 per SM
  return (int)(blocks < cap ? (blocks < 1 ? 1 : blocks) : cap);
}

}  // namespace

cudaError_t launch_reorder(const Geom& g, const __nv_bfloat16* x, __nv_bfloat16* xt, cudaStream_t s) {
  const long long total = (long long)g.B * g.NT * 64 * g.H * (g.d / 8);
  ReorderArgs a = make_args(g, total);
  reorder_kernel<<<grid_for(total), kThreads, 0, s>>>(a, reinterpret_cast<const uint4*>(x),
                                                      reinterpret_cast<uint4*>(xt));
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_reorder_pool(const Geom& g, const __nv_bfloat16* x, __nv_bfloat16* xt, float* xbar,
                                cudaStream_t s) {
  ReorderArgs a = make_args(g, 0);
  const dim3 grid(g.B * g.NT, ceil_div(g.H * (g.d / 8), kPoolThreads));
  reorder_pool_kernel<<<grid, kPoolThreads, 0, s>>>(a, reinterpret_cast<const uint4*>(x),
                                                    reinterpret_cast<uint4*>(xt), xbar);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_unreorder(const Geom& g, const __nv_bfloat16* xt, __nv_bfloat16* x, cudaStream_t s) {
  const long long total = (long long)g.B * g.N * g.H * (g.d / 8);
  ReorderArgs a = make_args(g, total);
  unreorder_kernel<<<grid_for(total), kThreads, 0, s>>>(a, reinterpret_cast<const uint4*>(xt),
                                                        reinterpret_cast<uint4*>(x));
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace bsa

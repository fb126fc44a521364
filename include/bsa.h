/*
 * bsa.h - C ABI of the B200 (sm_100a) block-sparse video attention library (libbsa.so).
 *
 * The library implements the data path of heterogeneous block-sparse self-attention over
 * the spatio-temporal token grid of a video diffusion transformer, as described across
 * the HetA-DiT abstract (dense global attention for difficult regions, local attention
 * elsewhere), the Token Radius Attention summary (tile-major token layout, budget from
 * attention entropy, radius with temporal distance decay, block-sparse masks for
 * execution), the VORTA summary (sliding-tile local branch, average pooling of tiles) and
 * the MOD-DiT poster abstract (block masks mixing diagonal, temporal and global patterns).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tokens of one video form a T x Hs x Ws grid in raster order, n = (t*Hs + y)*Ws + x.
 *  - A tile is a 4x4x4 cube of 64 tokens. Tiles per axis: nT = ceil(T/4), nY = ceil(Hs/4),
 *    nX = ceil(Ws/4); NT = nT*nY*nX. Tile j = (tt*nY + ty)*nX + tx; slot r inside a tile
 *    = (dt*4 + dy)*4 + dx. Edge tiles are partial: their missing slots are zero in the
 *    tile-major tensors and are never attended to or written back.
 *  - Query tiles and key tiles are the same tiles: NQT = NKT = NT.
 *  - All tensor pointers are DEVICE pointers to caller-owned memory, 16-byte aligned,
 *    densely packed in the stated layout. bf16 = IEEE bfloat16, row-major, last index
 *    fastest.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Every call is
 *    asynchronous on that stream, allocates no memory, never synchronises the host and
 *    copies nothing between host and device.
 *  - Every call returns a status code (BSA_OK = 0). On error nothing is launched, except
 *    BSA_ERR_CUDA, which reports a failed launch (cudaGetLastError) after earlier kernels
 *    of the same call may already have been queued.
 *  - The current CUDA device must be an sm_100 part (B200); otherwise
 *    BSA_ERR_UNSUPPORTED_DEVICE.
 *  - Kernel-side faults that the kernels detect (a bounded wait that ran out, an index
 *    out of range) never trap: they set bits of the 32-bit error word at byte 0 of the
 *    workspace (BSA_KERR_*), which the caller may read back after synchronising.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Shape of one attention call. d (head dim) must be 64 or 128; B, H >= 1;
 * T, Hs, Ws >= 1 and at most 4096 each, with NT <= 4096 tiles, B*H <= 65535 and
 * B*H*NT*64 < 2^31 tile rows. */
typedef struct bsa_geom {
    int B;   /* batch items */
    int H;   /* attention heads */
    int d;   /* head dimension */
    int T;   /* frames (latent) */
    int Hs;  /* latent height */
    int Ws;  /* latent width */
} bsa_geom;

/* Mask rule. Each query tile is either routed to dense attention (all key tiles) or to a
 * local support plus extra tiles chosen by pooled score.
 *   window_kind   0: cube window, max(|dt|,|dy|,|dx|) <= radius (tile units)
 *                 1: window with temporal decay, |dt| <= radius and
 *                    max(|dy|,|dx|) <= radius - |dt|
 *                 2: the tiles touched by a token-level circular support with temporal
 *                    decay (Token Radius Attention summary: query-centred circular
 *                    neighbourhoods, base radius applied across frames with decay): key
 *                    token m supports query token n when |t_m - t_n| <= radius and
 *                    (y_m - y_n)^2 + (x_m - x_n)^2 <= (radius - |t_m - t_n|)^2, in tokens;
 *                    key tile j is a window tile of query tile i when a valid token of j
 *                    supports a valid token of i. Budget modes 0 and 2 only. The mask is
 *                    tile-granular; bsa_sparse_attn_fwd_token masks the tokens outside the
 *                    support inside window tiles (bsa_sparse_attn_fwd attends every valid
 *                    token of each retained tile)
 *   radius        window radius (>= 0): in tiles for kinds 0 and 1, in tokens (at most
 *                 32767) for kind 2; ignored when budget_mode = 1
 *   topk          extra key tiles outside the window, by pooled score, ties to the lower
 *                 tile index; capped at the number of tiles outside the window (>= 0)
 *   dense_fraction rho in [0,1]: the floor(rho*NQT + 1/2) query tiles of highest
 *                 difficulty (ties to the lower index) of each batch item take every key
 *                 tile, in every head
 *   budget_mode   0: window + topk; 1: per-(head, query tile) budget from the entropy of
 *                 the pooled-score softmax, b_i = clamp(floor(tau*NKT*NQT*exp(H_i) /
 *                 sum_i' exp(H_i') + 1/2), 1, NKT); the window is the decayed window of the
 *                 largest radius that fits b_i, topped up to b_i tiles by pooled score
 *                 (window_kind must be 1);
 *                 2: cumulative mass: the window (window_kind, radius), then the tiles
 *                 outside it in decreasing pooled score (ties to the lower index) until
 *                 the row's pooled probability, softmax over all key tiles of the pooled
 *                 scores, reaches theta (Token Radius Attention summary: the keys needed
 *                 to capture a target attention mass); every tile outside the window when
 *                 theta is not reached; topk is ignored
 *   budget_target tau in (0,1] for budget_mode 1, theta in (0,1] for budget_mode 2 */
typedef struct bsa_mask_params {
    int window_kind;
    int radius;
    int topk;
    float dense_fraction;
    int budget_mode;
    float budget_target;
} bsa_mask_params;

enum {
    BSA_OK = 0,
    BSA_ERR_INVALID_ARG = 1,        /* null pointer, bad shape, bad alignment, bad param */
    BSA_ERR_WORKSPACE = 2,          /* workspace missing or smaller than required */
    BSA_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not sm_100 */
    BSA_ERR_CUDA = 4                /* a CUDA call or launch failed */
};

/* Bits of the kernel error word (uint32 at byte 0 of the workspace). */
enum {
    BSA_KERR_WAIT_TIMEOUT = 1u << 0, /* a bounded barrier wait in a kernel ran out */
    BSA_KERR_BAD_UNIT = 1u << 1,     /* attention work list entry out of range */
    BSA_KERR_BAD_MASK = 1u << 2      /* a mask row with no retained tile */
};

/* Human-readable name of a status code (static storage, never NULL). */
const char* bsa_status_string(int status);

/* Tile grid of a geometry. Any output pointer may be NULL. Returns BSA_ERR_INVALID_ARG for
 * an invalid geometry. Host-only, no CUDA call. */
int bsa_tile_grid(const bsa_geom* g, int* nT, int* nY, int* nX, int* NT);

/* Bytes of workspace needed by bsa_build_mask and bsa_sparse_attn_fwd for this
 * geometry (one workspace serves both; its first 256 bytes hold the error word).
 * Returns 0 for an invalid geometry. Host-only. */
size_t bsa_workspace_bytes(const bsa_geom* g, const bsa_mask_params* p);

/* Zero the kernel error word at byte 0 of `ws` (stream-ordered memset of 4 bytes). */
int bsa_clear_error(void* ws, void* stream);

/* Tile-major reorder (Token Radius Attention summary, "Efficient execution": tokens of a
 * tile are made contiguous so that a tile mask is a block-sparse mask).
 *   x  : bf16 [B, N, H, d], N = T*Hs*Ws, raster token order (input, read only)
 *   xt : bf16 [B, H, NT, 64, d] (output; padding slots are written as zeros)
 * Bit-exact copy; no arithmetic. */
int bsa_reorder(const bsa_geom* g, const void* x, void* xt, void* stream);

/* Tile-major reorder fused with the per-tile mean of the mask builder (Token Radius
 * Attention summary, "Efficient execution", tile-major layout; VORTA summary, "average
 * pooling" of tiles). One pass over x does both:
 *   x    : bf16 [B, N, H, d] raster (input, read only)
 *   xt   : bf16 [B, H, NT, 64, d] (output, exactly as bsa_reorder writes it)
 *   xbar : fp32 [B, H, NT, d] (output): the mean over the valid tokens of each tile, summed
 *          in fp32 in slot order
 * For Q and K ahead of bsa_build_mask_pooled, which then needs no second read of qt, kt. */
int bsa_reorder_pool(const bsa_geom* g, const void* x, void* xt, float* xbar, void* stream);

/* Inverse of bsa_reorder: xt bf16 [B, H, NT, 64, d] -> x bf16 [B, N, H, d]. Padding slots
 * of xt are ignored. Bit-exact. */
int bsa_unreorder(const bsa_geom* g, const void* xt, void* x, void* stream);

/* Block mask (Token Radius Attention summary, budget and radius steps; HetA-DiT abstract,
 * dense/local routing; VORTA summary, average pooling and sliding tiles).
 *   qt, kt     : bf16 [B, H, NT, 64, d] tile-major Q and K (from bsa_reorder)
 *   difficulty : fp32 [B, NQT] per-query-tile difficulty used for dense routing
 *   mask       : uint32 [B, H, NQT, ceil(NKT/32)] output; key tile j of a row is bit
 *                (j % 32) of word (j / 32); bits at j >= NKT are zero
 *   kv_count   : int32 [B, H, NQT] output; retained key tiles per row
 *   ws, ws_bytes : device workspace of at least bsa_workspace_bytes(g, p) bytes
 * Steps: mean of each tile's valid tokens (fp32); pooled scores qbar.kbar (fp32, ranked
 * unscaled; the 1/sqrt(d) scale enters the entropy and the pooled probabilities of the
 * cumulative-mass mode only); routing; window; extra tiles by pooled score.
 * Deterministic: repeated calls give identical bits. */
int bsa_build_mask(const bsa_geom* g, const bsa_mask_params* p, const void* qt,
                   const void* kt, const float* difficulty, uint32_t* mask,
                   int32_t* kv_count, void* ws, size_t ws_bytes, void* stream);

/* bsa_build_mask starting from the per-tile means of Q and K (as bsa_reorder_pool writes
 * them) instead of the tile-major tensors: the same routing, window and selection steps,
 * with the same arguments otherwise.
 *   qbar, kbar : fp32 [B, H, NT, d] per-tile means of the valid tokens of Q and K */
int bsa_build_mask_pooled(const bsa_geom* g, const bsa_mask_params* p, const float* qbar,
                          const float* kbar, const float* difficulty, uint32_t* mask,
                          int32_t* kv_count, void* ws, size_t ws_bytes, void* stream);

/* Block-sparse attention forward (Token Radius Attention summary, execution of
 * block-sparse masks; FlashAttention-style online softmax).
 *   qt, kt, vt : bf16 [B, H, NT, 64, d] tile-major Q, K, V
 *   mask, kv_count : as written by bsa_build_mask (any mask whose rows each retain at
 *                least one tile is accepted; kv_count[row] must equal the row's popcount)
 *   softmax_scale : multiplier of q.k (normally 1/sqrt(d))
 *   out        : bf16 [B, N, H, d] output in raster token order; every valid token of
 *                every (b, h) is written
 *   lse        : fp32 [B, H, N] natural-log sum of exp(scale*q.k) over the retained valid
 *                keys, raster order; may be NULL
 *   ws, ws_bytes : device workspace of at least bsa_workspace_bytes(g, NULL) bytes; the
 *                call rebuilds its work list there, so it may not be shared with a
 *                concurrently running call
 * For each query token: softmax over the valid tokens of its retained key tiles, fp32
 * scores and statistics, bf16 probabilities into the P.V product, fp32 accumulation. */
int bsa_sparse_attn_fwd(const bsa_geom* g, const void* qt, const void* kt, const void* vt,
                        const uint32_t* mask, const int32_t* kv_count, float softmax_scale,
                        void* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/* Block-sparse attention forward under a token-level circular support (window kind 2 of
 * bsa_mask_params; Token Radius Attention summary: query-centred circular neighbourhoods,
 * base radius applied across frames with temporal decay).
 *   Arguments as bsa_sparse_attn_fwd, plus
 *   dense        : device pointer, uint8 [B, NQT]; nonzero marks a dense row (see
 *                  bsa_route_flags_offset for the flags bsa_build_mask leaves in its
 *                  workspace)
 *   token_radius : the support radius rho in tokens, 0 <= rho <= 32767
 * A local row (dense == 0) sees, in each retained key tile that is a window tile of its
 * query tile (window kind 2 with radius rho), only the key tokens in the support of each
 * query token: |t_k - t_q| <= rho and (y_k - y_q)^2 + (x_k - x_q)^2 <= (rho - |t_k - t_q|)^2.
 * Other retained tiles, and every tile of a dense row, are seen whole. Every query token
 * sees at least itself, so no row is empty. Errors as bsa_sparse_attn_fwd; a null dense or
 * a radius out of range is BSA_ERR_INVALID_ARG. */
int bsa_sparse_attn_fwd_token(const bsa_geom* g, const void* qt, const void* kt, const void* vt,
                              const uint32_t* mask, const int32_t* kv_count, const uint8_t* dense,
                              int token_radius, float softmax_scale, void* out, float* lse, void* ws,
                              size_t ws_bytes, void* stream);

/* Byte offset in the workspace at which bsa_build_mask leaves the route flags of its call
 * (uint8 [B, NQT], 1 = dense row), valid until the workspace is given to another
 * bsa_build_mask call. The attention calls do not touch that region, so the flags may be
 * passed to bsa_sparse_attn_fwd_token together with the same workspace. 0 for an invalid
 * geometry. Host only. */
size_t bsa_route_flags_offset(const bsa_geom* g);

/* Block-sparse attention forward without a workspace argument. The papers have no
 * counterpart: this entry point exists for callers that cannot allocate device memory,
 * such as a plug-in inside a host application that owns all device memory through its own
 * allocator and hands the plug-in tensors but no allocator, or a serving loop that bans
 * cudaMalloc after start-up because it can block and synchronise the device.
 *   Arguments as bsa_sparse_attn_fwd, minus ws / ws_bytes, plus
 *   kernel_errors : optional device pointer to one uint32; if not NULL it receives the
 *                   call's kernel error word (BSA_KERR_* bits) at the end of the call
 * Scratch: a fixed 1 MiB array inside the library (a file-scope device array that every
 * GPU which loads the library holds until the process exits). A call needs
 * 256 + align256(16*B*H) + 32*B*H*(floor(NT/4) + 2) bytes of it (about 61 KB for 12 heads
 * of 624 tiles, 464 KB for 40 heads of 1440 tiles); a larger call is rejected with
 * BSA_ERR_WORKSPACE before anything is launched. The call allocates and frees nothing.
 * Every call uses the same array and leaves its contents there: each call zeroes the
 * array's header on its stream before use, and calls that overlap on the GPU (other
 * streams, other host threads, same device) race on the array and must not be issued.
 * Every call made outside stream capture looks the array's device address up again (with
 * the call's device current), so the address stays valid after a device reset, which
 * reloads the library's module. A call captured into a CUDA graph uses the address looked
 * up by the last uncaptured call on that device (make one before the first capture), and
 * the graph holds that address: re-capture it after a device reset. */
int bsa_sparse_attn_fwd_fixed_scratch(const bsa_geom* g, const void* qt, const void* kt, const void* vt,
                                      const uint32_t* mask, const int32_t* kv_count, float softmax_scale,
                                      void* out, float* lse, uint32_t* kernel_errors, void* stream);

/* Number of kernels the library launched since it was loaded (all entry points, all
 * threads). Host-side counter, for accounting only. */
uint64_t bsa_launch_count(void);

/* Self-test of the kernels' bounded waits (no counterpart in the papers). Launches one
 * warp that waits, with the same bounded mbarrier wait the attention kernel uses, on a
 * barrier that nothing ever arrives on, giving up after `limit_cycles` SM cycles (> 0, at
 * most 4e9). On time-out the wait sets BSA_KERR_WAIT_TIMEOUT in *err (device memory, 4-byte
 * aligned, OR-ed in) and the kernel returns: the CUDA context stays usable. This is how a
 * lost arrival (a producer that never delivers) surfaces to the caller, checked without
 * faulting or hanging a GPU. Asynchronous on `stream`; returns BSA_ERR_INVALID_ARG for a
 * null or misaligned err or an out-of-range limit. */
int bsa_selftest_bounded_wait(long long limit_cycles, uint32_t* err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */

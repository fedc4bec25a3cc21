/*
 * dsa.h - C ABI of a B200 (sm_100a) library for 3D Deformable Slide Attention (3D-DSA).
 *
 * The operator.  3D-DSA is the motion-adaptive local attention of "MegaSlide-DiT:
 * Memory-Centric Adaptation and Deformable Local Attention for Efficient Video Diffusion"
 * (abstract), which makes attention cost linear in the sequence length; its window is
 * tile-granular in the manner of "Fast Video Generation with Sliding Tile Attention"
 * (abstract: attention over a local spatial-temporal region).  The pages give the operator
 * in outline only; this library fixes the following concrete form.
 *
 *   - Tokens form a T x H x W grid, cut into tiles of tt x th x tw tokens; the tile grid is
 *     G = (T/tt, H/th, W/tw).  Per axis the window is w' = min(w, G) tiles long.
 *   - Query tile i carries an integer offset o (tile units).  Per axis its window starts at
 *         s = clamp(i + o - floor(w'/2), 0, G - w'),
 *     i.e. it is centred on i + o and then moved to lie fully inside the tile grid.
 *   - Every query token n of tile i attends to exactly the tokens K(i) of the tiles in that
 *     window:  O_n = sum_m softmax_m(scale * <q_n, k_m>) v_m,  LSE_n = ln sum_m exp(scale * <q_n, k_m>).
 *
 * Layouts (all contiguous, row-major):
 *   q, k, v, out, dout, dq, dk, dv : [B, heads, T, H, W, d]  (token n = (t*H + h)*W + w)
 *   lse                            : [B, heads, T, H, W] fp32, natural log
 *   tile_offsets                   : int32 [nTiles, 3] = (dt, dh, dw) per query tile, tiles in
 *                                    raster order (t outer, w inner); shared by all B and heads
 *   starts                         : int32 [nTiles, 3] window start per axis (tile units)
 *   kv_tiles                       : int32 [nTiles, Wt] key tiles of each window, ascending
 *   inv_row_ptr, inv_q_tiles       : CSR of the inverse map: row j lists, ascending, the query
 *                                    tiles whose window holds key tile j (nnz = nTiles * Wt)
 *
 * Ownership and execution.  Every pointer argument except `p` (and the host buffers of
 * dsa_fwd_host) is DEVICE memory owned by the caller.  The library allocates no memory:
 * scratch lives in the caller's workspace (dsa_workspace_size).  All work is enqueued on
 * `stream` (a cudaStream_t; NULL = the legacy default stream) and returns without waiting.
 * The library holds no per-call state and may be called from several threads.  The device-
 * buffer entry points allocate and synchronise nothing, so they can be captured in a CUDA
 * graph (after one call outside the capture); dsa_fwd_host creates streams and events and
 * cannot.
 *
 * Errors.  Argument errors are returned synchronously and nothing is launched.  A launch
 * error returns DSA_ERR_CUDA.  Kernels never trap: a device-side failure (a bounded wait
 * that ran out, an index outside its buffer) is recorded in a device status word that
 * dsa_device_status() reads.
 *
 * Supported: bf16 with d = 128 on the tensor-core path, where a tile's 128-token chunks and
 * the backward's 64-token query chunks must be whole (h, w) planes (th*tw divides 64 and
 * 128/(th*tw) divides tt), and for the backward tw a multiple of 4;
 * fp32 with d in {64, 128} on the exact-fp32 path (any tile shape).  Pointers of the bf16
 * path must be 16-byte aligned.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1, /* a size, pointer, alignment or shape is invalid */
  DSA_ERR_UNSUPPORTED = 2, /* valid, but outside what the kernels implement */
  DSA_ERR_CUDA = 3,        /* a CUDA call or launch failed */
  DSA_ERR_TIMEOUT = 4,     /* a device-side bounded wait ran out */
  DSA_ERR_WORKSPACE = 5,   /* workspace missing or smaller than dsa_workspace_size() */
  DSA_ERR_DEVICE = 6       /* a device-side bounds check failed */
} dsa_status_t;

typedef enum { DSA_F32 = 0, DSA_BF16 = 1 } dsa_dtype_t;

typedef struct {
  int32_t B, heads, d;  /* batch, heads, head dimension */
  int32_t T, H, W;      /* token grid */
  int32_t tile[3];      /* tt, th, tw: tokens per tile along T, H, W */
  int32_t window[3];    /* wt, wh, ww: window length in tiles (limited to the tile grid) */
  float scale;          /* softmax scale, > 0 (usually 1/sqrt(d)) */
  int32_t dtype;        /* dsa_dtype_t of q, k, v, out, dout, dq, dk, dv */
} dsa_problem_t;

/* Which call a workspace is sized for. */
typedef enum { DSA_WS_FWD = 0, DSA_WS_BWD = 1 } dsa_ws_kind_t;

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t dsa_version(void);

/* Human-readable name of a status code (static string). */
const char* dsa_status_string(dsa_status_t s);

/* Plan sizes of a problem: *n_tiles = nTiles, *window_tiles = Wt (per-axis min(w, G)
 * multiplied).  Host only; validates the shape (not the dtype-specific limits). */
dsa_status_t dsa_plan_shape(const dsa_problem_t* p, int32_t* n_tiles, int32_t* window_tiles);

/* Bytes of device workspace dsa_fwd (kind = DSA_WS_FWD) or dsa_bwd (DSA_WS_BWD) needs;
 * 0 if the problem is invalid. */
size_t dsa_workspace_size(const dsa_problem_t* p, int32_t kind);

/* Window planner (the window rule above).  Writes starts[nTiles,3] and kv_tiles[nTiles,Wt];
 * if both inv_row_ptr[nTiles+1] and inv_q_tiles[nTiles*Wt] are non-NULL also the inverse
 * CSR.  All pointers are device memory. */
dsa_status_t dsa_plan(const dsa_problem_t* p, const int32_t* tile_offsets, int32_t* starts, int32_t* kv_tiles,
                      int32_t* inv_row_ptr, int32_t* inv_q_tiles, void* stream);

/* Forward: plans the windows of tile_offsets, then writes out (dtype of p) and lse (fp32).
 * workspace: device memory of at least dsa_workspace_size(p, DSA_WS_FWD) bytes, 256-byte
 * aligned; its contents on entry do not matter.  bf16 tiles of an even number of 128-token
 * chunks run on clusters of two CTAs (one product per pair of SMs over two chunks of a
 * tile), other tiles on one CTA per chunk; every row's arithmetic is the same in both. */
dsa_status_t dsa_fwd(const dsa_problem_t* p, const void* q, const void* k, const void* v,
                     const int32_t* tile_offsets, void* out, float* lse, void* workspace, size_t ws_bytes,
                     void* stream);

/* Forward from and to HOST memory (pinned, for asynchronous copies): copies q, k, v and
 * tile_offsets into the caller's device buffer `dev`, runs dsa_fwd there, and copies out and
 * lse back.  The work is pipelined over up to 24 groups of (batch, head) slices: copies in
 * run on one internal stream, the forward of each group on `stream`, copies back on a
 * second internal stream, ordered by events, so both copy directions overlap the kernels.
 * Everything the call enqueues happens after the work already on `stream`, and `stream`
 * reaches the end of the call only after the last copy back.  dev: at least
 * dsa_fwd_host_bytes(p) bytes of device memory, 256-byte aligned.  The host buffers must
 * stay valid until the stream reaches the end of the call (after an error return, until
 * the device is idle). */
size_t dsa_fwd_host_bytes(const dsa_problem_t* p);
dsa_status_t dsa_fwd_host(const dsa_problem_t* p, const void* q_host, const void* k_host, const void* v_host,
                          const int32_t* tile_offsets_host, void* out_host, float* lse_host, void* dev,
                          size_t dev_bytes, void* stream);

/* Backward of L = sum(out * dout) (gradients of the forward above with respect to q, k, v;
 * the integer offsets have none; the full-parameter adaptation of the MegaSlide-DiT
 * abstract needs them).  out and lse are the forward's outputs for the same inputs.
 * Writes dq, dk, dv (dtype of p).  Two passes on the tensor cores: a key-major kernel sums
 * dk and dv of each key row over the query tiles whose window holds it, a query-major
 * kernel sums dq of each query row over its window; every sum runs in one CTA in a fixed
 * order, so the gradients are identical from run to run.  workspace: at least
 * dsa_workspace_size(p, DSA_WS_BWD) bytes; its contents on entry do not matter.
 * bf16 only. */
dsa_status_t dsa_bwd(const dsa_problem_t* p, const void* q, const void* k, const void* v, const void* out,
                     const float* lse, const void* dout, const int32_t* tile_offsets, void* dq, void* dk, void* dv,
                     void* workspace, size_t ws_bytes, void* stream);

/* Forward that allocates nothing and takes no workspace, for callers that cannot
 * allocate device memory (a plugin whose host engine owns all device memory, a loop that
 * must not call cudaMalloc because it can synchronize the device, a process with a memory
 * budget fixed at start-up).  It computes exactly what dsa_fwd computes; the paper has no
 * counterpart of this entry point.  The planner's scratch is a fixed 256 KB device array
 * inside the library, held by every GPU that loads it until the process exits, so a
 * problem must satisfy  roundup(3 * nTiles, 64) + nTiles * Wt <= 65536;  larger ones
 * return DSA_ERR_UNSUPPORTED before anything is launched.  The first call on each device
 * looks up the array's device address (make that first call before any stream capture);
 * the address is cached with the context it was found in and looked up again, on the next
 * call, if the device's context has changed (after cudaDeviceReset).  All calls on a
 * device share the array and each call's planner rewrites every entry its forward reads:
 * calls whose work overlaps on the GPU (other streams, other threads) race and must be
 * serialized by the caller. */
dsa_status_t dsa_fwd_noalloc(const dsa_problem_t* p, const void* q, const void* k, const void* v,
                             const int32_t* tile_offsets, void* out, float* lse, void* stream);

/* Key-tile lists: the block-sparse form of the operator.  Instead of the window box, query
 * tile i attends to every token of the key tiles kv_list[kv_row_ptr[i] .. kv_row_ptr[i+1]-1]
 * (tile indices in raster order of the tile grid, any order within a row).  This is the
 * generalisation MOD-DiT's online block masking uses (the MOD-DiT page, Method section,
 * Stage 2 "Online Block Masking": attention over selected key blocks); the window form is
 * the case kv_row_ptr[i] = i * Wt with the plan's key tiles.
 *   per_head = 0: one list for every (batch, head): kv_row_ptr is device int32 [nTiles + 1];
 *   per_head = 1: a list per (batch, head) (head-adaptive sparsity, or per-head offsets via
 *                 dsa_plan_heads): kv_row_ptr is [B * heads, nTiles + 1], row i of head h at
 *                 kv_row_ptr[h * (nTiles + 1) + i], with absolute positions in kv_list;
 *   in both cases kv_row_ptr, read as one sequence, starts at 0, never decreases and ends at
 *   nnz (so each head's rows follow the previous head's); kv_list: device int32 [nnz] (may
 *   be NULL when nnz = 0), entries in [0, nTiles).  A tile listed twice in a row counts
 *   twice (the softmax runs over the multiset); an empty row gives out = 0 and lse = -inf.
 *   p->window is not used (any positive values).
 * The lists are checked on the device: a violation is recorded in the status word
 * (DSA_ERR_DEVICE from dsa_device_status) and the results are then unspecified; every
 * index the kernels take from the lists is clamped, so an invalid list never makes them
 * read or write outside the buffers.  bf16 with d = 128, tile limits as dsa_fwd.
 * The forward needs no workspace; the backward builds the inverse lists in its workspace
 * of at least dsa_list_workspace_size(p, nnz, per_head, DSA_WS_BWD) bytes (256-byte
 * aligned, contents on entry do not matter). */
size_t dsa_list_workspace_size(const dsa_problem_t* p, int32_t nnz, int32_t per_head, int32_t kind);
dsa_status_t dsa_fwd_list(const dsa_problem_t* p, const void* q, const void* k, const void* v,
                          const int32_t* kv_row_ptr, const int32_t* kv_list, int32_t nnz, int32_t per_head, void* out,
                          float* lse, void* stream);
dsa_status_t dsa_bwd_list(const dsa_problem_t* p, const void* q, const void* k, const void* v, const void* out,
                          const float* lse, const void* dout, const int32_t* kv_row_ptr, const int32_t* kv_list,
                          int32_t nnz, int32_t per_head, void* dq, void* dk, void* dv, void* workspace,
                          size_t ws_bytes, void* stream);

/* Text prefix (token-type-aware attention; the MOD-DiT page, "Token-Type-Aware Masking":
 * in unified text + video attention, text tokens get full attention and only video-video
 * attention is sparse).  With L_text text tokens q_text, k_text, v_text (device bf16
 * [B, heads, L_text, 128]) beside the video tokens q, k, v of p:
 *   every video query attends to the keys of its window (tile_offsets, as dsa_fwd) and to
 *   every text key;  every text query attends to every text key and every video key.
 * Writes out, lse (video, as dsa_fwd) and out_text [B, heads, L_text, 128] bf16, lse_text
 * [B, heads, L_text] fp32.  The parts are computed on the tensor cores separately (the
 * window kernel, and dense attention between flat token sequences) and merged exactly by
 * their LSEs.  L_text = 0 is dsa_fwd (the text pointers may then be NULL).  workspace: at
 * least dsa_prefix_workspace_size(p, L_text) bytes, 256-byte aligned.  bf16, d = 128. */
size_t dsa_prefix_workspace_size(const dsa_problem_t* p, int32_t L_text);
dsa_status_t dsa_fwd_prefix(const dsa_problem_t* p, const void* q, const void* k, const void* v,
                            const int32_t* tile_offsets, int32_t L_text, const void* q_text, const void* k_text,
                            const void* v_text, void* out, float* lse, void* out_text, float* lse_text,
                            void* workspace, size_t ws_bytes, void* stream);

/* Backward of dsa_fwd_prefix: gradients of L = sum(O * dO) over both token types, each
 * query's softmax over its key set as in dsa_fwd_prefix, given that call's out, lse,
 * out_text, lse_text and the output gradients dout [B, heads, T, H, W, 128] and dout_text
 * [B, heads, L_text, 128] (bf16).  Writes dq, dk, dv (video, the layout of q) and dq_text,
 * dk_text, dv_text (the layout of q_text), bf16.  Video keys are reduced over their windows'
 * queries and every text query by the key-major backward kernel; text keys over every video
 * and text query by the same kernel in a flat-key mode (query chunks cut into parts for
 * load balance); video queries' dQ over their windows' keys and every text key by the
 * query-major kernel; text queries' dQ over every key by that kernel in a flat mode (key
 * chunks cut into parts).  The parts' fp32 sums are added in part order and nothing is
 * summed with atomics, so the gradients are identical from run to run.  L_text = 0 is dsa_bwd
 * (text pointers may be NULL).  workspace: at least dsa_bwd_prefix_workspace_size(p, L_text)
 * bytes, 256-byte aligned.  bf16, d = 128. */
size_t dsa_bwd_prefix_workspace_size(const dsa_problem_t* p, int32_t L_text);
dsa_status_t dsa_bwd_prefix(const dsa_problem_t* p, const void* q, const void* k, const void* v, const void* out,
                            const float* lse, const void* dout, const int32_t* tile_offsets, int32_t L_text,
                            const void* q_text, const void* k_text, const void* v_text, const void* out_text,
                            const float* lse_text, const void* dout_text, void* dq, void* dk, void* dv,
                            void* dq_text, void* dk_text, void* dv_text, void* workspace, size_t ws_bytes,
                            void* stream);

/* Block attention mass (the sparsity map that block masks are chosen from; MOD-DiT page,
 * Method section and project structure: attention fused with a sparsity map): for every
 * (batch, head) h, query tile i and key tile j,
 *   map[h][i][j] = (1 / tile tokens) * sum over the query tokens n of tile i and the
 *                  tokens m of key tile j in i's list of exp(scale * q_n . k_m - lse_n),
 * the mean attention probability tile i's queries put on tile j (each listed occurrence of
 * j counts; j not listed: 0).  lse: the LSE dsa_fwd_list wrote for the same inputs and lists
 * (then every non-empty row of the map sums to one); dense attention is the list of every
 * tile.  Lists as dsa_fwd_list.  map: device fp32 [B * heads, nTiles, nTiles], overwritten.
 * The scores are recomputed on the tensor cores; one CTA sums each row of the map (all
 * chunks of query tile i) in fp32 in a fixed order, so the map is the same from run to run.
 * A row of the lists may hold at most 1024 entries here (a longer row is recorded as
 * DSA_ERR_DEVICE, site 48, and its map row left zero).  bf16, d = 128. */
dsa_status_t dsa_block_map(const dsa_problem_t* p, const void* q, const void* k, const float* lse,
                           const int32_t* kv_row_ptr, const int32_t* kv_list, int32_t nnz, int32_t per_head, float* map,
                           void* stream);

/* Per-(batch, head) window offsets as per-head key-tile lists: head h = b * heads + j
 * plans its own offsets tile_offsets[h][i][3] (device int32 [B * heads, nTiles, 3], the
 * window rule of dsa_plan) into kv_list[(h * nTiles + i) * Wt ...] (device int32
 * [B * heads * nTiles * Wt]) with kv_row_ptr[h][i] = (h * nTiles + i) * Wt (device int32
 * [B * heads, nTiles + 1]), ready for dsa_fwd_list / dsa_bwd_list with per_head = 1 and
 * nnz = B * heads * nTiles * Wt. */
dsa_status_t dsa_plan_heads(const dsa_problem_t* p, const int32_t* tile_offsets, int32_t* kv_row_ptr, int32_t* kv_list,
                            void* stream);

/* Regularised least squares with a cached factorisation (the MOD-DiT page, Method
 * section, Stage 1 "Sparsity Map Reconstruction": pattern intensities X from
 * (M^T M + lambda I) X = M^T S_t, where the design matrix M depends only on the sequence
 * geometry, so its factorisation is computed once and reused across heads and steps).
 * The page does not define the structural bases that make up M, so M is the caller's:
 *   M: device fp32 [m, p] row-major (m observations, e.g. the entries of a block map;
 *      p patterns, 1 <= p <= 32); lambda >= 0.
 * dsa_lstsq_factor writes the Cholesky factor L of M^T M + lambda I (lower triangle, device
 * fp64 [p, p], upper triangle zero); a matrix that is not positive definite is recorded as
 * DSA_ERR_DEVICE (site 95).  dsa_lstsq_solve solves for a batch of right-hand sides
 * S (device fp32 [batch, m], one map per row, batch <= 65535) into X (device fp32
 * [batch, p]) with L from dsa_lstsq_factor, in one launch (a cluster of 8 CTAs per map sums
 * M^T s in fp64 and combines the partial sums through distributed shared memory).  It needs
 * no workspace: dsa_lstsq_workspace_size returns 0 and workspace may be NULL.  Sums and
 * solves run in fp64 in a fixed order, so X is the same from run to run. */
size_t dsa_lstsq_workspace_size(int32_t m, int32_t p, int32_t batch);
dsa_status_t dsa_lstsq_factor(int32_t m, int32_t p, const float* M, float lambda, double* L, void* stream);
dsa_status_t dsa_lstsq_solve(int32_t m, int32_t p, int32_t batch, const float* M, const double* L, const float* S,
                             float* X, void* workspace, size_t ws_bytes, void* stream);

/* Waits for `stream`, then reads and clears the device status word of the current device.
 * Returns DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_DEVICE (or DSA_ERR_CUDA if the read failed);
 * site / block (either may be NULL) receive where the first failure was raised. */
dsa_status_t dsa_device_status(void* stream, int32_t* site, int32_t* block);

/* Failure-path self-test: enqueues one small kernel that waits on a barrier nothing ever
 * completes, through the same bounded wait every kernel of the library uses.  After the
 * wait's limit (2 s of the device clock) it records DSA_DEV_TIMEOUT at site 99 and returns,
 * so dsa_device_status() then reports DSA_ERR_TIMEOUT with *site = 99 and the context stays
 * usable.  Nothing faults, traps or hangs. */
#define DSA_SELFTEST_SITE 99
dsa_status_t dsa_selftest_wait(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */

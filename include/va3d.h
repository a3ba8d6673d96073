/*
 * va3d: 3D-RoPE video self-attention for NVIDIA B200 (sm_100a).
 *
 * C ABI of libva3d.so.  Plain pointers and sizes only; no CUDA or framework
 * types appear in the signatures (a CUDA stream is passed as void*).
 *
 * Operations and where they are defined:
 *  - token grid: "A video model's architecture: spatiotemporal attention and
 *    the 3D VAE" (anrans.github.io ai-infra-handbooks), section "The latents:
 *    the extra time axis": T' = 1 + (T-1)/4, H' = H/8/2, W' = W/8/2;
 *  - 3D RoPE: same page, section "Position: RoPE in three dimensions" (head
 *    dim split into t, h and w ranges, each rotated by its coordinate), and
 *    "CogVideoX Architecture ..." (aifetchly-blog) section 3, block-diagonal
 *    R_3D(t, y, x);
 *  - full, spatial and temporal attention: handbook page, section "How
 *    attention sees time: factorised or full";
 *  - joint video+text attention: "04 HunyuanVideo and Wan" (note.shouss.top)
 *    sections 2.3-2.4, and the handbook's diffusers example (video tokens +
 *    text tokens attended together in one sequence);
 *  - text cross-attention: the same page, section 3.1 (Wan's block);
 *  - local 3D-window attention: anthology-of-the-sota record sota-390
 *    (W.A.L.T's local 3D-window blocks, the one numbered comparison against
 *    full attention it cites);
 *  - context parallelism (Ulysses and ring exchanges, one process per GPU):
 *    the same record (long videos turn to context parallelism) and the
 *    handbook's RoPE section (each rank's token coordinates are absolute).
 *
 * Conventions shared by every entry point
 *  - Tensors are contiguous bf16 (bit patterns, va3d_bf16) of shape
 *    [B, heads, N, head_dim], row-major, head_dim innermost.  Every pointer
 *    must be 16-byte aligned.  head_dim must be 128.
 *  - Token n of a sequence is a video token when n < T'H'W', with
 *    t = n / (H'W'), h = (n / W') % H', w = n % W' (w fastest); tokens
 *    n >= T'H'W' are text tokens, which carry no position (identity RoPE).
 *    N must equal T'H'W' + n_text.
 *  - RoPE: the head dim is split into ranges [0, d_t), [d_t, d_t+d_h),
 *    [d_t+d_h, 128) turned by t, h and w; inside a range of width d the
 *    adjacent pair (2j, 2j+1) turns by pos * theta^(-2j/d).
 *  - Memory is owned by the caller.  No compute entry point allocates device
 *    memory; scratch space is the caller's `workspace` (size from
 *    va3d_workspace_bytes).  The one allocating call, va3d_region_alloc, is a
 *    set-up call for the context-parallel exchange regions.  Device pointers must belong to the current
 *    device.  Two calls that share a workspace must not overlap in time.
 *  - Calls are asynchronous on `stream` (NULL = legacy default stream).  The
 *    return value reports argument errors and launch errors only; device-side
 *    faults surface at the caller's next synchronisation.  A device-side
 *    watchdog (every wait in the kernels is bounded) records a code that
 *    va3d_device_error() returns.
 *  - Entry points are thread-safe.  They keep no mutable host state, except
 *    attn3d_full_fwd_noalloc's per-device address cache (mutex-guarded).
 */
#ifndef VA3D_H
#define VA3D_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t va3d_bf16;   /* bf16 bit pattern */

/* Post-patch token grid and RoPE split. */
typedef struct va3d_grid {
    int T, H, W;        /* latent grid after patchify: T', H', W' (each >= 1) */
    int n_text;         /* text tokens appended after the video tokens (>= 0) */
    int d_t, d_h, d_w;  /* RoPE ranges; each even and >= 0, sum == head_dim */
    double theta;       /* RoPE base (> 0), 10000 for the models on the pages */
} va3d_grid_t;

/* Status codes (0 = success, negative = error). */
enum {
    VA3D_OK = 0,
    VA3D_ERR_INVALID = -1,      /* null pointer, non-positive size, inconsistent grid */
    VA3D_ERR_UNSUPPORTED = -2,  /* head_dim != 128, or a size the kernels do not cover */
    VA3D_ERR_ALIGNMENT = -3,    /* a pointer is not 16-byte aligned */
    VA3D_ERR_WORKSPACE = -4,    /* workspace missing or smaller than va3d_workspace_bytes */
    VA3D_ERR_CUDA = -5,         /* a CUDA runtime or driver call failed */
    VA3D_ERR_DEVICE = -6,       /* current device is not compute capability 10.0 */
    VA3D_ERR_SCRATCH_LIMIT = -7 /* needs more than the built-in scratch of the no-alloc entry */
};

/* Flags for the attention entry points. */
enum {
    VA3D_K_ROTATED = 1          /* `k` already holds RoPE-rotated keys (no key pre-pass) */
};

/* Device-side watchdog codes returned by va3d_device_error(). */
enum {
    VA3D_DEVERR_NONE = 0,
    VA3D_DEVERR_TIMEOUT_LOAD = 1,     /* a wait in the tile-loading role timed out */
    VA3D_DEVERR_TIMEOUT_MMA = 2,      /* a wait in the MMA-issuing role timed out */
    VA3D_DEVERR_TIMEOUT_SOFTMAX = 3,  /* a wait in the softmax role timed out */
    VA3D_DEVERR_TIMEOUT_SELFTEST = 4, /* the wait of va3d_watchdog_selftest timed out (expected) */
    VA3D_DEVERR_TIMEOUT_PEER = 5      /* va3d_ulysses_wait gave up on its peers */
};

/* Human-readable text of a status code; never NULL. */
const char *va3d_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int va3d_version(void);

/*
 * Token grid of a clip (handbook, "The latents: the extra time axis"):
 * T' = 1 + (frames - 1)/4, H' = height/16, W' = width/16.  Requires
 * frames = 4k + 1 >= 1 and height, width positive multiples of 16 (the
 * causal VAE's 4k+1 frame rule, 8x spatial compression, 2x2 patches);
 * otherwise returns VA3D_ERR_INVALID and leaves *out untouched.  The RoPE
 * split and text length are copied into *out; theta is set to 10000.
 * Host-only; needs no device.
 */
int va3d_grid_from_video(int frames, int height, int width, int d_t, int d_h, int d_w,
                         int n_text, va3d_grid_t *out);

/*
 * Bytes of scratch space attn3d_full_fwd / attn_factorized_fwd need for
 * these arguments: a cos/sin table of the grid's rotation angles
 * (8 * (T'*d_t/2 + H'*d_h/2 + W'*d_w/2) bytes, rounded up to 256) plus,
 * unless flags has VA3D_K_ROTATED, the rotated keys (B*heads*N*head_dim*2
 * bytes), plus scratch for splitting the query tiles of the last partial wave
 * over two key halves (min(128, tiles) * 266,244 bytes, rounded up to 256,
 * with tiles = B*heads*ceil(N/256)).  Returns 0 for invalid arguments.
 * Host-only.
 */
size_t va3d_workspace_bytes(int B, int heads, int N, int head_dim, const va3d_grid_t *grid,
                            unsigned flags);

/*
 * 3D RoPE (handbook "Position: RoPE in three dimensions"; CogVideoX guide
 * section 3, R_3D block-diagonal matrix): y = R_3D(t, h, w) x for every
 * video token, y = x for text tokens.
 *   x, y    device, [B, heads, N, head_dim] bf16; x == y (in place) is allowed,
 *           other overlap is not.  Output rounded to bf16 (nearest even);
 *           angles are computed in fp32 from fp64 inverse frequencies.
 *   stream  cudaStream_t or NULL.
 * Errors: VA3D_ERR_INVALID, _UNSUPPORTED, _ALIGNMENT, _DEVICE, _CUDA.
 */
int rope3d_apply(const va3d_bf16 *x, va3d_bf16 *y, int B, int heads, int N, int head_dim,
                 const va3d_grid_t *grid, void *stream);

/*
 * Full 3D attention (handbook "How attention sees time": every token attends
 * to every token); with grid->n_text > 0 this is joint video+text attention
 * (HunyuanVideo/CogVideoX joint attention over the concatenated sequence,
 * text appended after the video tokens, no mask):
 *   o = softmax(scale * RoPE(q) RoPE(k)^T) v,   lse = log-sum-exp of the row.
 *   q, k, v   device, [B, heads, N, head_dim] bf16, read only.  When flags
 *             has VA3D_K_ROTATED, k must already be rotated (e.g. by
 *             rope3d_apply) and q is still rotated inside the kernel.
 *   o         device, [B, heads, N, head_dim] bf16, written; must not overlap
 *             the inputs or the workspace.
 *   lse       device fp32 [B, heads, N] (natural log), or NULL.
 *   softmax_scale  <= 0 selects 1/sqrt(head_dim).
 *   workspace, workspace_bytes  device scratch of at least
 *             va3d_workspace_bytes(B, heads, N, head_dim, grid, flags) bytes,
 *             256-byte aligned; contents are overwritten.
 * Accumulation is fp32; P is rounded to bf16 before the PV product; o is
 * rounded to bf16 (nearest even).
 * Errors: VA3D_ERR_INVALID, _UNSUPPORTED, _ALIGNMENT, _WORKSPACE, _DEVICE, _CUDA.
 */
int attn3d_full_fwd(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v,
                    va3d_bf16 *o, float *lse, int B, int heads, int N, int head_dim,
                    const va3d_grid_t *grid, float softmax_scale, unsigned flags,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * Factorised spatiotemporal attention (handbook "How attention sees time":
 * spatial attention inside each frame, T' sequences of H'W' tokens, then
 * temporal attention at each spatial position, H'W' sequences of T' tokens).
 * Both passes read the same rotated q, k and v and write separate outputs:
 *   o_spatial  [B, heads, N, head_dim]: token attends to tokens with equal t;
 *   o_temporal [B, heads, N, head_dim]: token attends to tokens with equal (h, w).
 * Either output may be NULL to skip that pass.  grid->n_text must be 0.  The
 * temporal pass needs T' <= 64.  Other arguments as in attn3d_full_fwd.
 * Errors: as attn3d_full_fwd.
 */
int attn_factorized_fwd(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v,
                        va3d_bf16 *o_spatial, va3d_bf16 *o_temporal, int B, int heads, int N,
                        int head_dim, const va3d_grid_t *grid, float softmax_scale,
                        unsigned flags, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Local 3D-window attention (anthology-of-the-sota record sota-390, the
 * W.A.L.T comparison: blocks whose tokens attend only inside local 3D
 * windows).  The grid is cut into non-overlapping windows of
 * win_t x win_h x win_w tokens (each must divide T', H', W'); every video
 * token attends to the tokens of its own window, with the same 3D RoPE
 * (absolute coordinates) as full attention:
 *   o_i = softmax_j(scale * RoPE(q_i) . RoPE(k_j)) v_j over j in window(i).
 * grid->n_text must be 0.  win = (T', H', W') is full attention, (1, H', W')
 * the spatial pass, (T', 1, 1) the temporal pass.  Other arguments, the
 * workspace size (va3d_workspace_bytes with the same grid and flags),
 * results and errors as in attn3d_full_fwd.
 */
int attn_window_fwd(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v, va3d_bf16 *o,
                    float *lse, int B, int heads, int N, int head_dim, const va3d_grid_t *grid,
                    int win_t, int win_h, int win_w, float softmax_scale, unsigned flags,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * Bytes of optional scratch attn_cross_fwd can use (for splitting the query
 * tiles of the last partial wave over two key halves):
 * min(128, B*heads*ceil(Nq/256)) * 266,244, rounded up to 256.  Returns 0
 * for invalid arguments.  Host-only.
 */
size_t va3d_cross_workspace_bytes(int B, int heads, int Nq, int Nkv, int head_dim);

/*
 * Text cross-attention of a video block ("04 HunyuanVideo and Wan",
 * note.shouss.top, section 3.1, the steps of one Wan block: queries from the
 * video tokens, keys and values from the text encoder's tokens, up to 512 of
 * them; the text side is not updated).  No RoPE on either side:
 *   o = softmax(scale * q k^T) v,   lse = log-sum-exp of the row.
 *   q     device, [B, heads, Nq, head_dim] bf16 (video tokens), read only.
 *   k, v  device, [B, heads, Nkv, head_dim] bf16 (text tokens), read only;
 *         any Nkv >= 1.
 *   o     device, [B, heads, Nq, head_dim] bf16, written; must not overlap
 *         the inputs or the workspace.
 *   lse   device fp32 [B, heads, Nq] (natural log), or NULL.
 *   softmax_scale  <= 0 selects 1/sqrt(head_dim).
 *   workspace, workspace_bytes  optional device scratch, 256-byte aligned:
 *         NULL (or too small) runs every tile whole; with
 *         va3d_cross_workspace_bytes(...) bytes the last partial wave is
 *         split.  Contents are overwritten.
 * Accumulation is fp32; P is rounded to bf16 before the PV product; o is
 * rounded to bf16 (nearest even).
 * Errors: VA3D_ERR_INVALID, _UNSUPPORTED, _ALIGNMENT, _DEVICE, _CUDA.
 */
int attn_cross_fwd(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v, va3d_bf16 *o,
                   float *lse, int B, int heads, int Nq, int Nkv, int head_dim,
                   float softmax_scale, void *workspace, size_t workspace_bytes, void *stream);

/* Capacity of the built-in scratch used by attn3d_full_fwd_noalloc. */
#define VA3D_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * attn3d_full_fwd for callers that cannot allocate device memory and so cannot
 * hand in a workspace: for example a plugin running inside a host framework
 * that owns all device memory and passes in only its input and output
 * pointers, or code on a path where calling cudaMalloc is not allowed or too
 * slow.  (The pages have no counterpart; this is a property of the library.)
 *
 * Same arguments, results and errors as attn3d_full_fwd, minus the workspace.
 * Its scratch lives in one static device array of VA3D_NOALLOC_SCRATCH_BYTES
 * (64 MiB) built into the library; every GPU that loads the library holds
 * that array until the process exits.  The array must hold the angle table
 * and, unless VA3D_K_ROTATED, the rotated keys (B*heads*N*256 bytes); a call
 * whose table plus rotated keys exceed 64 MiB returns VA3D_ERR_SCRATCH_LIMIT
 * and launches nothing.  Without VA3D_K_ROTATED that allows up to
 * B*heads*N of about 262,000 rows (e.g. 7 heads of 32,760 tokens, not 8);
 * with it, any size the workspace entry takes.  Whatever is left of the
 * array after those parts serves as scratch for splitting the last partial
 * wave of query tiles; when too little is left, that wave runs whole (same
 * results, a little slower).  The function calls no allocator.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it per CUDA context (by the context's unique
 * id), so a call under another context, or after cudaDeviceReset, looks it
 * up again; make the first call of each context before any stream capture.
 * All calls share the one array, and each call writes the parts it reads
 * before reading them (the table, the rotated keys and the split counters),
 * so leftovers of the previous call do no harm; but calls that overlap in
 * time on the GPU (different streams, or different host threads, without
 * ordering between them) race on the array and give wrong results.  Order
 * them on one stream or synchronise.
 */
int attn3d_full_fwd_noalloc(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v,
                            va3d_bf16 *o, float *lse, int B, int heads, int N, int head_dim,
                            const va3d_grid_t *grid, float softmax_scale, unsigned flags,
                            void *stream);

/*
 * Watchdog self-test: launches one CTA whose mbarrier wait can never
 * complete (the arrival it waits for is never made).  The bounded wait gives
 * up after its limit (2 s), records VA3D_DEVERR_TIMEOUT_SELFTEST in the
 * device error word (unless another code is already there) and the kernel
 * exits; no trap, no fault, the context stays usable.  Asynchronous on
 * `stream`; read the result with va3d_device_error().
 * Errors: VA3D_ERR_DEVICE, _CUDA.
 */
int va3d_watchdog_selftest(void *stream);

/*
 * Last device-side watchdog code recorded on the current device
 * (VA3D_DEVERR_*; 0 = none).  Synchronises the device.  With reset != 0 the
 * word is cleared afterwards.  Returns VA3D_ERR_CUDA if it cannot be read.
 */
int va3d_device_error(int reset);

/* ------------------------------------------------------------------------
 * Ulysses context parallelism over peer memory (one process per GPU).
 *
 * The pages on full 3D attention name context parallelism (Ulysses and
 * ring) as what long videos turn to (anthology record sota-390, "budget for
 * that cost"), and note that 3D RoPE needs no exchange under sequence
 * parallelism because each rank's token coordinates are absolute (handbook
 * "A video model's architecture", section "Position: RoPE in three
 * dimensions").  Rank r of `world` holds the contiguous token slice
 * [r*N/world, (r+1)*N/world) of every head, as [B, heads, N/world, 128].
 * va3d_ulysses_scatter sends each head group (heads/world heads) with all
 * its tokens to the rank that owns it, turning keys by their global
 * positions on the way; attn3d_full_fwd then runs on whole sequences (keys
 * already rotated, VA3D_K_ROTATED); va3d_ulysses_gather sends each token
 * slice of the output back.  Transfers are 16-byte stores into the peers'
 * regions; each copy kernel then signals every peer's counter, and
 * va3d_ulysses_wait (bounded) orders a rank's next step after its peers'.
 *
 * Region (one per rank, device memory from va3d_region_alloc, mapped into
 * every rank with the IPC calls): a 256-byte header holding two u64
 * counters (scatter, gather; zero at allocation and never reset), then
 * Qh, Kh, Vh, each [B, heads/world, N, 128] bf16 (this rank's heads, all
 * tokens), then the O shard [B, heads, N/world, 128] bf16 (all heads, this
 * rank's tokens).  Requirements: 1 <= world <= 8, heads and N divisible by
 * world, 0 <= rank < world; the same shapes on every rank.
 * ---------------------------------------------------------------------- */

#define VA3D_IPC_HANDLE_BYTES 64

/* Bytes of one rank's region; 0 if the sizes are invalid or unsupported. */
size_t va3d_ulysses_region_bytes(int B, int heads, int N, int head_dim, int world);

/*
 * Byte offsets of Qh, Kh, Vh and the O shard inside a region (each
 * 256-byte aligned).  Errors: VA3D_ERR_INVALID, _UNSUPPORTED.
 */
int va3d_ulysses_offsets(int B, int heads, int N, int head_dim, int world, size_t *off_q,
                         size_t *off_k, size_t *off_v, size_t *off_o);

/*
 * Allocate `bytes` of device memory on the current device with cudaMalloc
 * and zero it (set-up time, not in a hot call; the counters must start at
 * zero).  The caller owns it and frees it with va3d_region_free.
 * Errors: VA3D_ERR_INVALID (bytes == 0 or ptr NULL), _CUDA.
 */
int va3d_region_alloc(size_t bytes, void **ptr);
int va3d_region_free(void *ptr);

/*
 * CUDA IPC handle (VA3D_IPC_HANDLE_BYTES bytes, written to `handle`) of a
 * region returned by va3d_region_alloc; va3d_ipc_open maps a peer's region
 * into this process (peer access enabled lazily) and va3d_ipc_close unmaps
 * it.  The handle travels between processes as plain bytes.
 * Errors: VA3D_ERR_INVALID (NULL arguments), _CUDA.
 */
int va3d_ipc_export(const void *region, unsigned char *handle);
int va3d_ipc_open(const unsigned char *handle, void **ptr);
int va3d_ipc_close(void *ptr);

/*
 * Scatter this rank's slice: q, k, v are [B, heads, N/world, 128] bf16
 * (16-byte aligned), `regions` a host array of `world` region pointers
 * valid in this process, index j = rank j's region (this rank's own at
 * index `rank`).  Writes rank j's Qh, Kh, Vh rows [rank*N/world,
 * (rank+1)*N/world) of heads [j*heads/world, (j+1)*heads/world); keys are
 * turned by 3D RoPE at their global positions unless flags has
 * VA3D_K_ROTATED.  Then adds, per block of its grid, 1 to every region's
 * scatter counter.  Asynchronous on `stream`.
 * Errors: VA3D_ERR_INVALID, _UNSUPPORTED, _ALIGNMENT, _DEVICE, _CUDA.
 */
int va3d_ulysses_scatter(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v,
                         void *const *regions, int world, int rank, int B, int heads, int N,
                         int head_dim, const va3d_grid_t *grid, unsigned flags, void *stream);

/*
 * Gather: o_heads is this rank's attention output [B, heads/world, N, 128]
 * bf16 (16-byte aligned).  Writes, for every rank j, its O shard rows of
 * heads [rank*heads/world, (rank+1)*heads/world); then adds, per block, 1
 * to every region's gather counter.  Asynchronous on `stream`.
 * Errors: as va3d_ulysses_scatter.
 */
int va3d_ulysses_gather(const va3d_bf16 *o_heads, void *const *regions, int world, int rank,
                        int B, int heads, int N, int head_dim, void *stream);

/*
 * Stream-ordered wait until this rank's counter for `phase` (0 scatter,
 * 1 gather) has received every peer's signals of call number `epoch`
 * (1, 2, ...), i.e. reaches epoch * world * blocks of that copy kernel.
 * Bounded: after 2 s it records VA3D_DEVERR_TIMEOUT_PEER in the device
 * error word and returns, so a rank that never arrives cannot hang the GPU
 * (the data read after it is then incomplete; check va3d_device_error).
 * Errors: VA3D_ERR_INVALID, _UNSUPPORTED, _DEVICE, _CUDA.
 */
int va3d_ulysses_wait(const void *region, int phase, unsigned long long epoch, int world, int B,
                      int heads, int N, int head_dim, void *stream);

/* ------------------------------------------------------------------------
 * Ring context parallelism (no head split, so any number of heads).
 *
 * Rank r holds tokens [r*N/world, (r+1)*N/world) of every head.
 * va3d_ring_load turns this rank's q and k by 3D RoPE at their global
 * positions (positions are absolute: handbook "A video model's
 * architecture", section "Position: RoPE in three dimensions") into q_rot
 * and the region's block buffer 0, with v.  Then for steps s = 0..world-1
 * the rank attends q_rot to the block in buffer s % 2 and merges that
 * partial output into an fp32 accumulator by log-sum-exp weights, in one
 * call, va3d_ring_attend (the merge runs in the attention kernel's epilogue;
 * the two-call form, attn_cross_fwd with its LSE then va3d_ring_merge,
 * computes the same), and, except at the last step, copies the block to the
 * next rank's buffer (s + 1) % 2 with va3d_ring_pass.  Ordering, all stream-ordered and bounded (2 s, then
 * VA3D_DEVERR_TIMEOUT_PEER): before va3d_ring_pass of step s of call c,
 * va3d_ring_wait(free, (c-1)*world + s) (the next rank has finished the
 * products that read that buffer); after each product va3d_ring_free on the
 * previous rank's region; before the product of step s+1,
 * va3d_ring_wait(full, (c-1)*(world-1) + s + 1) (the block has landed).
 *
 * Region (one per rank, from va3d_region_alloc; mapped into the previous
 * rank with the IPC calls): a 256-byte header with two u64 counters (full,
 * free), then K0, V0, K1, V1, each [B, heads, N/world, 128] bf16.
 * Requirements: 1 <= world <= 8, N divisible by world, 0 <= rank < world.
 * ---------------------------------------------------------------------- */

/* Bytes of one rank's ring region; 0 if the sizes are invalid. */
size_t va3d_ring_region_bytes(int B, int heads, int N, int head_dim, int world);

/* Byte offsets of K0, V0, K1, V1 inside a ring region (256-byte aligned).
 * Errors: VA3D_ERR_INVALID, _UNSUPPORTED. */
int va3d_ring_offsets(int B, int heads, int N, int head_dim, int world, size_t *off_k0,
                      size_t *off_v0, size_t *off_k1, size_t *off_v1);

/*
 * q, k, v: this rank's slice [B, heads, N/world, 128] bf16; q_rot: output of
 * the same shape (device, 16-byte aligned); region: this rank's region.
 * Keys are copied as they are if flags has VA3D_K_ROTATED.  Text tokens
 * (global index >= T'H'W') are not turned.  Asynchronous on `stream`.
 * Errors: VA3D_ERR_INVALID, _UNSUPPORTED, _ALIGNMENT, _DEVICE, _CUDA.
 */
int va3d_ring_load(const va3d_bf16 *q, const va3d_bf16 *k, const va3d_bf16 *v, va3d_bf16 *q_rot,
                   void *region, int world, int rank, int B, int heads, int N, int head_dim,
                   const va3d_grid_t *grid, unsigned flags, void *stream);

/*
 * Copy block buffer `buf` (0 or 1) of this rank's region into buffer 1-buf
 * of `next_region` (the next rank's region, mapped here), then add one per
 * block of its grid to the next rank's `full` counter.
 * Errors: VA3D_ERR_INVALID, _UNSUPPORTED, _ALIGNMENT, _DEVICE, _CUDA.
 */
int va3d_ring_pass(const void *region, void *next_region, int buf, int world, int B, int heads,
                   int N, int head_dim, void *stream);

/* Add one to the `free` counter of `prev_region` (the previous rank's).
 * Errors: VA3D_ERR_INVALID, _ALIGNMENT, _DEVICE, _CUDA. */
int va3d_ring_free(void *prev_region, void *stream);

/*
 * Bounded stream-ordered wait on this rank's counter `counter` (0 full,
 * 1 free): until `count` passes have landed (full; count * the pass grid's
 * blocks signals) or `count` frees have arrived (free).
 * Errors: VA3D_ERR_INVALID, _UNSUPPORTED, _ALIGNMENT, _DEVICE, _CUDA.
 */
int va3d_ring_wait(const void *region, int counter, unsigned long long count, int world, int B,
                   int heads, int N, int head_dim, void *stream);

/*
 * Merge one block's output o_blk [B, heads, n_rows, 128] bf16 and its LSE
 * lse_blk [B, heads, n_rows] fp32 (natural log) into the accumulator acc
 * [B, heads, n_rows, 128] fp32 whose LSE is lse_in; writes the merged LSE to
 * lse_out (a different buffer).  first != 0: the accumulator starts as this
 * block (lse_in unused).  out (nullable): also write the merged output as
 * bf16.  Errors: VA3D_ERR_INVALID, _UNSUPPORTED, _ALIGNMENT, _DEVICE, _CUDA.
 */
int va3d_ring_merge(const va3d_bf16 *o_blk, const float *lse_blk, float *acc, const float *lse_in,
                    float *lse_out, va3d_bf16 *out, int B, int heads, int n_rows, int first,
                    void *stream);

/*
 * One block step of the ring form with the merge done in the attention
 * kernel's epilogue (the product of va3d_ring_merge's inputs, without the
 * block output ever reaching memory as bf16): the block attention
 *   o_blk = softmax(scale * q_rot k^T) v,  l_blk = its log-sum-exp,
 * over the n_keys keys of k, v (no RoPE: q_rot and k come turned at their
 * global positions), merged into the accumulator as in va3d_ring_merge:
 *   first != 0:  acc = o_blk, lse_out = l_blk;
 *   otherwise:   with m = max(lse_in, l_blk),
 *                acc = (e^(lse_in-m) acc + e^(l_blk-m) o_blk) / (e^(lse_in-m) + e^(l_blk-m)),
 *                lse_out = m + log(e^(lse_in-m) + e^(l_blk-m)).
 * The block output is the normalised fp32 accumulator of the kernel (one
 * rounding less than va3d_ring_merge, which reads a bf16 o_blk).
 * (Anthology record sota-390: ring context parallelism for long videos;
 * log-sum-exp merging of softmax blocks over disjoint key sets.)
 *   q_rot       device bf16 [B, heads, n_rows, head_dim], read only.
 *   k, v        device bf16 [B, heads, n_keys, head_dim], read only.
 *   acc         device fp32 [B, heads, n_rows, head_dim], read (unless first)
 *               and written.
 *   lse_in      device fp32 [B, heads, n_rows] (natural log); NULL when first;
 *               must not alias lse_out.
 *   lse_out     device fp32 [B, heads, n_rows], written.
 *   out         device bf16 [B, heads, n_rows, head_dim] receiving the merged
 *               output as well (the last block), or NULL.
 *   softmax_scale  <= 0 selects 1/sqrt(head_dim).
 * Asynchronous on `stream`.  Every query tile runs whole (no workspace).
 * Errors: VA3D_ERR_INVALID, _UNSUPPORTED, _ALIGNMENT, _DEVICE, _CUDA.
 */
int va3d_ring_attend(const va3d_bf16 *q_rot, const va3d_bf16 *k, const va3d_bf16 *v, float *acc,
                     const float *lse_in, float *lse_out, va3d_bf16 *out, int B, int heads,
                     int n_rows, int n_keys, int head_dim, float softmax_scale, int first,
                     void *stream);

#ifdef __cplusplus
}
#endif

#endif /* VA3D_H */
